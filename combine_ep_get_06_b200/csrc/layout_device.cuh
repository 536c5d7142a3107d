// Device building blocks of the layout step, shared by the layout kernels
// and the fused small-batch layout+dispatch kernel.
//
// One thread per slot.  Inside a chunk of slots a slot's rank among the
// earlier slots of the same expert is
//   (equal-expert lanes before it in its warp: __match_any_sync + popc)
// + (equal-expert slots in earlier warps: an exclusive column scan over the
//    32 per-warp counts of each expert),
// so no atomic decides a position and the slot map is deterministic.
#pragma once

#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {
namespace layout_dev {

constexpr int kThreads = kLayoutThreads;
constexpr int kWarps = kThreads / 32;

template <typename IdxT>
__device__ __forceinline__ int read_expert(const IdxT* idx, int64_t s, int E, bool& bad) {
    long long e = (long long)__ldg(idx + s);
    if (e < -1 || e >= E) {
        bad = true;
        return -1;
    }
    return (int)e;
}

// Tokens per segment for the tokens whose slots this CTA holds, one slot
// per thread (slot s = base_slot + threadIdx.x, expert e or -1): a token
// counts once in every segment that at least one of its valid slots goes
// to.  When k divides 32 a token's slots share a warp and one
// __match_any_sync on (token, segment) finds the first slot of each pair;
// otherwise one thread per token walks its k slots.
template <typename IdxT>
__device__ __forceinline__ void count_segments(const IdxT* idx, int t0, int t1, int k, int E, int S,
                                               int e, int* seg) {
    const int per_seg = E / S;
    if ((32 % k) == 0) {
        const int lane = threadIdx.x & 31;
        const int g = e >= 0 ? e / per_seg : 0;
        const int key = e >= 0 ? ((lane / k) << 16) | g : -1 - lane;
        const unsigned peers = __match_any_sync(0xffffffffu, key);
        if (e >= 0 && (peers & lanemask_lt()) == 0) atomicAdd(&seg[g], 1);
        return;
    }
    for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
        const IdxT* row = idx + (int64_t)t * k;
        bool ignore = false;
        if (S <= 64) {
            unsigned long long mask = 0;
            for (int j = 0; j < k; ++j) {
                const int ej = read_expert(row, j, E, ignore);
                if (ej >= 0) mask |= 1ull << (ej / per_seg);
            }
            while (mask) {
                atomicAdd(&seg[__ffsll((long long)mask) - 1], 1);
                mask &= mask - 1;
            }
        } else {
            for (int j = 0; j < k; ++j) {
                const int ej = read_expert(row, j, E, ignore);
                if (ej < 0) continue;
                const int g = ej / per_seg;
                bool seen = false;
                for (int jj = 0; jj < j && !seen; ++jj) {
                    const int e2 = read_expert(row, jj, E, ignore);
                    seen = e2 >= 0 && e2 / per_seg == g;
                }
                if (!seen) atomicAdd(&seg[g], 1);
            }
        }
    }
}

// Inclusive scan of two ints over the whole CTA (kThreads threads).
__device__ __forceinline__ int2 block_inclusive_scan2(int x, int y, int* tmp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int xo = __shfl_up_sync(0xffffffffu, x, o);
        const int yo = __shfl_up_sync(0xffffffffu, y, o);
        if (lane >= o) {
            x += xo;
            y += yo;
        }
    }
    if (lane == 31) {
        tmp[warp] = x;
        tmp[kWarps + warp] = y;
    }
    __syncthreads();
    if (warp == 0) {
        int wx = tmp[lane], wy = tmp[kWarps + lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int xo = __shfl_up_sync(0xffffffffu, wx, o);
            const int yo = __shfl_up_sync(0xffffffffu, wy, o);
            if (lane >= o) {
                wx += xo;
                wy += yo;
            }
        }
        tmp[lane] = wx;
        tmp[kWarps + lane] = wy;
    }
    __syncthreads();
    if (warp > 0) {
        x += tmp[warp - 1];
        y += tmp[kWarps + warp - 1];
    }
    return make_int2(x, y);
}

// Shared memory of a layout CTA.
struct Smem {
    int* tab;     // [kWarps][E] per-warp expert counts -> exclusive warp prefix
    int* base;    // [E] first row of each expert's slots in this chunk
    int* cnt;     // [E] c_e over all chunks
    int* off;     // [E+1] first row of each expert
    int* padoff;  // [E+1] first padding index of each expert
    int* seg;     // [S]
    int* tmp;     // [2*kWarps]
    __device__ Smem(int* p, int E, int S) {
        tab = p;
        base = tab + kWarps * E;
        cnt = base + E;
        off = cnt + E;
        padoff = off + E + 1;
        seg = padoff + E + 1;
        tmp = seg + S;
    }
};

__host__ __device__ inline size_t smem_bytes(int E, int S) {
    return sizeof(int) * ((size_t)kWarps * E + E + E + (E + 1) + (E + 1) + S + 2 * kWarps);
}

struct SlotRank {
    int e, rank;
};

// Rank of this thread's slot among equal-expert lanes of its warp; the
// lowest such lane records the warp's count of that expert in tab.
__device__ __forceinline__ SlotRank rank_in_warp(int e, int* tab, int E) {
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lanemask_lt());
    if (e >= 0 && rank == 0) tab[(threadIdx.x >> 5) * E + e] = __popc(peers);
    return {e, rank};
}

// Thread e < E: exclusive prefix of tab's column e over the warps, in
// place; returns the column total.
__device__ __forceinline__ int column_scan(int* tab, int E) {
    const int e = threadIdx.x;
    int v[kWarps];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v[w] = tab[w * E + e];
    int run = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        tab[w * E + e] = run;
        run += v[w];
    }
    return run;
}

// Column sums of a [C][N] int matrix the previous grid wrote (N <= kThreads):
// adds the sum over all rows to tot[n] and over rows < c_lim to bef[n]
// (bef may be null).  All threads take part, 8 loads in flight each.
__device__ __forceinline__ void reduce_columns(const int* ws, int C, int N, int c_lim, int* tot, int* bef) {
    const int tpn = kThreads / N;  // threads per column
    const int n = threadIdx.x % N, q = threadIdx.x / N;
    if (q >= tpn) return;
    int sum = 0, before = 0;
    for (int c0 = q; c0 < C; c0 += 8 * tpn) {
        int v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int cc = c0 + u * tpn;
            v[u] = cc < C ? ld_cg(ws + (int64_t)cc * N + n) : 0;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            sum += v[u];
            before += (c0 + u * tpn < c_lim) ? v[u] : 0;
        }
    }
    if (sum) atomicAdd(&tot[n], sum);
    if (bef != nullptr && before) atomicAdd(&bef[n], before);
}

// Aligned exclusive scan over experts of A(c_e) given cnt: fills off and
// padoff (both [E+1]).  Contains __syncthreads; all threads must call it.
__device__ __forceinline__ void aligned_offsets(Smem& m, int E, int align) {
    const int tid = threadIdx.x;
    int rows_e = 0, pad_e = 0;
    if (tid < E) {
        const int ce = m.cnt[tid];
        rows_e = (ce + align - 1) / align * align;
        pad_e = rows_e - ce;
    }
    const int2 incl = block_inclusive_scan2(rows_e, pad_e, m.tmp);
    if (tid < E) {
        m.off[tid] = incl.x - rows_e;
        m.padoff[tid] = incl.y - pad_e;
    }
    if (tid == blockDim.x - 1) {
        m.off[E] = incl.x;
        m.padoff[E] = incl.y;
    }
}

// Row of a slot, or -1 when dropped.
__device__ __forceinline__ int slot_row(const Smem& m, const SlotRank& r, int E) {
    return r.e >= 0 ? m.base[r.e] + m.tab[(threadIdx.x >> 5) * E + r.e] + r.rank : -1;
}

// Writes slot s's row to slot_map and the per-row arrays.
__device__ __forceinline__ void write_slot(const LayoutArgs& a, int64_t s, int row, int e, float wv) {
    if (row >= a.h.max_recv_rows) {
        atomicOr(a.h.error_word, EP_DEVERR_CAPACITY);
        row = -1;
    }
    if (row >= 0) {
        a.h.recv_src[row] = (int)s;
        if (a.recv_topk_idx) a.recv_topk_idx[row] = e;
        if (a.recv_topk_weights) a.recv_topk_weights[row] = wv;
    }
    a.h.slot_map[s] = row;
}

// Row of padding index p (expert by binary search on padoff).
__device__ __forceinline__ int pad_row(const Smem& m, int E, int p) {
    int lo = 0, hi = E;  // padoff[lo] <= p < padoff[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (m.padoff[mid] <= p) lo = mid;
        else hi = mid;
    }
    return m.off[lo] + m.cnt[lo] + (p - m.padoff[lo]);
}

// Padding rows with index in [p0, p1): the list and the per-row arrays.
__device__ __forceinline__ void write_padding(const LayoutArgs& a, const Smem& m, int E, int p0, int p1) {
    for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
        const int row = pad_row(m, E, p);
        a.h.pad_rows[p] = row;
        if (row < a.h.max_recv_rows) {
            a.h.recv_src[row] = -1;
            if (a.recv_topk_idx) a.recv_topk_idx[row] = -1;
            if (a.recv_topk_weights) a.recv_topk_weights[row] = 0.0f;
        } else {
            atomicOr(a.h.error_word, EP_DEVERR_CAPACITY);
        }
    }
}

// Handle-level outputs (one CTA writes them).
__device__ __forceinline__ void write_totals(const LayoutArgs& a, const Smem& m, int E) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        a.h.counts[e] = m.cnt[e];
        a.h.recv_counts[e] = m.off[e + 1] - m.off[e];
        a.h.offsets[e] = m.off[e];
    }
    if (threadIdx.x == 0) {
        a.h.offsets[E] = m.off[E];
        *a.h.num_pad_rows = m.padoff[E];
    }
}

// The whole layout of T*k <= kThreads slots inside one CTA: on return
// (after a __syncthreads) the smem holds cnt, off, padoff, seg, base and
// the warp prefixes, and *r is this thread's slot rank.  Writes nothing to
// global memory except the error bit.
template <typename IdxT>
__device__ __forceinline__ SlotRank small_layout(const LayoutArgs& a, Smem& m, int e, bool bad) {
    const int E = a.h.num_experts, S = a.h.num_segments, k = a.h.num_topk, T = a.h.num_tokens;
    const int tid = threadIdx.x;
    for (int i = tid; i < kWarps * E; i += blockDim.x) m.tab[i] = 0;
    for (int i = tid; i < S; i += blockDim.x) m.seg[i] = 0;
    if (bad) atomicOr(a.h.error_word, EP_DEVERR_BAD_TOPK_IDX);
    __syncthreads();
    const SlotRank r = rank_in_warp(e, m.tab, E);
    count_segments((const IdxT*)a.topk_idx, 0, T, k, E, S, e, m.seg);
    __syncthreads();
    if (tid < E) m.cnt[tid] = column_scan(m.tab, E);
    __syncthreads();
    aligned_offsets(m, E, a.h.expert_alignment);
    if (tid < E) m.base[tid] = m.off[tid];
    __syncthreads();
    return r;
}

}  // namespace layout_dev
}  // namespace ep
