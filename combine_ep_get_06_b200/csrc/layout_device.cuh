// Device building blocks of the layout kernels.
//
// One thread per slot, chunks of <= kThreads slots of whole tokens.  Each
// slot sets its lane's bit in a per-(warp, expert) word of shared memory
// (atomicOr: the result does not depend on the order).  A slot's rank among
// the earlier slots of the same expert in its chunk is then
//   popc(word & lanes below it)                          (same warp)
// + the exclusive column scan over warps of popc(word)  (earlier warps),
// so the slot map is deterministic.  Tokens per segment come from a
// per-token bit mask of the segments its slots reach.
//
// The per-row outputs (recv_src, recv_topk_idx, recv_topk_weights) are
// staged in shared memory in "compact" order -- the chunk's valid slots
// sorted by (expert, slot) -- and written from there, so consecutive
// threads write consecutive rows instead of scattering 4-byte stores.
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

// ------------------------------------------------------------------ segments

// Generic path (more than 64 segments): one thread per token [t0, t1)
// walks its k slots and counts each segment once.
template <typename IdxT>
__device__ __forceinline__ void count_segments_walk(const IdxT* idx, int t0, int t1, int k, int E, int S,
                                                    int* seg) {
    const int per_seg = E / S;
    for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
        const IdxT* row = idx + (int64_t)t * k;
        bool ignore = false;
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

// S <= 64: records in tmask (two 32-bit words per token) the segments the
// token's slots reach.  When k divides 32 a token's k slots are k
// consecutive lanes: their bits are OR-reduced with shuffles and the first
// lane stores them (no atomics); otherwise each slot ORs in its own bit.
// All lanes of the warp must call it.
__device__ __forceinline__ void mark_segment(unsigned* tmask, int token, int e, int E, int S, int k) {
    const int g = e >= 0 ? e / (E / S) : 0;
    unsigned lo = (e >= 0 && g < 32) ? 1u << g : 0u;
    unsigned hi = (e >= 0 && g >= 32) ? 1u << (g - 32) : 0u;
    if ((32 % k) == 0) {
        for (int o = 1; o < k; o <<= 1) {
            lo |= __shfl_xor_sync(0xffffffffu, lo, o);
            hi |= __shfl_xor_sync(0xffffffffu, hi, o);
        }
        if ((threadIdx.x & 31) % k == 0) {
            tmask[2 * token] = lo;
            tmask[2 * token + 1] = hi;
        }
    } else if (e >= 0) {
        atomicOr(&tmask[2 * token + (g >> 5)], g < 32 ? lo : hi);
    }
}

// S <= 64: tokens per segment from the masks of n_tokens tokens.  Per warp
// of 32 tokens, one ballot per segment; lane g keeps segment g's count in a
// register and all lanes then add theirs at once (one atomic per lane, so
// no lane waits on a chain of atomics).
__device__ __forceinline__ void count_segments_masks(const unsigned* tmask, int n_tokens, int S, int* seg) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int mine_lo = 0, mine_hi = 0;  // counts of segments lane and 32 + lane
    for (int t0 = warp * 32; t0 < n_tokens; t0 += kThreads) {
        const int t = t0 + lane;
        const unsigned lo = t < n_tokens ? tmask[2 * t] : 0u;
        const unsigned hi = t < n_tokens ? tmask[2 * t + 1] : 0u;
        for (int g = 0; g < S; ++g) {
            const unsigned bit = g < 32 ? (lo >> g) & 1u : (hi >> (g - 32)) & 1u;
            const int n = __popc(__ballot_sync(0xffffffffu, bit));
            if (g < 32) mine_lo += lane == g ? n : 0;
            else mine_hi += lane == g - 32 ? n : 0;
        }
    }
    if (lane < S && mine_lo) atomicAdd(&seg[lane], mine_lo);
    if (32 + lane < S && mine_hi) atomicAdd(&seg[32 + lane], mine_hi);
}

// -------------------------------------------------------------- block scans

// Inclusive scan of three ints over the whole CTA (kThreads threads).
__device__ __forceinline__ int3 block_inclusive_scan3(int x, int y, int z, int* tmp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int xo = __shfl_up_sync(0xffffffffu, x, o);
        const int yo = __shfl_up_sync(0xffffffffu, y, o);
        const int zo = __shfl_up_sync(0xffffffffu, z, o);
        if (lane >= o) {
            x += xo;
            y += yo;
            z += zo;
        }
    }
    if (lane == 31) {
        tmp[warp] = x;
        tmp[kWarps + warp] = y;
        tmp[2 * kWarps + warp] = z;
    }
    __syncthreads();
    if (warp == 0) {
        int wx = tmp[lane], wy = tmp[kWarps + lane], wz = tmp[2 * kWarps + lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int xo = __shfl_up_sync(0xffffffffu, wx, o);
            const int yo = __shfl_up_sync(0xffffffffu, wy, o);
            const int zo = __shfl_up_sync(0xffffffffu, wz, o);
            if (lane >= o) {
                wx += xo;
                wy += yo;
                wz += zo;
            }
        }
        tmp[lane] = wx;
        tmp[kWarps + lane] = wy;
        tmp[2 * kWarps + lane] = wz;
    }
    __syncthreads();
    if (warp > 0) {
        x += tmp[warp - 1];
        y += tmp[kWarps + warp - 1];
        z += tmp[2 * kWarps + warp - 1];
    }
    return make_int3(x, y, z);
}

// ----------------------------------------------------------- shared memory

// Shared memory of a layout CTA (E experts, S segments), carved in order.
struct Smem {
    int* tab;         // [kWarps][E] (warp, expert) lane-bit words -> exclusive warp prefix
    int* base;        // [E] first row of each expert's slots of this chunk
    int* cnt;         // [E] c_e over all chunks
    int* lc;          // [E] this chunk's count of each expert
    int* lcoff;       // [E+1] exclusive prefix of lc: compact index of each expert
    int* off;         // [E+1] first row of each expert
    int* padoff;      // [E+1] first padding index of each expert
    int* seg;         // [S]
    int* tmp;         // [3*kWarps]
    unsigned* tmask;  // [2*kThreads] segment bits of each token of the chunk
    int* cq_slot;     // [kThreads] compact order: slot,
    int* cq_expert;   //            its expert,
    float* cq_w;      //            its weight
    __device__ Smem(int* p, int E, int S) {
        tab = p;
        base = tab + kWarps * E;
        cnt = base + E;
        lc = cnt + E;
        lcoff = lc + E;
        off = lcoff + E + 1;
        padoff = off + E + 1;
        seg = padoff + E + 1;
        tmp = seg + S;
        tmask = reinterpret_cast<unsigned*>(tmp + 3 * kWarps);
        cq_slot = reinterpret_cast<int*>(tmask + 2 * kThreads);
        cq_expert = cq_slot + kThreads;
        cq_w = reinterpret_cast<float*>(cq_expert + kThreads);
    }
};

__host__ __device__ inline size_t smem_bytes(int E, int S) {
    return sizeof(int) * ((size_t)kWarps * E + 3 * (size_t)E + 3 * ((size_t)E + 1) + S + 3 * kWarps +
                          2 * kThreads + 3 * kThreads);
}

// Zeroes tab (kWarps*E words, 16-byte aligned) with 16-byte stores.
__device__ __forceinline__ void zero_tab(int* tab, int E) {
    uint4* t4 = reinterpret_cast<uint4*>(tab);
    for (int i = threadIdx.x; i < kWarps * E / 4; i += blockDim.x) t4[i] = make_uint4(0, 0, 0, 0);
}

// ---------------------------------------------------------------- ranking

// Marks this thread's slot in the (warp, expert) bit word.
__device__ __forceinline__ void mark_slot(int e, int* tab, int E) {
    if (e >= 0) atomicOr(reinterpret_cast<unsigned*>(tab) + (threadIdx.x >> 5) * E + e, 1u << (threadIdx.x & 31));
}

// Rank among the equal-expert slots of the warp (after mark_slot and a barrier).
__device__ __forceinline__ int rank_in_warp(int e, const int* tab, int E) {
    return e >= 0 ? __popc((unsigned)tab[(threadIdx.x >> 5) * E + e] & lanemask_lt()) : 0;
}

// Thread e < E: turns tab's column e (bit words) into the exclusive prefix
// over warps of their popcounts, in place; returns the column total.
__device__ __forceinline__ int column_scan(int* tab, int E) {
    const int e = threadIdx.x;
    int v[kWarps];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v[w] = __popc((unsigned)tab[w * E + e]);
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
// (bef may be null).  All threads take part, 16 loads in flight each.
__device__ __forceinline__ void reduce_columns(const int* ws, int C, int N, int c_lim, int* tot, int* bef) {
    const int tpn = kThreads / N;  // threads per column
    const int n = threadIdx.x % N, q = threadIdx.x / N;
    if (q >= tpn) return;
    int sum = 0, before = 0;
    for (int c0 = q; c0 < C; c0 += 16 * tpn) {
        int v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int cc = c0 + u * tpn;
            v[u] = cc < C ? ld_cg(ws + (int64_t)cc * N + n) : 0;
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            sum += v[u];
            before += (c0 + u * tpn < c_lim) ? v[u] : 0;
        }
    }
    if (sum) atomicAdd(&tot[n], sum);
    if (bef != nullptr && before) atomicAdd(&bef[n], before);
}

// Scans over experts, given cnt (c_e over all chunks) and lc (this chunk's
// counts): off / padoff (aligned rows and padding indices) and lcoff
// (compact index of each expert in this chunk).  All threads must call it.
__device__ __forceinline__ void expert_offsets(Smem& m, int E, int align) {
    const int tid = threadIdx.x;
    int rows_e = 0, pad_e = 0, l_e = 0;
    if (tid < E) {
        const int ce = m.cnt[tid];
        rows_e = (ce + align - 1) / align * align;
        pad_e = rows_e - ce;
        l_e = m.lc[tid];
    }
    const int3 incl = block_inclusive_scan3(rows_e, pad_e, l_e, m.tmp);
    if (tid < E) {
        m.off[tid] = incl.x - rows_e;
        m.padoff[tid] = incl.y - pad_e;
        m.lcoff[tid] = incl.z - l_e;
    }
    if (tid == blockDim.x - 1) {
        m.off[E] = incl.x;
        m.padoff[E] = incl.y;
        m.lcoff[E] = incl.z;
    }
}

// ------------------------------------------------------------------ writes

// Rank of the slot within its expert in this chunk (0-based), or -1.
__device__ __forceinline__ int chunk_rank(const Smem& m, int e, int warp_rank, int E) {
    return e >= 0 ? m.tab[(threadIdx.x >> 5) * E + e] + warp_rank : -1;
}

// The slot's row (base[e] + chunk rank); -1 when dropped or past the capacity.
__device__ __forceinline__ int slot_row(const LayoutArgs& a, const Smem& m, int e, int crank) {
    if (e < 0) return -1;
    const int row = m.base[e] + crank;
    if (row >= a.h.max_recv_rows) {
        atomicOr(a.h.error_word, EP_DEVERR_CAPACITY);
        return -1;
    }
    return row;
}

// Puts the slot into the compact staging arrays (a barrier must follow).
__device__ __forceinline__ void stage_slot(Smem& m, int64_t s, int e, int crank, float wv) {
    if (e < 0) return;
    const int q = m.lcoff[e] + crank;
    m.cq_slot[q] = (int)s;
    m.cq_expert[q] = e;
    m.cq_w[q] = wv;
}

// Writes the per-row arrays of compact indices [q0, q1) of this chunk.
__device__ __forceinline__ void write_rows(const LayoutArgs& a, const Smem& m, int q0, int q1) {
    for (int q = q0 + threadIdx.x; q < q1; q += blockDim.x) {
        const int e = m.cq_expert[q];
        const int row = m.base[e] + (q - m.lcoff[e]);
        if (row >= a.h.max_recv_rows) continue;  // flagged by slot_row
        // the row lies in its expert's block, before its padding
        if (!EP_CHECK(e >= 0 && e < a.h.num_experts && row >= m.off[e] && row < m.off[e] + m.cnt[e],
                      a.h.error_word))
            continue;
        a.h.recv_src[row] = m.cq_slot[q];
        if (a.recv_topk_idx) a.recv_topk_idx[row] = e;
        if (a.recv_topk_weights) a.recv_topk_weights[row] = m.cq_w[q];
    }
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
        if (!EP_CHECK(p >= 0 && p < m.padoff[E] && row >= 0 && row < m.off[E], a.h.error_word)) continue;
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
__device__ __forceinline__ void write_totals(const LayoutArgs& a, const Smem& m, int E, int S) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        a.h.counts[e] = m.cnt[e];
        a.h.recv_counts[e] = m.off[e + 1] - m.off[e];
        a.h.offsets[e] = m.off[e];
    }
    for (int g = threadIdx.x; g < S; g += blockDim.x) a.h.seg_tokens[g] = m.seg[g];
    if (threadIdx.x == 0) {
        a.h.offsets[E] = m.off[E];
        *a.h.num_pad_rows = m.padoff[E];
    }
}

// ------------------------------------------------------- one-CTA layout

// The whole layout of T*k <= kThreads slots inside one CTA (thread = slot
// tid, expert e or -1).  On return (after a barrier) the smem holds cnt,
// off, padoff, seg, base, lcoff and the compact staging arrays; the result
// is the slot's row (-1 when dropped).  Writes nothing to global memory
// except error bits.
template <typename IdxT>
__device__ __forceinline__ int small_layout(const LayoutArgs& a, Smem& m, int e, bool bad, float wv) {
    const int E = a.h.num_experts, S = a.h.num_segments, k = a.h.num_topk, T = a.h.num_tokens;
    const int tid = threadIdx.x;
    zero_tab(m.tab, E);
    for (int i = tid; i < S; i += blockDim.x) m.seg[i] = 0;
    m.tmask[2 * tid] = 0;
    m.tmask[2 * tid + 1] = 0;
    if (bad) atomicOr(a.h.error_word, EP_DEVERR_BAD_TOPK_IDX);
    __syncthreads();
    mark_slot(e, m.tab, E);
    if (S <= 64) mark_segment(m.tmask, tid / k, e, E, S, k);
    __syncthreads();
    const int wrank = rank_in_warp(e, m.tab, E);
    if (S <= 64) count_segments_masks(m.tmask, T, S, m.seg);
    else count_segments_walk((const IdxT*)a.topk_idx, 0, T, k, E, S, m.seg);
    __syncthreads();
    if (tid < E) m.cnt[tid] = m.lc[tid] = column_scan(m.tab, E);
    __syncthreads();
    expert_offsets(m, E, a.h.expert_alignment);
    if (tid < E) m.base[tid] = m.off[tid];
    __syncthreads();
    const int crank = chunk_rank(m, e, wrank, E);
    stage_slot(m, tid, e, crank, wv);
    const int row = slot_row(a, m, e, crank);
    __syncthreads();
    return row;
}

}  // namespace layout_dev
}  // namespace ep
