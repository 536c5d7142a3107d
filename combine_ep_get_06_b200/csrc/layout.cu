// Layout step of MoE dispatch: per-expert counts, the aligned expert-major
// receive layout and the deterministic slot map (DeepEP V2 README,
// "Interfaces and examples": the dispatch handle carries the routing
// metadata and the per-expert counts that feed the expert GEMM;
// expert_alignment pads each expert's block).
//
// Slots are split into chunks of whole tokens, one CTA per chunk.
//   count  (one CTA per chunk): validate topk_idx, per-chunk expert
//          histogram and per-chunk segment token counts -> workspace.
//   assign (one CTA per chunk): every CTA re-reduces the small histogram
//          table to get each expert's total and the part that precedes its
//          chunk, runs the aligned exclusive scan over experts, writes its
//          share of the padding rows, then hands out rows to its chunk's
//          slots in flat order: a warp groups equal experts with
//          __match_any_sync (rank in warp = earlier equal lanes), and a
//          per-expert column scan over the 32 warps orders the warps.  No
//          atomics decide a position, so the result is deterministic.
// When all slots fit one chunk (decode), one fused CTA does both.
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {
namespace {

constexpr int kWarps = kLayoutThreads / 32;

template <typename IdxT>
__device__ __forceinline__ int read_expert(const IdxT* idx, int64_t s, int E, bool& bad) {
    long long e = (long long)__ldg(idx + s);
    if (e < -1 || e >= E) {
        bad = true;
        return -1;
    }
    return (int)e;
}

// Counts token t into the expert histogram and, once per segment it
// reaches, into the segment token counts.
template <typename IdxT>
__device__ __forceinline__ void count_token_segments(const IdxT* idx, int t, int k, int E,
                                                     int per_seg, int* seg) {
    const IdxT* row = idx + (int64_t)t * k;
    bool ignore = false;
    for (int j = 0; j < k; ++j) {
        int e = read_expert(row, j, E, ignore);
        if (e < 0) continue;
        int g = e / per_seg;
        bool seen = false;
        for (int jj = 0; jj < j && !seen; ++jj) {
            int e2 = read_expert(row, jj, E, ignore);
            seen = e2 >= 0 && e2 / per_seg == g;
        }
        if (!seen) atomicAdd(&seg[g], 1);
    }
}

template <typename IdxT>
__device__ __forceinline__ void count_range(const IdxT* idx, int t0, int t1, int k, int E, int S,
                                            int* hist, int* seg, uint32_t* error_word) {
    bool bad = false;
    const int64_t s1 = (int64_t)t1 * k;
    for (int64_t s = (int64_t)t0 * k + threadIdx.x; s < s1; s += blockDim.x) {
        int e = read_expert(idx, s, E, bad);
        if (e >= 0) atomicAdd(&hist[e], 1);
    }
    for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x)
        count_token_segments(idx, t, k, E, E / S, seg);
    if (bad) atomicOr(error_word, EP_DEVERR_BAD_TOPK_IDX);
}

template <typename IdxT>
__global__ void __launch_bounds__(kLayoutThreads) layout_count_kernel(LayoutArgs a) {
    extern __shared__ int smem[];
    const int E = a.h.num_experts, S = a.h.num_segments;
    int* hist = smem;
    int* seg = smem + E;
    for (int i = threadIdx.x; i < E + S; i += blockDim.x) smem[i] = 0;
    __syncthreads();
    const int c = blockIdx.x;
    const int t0 = c * a.chunk_tokens;
    const int t1 = min(a.h.num_tokens, t0 + a.chunk_tokens);
    count_range((const IdxT*)a.topk_idx, t0, t1, a.h.num_topk, E, S, hist, seg, a.h.error_word);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) a.ws_hist[(int64_t)c * E + e] = hist[e];
    for (int g = threadIdx.x; g < S; g += blockDim.x) a.ws_seg[(int64_t)c * S + g] = seg[g];
}

// Inclusive scan of two ints over the whole CTA (kLayoutThreads threads).
__device__ __forceinline__ int2 block_inclusive_scan2(int x, int y, int* tmp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int xo = __shfl_up_sync(0xffffffffu, x, o);
        int yo = __shfl_up_sync(0xffffffffu, y, o);
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
            int xo = __shfl_up_sync(0xffffffffu, wx, o);
            int yo = __shfl_up_sync(0xffffffffu, wy, o);
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

template <typename IdxT, bool kFused>
__global__ void __launch_bounds__(kLayoutThreads) layout_assign_kernel(LayoutArgs a) {
    extern __shared__ int smem[];
    const int E = a.h.num_experts, S = a.h.num_segments, k = a.h.num_topk;
    const int T = a.h.num_tokens, align = a.h.expert_alignment, max_rows = a.h.max_recv_rows;
    const int c = blockIdx.x, C = gridDim.x;
    const int tid = threadIdx.x, warp = tid >> 5;
    int* tab = smem;                 // [kWarps][E] per-warp counts, then row bases
    int* cursor = tab + kWarps * E;  // [E] next free row of each expert in this chunk
    int* cnt = cursor + E;           // [E] c_e
    int* off = cnt + E;              // [E+1] first row of each expert
    int* padoff = off + E + 1;       // [E+1] first padding index of each expert
    int* seg = padoff + E + 1;       // [S]
    int* scan_tmp = seg + S;         // [2*kWarps]
    const IdxT* idx = (const IdxT*)a.topk_idx;

    for (int i = tid; i < kWarps * E; i += blockDim.x) tab[i] = 0;

    // Expert totals, and the slots of lower chunks (they come first).
    int before = 0;
    if (kFused) {
        for (int i = tid; i < E; i += blockDim.x) cnt[i] = 0;
        for (int i = tid; i < S; i += blockDim.x) seg[i] = 0;
        __syncthreads();
        count_range(idx, 0, T, k, E, S, cnt, seg, a.h.error_word);
    } else {
        if (tid < E) {
            int total = 0;
            for (int cc = 0; cc < a.num_chunks; ++cc) {
                int v = __ldg(a.ws_hist + (int64_t)cc * E + tid);
                before += (cc < c) ? v : 0;
                total += v;
            }
            cnt[tid] = total;
        }
    }
    __syncthreads();

    // Aligned exclusive scan: expert e gets A(c_e) rows, A(c_e) - c_e of them padding.
    int rows_e = 0, pad_e = 0;
    if (tid < E) {
        int ce = cnt[tid];
        rows_e = (ce + align - 1) / align * align;
        pad_e = rows_e - ce;
    }
    const int2 incl = block_inclusive_scan2(rows_e, pad_e, scan_tmp);
    if (tid < E) {
        off[tid] = incl.x - rows_e;
        padoff[tid] = incl.y - pad_e;
        cursor[tid] = incl.x - rows_e + before;
    }
    if (tid == blockDim.x - 1) {
        off[E] = incl.x;
        padoff[E] = incl.y;
    }
    __syncthreads();

    if (c == 0) {
        for (int e = tid; e < E; e += blockDim.x) {
            a.h.counts[e] = cnt[e];
            a.h.recv_counts[e] = off[e + 1] - off[e];
            a.h.offsets[e] = off[e];
        }
        if (tid == 0) {
            a.h.offsets[E] = off[E];
            *a.h.num_pad_rows = padoff[E];
        }
        for (int g = tid; g < S; g += blockDim.x) {
            int v = 0;
            if (kFused) {
                v = seg[g];
            } else {
                for (int cc = 0; cc < a.num_chunks; ++cc) v += __ldg(a.ws_seg + (int64_t)cc * S + g);
            }
            a.h.seg_tokens[g] = v;
        }
    }

    // This CTA's even share of the padding rows.
    const int P = padoff[E];
    const int p0 = (int)((int64_t)P * c / C), p1 = (int)((int64_t)P * (c + 1) / C);
    for (int p = p0 + tid; p < p1; p += blockDim.x) {
        int lo = 0, hi = E;  // padoff[lo] <= p < padoff[hi]
        while (hi - lo > 1) {
            int mid = (lo + hi) >> 1;
            if (padoff[mid] <= p) lo = mid;
            else hi = mid;
        }
        const int row = off[lo] + cnt[lo] + (p - padoff[lo]);
        a.h.pad_rows[p] = row;
        if (row < max_rows) {
            a.h.recv_src[row] = -1;
            if (a.recv_topk_idx) a.recv_topk_idx[row] = -1;
            if (a.recv_topk_weights) a.recv_topk_weights[row] = 0.0f;
        } else {
            atomicOr(a.h.error_word, EP_DEVERR_CAPACITY);
        }
    }

    // Rows for this chunk's slots, in flat slot order.
    const int t0 = kFused ? 0 : c * a.chunk_tokens;
    const int t1 = kFused ? T : min(T, t0 + a.chunk_tokens);
    const int64_t s_end = (int64_t)t1 * k;
    const unsigned lt = lanemask_lt();
    for (int64_t base = (int64_t)t0 * k; base < s_end; base += blockDim.x) {
        const int64_t s = base + tid;
        int e = -1;
        if (s < s_end) {
            bool ignore = false;
            e = read_expert(idx, s, E, ignore);
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & lt);
        const bool leader = rank == 0;
        if (e >= 0 && leader) tab[warp * E + e] = __popc(peers);
        __syncthreads();
        if (tid < E) {
            int run = cursor[tid];
            for (int w = 0; w < kWarps; ++w) {
                int v = tab[w * E + tid];
                if (v) {
                    tab[w * E + tid] = run;
                    run += v;
                }
            }
            cursor[tid] = run;
        }
        __syncthreads();
        if (s < s_end) {
            int row = -1;
            if (e >= 0) {
                row = tab[warp * E + e] + rank;
                if (row < max_rows) {
                    a.h.recv_src[row] = (int)s;
                    if (a.recv_topk_idx) a.recv_topk_idx[row] = e;
                    if (a.recv_topk_weights)
                        a.recv_topk_weights[row] = a.topk_weights ? __ldg(a.topk_weights + s) : 0.0f;
                } else {
                    atomicOr(a.h.error_word, EP_DEVERR_CAPACITY);
                    row = -1;
                }
            }
            a.h.slot_map[s] = row;
        }
        __syncthreads();
        if (e >= 0 && leader) tab[warp * E + e] = 0;
    }
}

size_t assign_smem_bytes(int E, int S) {
    return sizeof(int) * ((size_t)kWarps * E + E + E + (E + 1) + (E + 1) + S + 2 * kWarps);
}

template <typename IdxT>
cudaError_t launch_layout_t(const LayoutArgs& a, cudaStream_t stream) {
    const int E = a.h.num_experts, S = a.h.num_segments;
    const size_t smem_assign = assign_smem_bytes(E, S);
    auto fused = layout_assign_kernel<IdxT, true>;
    auto split = layout_assign_kernel<IdxT, false>;
    cudaError_t err;
    if (smem_assign > 48 * 1024) {
        err = cudaFuncSetAttribute(fused, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_assign);
        if (err != cudaSuccess) return err;
        err = cudaFuncSetAttribute(split, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_assign);
        if (err != cudaSuccess) return err;
    }
    if (a.num_chunks == 1) {
        fused<<<1, kLayoutThreads, smem_assign, stream>>>(a);
        return cudaGetLastError();
    }
    layout_count_kernel<IdxT><<<a.num_chunks, kLayoutThreads, sizeof(int) * (E + S), stream>>>(a);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    split<<<a.num_chunks, kLayoutThreads, smem_assign, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_layout(const LayoutArgs& a, bool idx_is_int64, cudaStream_t stream) {
    return idx_is_int64 ? launch_layout_t<long long>(a, stream) : launch_layout_t<int>(a, stream);
}

}  // namespace ep
