// Dispatch and combine across the GPUs of one NVLink domain (DeepEP V2
// README, "Performance": EP over an NVLink domain; "Interfaces and
// examples": dispatch_forward / combine_forward).  Segments are ranks.
//
// Dispatch.  From the gathered per-rank counts all_counts[W][E], every CTA
// builds the same tables in shared memory.  For each expert e:
//   C_e = sum_r all_counts[r][e]
//   A_e = ceil(C_e/a)*a
//   first_e = (sum of A over the owner's experts below e)
//           + (sum of all_counts[r][e] over the ranks r below this one)
// first_e is the owner's row of this rank's first slot of e.  A valid slot
// s = t*k+j with expert e, at local row slot_map[s] (alignment-1 layout,
// ascending slots), goes to row first_e + slot_map[s] - offsets[e] of rank
// e/(E/W).  Warp units, as in the one-GPU dispatch: a unit is 1024
// elements of one token row (or one of this rank's padding rows).  The warp
// loads and converts the slice into its shared-memory stage, then copies it
// with 16-byte stores to the slice's k destinations: peers' blocks through
// the peer table, as plain stores over NVLink.  The warp that takes a
// token's first slice also writes the token's slot metadata.  Padding rows
// are zeroed in this rank's own block, and CTA 0 writes its receive totals.
// No barrier after the tables: warps never wait on one another.

// Combine.  The one-GPU combine with rows (rank, row) from dest: y is
// loaded from the owners' blocks.  The arithmetic is the same: fp32 FMA
// in ascending j from +0, one bf16 rounding.
//
// Neither kernel waits on another GPU.  The caller's collectives order the
// ranks' launches.
#include "dispatch_warp.cuh"

namespace ep {
namespace {

using namespace warp_units;

constexpr int kThreads = 256;

constexpr int kWarps = kThreads / 32;
constexpr int kMinUnitsPerWarp = 8;

struct MgpuSmem {
    int* first;      // [E]
    int* lofs;       // [E]
    int* asz;        // [E] A_e
    int* own_c;      // [epr]
    int* own_off;    // [epr]
    int* padoff;     // [epr + 1]
    char** peer;     // [W]
    unsigned char* stages;  // [kWarps][stage_bytes]
};

__host__ __device__ inline size_t align16(size_t n) { return (n + 15) & ~(size_t)15; }

__host__ __device__ inline size_t mgpu_smem(int E, int epr, int W, int stage_bytes, MgpuSmem* m,
                                            unsigned char* base) {
    size_t at = 0;
    auto take = [&](size_t n) {
        size_t here = at;
        at += align16(n);
        return base + here;
    };
    unsigned char* first = take((size_t)E * 4);
    unsigned char* lofs = take((size_t)E * 4);
    unsigned char* asz = take((size_t)E * 4);
    unsigned char* own_c = take((size_t)epr * 4);
    unsigned char* own_off = take((size_t)epr * 4);
    unsigned char* padoff = take((size_t)(epr + 1) * 4);
    unsigned char* peer = take((size_t)W * sizeof(char*));
    unsigned char* stages = take((size_t)kWarps * stage_bytes);
    if (m != nullptr) {
        m->first = (int*)first;
        m->lofs = (int*)lofs;
        m->asz = (int*)asz;
        m->own_c = (int*)own_c;
        m->own_off = (int*)own_off;
        m->padoff = (int*)padoff;
        m->peer = (char**)peer;
        m->stages = stages;
    }
    return at;
}

__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Builds the tables (see the file comment); ends with a barrier.
__device__ void build_tables(const MgpuArgs& a, const MgpuSmem& m) {
    const ep_mgpu_geometry& g = a.g;
    const int E = g.num_experts, W = g.world, epr = g.experts_per_rank, al = g.expert_alignment;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int32_t* all_counts = (const int32_t*)(a.local_block + g.off_all_counts);
    for (int i = tid; i < W; i += blockDim.x) m.peer[i] = a.peer_blocks[i];
    for (int e = tid; e < E; e += blockDim.x) {
        int C = 0, below = 0;
        for (int r = 0; r < W; ++r) {
            const int c = all_counts[(size_t)r * E + e];
            C += c;
            if (r < g.rank) below += c;
        }
        m.first[e] = below;
        m.asz[e] = (C + al - 1) / al * al;
        m.lofs[e] = a.offsets[e];
        const int i = e - g.rank * epr;
        if (i >= 0 && i < epr) m.own_c[i] = C;
    }
    __syncthreads();
    // Exclusive scan of A within each owner's experts.
    for (int d = warp; d < W; d += nwarps) {
        int run = 0;
        for (int b = 0; b < epr; b += 32) {
            const int i = b + lane;
            const int v = i < epr ? m.asz[d * epr + i] : 0;
            const int inc = warp_incl_scan(v);
            if (i < epr) {
                m.first[d * epr + i] += run + inc - v;
                if (d == g.rank) m.own_off[i] = run + inc - v;
            }
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
    }
    // Exclusive scan of this rank's padding rows per local expert.
    if (warp == 0) {
        int run = 0;
        for (int b = 0; b < epr; b += 32) {
            const int i = b + lane;
            const int v = i < epr ? m.asz[g.rank * epr + i] - m.own_c[i] : 0;
            const int inc = warp_incl_scan(v);
            if (i < epr) m.padoff[i] = run + inc - v;
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) m.padoff[epr] = run;
    }
    __syncthreads();
}

__device__ __forceinline__ int local_expert_of_pad(const MgpuSmem& m, int epr, int p) {
    int lo = 0, hi = epr;  // padoff[lo] <= p < padoff[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (m.padoff[mid] <= p) lo = mid;
        else hi = mid;
    }
    return lo;
}

// The lanes of a warp copy n bytes from shared memory (16-byte aligned) to
// global memory, in the widest units that divide both n and the
// destination's alignment.
__device__ __forceinline__ void warp_copy_out(char* dst, const unsigned char* src, int n, int lane) {
    const uintptr_t al = (uintptr_t)dst;
    if ((n & 15) == 0 && (al & 15) == 0) {
        for (int i = lane; i < n / 16; i += 32)
            reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(src)[i];
    } else if ((n & 3) == 0 && (al & 3) == 0) {
        for (int i = lane; i < n / 4; i += 32)
            reinterpret_cast<uint32_t*>(dst)[i] = reinterpret_cast<const uint32_t*>(src)[i];
    } else {
        for (int i = lane; i < n; i += 32) dst[i] = (char)src[i];
    }
}

__device__ __forceinline__ void warp_zero_out(char* dst, int n, int lane) {
    const uintptr_t al = (uintptr_t)dst;
    if ((n & 15) == 0 && (al & 15) == 0) {
        for (int i = lane; i < n / 16; i += 32) reinterpret_cast<uint4*>(dst)[i] = make_uint4(0, 0, 0, 0);
    } else if ((n & 3) == 0 && (al & 3) == 0) {
        for (int i = lane; i < n / 4; i += 32) reinterpret_cast<uint32_t*>(dst)[i] = 0u;
    } else {
        for (int i = lane; i < n; i += 32) dst[i] = 0;
    }
}

template <int kMode>
__global__ void __launch_bounds__(kThreads, 3) mgpu_dispatch_kernel(MgpuArgs a) {
    using M = Mode<kMode>;
    extern __shared__ __align__(128) unsigned char smem[];
    const ep_mgpu_geometry& g = a.g;
    const SliceGeo sg = slice_geo(kMode, g.hidden);
    MgpuSmem m;
    mgpu_smem(g.num_experts, g.experts_per_rank, g.world, sg.stage_bytes, &m, smem);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = a.T, k = g.num_topk, epr = g.experts_per_rank;
    const int rb_bytes = g.row_bytes, sc_bytes = g.scale_bytes;
    uint32_t* const err = (uint32_t*)(a.local_block + g.off_error_word);
    int2* const dest = (int2*)(a.local_block + g.off_dest);
    unsigned char* const st = m.stages + (size_t)warp * sg.stage_bytes;
    unsigned char* const sst = st + sg.out_bytes;

    build_tables(a, m);
    const int n_pad = m.padoff[epr];

    if (blockIdx.x == 0) {
        int32_t* raw = (int32_t*)(a.local_block + g.off_raw_counts);
        int32_t* cnt = (int32_t*)(a.local_block + g.off_recv_counts);
        int32_t* off = (int32_t*)(a.local_block + g.off_recv_offsets);
        for (int i = tid; i < epr; i += kThreads) {
            raw[i] = m.own_c[i];
            cnt[i] = m.asz[g.rank * epr + i];
            off[i] = m.own_off[i];
        }
        if (tid == 0) {
            off[epr] = m.own_off[epr - 1] + m.asz[g.rank * epr + epr - 1];
            *(int32_t*)(a.local_block + g.off_num_pad_rows) = n_pad;
        }
    }

    const int64_t n_tok_units = (int64_t)T * sg.ns;
    const int64_t n_units = n_tok_units + n_pad;
    for (int64_t u = (int64_t)blockIdx.x * kWarps + warp; u < n_units; u += (int64_t)gridDim.x * kWarps) {
        if (u >= n_tok_units) {
            // one of this rank's padding rows, in its own block
            const int p = (int)(u - n_tok_units);
            const int i = local_expert_of_pad(m, epr, p);
            const int row = m.own_off[i] + m.own_c[i] + (p - m.padoff[i]);
            if (row >= g.max_recv_rows) {
                if (lane == 0) atomicOr(err, EP_DEVERR_CAPACITY);
                continue;
            }
            warp_zero_out(a.local_block + g.off_recv_x + (size_t)row * rb_bytes, rb_bytes, lane);
            if (sc_bytes > 0) warp_zero_out(a.local_block + g.off_recv_scales + (size_t)row * sc_bytes, sc_bytes, lane);
            if (lane == 0) {
                ((int32_t*)(a.local_block + g.off_recv_src))[row] = -1;
                ((int32_t*)(a.local_block + g.off_recv_topk_idx))[row] = -1;
                ((float*)(a.local_block + g.off_recv_topk_weights))[row] = 0.0f;
            }
            continue;
        }

        // A token slice: its loads first, so they fly while the routing resolves.
        const int t = (int)(u / sg.ns), s = (int)(u - (int64_t)t * sg.ns);
        const int ne = min(kSliceElems, g.hidden - s * kSliceElems);
        const Loads<kMode> l = load_x<kMode>(a.src, sg, u, n_tok_units, lane);
        Meta mt;
        mt.row = -1;
        mt.xs = 0.0f;
        if (kMode == EP_X_FP8 && lane < ne / 128)
            mt.xs = a.src.x_scales[(size_t)t * (g.hidden / 128) + s * (kSliceElems / 128) + lane];
        int d = -1, row = -1;
        if (lane < k) {
            const size_t sl = (size_t)t * k + lane;
            const int lr = a.slot_map[sl];
            if (lr >= 0) {
                const int64_t e64 =
                    a.idx_is_int64 ? ((const int64_t*)a.topk_idx)[sl] : ((const int32_t*)a.topk_idx)[sl];
                const int e = (int)e64;
                if (e64 < 0 || e64 >= g.num_experts) {
                    // not the topk_idx the layout saw: drop the slot
                    if (s == 0) atomicOr(err, EP_DEVERR_BAD_TOPK_IDX);
                } else {
                    d = e / epr;
                    row = m.first[e] + (lr - m.lofs[e]);
                }
                if (d < 0) {
                    row = -1;
                } else if (row < 0 || row >= g.max_recv_rows) {
                    if (s == 0) atomicOr(err, EP_DEVERR_CAPACITY);
                    d = row = -1;
                } else if (s == 0) {
                    char* pb = m.peer[d];
                    ((int32_t*)(pb + g.off_recv_src))[row] = (int32_t)((int64_t)g.rank * g.max_tokens * k + sl);
                    ((int32_t*)(pb + g.off_recv_topk_idx))[row] = e;
                    ((float*)(pb + g.off_recv_topk_weights))[row] = a.topk_weights ? a.topk_weights[sl] : 0.0f;
                }
            }
            if (s == 0) dest[sl] = make_int2(d, row);
        }
        __syncwarp();  // the previous unit's copies have read the stage
        fill_stage<kMode>(l, mt, ne, lane, st, sst);
        __syncwarp();
        const int db = ne * sg.out_bytes / kSliceElems;
        const int sb = M::kScales ? ne / M::kScaleBlock * M::kScaleBytes : 0;
        for (int j = 0; j < k; ++j) {
            const int dj = __shfl_sync(0xffffffffu, d, j), rj = __shfl_sync(0xffffffffu, row, j);
            if (dj < 0) continue;
            char* pb = m.peer[dj];
            warp_copy_out(pb + g.off_recv_x + (size_t)rj * rb_bytes + (size_t)s * sg.out_bytes, st, db, lane);
            if (sb > 0)
                warp_copy_out(pb + g.off_recv_scales + (size_t)rj * sc_bytes + (size_t)s * sg.sout_bytes, sst, sb,
                              lane);
        }
    }
    // The CTA's stores to peers' memory are ordered before the grid's end:
    // the barrier makes them precede thread 0's system-scope fence, which is
    // cumulative.  (A fence in every thread measured as the top stall.)
    __syncthreads();
    if (tid == 0) __threadfence_system();
}

template <int G>
__global__ void __launch_bounds__(kThreads) mgpu_combine_kernel(MgpuArgs a, int ipr, int upr) {
    __shared__ const char* peer_y[kMaxWorld];
    const ep_mgpu_geometry& g = a.g;
    const int tid = threadIdx.x;
    const int T = a.T, k = g.num_topk, W = g.world;
    const size_t row_bytes = (size_t)g.hidden * 2;
    const int2* const dest = (const int2*)(a.local_block + g.off_dest);
    uint32_t* const err = (uint32_t*)(a.local_block + g.off_error_word);
    for (int i = tid; i < W; i += blockDim.x) peer_y[i] = a.peer_blocks[i] + g.off_y;
    __syncthreads();

    const int64_t n_units = (int64_t)T * upr;
    for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
        const int t = (int)(u / upr);
        const int c = (int)(u - (int64_t)t * upr) * blockDim.x + tid;
        if (c >= ipr) continue;

        const char* src[8 * G];
        float w[8 * G];
#pragma unroll
        for (int j = 0; j < 8 * G; ++j) {
            const char* p = nullptr;
            float wj = 1.0f;
            if (j < k) {
                const int2 dr = dest[(size_t)t * k + j];
                if (a.topk_weights != nullptr) wj = a.topk_weights[(size_t)t * k + j];
                if (dr.x >= 0) {
                    if (dr.x < W && dr.y >= 0 && dr.y < g.max_recv_rows)
                        p = peer_y[dr.x] + (size_t)dr.y * row_bytes + (size_t)c * 16;
                    else
                        atomicOr(err, EP_DEVERR_CAPACITY);
                }
            }
            src[j] = p;
            w[j] = wj;
        }

        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
        for (int gi = 0; gi < G; ++gi) {
            uint4 v[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const char* p = src[8 * gi + jj];
                v[jj] = p != nullptr ? ld_stream(p) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                if (src[8 * gi + jj] == nullptr) continue;
                const float wj = w[8 * gi + jj];
                acc[0] = __fmaf_rn(wj, bf16_lo(v[jj].x), acc[0]);
                acc[1] = __fmaf_rn(wj, bf16_hi(v[jj].x), acc[1]);
                acc[2] = __fmaf_rn(wj, bf16_lo(v[jj].y), acc[2]);
                acc[3] = __fmaf_rn(wj, bf16_hi(v[jj].y), acc[3]);
                acc[4] = __fmaf_rn(wj, bf16_lo(v[jj].z), acc[4]);
                acc[5] = __fmaf_rn(wj, bf16_hi(v[jj].z), acc[5]);
                acc[6] = __fmaf_rn(wj, bf16_lo(v[jj].w), acc[6]);
                acc[7] = __fmaf_rn(wj, bf16_hi(v[jj].w), acc[7]);
            }
        }
        const uint4 o = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                   pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
        st_stream((char*)a.out + (size_t)t * row_bytes + (size_t)c * 16, o);
    }
}

template <int kMode>
cudaError_t launch_dispatch_t(const MgpuArgs& a, cudaStream_t stream) {
    const SliceGeo sg = slice_geo(kMode, a.g.hidden);
    const size_t smem = mgpu_smem(a.g.num_experts, a.g.experts_per_rank, a.g.world, sg.stage_bytes, nullptr, nullptr);
    auto kernel = mgpu_dispatch_kernel<kMode>;
    cudaError_t err;
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    // Every CTA first builds its tables from the gathered counts (W x E
    // loads and scans): give each warp at least kMinUnitsPerWarp units so
    // that this set-up is amortised (measured with 8 ranks of 1024 tokens on
    // one GPU: 204 -> 180 us for the dispatch phase); large batches still
    // fill every SM.
    const int64_t cap = (int64_t)device_sm_count() * per_sm;
    const int64_t units = (int64_t)a.T * sg.ns + (int64_t)a.g.experts_per_rank * (a.g.expert_alignment - 1);
    const int64_t want = (units + kWarps * kMinUnitsPerWarp - 1) / (kWarps * kMinUnitsPerWarp);
    const int64_t grid = want < 1 ? 1 : (want < cap ? want : cap);
    debug_launch("mgpu_dispatch_kernel", kMode, dim3((unsigned)grid), dim3(kThreads), smem, stream);
    kernel<<<(unsigned)grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

int combine_threads(int ipr) {
    for (int bd = kThreads; bd >= 32; bd -= 32)
        if (ipr % bd == 0) return bd;
    return ipr < kThreads ? ((ipr + 31) / 32) * 32 : kThreads;
}

template <int G>
cudaError_t launch_combine_t(const MgpuArgs& a, cudaStream_t stream) {
    const int ipr = a.g.hidden / 8;
    const int bd = combine_threads(ipr);
    const int upr = (ipr + bd - 1) / bd;
    int per_sm = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, mgpu_combine_kernel<G>, bd, 0);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) per_sm = 1;
    const int64_t cap = (int64_t)device_sm_count() * per_sm;
    const int64_t want = (int64_t)a.T * upr;
    const int64_t grid = want < 1 ? 1 : (want < cap ? want : cap);
    debug_launch("mgpu_combine_kernel", G, dim3((unsigned)grid), dim3(bd), 0, stream);
    mgpu_combine_kernel<G><<<(unsigned)grid, bd, 0, stream>>>(a, ipr, upr);
    return cudaGetLastError();
}

}  // namespace

size_t mgpu_dispatch_smem_bytes(const ep_mgpu_geometry& g) {
    const SliceGeo sg = slice_geo(g.x_mode, g.hidden);
    return mgpu_smem(g.num_experts, g.experts_per_rank, g.world, sg.stage_bytes, nullptr, nullptr);
}

cudaError_t launch_mgpu_dispatch(const MgpuArgs& a, ep_x_mode mode, cudaStream_t stream) {
    switch (mode) {
        case EP_X_BF16: return launch_dispatch_t<EP_X_BF16>(a, stream);
        case EP_X_FP8: return launch_dispatch_t<EP_X_FP8>(a, stream);
        case EP_X_BF16_TO_FP8: return launch_dispatch_t<EP_X_BF16_TO_FP8>(a, stream);
        case EP_X_BF16_TO_NVFP4: return launch_dispatch_t<EP_X_BF16_TO_NVFP4>(a, stream);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_mgpu_combine(const MgpuArgs& a, cudaStream_t stream) {
    switch ((a.g.num_topk + 7) / 8) {
        case 1: return launch_combine_t<1>(a, stream);
        case 2: return launch_combine_t<2>(a, stream);
        case 3: return launch_combine_t<3>(a, stream);
        case 4: return launch_combine_t<4>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ep
