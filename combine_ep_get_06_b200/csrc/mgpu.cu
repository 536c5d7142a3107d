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
// keeps its next unit's x loads and routing loads in flight, converts the
// slice into one of its kStages shared-memory stages, and lanes j < k copy
// the stage to the slice's k destinations in peers' blocks (through the
// peer table) with TMA bulk copies, shared -> global, one destination each.
// Where a destination is not 16-byte aligned the warp stores it with plain
// stores instead.  The warp that takes a token's first slice also writes
// the token's slot metadata.  Padding rows are zeroed in this rank's own
// block from a zero buffer, and CTA 0 writes its receive totals.  No
// barrier after the tables: warps never wait on one another.

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
constexpr int kStages = 4;  // shared-memory stages per warp

struct MgpuSmem {
    int* first;      // [E]
    int* lofs;       // [E]
    int* asz;        // [E] A_e
    int* own_c;      // [epr]
    int* own_off;    // [epr]
    int* padoff;     // [epr + 1]
    char** peer;     // [W]
    unsigned char* zeros;   // [stage_bytes] of zeros
    unsigned char* stages;  // [kWarps][kStages][stage_bytes]
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
    unsigned char* zeros = take((size_t)stage_bytes);
    unsigned char* stages = take((size_t)kWarps * kStages * stage_bytes);
    if (m != nullptr) {
        m->first = (int*)first;
        m->lofs = (int*)lofs;
        m->asz = (int*)asz;
        m->own_c = (int*)own_c;
        m->own_off = (int*)own_off;
        m->padoff = (int*)padoff;
        m->peer = (char**)peer;
        m->zeros = zeros;
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

// The raw routing loads of unit u, issued a unit ahead: per lane j < k the
// slot's local row and expert (and on a token's first slice its weight);
// for pre-quantised FP8 the slice's block scales.
struct Route {
    int lr;
    long long e;
    float w;
    float xs;
};

template <int kMode>
__device__ __forceinline__ Route load_route(const MgpuArgs& a, const SliceGeo& sg, int64_t u, int64_t n_tok_units,
                                            int lane) {
    Route r;
    r.lr = -1;
    r.e = -1;
    r.w = 0.0f;
    r.xs = 0.0f;
    if (u >= n_tok_units) return r;
    const int k = a.g.num_topk;
    const int t = (int)(u / sg.ns), s = (int)(u - (int64_t)t * sg.ns);
    if (lane < k) {
        const size_t sl = (size_t)t * k + lane;
        r.lr = a.slot_map[sl];
        r.e = a.idx_is_int64 ? ((const int64_t*)a.topk_idx)[sl] : ((const int32_t*)a.topk_idx)[sl];
        if (s == 0 && a.topk_weights) r.w = a.topk_weights[sl];
    }
    if (kMode == EP_X_FP8) {
        const int ne = min(kSliceElems, a.g.hidden - s * kSliceElems);
        if (lane < ne / 128) r.xs = a.src.x_scales[(size_t)t * (a.g.hidden / 128) + s * (kSliceElems / 128) + lane];
    }
    return r;
}

__device__ __forceinline__ bool bulk_ok(const void* dst, int n) {
    return ((reinterpret_cast<uintptr_t>(dst) | (uintptr_t)n) & 15) == 0;
}

template <int kMode>
__global__ void __launch_bounds__(kThreads, 2) mgpu_dispatch_kernel(MgpuArgs a) {
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
    unsigned char* const stages = m.stages + (size_t)warp * kStages * sg.stage_bytes;

    // The first unit's loads fly while the tables are built (the grid
    // starts after the layout and the counts exchange have completed).
    const int64_t n_tok_units = (int64_t)T * sg.ns;
    const int64_t stride = (int64_t)gridDim.x * kWarps;
    int64_t u = (int64_t)blockIdx.x * kWarps + warp;
    Loads<kMode> nxt = load_x<kMode>(a.src, sg, u, n_tok_units, lane);
    Route nrt = load_route<kMode>(a, sg, u, n_tok_units, lane);

    for (int i = tid; i < sg.stage_bytes / 16; i += kThreads) reinterpret_cast<uint4*>(m.zeros)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    build_tables(a, m);  // ends with a barrier
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

    const int64_t n_units = n_tok_units + n_pad;
    int it = 0;  // token units of this warp (selects the stage)
    for (; u < n_units; u += stride) {
        const Loads<kMode> cur = nxt;
        const Route rt = nrt;
        {
            const int64_t un = u + stride;
            nxt = load_x<kMode>(a.src, sg, un, n_tok_units, lane);
            nrt = load_route<kMode>(a, sg, un, n_tok_units, lane);
        }
        if (u >= n_tok_units) {
            // one of this rank's padding rows, in its own block
            const int p = (int)(u - n_tok_units);
            const int i = local_expert_of_pad(m, epr, p);
            const int row = m.own_off[i] + m.own_c[i] + (p - m.padoff[i]);
            if (row >= g.max_recv_rows) {
                if (lane == 0) atomicOr(err, EP_DEVERR_CAPACITY);
                continue;
            }
            char* const dx = a.local_block + g.off_recv_x + (size_t)row * rb_bytes;
            char* const ds = a.local_block + g.off_recv_scales + (size_t)row * sc_bytes;
            bool plain_x = false, plain_s = false;
            for (int s = lane; s < sg.ns; s += 32) {
                const int ne = min(kSliceElems, g.hidden - s * kSliceElems);
                const int db = ne * sg.out_bytes / kSliceElems;
                char* const px = dx + (size_t)s * sg.out_bytes;
                if (bulk_ok(px, db)) bulk_s2g(px, m.zeros, db);
                else plain_x = true;
                if (sc_bytes > 0) {
                    const int sb = ne / M::kScaleBlock * M::kScaleBytes;
                    char* const ps = ds + (size_t)s * sg.sout_bytes;
                    if (bulk_ok(ps, sb)) bulk_s2g(ps, m.zeros, sb);
                    else plain_s = true;
                }
            }
            bulk_commit();
            if (__any_sync(0xffffffffu, plain_x)) warp_zero_out(dx, rb_bytes, lane);
            if (__any_sync(0xffffffffu, plain_s)) warp_zero_out(ds, sc_bytes, lane);
            if (lane == 0) {
                ((int32_t*)(a.local_block + g.off_recv_src))[row] = -1;
                ((int32_t*)(a.local_block + g.off_recv_topk_idx))[row] = -1;
                ((float*)(a.local_block + g.off_recv_topk_weights))[row] = 0.0f;
            }
            continue;
        }

        // A token slice: resolve its routing (loaded a unit ago).
        const int t = (int)(u / sg.ns), s = (int)(u - (int64_t)t * sg.ns);
        const int ne = min(kSliceElems, g.hidden - s * kSliceElems);
        int d = -1, row = -1;
        if (lane < k) {
            const size_t sl = (size_t)t * k + lane;
            if (rt.lr >= 0) {
                if (rt.e < 0 || rt.e >= g.num_experts) {
                    // not the topk_idx the layout saw: drop the slot
                    if (s == 0) atomicOr(err, EP_DEVERR_BAD_TOPK_IDX);
                } else {
                    const int e = (int)rt.e;
                    d = e / epr;
                    row = m.first[e] + (rt.lr - m.lofs[e]);
                }
                if (d < 0) {
                    row = -1;
                } else if (row < 0 || row >= g.max_recv_rows) {
                    if (s == 0) atomicOr(err, EP_DEVERR_CAPACITY);
                    d = row = -1;
                } else if (s == 0) {
                    char* pb = m.peer[d];
                    ((int32_t*)(pb + g.off_recv_src))[row] = (int32_t)((int64_t)g.rank * g.max_tokens * k + sl);
                    ((int32_t*)(pb + g.off_recv_topk_idx))[row] = (int)rt.e;
                    ((float*)(pb + g.off_recv_topk_weights))[row] = rt.w;
                }
            }
            if (s == 0) dest[sl] = make_int2(d, row);
        }

        unsigned char* const st = stages + (size_t)(it % kStages) * sg.stage_bytes;
        unsigned char* const sst = st + sg.out_bytes;
        ++it;
        // The copies issued from this stage kStages units ago must have read it.
        if (lane < k) bulk_wait_read<kStages - 1>();
        __syncwarp();
        Meta mt;
        mt.row = -1;
        mt.xs = rt.xs;
        fill_stage<kMode>(cur, mt, ne, lane, st, sst);
        fence_proxy_async_smem();
        __syncwarp();
        const int db = ne * sg.out_bytes / kSliceElems;
        const int sb = M::kScales ? ne / M::kScaleBlock * M::kScaleBytes : 0;
        bool plain_x = false, plain_s = false;
        if (lane < k) {
            if (d >= 0) {
                char* const pb = m.peer[d];
                char* const px = pb + g.off_recv_x + (size_t)row * rb_bytes + (size_t)s * sg.out_bytes;
                if (bulk_ok(px, db)) bulk_s2g(px, st, db);
                else plain_x = true;
                if (sb > 0) {
                    char* const ps = pb + g.off_recv_scales + (size_t)row * sc_bytes + (size_t)s * sg.sout_bytes;
                    if (bulk_ok(ps, sb)) bulk_s2g(ps, sst, sb);
                    else plain_s = true;
                }
            }
            bulk_commit();
        }
        // Destinations a bulk copy cannot take: the whole warp stores them.
        unsigned px_mask = __ballot_sync(0xffffffffu, plain_x), ps_mask = __ballot_sync(0xffffffffu, plain_s);
        while (px_mask | ps_mask) {
            const int j = __ffs(px_mask | ps_mask) - 1;
            const int dj = __shfl_sync(0xffffffffu, d, j), rj = __shfl_sync(0xffffffffu, row, j);
            char* const pb = m.peer[dj];
            if (px_mask >> j & 1)
                warp_copy_out(pb + g.off_recv_x + (size_t)rj * rb_bytes + (size_t)s * sg.out_bytes, st, db, lane);
            if (ps_mask >> j & 1)
                warp_copy_out(pb + g.off_recv_scales + (size_t)rj * sc_bytes + (size_t)s * sg.sout_bytes, sst, sb,
                              lane);
            px_mask &= ~(1u << j);
            ps_mask &= ~(1u << j);
        }
    }
    // The CTA's writes to peers' memory are ordered before the grid's end:
    // each thread waits for its bulk copies to complete and orders them
    // (async proxy) before its own later accesses (proxy fence); the
    // barrier makes all of them precede thread 0's system-scope fence,
    // which is cumulative.  (A system fence in every thread measured as the
    // top stall.)
    bulk_wait_all();
    fence_proxy_async_global();
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
