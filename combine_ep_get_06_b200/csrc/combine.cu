// MoE combine on one device (DeepEP V2 README, "Interfaces and examples",
// combine_forward, and dispatch_backward when unweighted).
//
// out[t] = bf16( sum_j w[t,j] * y[slot_map[t*k+j]] ) over the valid slots,
// fp32 FMA from +0 in ascending j, one bf16 rounding at the end.  A unit is
// `ut` 16-byte column items (8 bf16) of one token, one item per thread: each
// thread issues its (up to 8 per group) row loads before the FMAs, so a
// thread keeps k 16-byte loads in flight.  A CTA is blockDim / ut groups of
// ut threads, each working through units on its own (one group normally;
// under an SM budget enough groups to fill an SM with one CTA).  Launched with programmatic
// dependent launch: the CTAs start while the previous grid finishes and
// wait for it before reading anything; each lets the next grid start
// launching once its own work is issued.
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {
namespace {

constexpr int kMaxThreads = 448;   // threads of a unit at most (V3: two units of 448 per token row)
constexpr int kSmallThreads = 256; // launch bound of the kernel for units of at most this many threads

// Threads of a unit under an SM budget at most (a CTA holds several).
constexpr int kBudgetUnitThreads = 256;

// Threads of a CTA under an SM budget, for k <= 8*G: as many as fit an SM
// without spilling the k row values a thread holds.
template <int G>
constexpr int budget_threads() {
    return G == 1 ? 1024 : 256;
}

template <int G, int kMaxT>  // groups of 8 slots: k <= 8 * G; at most kMaxT threads
__global__ void __launch_bounds__(kMaxT) combine_kernel(CombineArgs a, int ipr, int upr, int ut) {
    const int tid = threadIdx.x;
    const int nsub = blockDim.x / ut, sub = tid / ut, lt = tid - sub * ut;
    const int T = a.T, k = a.k, H = a.H;
    const char* const y = (const char*)a.y;
    const size_t row_bytes = (size_t)H * 2;
    const int64_t n_units = (int64_t)T * upr;
    // With more units than the grid holds at once (a persistent grid), the
    // slot map and weights of the CTA's first units are asked into L2 while
    // the previous grid drains: a prefetch returns no value and every write
    // lands in L2, so nothing stale is observed (the loads come after the
    // wait).  Only the 16-byte aligned interior of each range.  (A one-wave
    // batch, as at decode, measured slower with it.)
    if (tid == 0 && n_units > (int64_t)gridDim.x * nsub) {
        const int64_t u_lo = (int64_t)blockIdx.x * nsub, u_hi = min(n_units, u_lo + nsub);
        if (u_hi > u_lo) {
            const int64_t s_lo = u_lo / upr * k, s_hi = ((u_hi - 1) / upr + 1) * k;
            prefetch_interior_l2(a.slot_map + s_lo, a.slot_map + s_hi);
            if (a.topk_weights != nullptr) prefetch_interior_l2(a.topk_weights + s_lo, a.topk_weights + s_hi);
        }
    }
    pdl_wait();

    // dispatch_backward's weight gradient: gather each slot's row value.
    if (a.out_weights != nullptr) {
        const int64_t n = (int64_t)T * k;
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + tid; i < n; i += (int64_t)gridDim.x * blockDim.x) {
            const int row = ld_cg(a.slot_map + i);
            a.out_weights[i] = (row >= 0 && row < a.max_rows) ? ld_cg(a.recv_weights_in + row) : 0.0f;
        }
    }

    const int64_t u0 = sub < nsub ? (int64_t)blockIdx.x * nsub + sub : n_units;
    for (int64_t u = u0; u < n_units; u += (int64_t)gridDim.x * nsub) {
        const int t = (int)(u / upr);
        const int c = (int)(u - (int64_t)t * upr) * ut + lt;
        if (c >= ipr) continue;

        int rows[8 * G];
        float w[8 * G];
#pragma unroll
        for (int j = 0; j < 8 * G; ++j) {
            int row = -1;
            float wj = 1.0f;
            if (j < k) {
                row = a.slot_map[(size_t)t * k + j];
                if (a.topk_weights != nullptr) wj = a.topk_weights[(size_t)t * k + j];
                if (row >= a.max_rows) {
                    atomicOr(a.error_word, EP_DEVERR_CAPACITY);
                    row = -1;
                }
            }
            rows[j] = row;
            w[j] = wj;
        }

        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            uint4 v[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int row = rows[8 * g + jj];
                v[jj] = row >= 0 ? ld_stream(y + (size_t)row * row_bytes + (size_t)c * 16)
                                 : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                if (rows[8 * g + jj] < 0) continue;
                const float wj = w[8 * g + jj];
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
    pdl_launch_dependents();
}

// Threads of a unit: the largest multiple of 32 up to `most` that divides
// the row's items, else the row rounded up to a warp (or `most`).
int unit_threads(int ipr, int most) {
    for (int bd = most; bd >= 32; bd -= 32)
        if (ipr % bd == 0) return bd;
    return ipr < most ? ((ipr + 31) / 32) * 32 : most;
}

// Below this many units per SM a batch is one short wave (decode sizes):
// units of at most 128 threads then spread its rows over more CTAs, so
// that every SM gets a similar share of the row loads.
constexpr int kSmallUnitsPerSm = 8;

template <int G, int kMaxT>
cudaError_t launch_bd(const CombineArgs& a, int ipr, int ut, int bd, int max_ctas, cudaStream_t stream) {
    const int upr = (ipr + ut - 1) / ut;
    auto kernel = combine_kernel<G, kMaxT>;
    int per_sm = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, bd, 0);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) per_sm = 1;
    // Persistent grid, no larger than the work.
    const int64_t cap = max_ctas > 0 ? max_ctas : (int64_t)device_sm_count() * per_sm;
    int64_t want = ((int64_t)a.T * upr + bd / ut - 1) / (bd / ut);
    if (a.out_weights != nullptr) {
        const int64_t gather = ((int64_t)a.T * a.k + bd - 1) / bd;
        if (gather > want) want = gather;
    }
    const int64_t grid = want < 1 ? 1 : (want < cap ? want : cap);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(bd);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    debug_launch("combine_kernel", G, cfg);
    return cudaLaunchKernelEx(&cfg, kernel, a, ipr, upr, ut);
}

// One unit group per CTA and as many CTAs as fit; under an SM budget of n,
// n CTAs of as many unit groups as fit budget_threads<G>(), one CTA to an SM.
template <int G>
cudaError_t launch_t(const CombineArgs& a, cudaStream_t stream) {
    const int ipr = a.H / 8;
    const int budget = sm_budget();
    if (budget > 0) {
        // units of at most kBudgetUnitThreads, several to a CTA of kT threads
        constexpr int kT = budget_threads<G>();
        const int ut = unit_threads(ipr, kBudgetUnitThreads);
        return launch_bd<G, kT>(a, ipr, ut, (kT / ut) * ut, budget, stream);
    }
    int ut = unit_threads(ipr, kMaxThreads);
    if ((int64_t)a.T * ((ipr + ut - 1) / ut) < (int64_t)kSmallUnitsPerSm * device_sm_count())
        ut = unit_threads(ipr, 128);
    // Units of up to 256 threads keep the kernel built for 256-thread
    // blocks: the looser bound of the 448-thread build lets the compiler
    // take registers that cost those launches an SM's worth of occupancy.
    if (ut <= kSmallThreads) return launch_bd<G, kSmallThreads>(a, ipr, ut, ut, 0, stream);
    return launch_bd<G, kMaxThreads>(a, ipr, ut, ut, 0, stream);
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream) {
    const int G = (a.k + 7) / 8;
    switch (G) {
        case 1: return launch_t<1>(a, stream);
        case 2: return launch_t<2>(a, stream);
        case 3: return launch_t<3>(a, stream);
        case 4: return launch_t<4>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ep
