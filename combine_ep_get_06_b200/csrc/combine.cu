// MoE combine on one device (DeepEP V2 README, "Interfaces and examples",
// combine_forward, and dispatch_backward when unweighted).
//
// out[t] = bf16( sum_j w[t,j] * y[slot_map[t*k+j]] ) over the valid slots,
// fp32 FMA from +0 in ascending j, one bf16 rounding at the end.  A CTA
// works on one unit = blockDim 16-byte column items (8 bf16) of one token:
// each thread issues its (up to 8 per group) row loads before the FMAs, so
// a thread keeps k 16-byte loads in flight.  Launched with programmatic
// dependent launch: the CTAs start while the previous grid finishes and
// wait for it before reading anything; each lets the next grid start
// launching once its own work is issued.
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {
namespace {

constexpr int kMaxThreads = 256;

template <int G>  // groups of 8 slots: k <= 8 * G
__global__ void __launch_bounds__(kMaxThreads) combine_kernel(CombineArgs a, int ipr, int upr) {
    const int tid = threadIdx.x;
    const int T = a.T, k = a.k, H = a.H;
    const char* const y = (const char*)a.y;
    const size_t row_bytes = (size_t)H * 2;
    pdl_wait();

    // dispatch_backward's weight gradient: gather each slot's row value.
    if (a.out_weights != nullptr) {
        const int64_t n = (int64_t)T * k;
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + tid; i < n; i += (int64_t)gridDim.x * blockDim.x) {
            const int row = ld_cg(a.slot_map + i);
            a.out_weights[i] = (row >= 0 && row < a.max_rows) ? ld_cg(a.recv_weights_in + row) : 0.0f;
        }
    }

    const int64_t n_units = (int64_t)T * upr;
    for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
        const int t = (int)(u / upr);
        const int c = (int)(u - (int64_t)t * upr) * blockDim.x + tid;
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

int unit_threads(int ipr) {
    for (int bd = kMaxThreads; bd >= 32; bd -= 32)
        if (ipr % bd == 0) return bd;
    return ipr < kMaxThreads ? ((ipr + 31) / 32) * 32 : kMaxThreads;
}

template <int G>
cudaError_t launch_t(const CombineArgs& a, cudaStream_t stream) {
    const int ipr = a.H / 8;
    const int bd = unit_threads(ipr);
    const int upr = (ipr + bd - 1) / bd;
    int per_sm = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, combine_kernel<G>, bd, 0);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) per_sm = 1;
    // Persistent grid, no larger than the work.
    const int64_t cap = (int64_t)device_sm_count() * per_sm;
    int64_t want = (int64_t)a.T * upr;
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
    return cudaLaunchKernelEx(&cfg, combine_kernel<G>, a, ipr, upr);
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
