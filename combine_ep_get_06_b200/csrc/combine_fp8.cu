// Combine of FP8 expert outputs (the low-precision combine; DeepEP V2
// README, introduction: the kernels support low precision, FP8 included).
//
// y arrives as e4m3 codes [rows, H] with one f32 scale per 1x128 block
// [rows, H/128], the layout the FP8 dispatch produces.  Each value is
// decoded (e4m3 -> half -> float, exact) and multiplied by its block scale
// in binary32, then summed exactly as the bf16 combine does:
//   out[t] = bf16( acc ),  acc = fma(w[t,j], decode(q) * scale, acc)
// from +0 over the valid slots in ascending j.
//
// A thread handles 16-byte items: 16 codes, all in one 1x128 block (8
// consecutive items share a scale), 16 bf16 outputs (two 16-byte stores).
// (The packed f32x2 multiply / FMA give the same bits but measured slower.)
// A CTA covers a slice of one token's items; each thread issues its k code
// loads and k scale loads before the math.  Launched with programmatic
// dependent launch, like the other kernels.
#include <cuda_fp8.h>

#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {
namespace {

constexpr int kMaxThreads = 256;

__device__ __forceinline__ void decode4(uint32_t w, float (&f)[16], int o) {
    const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xFFFFu), __NV_E4M3);
    const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3);
    const float2 a = __half22float2(__half2(lo));
    const float2 b = __half22float2(__half2(hi));
    f[o] = a.x;
    f[o + 1] = a.y;
    f[o + 2] = b.x;
    f[o + 3] = b.y;
}

template <int G>  // groups of 8 slots: k <= 8 * G
__global__ void __launch_bounds__(kMaxThreads) combine_fp8_kernel(CombineFp8Args a, int ipr, int upr) {
    const int tid = threadIdx.x;
    const int T = a.T, k = a.k, H = a.H, B = H / 128;
    const char* const yq = (const char*)a.y_q;
    pdl_wait();

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

        float acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            uint4 v[8];
            float s[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int row = rows[8 * g + jj];
                v[jj] = row >= 0 ? ld_stream(yq + (size_t)row * H + (size_t)c * 16) : make_uint4(0, 0, 0, 0);
                s[jj] = row >= 0 ? a.y_scales[(size_t)row * B + (c >> 3)] : 0.0f;
            }
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                if (rows[8 * g + jj] < 0) continue;
                float f[16];
                decode4(v[jj].x, f, 0);
                decode4(v[jj].y, f, 4);
                decode4(v[jj].z, f, 8);
                decode4(v[jj].w, f, 12);
                const float wj = w[8 * g + jj], sj = s[jj];
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[i] = __fmaf_rn(wj, __fmul_rn(f[i], sj), acc[i]);
            }
        }
        char* const o = (char*)a.out + (size_t)t * H * 2 + (size_t)c * 32;
        st_stream(o, make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7])));
        st_stream(o + 16, make_uint4(pack_bf16x2(acc[8], acc[9]), pack_bf16x2(acc[10], acc[11]),
                                     pack_bf16x2(acc[12], acc[13]), pack_bf16x2(acc[14], acc[15])));
    }
    pdl_launch_dependents();
}

int unit_threads(int ipr) {
    for (int bd = kMaxThreads; bd >= 32; bd -= 32)
        if (ipr % bd == 0) return bd;
    return ipr < kMaxThreads ? ((ipr + 31) / 32) * 32 : kMaxThreads;
}

template <int G>
cudaError_t launch_t(const CombineFp8Args& a, cudaStream_t stream) {
    const int ipr = a.H / 16;
    const int bd = unit_threads(ipr);
    const int upr = (ipr + bd - 1) / bd;
    int per_sm = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, combine_fp8_kernel<G>, bd, 0);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) per_sm = 1;
    const int64_t cap = (int64_t)device_sm_count() * per_sm;
    const int64_t want = (int64_t)a.T * upr;
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
    debug_launch("combine_fp8_kernel", G, cfg);
    return cudaLaunchKernelEx(&cfg, combine_fp8_kernel<G>, a, ipr, upr);
}

}  // namespace

cudaError_t launch_combine_fp8(const CombineFp8Args& a, cudaStream_t stream) {
    switch ((a.k + 7) / 8) {
        case 1: return launch_t<1>(a, stream);
        case 2: return launch_t<2>(a, stream);
        case 3: return launch_t<3>(a, stream);
        case 4: return launch_t<4>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ep
