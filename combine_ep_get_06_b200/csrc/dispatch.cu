// MoE dispatch on one device (DeepEP V2 README, "Interfaces and examples",
// dispatch_forward; FP8 dispatching as in its section "Performance").
//
// Token-major: each token row is read from HBM once and, in the FP8 mode,
// quantised once, then stored to each of its k receive rows.  A CTA works
// on one unit = a slice of blockDim 16-byte items of one row; units are
// handed out grid-stride over the token rows followed by the padding rows
// (which are zero-filled).  In the quantising mode a 1x128 block is 8
// consecutive lanes (16 bf16 values each): its amax is a 3-step xor
// shuffle, and lane 0 of the group stores the block's scale.
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {
namespace {

constexpr int kMaxThreads = 256;
constexpr float kE4m3Max = 448.0f;
constexpr float kAmaxFloor = 1e-4f;

template <int kMode>
__global__ void __launch_bounds__(kMaxThreads) dispatch_kernel(DispatchArgs a, int ipr, int upr) {
    constexpr bool kFp8Out = kMode != EP_X_BF16;
    const int tid = threadIdx.x;
    const int T = a.T, k = a.k, H = a.H, B = H / 128;
    const size_t row_bytes = kFp8Out ? (size_t)H : (size_t)H * 2;
    const int n_pad = *a.num_pad_rows;
    const int64_t n_units = (int64_t)(T + n_pad) * upr;
    char* const recv = (char*)a.recv_x;

    for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
        const int r = (int)(u / upr);
        const int c = (int)(u - (int64_t)r * upr) * blockDim.x + tid;  // 16-byte item of the row
        const bool active = c < ipr;

        if (r >= T) {  // padding row: zero data and scales
            const int row = __ldg(a.pad_rows + (r - T));
            if (active && row < a.max_rows) {
                st_stream(recv + (size_t)row * row_bytes + (size_t)c * 16, make_uint4(0, 0, 0, 0));
                if (kFp8Out && (c & 7) == 0) a.recv_scales[(size_t)row * B + (c >> 3)] = 0.0f;
            }
            continue;
        }

        const int t = r;
        uint4 out;
        float scale = 0.0f;
        if (kMode == EP_X_BF16_TO_FP8) {
            const char* src = (const char*)a.x + (size_t)t * H * 2 + (size_t)c * 32;
            uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
            if (active) {
                v0 = ld_stream(src);
                v1 = ld_stream(src + 16);
            }
            float f[16] = {bf16_lo(v0.x), bf16_hi(v0.x), bf16_lo(v0.y), bf16_hi(v0.y),
                           bf16_lo(v0.z), bf16_hi(v0.z), bf16_lo(v0.w), bf16_hi(v0.w),
                           bf16_lo(v1.x), bf16_hi(v1.x), bf16_lo(v1.y), bf16_hi(v1.y),
                           bf16_lo(v1.z), bf16_hi(v1.z), bf16_lo(v1.w), bf16_hi(v1.w)};
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
            amax = fmaxf(amax, kAmaxFloor);
            scale = __fdiv_rn(amax, kE4m3Max);
            const float inv = __fdiv_rn(kE4m3Max, amax);
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                w[i] = pack_e4m3x2(__fmul_rn(f[4 * i], inv), __fmul_rn(f[4 * i + 1], inv)) |
                       (pack_e4m3x2(__fmul_rn(f[4 * i + 2], inv), __fmul_rn(f[4 * i + 3], inv)) << 16);
            out = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
            out = make_uint4(0, 0, 0, 0);
            if (active) out = ld_stream((const char*)a.x + (size_t)t * row_bytes + (size_t)c * 16);
            if (kMode == EP_X_FP8 && active && (c & 7) == 0)
                scale = __ldg(a.x_scales + (size_t)t * B + (c >> 3));
        }
        if (!active) continue;

        const int32_t* sm = a.slot_map + (size_t)t * k;
        for (int j = 0; j < k; ++j) {
            const int row = __ldg(sm + j);
            if (row < 0) continue;
            if (row >= a.max_rows) {
                atomicOr(a.error_word, EP_DEVERR_CAPACITY);
                continue;
            }
            st_stream(recv + (size_t)row * row_bytes + (size_t)c * 16, out);
            if (kFp8Out && (c & 7) == 0) a.recv_scales[(size_t)row * B + (c >> 3)] = scale;
        }
    }
}

// Threads per CTA: the largest multiple of 32 (<= 256) that divides the
// row's item count, so that units tile rows exactly; else 256.
int unit_threads(int ipr) {
    for (int bd = kMaxThreads; bd >= 32; bd -= 32)
        if (ipr % bd == 0) return bd;
    return ipr < kMaxThreads ? ((ipr + 31) / 32) * 32 : kMaxThreads;
}

template <int kMode>
cudaError_t launch_t(const DispatchArgs& a, cudaStream_t stream) {
    const int ipr = (kMode == EP_X_BF16) ? a.H / 8 : a.H / 16;
    const int bd = unit_threads(ipr);
    const int upr = (ipr + bd - 1) / bd;
    int per_sm = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dispatch_kernel<kMode>, bd, 0);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) per_sm = 1;
    // Persistent grid: the padding-row count is only known on the device.
    const unsigned grid = (unsigned)(device_sm_count() * per_sm);
    dispatch_kernel<kMode><<<grid, bd, 0, stream>>>(a, ipr, upr);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dispatch(const DispatchArgs& a, ep_x_mode mode, cudaStream_t stream) {
    switch (mode) {
        case EP_X_BF16: return launch_t<EP_X_BF16>(a, stream);
        case EP_X_FP8: return launch_t<EP_X_FP8>(a, stream);
        case EP_X_BF16_TO_FP8: return launch_t<EP_X_BF16_TO_FP8>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ep
