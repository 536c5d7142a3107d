// Per-item work of the dispatch kernel.  An item is 16 bytes of one receive
// row -- 8 bf16 values (EP_X_BF16), 16 e4m3 values copied (EP_X_FP8), 16
// bf16 values quantised to 16 e4m3 bytes (EP_X_BF16_TO_FP8) -- or, for
// NVFP4, one 1x16 block: 16 bf16 values quantised to 8 bytes of E2M1 pairs
// and one E4M3 scale byte.
#pragma once

#include <cuda_fp4.h>

#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {
namespace dispatch_dev {

constexpr float kE4m3Max = 448.0f;
constexpr float kAmaxFloor = 1e-4f;

constexpr float kE2m1Max = 6.0f;
constexpr float kFp4AmaxFloor = 6.0f / 512.0f;  // 6 * 2^-9: the smallest e4m3 scale

struct Geometry {
    int row_bytes;    // bytes of one receive row
    int ipr;          // items per receive row
    int scale_bytes;  // bytes of one row of scales (0 in bf16 mode)
    int scale_pad;    // scale_bytes rounded up to 16
};

__host__ __device__ inline Geometry geometry(int mode, int H) {
    Geometry g;
    if (mode == EP_X_BF16_TO_NVFP4) {
        g.row_bytes = H / 2;
        g.ipr = H / 16;
        g.scale_bytes = H / 16;
    } else {
        const bool fp8 = mode != EP_X_BF16;
        g.row_bytes = fp8 ? H : 2 * H;
        g.ipr = g.row_bytes / 16;
        g.scale_bytes = fp8 ? (H / 128) * 4 : 0;
    }
    g.scale_pad = (g.scale_bytes + 15) & ~15;
    return g;
}

// The source of item c of token t (zeros when inactive).
struct Item {
    uint4 v0, v1;
};

template <int kMode>
__device__ __forceinline__ Item load_item(const DispatchArgs& d, int t, int c, bool active) {
    Item it;
    it.v0 = it.v1 = make_uint4(0, 0, 0, 0);
    if (!active) return it;
    if (kMode == EP_X_BF16_TO_FP8 || kMode == EP_X_BF16_TO_NVFP4) {
        const char* src = (const char*)d.x + (size_t)t * d.H * 2 + (size_t)c * 32;
        it.v0 = ld_stream(src);
        it.v1 = ld_stream(src + 16);
    } else {
        const size_t rb = kMode == EP_X_BF16 ? (size_t)d.H * 2 : (size_t)d.H;
        it.v0 = ld_stream((const char*)d.x + (size_t)t * rb + (size_t)c * 16);
    }
    return it;
}

// Two floats -> two E2M1 codes in one byte (a in the low nibble), nearest-even, saturating.
__device__ __forceinline__ uint32_t pack_e2m1x2(float a, float b) {
    return (uint32_t)__nv_cvt_float2_to_fp4x2(make_float2(a, b), __NV_E2M1, cudaRoundNearest);
}

// Writes item c of token t into the row buffer rb (and its block scale
// into sb).  In the FP8 quantising mode all 32 lanes of the warp must call
// it together: a 1x128 block is 8 consecutive lanes and its amax is a
// 3-step xor shuffle; lane 0 of the group stores the scale.  In the NVFP4
// mode a lane holds a whole 1x16 block and stores its e4m3 scale byte.

template <int kMode>
__device__ __forceinline__ void fill_item(const DispatchArgs& d, int t, int c, bool active, const Item& it,
                                          unsigned char* rb, float* sb) {
    if (kMode == EP_X_BF16_TO_NVFP4) {
        // one 1x16 block per lane: no shuffles
        const uint4 v0 = it.v0, v1 = it.v1;
        const float f[16] = {bf16_lo(v0.x), bf16_hi(v0.x), bf16_lo(v0.y), bf16_hi(v0.y),
                             bf16_lo(v0.z), bf16_hi(v0.z), bf16_lo(v0.w), bf16_hi(v0.w),
                             bf16_lo(v1.x), bf16_hi(v1.x), bf16_lo(v1.y), bf16_hi(v1.y),
                             bf16_lo(v1.z), bf16_hi(v1.z), bf16_lo(v1.w), bf16_hi(v1.w)};
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
        amax = fmaxf(amax, kFp4AmaxFloor);
        const __nv_fp8_storage_t code = __nv_cvt_float_to_fp8(__fdiv_rn(amax, kE2m1Max), __NV_SATFINITE, __NV_E4M3);
        const float scale = __half2float(__half(__nv_cvt_fp8_to_halfraw(code, __NV_E4M3)));
        const float inv = __fdiv_rn(1.0f, scale);
        uint32_t w[2] = {0, 0};
#pragma unroll
        for (int i = 0; i < 8; ++i)
            w[i >> 2] |= pack_e2m1x2(__fmul_rn(f[2 * i], inv), __fmul_rn(f[2 * i + 1], inv)) << (8 * (i & 3));
        if (active) {
            reinterpret_cast<uint2*>(rb)[c] = make_uint2(w[0], w[1]);
            reinterpret_cast<unsigned char*>(sb)[c] = code;
        }
    } else if (kMode == EP_X_BF16_TO_FP8) {
        const uint4 v0 = it.v0, v1 = it.v1;
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
        const float scale = __fdiv_rn(amax, kE4m3Max);
        const float inv = __fdiv_rn(kE4m3Max, amax);
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = pack_e4m3x2(__fmul_rn(f[4 * i], inv), __fmul_rn(f[4 * i + 1], inv)) |
                   (pack_e4m3x2(__fmul_rn(f[4 * i + 2], inv), __fmul_rn(f[4 * i + 3], inv)) << 16);
        if (active) {
            reinterpret_cast<uint4*>(rb)[c] = make_uint4(w[0], w[1], w[2], w[3]);
            if ((c & 7) == 0) sb[c >> 3] = scale;
        }
    } else if (active) {
        reinterpret_cast<uint4*>(rb)[c] = it.v0;
        if (kMode == EP_X_FP8 && (c & 7) == 0) sb[c >> 3] = ld_cg(d.x_scales + (size_t)t * (d.H / 128) + (c >> 3));
    }
}

}  // namespace dispatch_dev
}  // namespace ep
