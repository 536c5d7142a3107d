// Warp units of the dispatch kernels (dispatch.cu, mgpu.cu): the shape of a
// unit -- 1024 consecutive elements of one token row, loaded 16 bytes a lane
// (a warp load covers 512 contiguous bytes) -- its x loads, and its
// conversion into a shared-memory stage: bf16 or e4m3 copied, bf16
// quantised to e4m3 with one f32 scale per 1x128 block (16 lanes; amax by
// xor shuffles, scale and inverse by IEEE division), or to NVFP4 E2M1 codes
// with one e4m3 scale per 1x16 block (a lane pair).
#pragma once

#include <cuda_fp4.h>

#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {
namespace warp_units {

constexpr int kSliceElems = 1024;
constexpr float kE4m3Max = 448.0f;
constexpr float kAmaxFloor = 1e-4f;
constexpr float kE2m1Max = 6.0f;
constexpr float kFp4AmaxFloor = 6.0f / 512.0f;  // 6 * 2^-9: the smallest e4m3 scale

// Per-mode shape of a unit: 16-byte loads per lane and the elements in each.
template <int kMode>
struct Mode {
    static constexpr int kLoads = kMode == EP_X_FP8 ? 2 : 4;
    static constexpr int kElemsPerLoad = kMode == EP_X_FP8 ? 16 : 8;
    static constexpr bool kScales = kMode != EP_X_BF16;
    static constexpr int kScaleBlock = kMode == EP_X_BF16_TO_NVFP4 ? 16 : 128;  // elements per scale
    static constexpr int kScaleBytes = kMode == EP_X_BF16_TO_NVFP4 ? 1 : 4;    // bytes per scale
    static_assert(kLoads * kElemsPerLoad * 32 == kSliceElems, "a unit is one slice");
};

// Bytes of the receive row and of its slices, for a mode and hidden size.
struct SliceGeo {
    int ns;          // slices per row, ceil(H / 1024)
    int row_bytes;   // bytes of a receive row
    int srow_bytes;  // bytes of a receive row's scales (0: bf16)
    int out_bytes;   // data bytes of a full slice
    int sout_bytes;  // scale bytes of a full slice
    int stage_bytes; // out_bytes + sout_bytes (both multiples of 16)
};

__host__ __device__ inline SliceGeo slice_geo(int mode, int H) {
    SliceGeo g;
    g.ns = (H + kSliceElems - 1) / kSliceElems;
    if (mode == EP_X_BF16) {
        g.row_bytes = 2 * H;
        g.srow_bytes = 0;
        g.out_bytes = 2 * kSliceElems;
        g.sout_bytes = 0;
    } else if (mode == EP_X_BF16_TO_NVFP4) {
        g.row_bytes = H / 2;
        g.srow_bytes = H / 16;
        g.out_bytes = kSliceElems / 2;
        g.sout_bytes = kSliceElems / 16;
    } else {
        g.row_bytes = H;
        g.srow_bytes = (H / 128) * 4;
        g.out_bytes = kSliceElems;
        g.sout_bytes = (kSliceElems / 128) * 4;
    }
    g.stage_bytes = g.out_bytes + g.sout_bytes;
    return g;
}

template <int kMode>
struct Loads {
    uint4 v[Mode<kMode>::kLoads];
};

// Routing of a unit: a token slice's receive row for lane j < k (or the
// padding row, for every lane), and for pre-quantised x the slice's input
// scale for lane b < blocks in the slice.
struct Meta {
    int row;
    float xs;
};

// x loads of unit u (zeros for lanes past the row's end and for padding units).
template <int kMode>
__device__ __forceinline__ Loads<kMode> load_x(const DispatchArgs& a, const SliceGeo& g, int64_t u,
                                               int64_t n_tok_units, int lane) {
    using M = Mode<kMode>;
    Loads<kMode> l;
#pragma unroll
    for (int i = 0; i < M::kLoads; ++i) l.v[i] = make_uint4(0, 0, 0, 0);
    if (u >= n_tok_units) return l;
    const int t = (int)(u / g.ns), s = (int)(u - (int64_t)t * g.ns);
    const int ne = min(kSliceElems, a.H - s * kSliceElems);
    const size_t in_row = kMode == EP_X_FP8 ? (size_t)a.H : (size_t)a.H * 2;
    const char* base = (const char*)a.x + (size_t)t * in_row + (size_t)s * kSliceElems * (in_row / a.H);
#pragma unroll
    for (int i = 0; i < M::kLoads; ++i) {
        const int idx = i * 32 + lane;
        if (idx * M::kElemsPerLoad < ne) l.v[i] = ld_stream(base + (size_t)idx * 16);
    }
    return l;
}

// ---- conversions shared by the warp units and the row path

// bf16 pairs (low half first) of four 32-bit words -> 8 floats, exactly.
__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z); f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// FP8 block scale from the block's amax: scale = amax/448 and inv = 448/amax
// (amax floored at 1e-4), each one IEEE division.
__device__ __forceinline__ void fp8_scale(float amax, float& scale, float& inv) {
    amax = fmaxf(amax, kAmaxFloor);
    scale = __fdiv_rn(amax, kE4m3Max);
    inv = __fdiv_rn(kE4m3Max, amax);
}

// 4 floats times inv (one rounding each) -> 4 e4m3 bytes, nearest-even, saturating.
__device__ __forceinline__ uint32_t e4m3x4(const float* f, float inv) {
    return pack_e4m3x2(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv)) |
           (pack_e4m3x2(__fmul_rn(f[2], inv), __fmul_rn(f[3], inv)) << 16);
}

// NVFP4 block scale from the 1x16 block's amax (floored at 6*2^-9): the
// e4m3 code of amax/6 and the inverse of the decoded scale.
__device__ __forceinline__ __nv_fp8_storage_t nvfp4_scale(float amax, float& inv) {
    amax = fmaxf(amax, kFp4AmaxFloor);
    const __nv_fp8_storage_t code = __nv_cvt_float_to_fp8(__fdiv_rn(amax, kE2m1Max), __NV_SATFINITE, __NV_E4M3);
    inv = __fdiv_rn(1.0f, __half2float(__half(__nv_cvt_fp8_to_halfraw(code, __NV_E4M3))));
    return code;
}

// 8 floats times inv -> 8 E2M1 codes in 4 bytes, the even element in the low nibble.
__device__ __forceinline__ uint32_t e2m1x8(const float* f, float inv) {
    uint32_t w = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e)
        w |= (uint32_t)__nv_cvt_float2_to_fp4x2(make_float2(__fmul_rn(f[2 * e], inv), __fmul_rn(f[2 * e + 1], inv)),
                                                 __NV_E2M1, cudaRoundNearest)
             << (8 * e);
    return w;
}

__device__ __forceinline__ float amax8(const float* f) {
    float m = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
    return m;
}

// Converts the unit's loads into the stage: data at st, scales at sst.
template <int kMode>
__device__ __forceinline__ void fill_stage(const Loads<kMode>& l, const Meta& m, int ne, int lane,
                                           unsigned char* st, unsigned char* sst) {
    using M = Mode<kMode>;
#pragma unroll
    for (int i = 0; i < M::kLoads; ++i) {
        const int idx = i * 32 + lane;
        const bool active = idx * M::kElemsPerLoad < ne;
        const uint4 v = l.v[i];
        if (kMode == EP_X_BF16 || kMode == EP_X_FP8) {
            if (active) reinterpret_cast<uint4*>(st)[idx] = v;
        } else {
            float f[8];
            unpack8(v, f);
            float amax = amax8(f);
            if (kMode == EP_X_BF16_TO_FP8) {
                // a 1x128 block is 16 lanes (all active or all inactive: H % 128 == 0)
#pragma unroll
                for (int o = 1; o < 16; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                float scale, inv;
                fp8_scale(amax, scale, inv);
                const uint32_t w0 = e4m3x4(f, inv), w1 = e4m3x4(f + 4, inv);
                if (active) {
                    reinterpret_cast<uint2*>(st)[idx] = make_uint2(w0, w1);
                    if ((lane & 15) == 0) reinterpret_cast<float*>(sst)[idx >> 4] = scale;
                }
            } else {
                // NVFP4: a 1x16 block is a lane pair (H % 32 == 0)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
                float inv;
                const __nv_fp8_storage_t code = nvfp4_scale(amax, inv);
                const uint32_t w = e2m1x8(f, inv);
                if (active) {
                    reinterpret_cast<uint32_t*>(st)[idx] = w;
                    if ((lane & 1) == 0) sst[idx >> 1] = code;
                }
            }
        }
    }
    if (kMode == EP_X_FP8 && lane < ne / 128) reinterpret_cast<float*>(sst)[lane] = m.xs;
}

}  // namespace warp_units
}  // namespace ep
