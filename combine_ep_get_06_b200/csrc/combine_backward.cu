// Backward of the weighted combine (DeepEP V2 README, "Interfaces and
// examples": the backward of combine runs as a dispatch of the output
// gradient; with topk_weights in the forward, each receive row is scaled by
// its slot's weight, and the weights get their own gradient).
//
// For the output gradient g [T,H] bf16:
//   grad_y[slot_map[t*k+j], :] = bf16(w[t,j] * g[t, :])      (binary32 product)
//   grad_w[t, j]               = sum_h g[t,h] * y[slot_map[t*k+j], h]
// Padding rows of grad_y are zeroed; a dropped slot gets grad_w = 0.
//
// One kernel reads g[t] once and each valid y row once, writes each scaled
// grad_y row once: a CTA walks tokens grid-stride, each thread covering
// 16-byte column items of the token; per item it issues the k row loads
// before using them, stores the k scaled rows, and accumulates the k dot
// products in binary32 (FMA, item by item).  Per token the k partial sums
// are reduced in a fixed order (xor shuffles within warps, then warps in
// order), so the result is deterministic.  Padding rows follow the tokens.
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {
namespace {

constexpr int kMaxThreads = 256;

template <int G>  // groups of 8 slots: k <= 8 * G
__global__ void __launch_bounds__(kMaxThreads) combine_backward_kernel(CombineBackwardArgs a, int ipr) {
    __shared__ float red[kMaxThreads / 32][8 * G];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int T = a.T, k = a.k, H = a.H;
    const size_t row_bytes = (size_t)H * 2;
    const char* const gbase = (const char*)a.grad_out;
    const char* const ybase = (const char*)a.y;
    char* const gy = (char*)a.grad_y;

    pdl_wait();
    const int n_pad = ld_cg(a.num_pad_rows);

    for (int u = blockIdx.x; u < T + n_pad; u += gridDim.x) {
        if (u >= T) {  // a padding row of grad_y: zeros
            const int row = ld_cg(a.pad_rows + (u - T));
            if (row >= 0 && row < a.max_rows)
                for (int c = tid; c < ipr; c += blockDim.x)
                    st_stream(gy + (size_t)row * row_bytes + (size_t)c * 16, make_uint4(0, 0, 0, 0));
            continue;
        }
        const int t = u;
        int rows[8 * G];
        float w[8 * G], dot[8 * G];
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
            dot[j] = 0.0f;
        }

        for (int c = tid; c < ipr; c += blockDim.x) {
            const uint4 gv = ld_stream(gbase + (size_t)t * row_bytes + (size_t)c * 16);
            const float g[8] = {bf16_lo(gv.x), bf16_hi(gv.x), bf16_lo(gv.y), bf16_hi(gv.y),
                                bf16_lo(gv.z), bf16_hi(gv.z), bf16_lo(gv.w), bf16_hi(gv.w)};
#pragma unroll
            for (int grp = 0; grp < G; ++grp) {
                uint4 v[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int row = rows[8 * grp + jj];
                    v[jj] = row >= 0 ? ld_stream(ybase + (size_t)row * row_bytes + (size_t)c * 16)
                                     : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int j = 8 * grp + jj;
                    if (rows[j] < 0) continue;
                    const float wj = w[j];
                    const uint4 o = make_uint4(pack_bf16x2(__fmul_rn(wj, g[0]), __fmul_rn(wj, g[1])),
                                               pack_bf16x2(__fmul_rn(wj, g[2]), __fmul_rn(wj, g[3])),
                                               pack_bf16x2(__fmul_rn(wj, g[4]), __fmul_rn(wj, g[5])),
                                               pack_bf16x2(__fmul_rn(wj, g[6]), __fmul_rn(wj, g[7])));
                    st_stream(gy + (size_t)rows[j] * row_bytes + (size_t)c * 16, o);
                    float d = dot[j];
                    d = __fmaf_rn(g[0], bf16_lo(v[jj].x), d);
                    d = __fmaf_rn(g[1], bf16_hi(v[jj].x), d);
                    d = __fmaf_rn(g[2], bf16_lo(v[jj].y), d);
                    d = __fmaf_rn(g[3], bf16_hi(v[jj].y), d);
                    d = __fmaf_rn(g[4], bf16_lo(v[jj].z), d);
                    d = __fmaf_rn(g[5], bf16_hi(v[jj].z), d);
                    d = __fmaf_rn(g[6], bf16_lo(v[jj].w), d);
                    d = __fmaf_rn(g[7], bf16_hi(v[jj].w), d);
                    dot[j] = d;
                }
            }
        }

        // Per-token reduction of the k partial dot products, in a fixed order.
#pragma unroll
        for (int j = 0; j < 8 * G; ++j) {
            float d = dot[j];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            if (lane == 0) red[warp][j] = d;
        }
        __syncthreads();
        if (tid < k) {
            float s = 0.0f;
            for (int wi = 0; wi < nwarps; ++wi) s += red[wi][tid];
            const int row = a.slot_map[(size_t)t * k + tid];
            a.grad_weights[(size_t)t * k + tid] = (row >= 0 && row < a.max_rows) ? s : 0.0f;
        }
        __syncthreads();
    }
    pdl_launch_dependents();
}

int unit_threads(int ipr) {
    // the whole row per CTA: up to 256 threads, a multiple of 32
    return ipr >= kMaxThreads ? kMaxThreads : ((ipr + 31) / 32) * 32;
}

template <int G>
cudaError_t launch_t(const CombineBackwardArgs& a, cudaStream_t stream) {
    const int ipr = a.H / 8;
    const int bd = unit_threads(ipr);
    int per_sm = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, combine_backward_kernel<G>, bd, 0);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) per_sm = 1;
    const int64_t cap = (int64_t)device_sm_count() * per_sm;
    const int64_t want = (int64_t)a.T + a.max_pad_rows;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(want < 1 ? 1 : (want < cap ? want : cap)));
    cfg.blockDim = dim3(bd);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    debug_launch("combine_backward_kernel", G, cfg);
    return cudaLaunchKernelEx(&cfg, combine_backward_kernel<G>, a, ipr);
}

}  // namespace

cudaError_t launch_combine_backward(const CombineBackwardArgs& a, cudaStream_t stream) {
    switch ((a.k + 7) / 8) {
        case 1: return launch_t<1>(a, stream);
        case 2: return launch_t<2>(a, stream);
        case 3: return launch_t<3>(a, stream);
        case 4: return launch_t<4>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ep
