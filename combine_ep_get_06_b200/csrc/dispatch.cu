// MoE dispatch on one device (DeepEP V2 README, "Interfaces and examples",
// dispatch_forward; FP8 dispatching as in its section "Performance").
//
// Token-major: each token row is read from HBM once and, in the FP8 mode,
// quantised once, into a shared-memory row buffer; the TMA engine then
// copies that buffer to each of the token's k receive rows with bulk
// shared->global copies (cp.async.bulk, never multicast), so the SMs issue
// a handful of copy instructions per row instead of k stores per 16 bytes.
// Two row buffers alternate, so quantising row i+1 overlaps the copies of
// row i.  Padding rows are written by bulk copies of a zeroed buffer, one
// row per lane of warp 0.  Launched with programmatic dependent launch: a
// CTA waits for the previous grid before reading anything, and lets the
// next grid start launching once it has issued all its copies.
//
// A CTA walks rows grid-stride: token rows [0, T), then padding batches of
// 32 rows.  In the quantising mode a 1x128 block is 8 consecutive lanes
// (16 bf16 values each): its amax is a 3-step xor shuffle, and lane 0 of
// the group stores the block's scale.
#include "ep_device.cuh"
#include "ep_internal.h"

namespace ep {
namespace {

constexpr int kThreads = 256;
constexpr float kE4m3Max = 448.0f;
constexpr float kAmaxFloor = 1e-4f;

struct Geometry {
    int row_bytes;     // bytes of one receive row
    int ipr;           // 16-byte items per receive row
    int scale_bytes;   // bytes of one row of scales (0 in bf16 mode)
    int scale_pad;     // scale_bytes rounded up to 16
};

__host__ __device__ inline Geometry geometry(int mode, int H) {
    Geometry g;
    const bool fp8 = mode != EP_X_BF16;
    g.row_bytes = fp8 ? H : 2 * H;
    g.ipr = g.row_bytes / 16;
    g.scale_bytes = fp8 ? (H / 128) * 4 : 0;
    g.scale_pad = (g.scale_bytes + 15) & ~15;
    return g;
}

// smem: [2][row_bytes] row buffers | [2][scale_pad] scale buffers |
//       [row_bytes] zeros | [scale_pad] zeros | [2][kMaxTopk] int rows
__host__ __device__ inline size_t smem_bytes(const Geometry& g) {
    return (size_t)3 * g.row_bytes + (size_t)3 * g.scale_pad + 2 * kMaxTopk * sizeof(int);
}

template <int kMode>
__global__ void __launch_bounds__(kThreads) dispatch_kernel(DispatchArgs a) {
    constexpr bool kFp8Out = kMode != EP_X_BF16;
    extern __shared__ __align__(128) unsigned char smem[];
    const Geometry geo = geometry(kMode, a.H);
    unsigned char* rowbuf = smem;                                  // [2][row_bytes]
    unsigned char* sclbuf = smem + 2 * geo.row_bytes;              // [2][scale_pad]
    unsigned char* zeros = sclbuf + 2 * geo.scale_pad;             // [row_bytes + scale_pad]
    int* rows_s = (int*)(zeros + geo.row_bytes + geo.scale_pad);   // [2][kMaxTopk]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = a.T, k = a.k, H = a.H, B = H / 128;
    char* const recv = (char*)a.recv_x;
    char* const rscl = (char*)a.recv_scales;

    for (int i = tid; i < (geo.row_bytes + geo.scale_pad) / 16; i += kThreads)
        reinterpret_cast<uint4*>(zeros)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();

    // Everything below may read what the layout (the previous grid) wrote.
    pdl_wait();
    const int n_pad = ld_cg(a.num_pad_rows);
    const int n_pad_batches = (n_pad + 31) / 32;
    __syncthreads();

    int it = 0;  // token rows handled by this CTA (selects the buffer)
    for (int r = blockIdx.x; r < T + n_pad_batches; r += gridDim.x) {
        if (r >= T) {
            // 32 padding rows: one bulk copy of zeros per row (lanes of warp 0).
            const int p = (r - T) * 32 + lane;
            if (warp == 0 && p < n_pad) {
                const int row = ld_cg(a.pad_rows + p);
                if (row >= 0 && row < a.max_rows) {
                    bulk_s2g(recv + (size_t)row * geo.row_bytes, zeros, geo.row_bytes);
                    if (a.bulk_scales)
                        bulk_s2g(rscl + (size_t)row * geo.scale_bytes, zeros + geo.row_bytes, geo.scale_bytes);
                    bulk_commit();
                }
                if (kFp8Out && !a.bulk_scales && row >= 0 && row < a.max_rows)
                    for (int b = 0; b < B; ++b) a.recv_scales[(size_t)row * B + b] = 0.0f;
            }
            continue;
        }

        const int t = r;
        const int buf = it & 1;
        ++it;
        unsigned char* rb = rowbuf + buf * geo.row_bytes;
        float* sb = reinterpret_cast<float*>(sclbuf + buf * geo.scale_pad);
        int* rows = rows_s + buf * kMaxTopk;

        // The copies issued two rows ago from this buffer must have read it.
        if (warp == 0) bulk_wait_read<1>();
        __syncthreads();

        if (tid < k) rows[tid] = ld_cg(a.slot_map + (size_t)t * k + tid);

        // Fill the row buffer: warp-uniform loop over 32-item slices.
        for (int c0 = warp * 32; c0 < geo.ipr; c0 += kThreads) {
            const int c = c0 + lane;
            const bool active = c < geo.ipr;
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
                reinterpret_cast<uint4*>(rb)[c] = ld_stream((const char*)a.x + (size_t)t * geo.row_bytes + (size_t)c * 16);
                if (kMode == EP_X_FP8 && (c & 7) == 0) sb[c >> 3] = ld_cg(a.x_scales + (size_t)t * B + (c >> 3));
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        if (warp == 0 && lane < k) {
            const int row = rows[lane];
            if (row >= 0 && row < a.max_rows) {
                bulk_s2g(recv + (size_t)row * geo.row_bytes, rb, geo.row_bytes);
                if (a.bulk_scales) bulk_s2g(rscl + (size_t)row * geo.scale_bytes, sb, geo.scale_bytes);
            } else if (row >= a.max_rows) {
                atomicOr(a.error_word, EP_DEVERR_CAPACITY);
            }
            bulk_commit();
        }
        if (kFp8Out && !a.bulk_scales) {
            // Scale rows not a multiple of 16 bytes: plain stores.
            for (int i = tid; i < k * B; i += kThreads) {
                const int row = rows[i / B];
                if (row >= 0 && row < a.max_rows) a.recv_scales[(size_t)row * B + i % B] = sb[i % B];
            }
        }
    }
    // Let the next grid start launching while the copies drain.
    pdl_launch_dependents();
    if (warp == 0) bulk_wait_all();
}

template <int kMode>
cudaError_t launch_t(const DispatchArgs& a, cudaStream_t stream) {
    const Geometry g = geometry(kMode, a.H);
    const size_t smem = smem_bytes(g);
    auto kernel = dispatch_kernel<kMode>;
    cudaError_t err;
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    // Persistent grid, no larger than the work: the number of padding rows
    // is only known on the device, E*(alignment-1) bounds it.
    const int64_t cap = (int64_t)device_sm_count() * per_sm;
    const int64_t want = (int64_t)a.T + ((int64_t)a.max_pad_rows + 31) / 32;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(want < 1 ? 1 : (want < cap ? want : cap)));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, a);
}

}  // namespace

size_t dispatch_smem_bytes(ep_x_mode mode, int H) { return smem_bytes(geometry(mode, H)); }

cudaError_t launch_dispatch(const DispatchArgs& a, ep_x_mode mode, cudaStream_t stream) {
    switch (mode) {
        case EP_X_BF16: return launch_t<EP_X_BF16>(a, stream);
        case EP_X_FP8: return launch_t<EP_X_FP8>(a, stream);
        case EP_X_BF16_TO_FP8: return launch_t<EP_X_BF16_TO_FP8>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ep
