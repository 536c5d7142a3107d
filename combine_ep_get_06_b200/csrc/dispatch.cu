// MoE dispatch on one device (DeepEP V2 README, "Interfaces and examples",
// dispatch_forward; FP8 dispatching as in its section "Performance").
//
// Token-major: each token row is read from HBM once and, in the FP8 mode,
// quantised once, into a shared-memory row buffer; the TMA engine then
// copies that buffer to each of the token's k receive rows with bulk
// shared->global copies (cp.async.bulk, never multicast), so the SMs issue
// a handful of copy instructions per row instead of k stores per 16 bytes.
// Two row buffers alternate, so filling row i+1 overlaps the copies of row
// i, and the loads of a CTA's next row are issued as soon as the current
// row is in shared memory, so they are in flight across the barrier and
// the copy issue.  Padding rows are written by bulk copies of a zeroed
// buffer, one row per lane of warp 0.
//
// A CTA walks rows grid-stride: token rows [0, T), then padding batches of
// 32 rows.  Launched with programmatic dependent launch: a CTA waits for
// the previous grid before reading what it may have written (directly after
// the layout, only the routing), and lets the next grid start launching
// once it has issued all its copies.
#include "dispatch_device.cuh"

namespace ep {
namespace {

using namespace dispatch_dev;

constexpr int kThreads = 256;
constexpr int kPre = 2;  // 32-item slices per warp whose loads are prefetched
constexpr int kBuf = 2;  // row buffers: a buffer is refilled once the copies from kBuf rows ago have read it

// smem: [kBuf][row_bytes] row buffers | [kBuf][scale_pad] scale buffers |
//       [row_bytes] zeros | [scale_pad] zeros | [kBuf][kMaxTopk] int rows
__host__ __device__ inline size_t smem_bytes(const Geometry& g) {
    return (size_t)(kBuf + 1) * g.row_bytes + (size_t)(kBuf + 1) * g.scale_pad + kBuf * kMaxTopk * sizeof(int);
}

// Stores the scale of block b of receive row `row` (f32 row- or MN-major,
// or an e4m3 byte for NVFP4), taken from the row's scale buffer sb.
// MN-major scales are stored with an L2 evict-last policy: each token's
// scales land in B different columns, 4 bytes per 32-byte sector, and the
// whole array fits in L2, so its sectors fill up there before write-back
// (measured: 158 -> 134 us at the V3 shape).  A hint on the row copies
// measured slower and is not used.
template <int kMode>
__device__ __forceinline__ void store_scale(const DispatchArgs& a, int row, int b, const float* sb, bool zero,
                                            uint64_t keep) {
    if (kMode == EP_X_BF16_TO_NVFP4) {
        reinterpret_cast<unsigned char*>(a.recv_scales)[(size_t)row * (a.H / 16) + b] =
            zero ? 0 : reinterpret_cast<const unsigned char*>(sb)[b];
    } else if (a.scales_ld > 0) {
        st_f32_hint(reinterpret_cast<float*>(a.recv_scales) + (size_t)b * a.scales_ld + row, zero ? 0.0f : sb[b],
                    keep);
    } else {
        reinterpret_cast<float*>(a.recv_scales)[(size_t)row * (a.H / 128) + b] = zero ? 0.0f : sb[b];
    }
}


template <int kMode>
__device__ __forceinline__ void prefetch(const DispatchArgs& a, int t, int ipr, Item (&p)[kPre]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < kPre; ++i) {
        const int c = warp * 32 + i * kThreads + lane;
        p[i] = load_item<kMode>(a, t, c, t < a.T && c < ipr);
    }
}

template <int kMode>
__global__ void __launch_bounds__(kThreads) dispatch_kernel(DispatchArgs a) {
    constexpr bool kFp8Out = kMode != EP_X_BF16;
    extern __shared__ __align__(128) unsigned char smem[];
    const Geometry geo = geometry(kMode, a.H);
    unsigned char* rowbuf = smem;                                  // [kBuf][row_bytes]
    unsigned char* sclbuf = smem + kBuf * geo.row_bytes;           // [kBuf][scale_pad]
    unsigned char* zeros = sclbuf + kBuf * geo.scale_pad;          // [row_bytes + scale_pad]
    int* rows_s = (int*)(zeros + geo.row_bytes + geo.scale_pad);   // [kBuf][kMaxTopk]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = a.T, k = a.k;
    const int B = kMode == EP_X_BF16_TO_NVFP4 ? a.H / 16 : a.H / 128;  // scales per row
    char* const recv = (char*)a.recv_x;
    char* const rscl = (char*)a.recv_scales;

    for (int i = tid; i < (geo.row_bytes + geo.scale_pad) / 16; i += kThreads)
        reinterpret_cast<uint4*>(zeros)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    const uint64_t keep = a.scales_ld > 0 ? l2_evict_last_policy() : 0;

    // Right after the layout x is already complete (every layout kernel waits
    // for the grid before it before letting this one launch), so the first
    // row's loads can fly while the layout finishes.  Everything the layout
    // writes is read only after the wait.
    Item next[kPre];
    if (a.x_ready) prefetch<kMode>(a, blockIdx.x, geo.ipr, next);
    pdl_wait();
    if (!a.x_ready) prefetch<kMode>(a, blockIdx.x, geo.ipr, next);
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
                    if (kFp8Out && !a.bulk_scales)
                        for (int b = 0; b < B; ++b) store_scale<kMode>(a, row, b, nullptr, true, keep);
                }
            }
            continue;
        }

        const int t = r;
        const int buf = it % kBuf;
        ++it;
        unsigned char* rb = rowbuf + buf * geo.row_bytes;
        float* sb = reinterpret_cast<float*>(sclbuf + buf * geo.scale_pad);
        int* rows = rows_s + buf * kMaxTopk;

        // The copies issued kBuf rows ago from this buffer must have read it
        // (each lane below k commits one bulk group per token row).
        if (warp == 0) bulk_wait_read<kBuf - 1>();
        __syncthreads();

        if (tid < k) rows[tid] = ld_cg(a.slot_map + (size_t)t * k + tid);

        // Fill the row buffer: the prefetched slices, then any further ones.
#pragma unroll
        for (int i = 0; i < kPre; ++i) {
            const int c0 = warp * 32 + i * kThreads;
            if (c0 < geo.ipr) fill_item<kMode>(a, t, c0 + lane, c0 + lane < geo.ipr, next[i], rb, sb);
        }
        for (int c0 = warp * 32 + kPre * kThreads; c0 < geo.ipr; c0 += kThreads) {
            const int c = c0 + lane;
            fill_item<kMode>(a, t, c, c < geo.ipr, load_item<kMode>(a, t, c, c < geo.ipr), rb, sb);
        }
        // This CTA's next token row: its loads fly across the barrier and copy issue.
        prefetch<kMode>(a, r + gridDim.x, geo.ipr, next);
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
            // MN-major scales, or rows not a multiple of 16 bytes: plain stores.
            for (int i = tid; i < k * B; i += kThreads) {
                const int row = rows[i / B];
                if (row >= 0 && row < a.max_rows) store_scale<kMode>(a, row, i % B, sb, false, keep);
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
        case EP_X_BF16_TO_NVFP4: return launch_t<EP_X_BF16_TO_NVFP4>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ep
