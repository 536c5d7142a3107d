// Fused layout + dispatch for small batches (T*k <= 1024 slots, e.g. the
// decode step): the dispatch(x, topk_idx, topk_weights, ...) call of the
// DeepEP V2 README ("Interfaces and examples") in one launch.
//
// Every CTA (1024 threads, one per slot) computes the whole small layout in
// shared memory -- the same steps as the single-CTA layout kernel -- so no
// CTA waits for another.  CTA c then owns the tokens t = c, c+G, ...: it
// writes their slot-map entries and per-row arrays, quantises or copies
// their x rows into a shared row buffer and bulk-copies (TMA, no multicast)
// that buffer to the k receive rows; it also writes its share of the
// padding rows.  Each CTA loads and quantises the x row of its first token
// before the layout, so that work overlaps the layout's latency.
#include "dispatch_device.cuh"
#include "layout_device.cuh"

namespace ep {
namespace {

using namespace layout_dev;
using dispatch_dev::Item;
using dispatch_dev::fill_item;
using dispatch_dev::load_item;

struct FusedGeometry {
    int row_bytes, ipr, scale_bytes, scale_pad;
    size_t layout_off, row_off, scale_off, zero_off, srow_off, total;
};

__host__ __device__ inline FusedGeometry fused_geometry(int mode, int H, int E, int S) {
    FusedGeometry g;
    const bool fp8 = mode != EP_X_BF16;
    g.row_bytes = fp8 ? H : 2 * H;
    g.ipr = g.row_bytes / 16;
    g.scale_bytes = fp8 ? (H / 128) * 4 : 0;
    g.scale_pad = (g.scale_bytes + 15) & ~15;
    g.layout_off = 0;
    g.row_off = (layout_dev::smem_bytes(E, S) + 127) & ~(size_t)127;
    g.scale_off = g.row_off + g.row_bytes;
    g.zero_off = g.scale_off + g.scale_pad;
    g.srow_off = g.zero_off + g.row_bytes + g.scale_pad;
    g.total = g.srow_off + sizeof(int) * kThreads;
    return g;
}

template <typename IdxT, int kMode>
__global__ void __launch_bounds__(kThreads) layout_dispatch_kernel(LayoutArgs a, DispatchArgs d) {
    constexpr bool kFp8Out = kMode != EP_X_BF16;
    extern __shared__ __align__(128) unsigned char smem[];
    const int E = a.h.num_experts, S = a.h.num_segments, k = a.h.num_topk, T = a.h.num_tokens;
    const FusedGeometry geo = fused_geometry(kMode, d.H, E, S);
    Smem m(reinterpret_cast<int*>(smem + geo.layout_off), E, S);
    unsigned char* rb = smem + geo.row_off;
    float* sb = reinterpret_cast<float*>(smem + geo.scale_off);
    unsigned char* zeros = smem + geo.zero_off;
    int* srow = reinterpret_cast<int*>(smem + geo.srow_off);  // [kThreads] row of each slot

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c_cta = blockIdx.x, G = gridDim.x;
    const int64_t s = tid;
    const bool has_slot = s < (int64_t)T * k;
    char* const recv = (char*)d.recv_x;
    char* const rscl = (char*)d.recv_scales;

    // Launched with programmatic dependent launch: wait for the previous
    // grid before touching global memory.  Then the loads: this thread's
    // slot, and its item of the first token row.
    pdl_wait();
    bool bad = false;
    int e = -1;
    float wv = 0.0f;
    if (has_slot) {
        e = read_expert((const IdxT*)a.topk_idx, s, E, bad);
        if (a.topk_weights) wv = __ldg(a.topk_weights + s);
    }
    const Item pre = load_item<kMode>(d, c_cta, tid, c_cta < T && tid < geo.ipr);
    for (int i = tid; i < (geo.row_bytes + geo.scale_pad) / 16; i += kThreads)
        reinterpret_cast<uint4*>(zeros)[i] = make_uint4(0, 0, 0, 0);
    // The first token row needs no routing: quantise (or copy) it into the
    // row buffer now, so that work overlaps the layout below.
    if (c_cta < T) {
        for (int c0 = warp * 32; c0 < geo.ipr; c0 += kThreads) {
            const int c = c0 + lane;
            const bool active = c < geo.ipr;
            const Item it = c0 == warp * 32 ? pre : load_item<kMode>(d, c_cta, c, active);
            fill_item<kMode>(d, c_cta, c, active, it, rb, sb);
        }
    }
    fence_proxy_async_smem();

    const int row_s = small_layout<IdxT>(a, m, e, bad, wv);
    srow[tid] = row_s;
    {   // this CTA's share of the slot map, the per-row arrays and the padding rows
        const int64_t n = (int64_t)T * k;
        if (has_slot && s >= n * c_cta / G && s < n * (c_cta + 1) / G) a.h.slot_map[s] = row_s;
        const int V = m.lcoff[E];
        write_rows(a, m, (int)((int64_t)V * c_cta / G), (int)((int64_t)V * (c_cta + 1) / G));
    }
    if (c_cta == 0) write_totals(a, m, E, S);
    const int P = m.padoff[E];
    const int p0 = (int)((int64_t)P * c_cta / G), p1 = (int)((int64_t)P * (c_cta + 1) / G);
    write_padding(a, m, E, p0, p1);
    __syncthreads();

    // Padding rows of this CTA's share: bulk copies of zeros.
    if (warp == 0) {
        for (int p = p0 + lane; p < p1; p += 32) {
            const int row = pad_row(m, E, p);
            if (row >= a.h.max_recv_rows) continue;
            bulk_s2g(recv + (size_t)row * geo.row_bytes, zeros, geo.row_bytes);
            if (d.bulk_scales) bulk_s2g(rscl + (size_t)row * geo.scale_bytes, zeros + geo.row_bytes, geo.scale_bytes);
            bulk_commit();
            if (kFp8Out && !d.bulk_scales)
                for (int b = 0; b < d.H / 128; ++b) d.recv_scales[(size_t)row * (d.H / 128) + b] = 0.0f;
        }
    }

    for (int t = c_cta; t < T; t += G) {
        if (t != c_cta) {   // the first row is already in the buffer
            if (warp == 0) bulk_wait_read<0>();
            __syncthreads();
            for (int c0 = warp * 32; c0 < geo.ipr; c0 += kThreads) {
                const int c = c0 + lane;
                const bool active = c < geo.ipr;
                fill_item<kMode>(d, t, c, active, load_item<kMode>(d, t, c, active), rb, sb);
            }
            fence_proxy_async_smem();
            __syncthreads();
        }
        if (warp == 0 && lane < k) {
            const int row = srow[t * k + lane];
            if (row >= 0) {
                bulk_s2g(recv + (size_t)row * geo.row_bytes, rb, geo.row_bytes);
                if (d.bulk_scales) bulk_s2g(rscl + (size_t)row * geo.scale_bytes, sb, geo.scale_bytes);
            }
            bulk_commit();
        }
        if (kFp8Out && !d.bulk_scales) {
            const int B = d.H / 128;
            for (int i = tid; i < k * B; i += kThreads) {
                const int row = srow[t * k + i / B];
                if (row >= 0) d.recv_scales[(size_t)row * B + i % B] = sb[i % B];
            }
        }
    }
    pdl_launch_dependents();
    if (warp == 0) bulk_wait_all();
}

template <typename IdxT, int kMode>
cudaError_t launch_t(const LayoutArgs& a, const DispatchArgs& d, cudaStream_t stream) {
    const FusedGeometry g = fused_geometry(kMode, d.H, a.h.num_experts, a.h.num_segments);
    auto kernel = layout_dispatch_kernel<IdxT, kMode>;
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)g.total);
    if (err != cudaSuccess) return err;
    int grid = a.h.num_tokens < device_sm_count() ? a.h.num_tokens : device_sm_count();
    if (grid < 1) grid = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = g.total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, a, d);
}

template <typename IdxT>
cudaError_t launch_mode(const LayoutArgs& a, const DispatchArgs& d, ep_x_mode mode, cudaStream_t stream) {
    switch (mode) {
        case EP_X_BF16: return launch_t<IdxT, EP_X_BF16>(a, d, stream);
        case EP_X_FP8: return launch_t<IdxT, EP_X_FP8>(a, d, stream);
        case EP_X_BF16_TO_FP8: return launch_t<IdxT, EP_X_BF16_TO_FP8>(a, d, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

size_t layout_dispatch_smem_bytes(ep_x_mode mode, int H, int E, int S) {
    return fused_geometry(mode, H, E, S).total;
}

cudaError_t launch_layout_dispatch(const LayoutArgs& a, const DispatchArgs& d, ep_x_mode mode, bool idx_is_int64,
                                   cudaStream_t stream) {
    return idx_is_int64 ? launch_mode<long long>(a, d, mode, stream) : launch_mode<int>(a, d, mode, stream);
}

}  // namespace ep
