// C-ABI front end: argument checks on the host, then kernel launches on
// the caller's stream.  Allocates nothing; synchronises only in
// ep_read_total_rows and ep_check_error.
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <string>

#include "ep_internal.h"

namespace {

thread_local std::string g_last_error;
thread_local int32_t g_num_sms = 0;  // SM budget of this host thread; 0 = none

ep_status invalid(const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return EP_ERR_INVALID_ARG;
}

ep_status cuda_failed(const char* what, cudaError_t err) {
    g_last_error = std::string(what) + ": " + cudaGetErrorString(err);
    return EP_ERR_CUDA;
}

ep_status ok() {
    g_last_error.clear();
    return EP_OK;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

size_t round256(size_t n) { return (n + 255) & ~(size_t)255; }

// Checks the routing shape; on success *need gets T*k + E*(a-1).
ep_status check_shape(int32_t T, int32_t k, int32_t E, int32_t S, int32_t a, int64_t* need) {
    if (T < 0) return invalid("num_tokens must be >= 0 (got %d)", T);
    if (k < 1 || k > ep::kMaxTopk) return invalid("num_topk must be in [1, %d] (got %d)", ep::kMaxTopk, k);
    if (E < 1 || E > ep::kMaxExperts)
        return invalid("num_experts must be in [1, %d] (got %d)", ep::kMaxExperts, E);
    if (S < 1 || E % S != 0)
        return invalid("num_segments must be >= 1 and divide num_experts (got %d for %d experts)", S, E);
    if (a < 1) return invalid("expert_alignment must be >= 1 (got %d)", a);
    int64_t n = (int64_t)T * k + (int64_t)E * (a - 1);
    if (n > INT32_MAX) return invalid("T*k + E*(alignment-1) = %lld exceeds int32", (long long)n);
    *need = n;
    return EP_OK;
}

struct BlockLayout {
    size_t counts, recv_counts, offsets, seg_tokens, slot_map, recv_src, pad_rows, num_pad_rows,
        error_word, total;
};

BlockLayout block_layout(int32_t T, int32_t k, int32_t E, int32_t S, int32_t a, int32_t max_rows) {
    BlockLayout b;
    size_t at = 0;
    auto take = [&](size_t n_int32) {
        size_t here = at;
        at += round256(n_int32 * sizeof(int32_t));
        return here;
    };
    b.counts = take(E);
    b.recv_counts = take(E);
    b.offsets = take((size_t)E + 1);
    b.seg_tokens = take(S);
    b.slot_map = take((size_t)T * k > 0 ? (size_t)T * k : 1);
    b.recv_src = take(max_rows > 0 ? (size_t)max_rows : 1);
    b.pad_rows = take((size_t)E * (a - 1) > 0 ? (size_t)E * (a - 1) : 1);
    b.num_pad_rows = take(1);
    b.error_word = take(1);
    b.total = at;
    return b;
}

ep_status check_handle(const ep_handle* h) {
    if (h == nullptr) return invalid("handle is NULL");
    int64_t need = 0;
    ep_status st = check_shape(h->num_tokens, h->num_topk, h->num_experts, h->num_segments,
                               h->expert_alignment, &need);
    if (st != EP_OK) return st;
    if (h->max_recv_rows < need) return invalid("handle max_recv_rows %d < required %lld", h->max_recv_rows, (long long)need);
    const void* ptrs[] = {h->counts,   h->recv_counts, h->offsets,      h->seg_tokens, h->slot_map,
                          h->recv_src, h->pad_rows,    h->num_pad_rows, h->error_word};
    for (const void* p : ptrs)
        if (p == nullptr || !aligned(p, 4)) return invalid("handle has a NULL or misaligned array; use ep_handle_init");
    return EP_OK;
}

}  // namespace

namespace ep {

ep_status fail(ep_status status, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return status;
}

int device_sm_count() {
    static std::atomic<int> cache[128];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) dev = 0;
    if (dev < 128) {
        int v = cache[dev].load(std::memory_order_relaxed);
        if (v > 0) return v;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 1;
    if (dev < 128) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

void debug_launch(const char* kernel, int variant, dim3 grid, dim3 block, size_t smem, cudaStream_t stream) {
    static const bool on = [] {
        const char* v = getenv("EP_DEBUG");
        return v != nullptr && v[0] != '\0' && v[0] != '0';
    }();
    if (!on) return;
    fprintf(stderr, "[ep] %s<%d>: grid %u x %u x %u, block %u, smem %zu B, stream %p, sm budget %d\n", kernel,
            variant, grid.x, grid.y, grid.z, block.x, smem, (void*)stream, sm_budget());
}

int sm_budget() {
    const int n = g_num_sms;
    if (n <= 0) return 0;
    const int sms = device_sm_count();
    return n < sms ? n : sms;
}

}  // namespace ep

extern "C" {

EP_API int32_t ep_abi_version(void) { return EP_ABI_VERSION; }

EP_API ep_status ep_set_num_sms(int32_t num_sms) {
    if (num_sms < 0) return invalid("num_sms must be >= 0 (got %d); 0 means every SM", num_sms);
    g_num_sms = num_sms;
    return ok();
}

EP_API int32_t ep_get_num_sms(void) { return g_num_sms; }

EP_API const char* ep_status_string(ep_status s) {
    switch (s) {
        case EP_OK: return "EP_OK";
        case EP_ERR_INVALID_ARG: return "EP_ERR_INVALID_ARG";
        case EP_ERR_DEVICE: return "EP_ERR_DEVICE";
        case EP_ERR_CUDA: return "EP_ERR_CUDA";
    }
    return "EP_UNKNOWN_STATUS";
}

EP_API const char* ep_last_error(void) { return g_last_error.c_str(); }

EP_API int32_t ep_max_recv_rows(int32_t T, int32_t k, int32_t E, int32_t a) {
    if (T < 0 || k < 1 || E < 1 || a < 1) return -1;
    int64_t n = (int64_t)T * k + (int64_t)E * (a - 1);
    return n > INT32_MAX ? -1 : (int32_t)n;
}

EP_API size_t ep_handle_bytes(int32_t T, int32_t k, int32_t E, int32_t S, int32_t a, int32_t max_rows) {
    int64_t need = 0;
    if (check_shape(T, k, E, S, a, &need) != EP_OK || max_rows < need) return 0;
    return block_layout(T, k, E, S, a, max_rows).total;
}

EP_API ep_status ep_handle_init(ep_handle* h, int32_t T, int32_t k, int32_t E, int32_t S, int32_t a,
                                int32_t max_rows, void* block, size_t bytes) {
    if (h == nullptr) return invalid("handle is NULL");
    int64_t need = 0;
    ep_status st = check_shape(T, k, E, S, a, &need);
    if (st != EP_OK) return st;
    if (max_rows < need)
        return invalid("max_recv_rows %d < T*k + E*(alignment-1) = %lld", max_rows, (long long)need);
    BlockLayout b = block_layout(T, k, E, S, a, max_rows);
    if (block == nullptr || !aligned(block, 256)) return invalid("device_block must be non-NULL and 256-byte aligned");
    if (bytes < b.total) return invalid("device_block has %zu bytes, %zu needed", bytes, b.total);
    char* base = (char*)block;
    h->num_tokens = T;
    h->num_topk = k;
    h->num_experts = E;
    h->num_segments = S;
    h->expert_alignment = a;
    h->max_recv_rows = max_rows;
    h->counts = (int32_t*)(base + b.counts);
    h->recv_counts = (int32_t*)(base + b.recv_counts);
    h->offsets = (int32_t*)(base + b.offsets);
    h->seg_tokens = (int32_t*)(base + b.seg_tokens);
    h->slot_map = (int32_t*)(base + b.slot_map);
    h->recv_src = (int32_t*)(base + b.recv_src);
    h->pad_rows = (int32_t*)(base + b.pad_rows);
    h->num_pad_rows = (int32_t*)(base + b.num_pad_rows);
    h->error_word = (uint32_t*)(base + b.error_word);
    return ok();
}

EP_API size_t ep_layout_workspace_bytes(const ep_handle* h) {
    if (check_handle(h) != EP_OK) return 0;
    const size_t C = (size_t)ep::layout_num_chunks(h->num_tokens, h->num_topk);
    return round256(C * h->num_experts * sizeof(int32_t)) + round256(C * h->num_segments * sizeof(int32_t));
}

}  // extern "C"

namespace {

// Checks the layout arguments and fills a.
ep_status prepare_layout(ep_handle* h, const void* topk_idx, int32_t idx_is_int64, const float* topk_weights,
                         int32_t* recv_topk_idx, float* recv_topk_weights, void* workspace,
                         size_t workspace_bytes, ep::LayoutArgs* a) {
    ep_status st = check_handle(h);
    if (st != EP_OK) return st;
    if (idx_is_int64 != 0 && idx_is_int64 != 1) return invalid("idx_is_int64 must be 0 or 1");
    if (h->num_tokens > 0 && (topk_idx == nullptr || !aligned(topk_idx, idx_is_int64 ? 8 : 4)))
        return invalid("topk_idx is NULL or misaligned");
    if (topk_weights && !aligned(topk_weights, 4)) return invalid("topk_weights misaligned");
    if (recv_topk_idx && !aligned(recv_topk_idx, 4)) return invalid("recv_topk_idx misaligned");
    if (recv_topk_weights && !aligned(recv_topk_weights, 4)) return invalid("recv_topk_weights misaligned");
    const size_t need = ep_layout_workspace_bytes(h);
    if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need)
        return invalid("workspace must be 256-byte aligned with >= %zu bytes (got %zu)", need, workspace_bytes);
    a->topk_idx = topk_idx;
    a->topk_weights = topk_weights;
    a->recv_topk_idx = recv_topk_idx;
    a->recv_topk_weights = recv_topk_weights;
    a->h = *h;
    a->chunk_tokens = ep::layout_chunk_tokens(h->num_topk);
    a->num_chunks = ep::layout_num_chunks(h->num_tokens, h->num_topk);
    a->ws_hist = (int32_t*)workspace;
    a->ws_seg = (int32_t*)((char*)workspace + round256((size_t)a->num_chunks * h->num_experts * sizeof(int32_t)));
    return EP_OK;
}

// Checks the dispatch arguments and fills a.
ep_status prepare_dispatch(const ep_handle* h, ep_x_mode mode, const void* x, const float* x_scales, int32_t H,
                           void* recv_x, void* recv_scales, ep::DispatchArgs* a) {
    ep_status st = check_handle(h);
    if (st != EP_OK) return st;
    if (mode != EP_X_BF16 && mode != EP_X_FP8 && mode != EP_X_BF16_TO_FP8 && mode != EP_X_BF16_TO_NVFP4)
        return invalid("unknown x mode %d", (int)mode);
    const bool nvfp4 = mode == EP_X_BF16_TO_NVFP4;
    const bool fp8 = mode == EP_X_FP8 || mode == EP_X_BF16_TO_FP8;
    const int hmul = nvfp4 ? 32 : fp8 ? 128 : 8;
    if (H < 1 || H % hmul != 0)
        return invalid("hidden %d must be a positive multiple of %d in this mode", H, hmul);
    if (h->num_tokens > 0 && (x == nullptr || !aligned(x, 16))) return invalid("x must be non-NULL and 16-byte aligned");
    if (recv_x == nullptr || !aligned(recv_x, 16)) return invalid("recv_x must be non-NULL and 16-byte aligned");
    if (fp8 && (recv_scales == nullptr || !aligned(recv_scales, 4)))
        return invalid("recv_scales must be non-NULL and 4-byte aligned in the FP8 modes");
    if (nvfp4 && recv_scales == nullptr) return invalid("recv_scales must be non-NULL in the NVFP4 mode");
    if (mode == EP_X_FP8 && h->num_tokens > 0 && (x_scales == nullptr || !aligned(x_scales, 4)))
        return invalid("x_scales must be non-NULL and 4-byte aligned for pre-quantised x");
    if (ep::dispatch_smem_bytes(mode, H) > ep::kMaxDispatchSmem)
        return invalid("hidden %d: the dispatch stages exceed shared memory", H);
    a->x = x;
    a->x_scales = x_scales;
    a->recv_x = recv_x;
    a->recv_scales = recv_scales;
    a->slot_map = h->slot_map;
    a->pad_rows = h->pad_rows;
    a->num_pad_rows = h->num_pad_rows;
    a->error_word = h->error_word;
    a->T = h->num_tokens;
    a->k = h->num_topk;
    a->H = H;
    a->max_rows = h->max_recv_rows;
    a->max_pad_rows = h->num_experts * (h->expert_alignment - 1);
    a->bulk_scales = (fp8 && ((H / 128) * 4) % 16 == 0 && aligned(recv_scales, 16)) ||
                     (nvfp4 && (H / 16) % 16 == 0 && aligned(recv_scales, 16));
    a->x_ready = 0;
    a->scales_ld = 0;
    return EP_OK;
}

}  // namespace

extern "C" {

EP_API ep_status ep_get_layout(ep_handle* h, const void* topk_idx, int32_t idx_is_int64,
                               const float* topk_weights, int32_t* recv_topk_idx,
                               float* recv_topk_weights, void* workspace, size_t workspace_bytes,
                               ep_stream_t stream) {
    ep::LayoutArgs a;
    ep_status st = prepare_layout(h, topk_idx, idx_is_int64, topk_weights, recv_topk_idx, recv_topk_weights,
                                  workspace, workspace_bytes, &a);
    if (st != EP_OK) return st;
    cudaError_t err = ep::launch_layout(a, idx_is_int64 == 1, (cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("layout launch", err);
    return ok();
}

EP_API ep_status ep_dispatch(const ep_handle* h, ep_x_mode mode, const void* x, const float* x_scales,
                             int32_t H, void* recv_x, void* recv_scales, ep_stream_t stream) {
    ep::DispatchArgs a;
    ep_status st = prepare_dispatch(h, mode, x, x_scales, H, recv_x, recv_scales, &a);
    if (st != EP_OK) return st;
    cudaError_t err = ep::launch_dispatch(a, mode, (cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("dispatch launch", err);
    return ok();
}

EP_API ep_status ep_dispatch_mn_scales(const ep_handle* h, ep_x_mode mode, const void* x, const float* x_scales,
                                       int32_t H, void* recv_x, float* recv_scales_mn, int32_t scales_ld,
                                       ep_stream_t stream) {
    ep::DispatchArgs a;
    ep_status st = prepare_dispatch(h, mode, x, x_scales, H, recv_x, recv_scales_mn, &a);
    if (st != EP_OK) return st;
    if (mode != EP_X_FP8 && mode != EP_X_BF16_TO_FP8) return invalid("MN-major scales need an FP8 mode");
    if (scales_ld < h->max_recv_rows || scales_ld % 4 != 0)
        return invalid("scales_ld %d must be >= max_recv_rows (%d) and a multiple of 4", scales_ld,
                       h->max_recv_rows);
    if (!aligned(recv_scales_mn, 16)) return invalid("recv_scales_mn must be 16-byte aligned");
    a.scales_ld = scales_ld;
    a.bulk_scales = 0;
    cudaError_t err = ep::launch_dispatch(a, mode, (cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("dispatch launch", err);
    return ok();
}

EP_API ep_status ep_layout_dispatch(ep_handle* h, const void* topk_idx, int32_t idx_is_int64,
                                    const float* topk_weights, int32_t* recv_topk_idx,
                                    float* recv_topk_weights, void* workspace, size_t workspace_bytes,
                                    ep_x_mode mode, const void* x, const float* x_scales, int32_t H,
                                    void* recv_x, void* recv_scales, ep_stream_t stream) {
    ep::LayoutArgs la;
    ep::DispatchArgs da;
    ep_status st = prepare_layout(h, topk_idx, idx_is_int64, topk_weights, recv_topk_idx, recv_topk_weights,
                                  workspace, workspace_bytes, &la);
    if (st != EP_OK) return st;
    st = prepare_dispatch(h, mode, x, x_scales, H, recv_x, recv_scales, &da);
    if (st != EP_OK) return st;
    // One layout chunk (e.g. decode): one grid, each CTA computing the layout
    // it needs.  Otherwise the dispatch launches while the layout runs and
    // loads its x rows before waiting for it (x_ready); only the routing is
    // read after the wait.
    cudaError_t err = ep::launch_layout_dispatch_fused(la, da, mode, idx_is_int64 == 1, (cudaStream_t)stream);
    if (err == cudaSuccess) return ok();
    if (err != cudaErrorNotSupported) return cuda_failed("layout + dispatch launch", err);
    da.x_ready = 1;
    err = ep::launch_layout(la, idx_is_int64 == 1, (cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("layout launch", err);
    err = ep::launch_dispatch(da, mode, (cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("dispatch launch", err);
    return ok();
}

EP_API ep_status ep_combine(const ep_handle* h, const void* y, int32_t H, const float* topk_weights,
                            const float* recv_weights_in, float* out_weights, void* out, ep_stream_t stream) {
    ep_status st = check_handle(h);
    if (st != EP_OK) return st;
    if (H < 1 || H % 8 != 0) return invalid("hidden %d must be a positive multiple of 8", H);
    if (y == nullptr || !aligned(y, 16)) return invalid("y must be non-NULL and 16-byte aligned");
    if (h->num_tokens > 0 && (out == nullptr || !aligned(out, 16))) return invalid("out must be non-NULL and 16-byte aligned");
    if (topk_weights && !aligned(topk_weights, 4)) return invalid("topk_weights misaligned");
    if ((out_weights == nullptr) != (recv_weights_in == nullptr))
        return invalid("recv_weights_in and out_weights must be given together");
    if (out_weights && (!aligned(out_weights, 4) || !aligned(recv_weights_in, 4)))
        return invalid("out_weights / recv_weights_in misaligned");

    ep::CombineArgs a;
    a.y = y;
    a.topk_weights = topk_weights;
    a.recv_weights_in = recv_weights_in;
    a.out_weights = out_weights;
    a.out = out;
    a.slot_map = h->slot_map;
    a.error_word = h->error_word;
    a.T = h->num_tokens;
    a.k = h->num_topk;
    a.H = H;
    a.max_rows = h->max_recv_rows;
    if (a.T == 0) return ok();
    cudaError_t err = ep::launch_combine(a, (cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("combine launch", err);
    return ok();
}

EP_API ep_status ep_combine_fp8(const ep_handle* h, const void* y_q, const float* y_scales, int32_t H,
                                const float* topk_weights, void* out, ep_stream_t stream) {
    ep_status st = check_handle(h);
    if (st != EP_OK) return st;
    if (H < 1 || H % 128 != 0) return invalid("hidden %d must be a positive multiple of 128", H);
    if (y_q == nullptr || !aligned(y_q, 16)) return invalid("y_q must be non-NULL and 16-byte aligned");
    if (y_scales == nullptr || !aligned(y_scales, 4)) return invalid("y_scales must be non-NULL and 4-byte aligned");
    if (h->num_tokens > 0 && (out == nullptr || !aligned(out, 16))) return invalid("out must be non-NULL and 16-byte aligned");
    if (topk_weights && !aligned(topk_weights, 4)) return invalid("topk_weights misaligned");

    ep::CombineFp8Args a;
    a.y_q = y_q;
    a.y_scales = y_scales;
    a.topk_weights = topk_weights;
    a.out = out;
    a.slot_map = h->slot_map;
    a.error_word = h->error_word;
    a.T = h->num_tokens;
    a.k = h->num_topk;
    a.H = H;
    a.max_rows = h->max_recv_rows;
    if (a.T == 0) return ok();
    cudaError_t err = ep::launch_combine_fp8(a, (cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("combine_fp8 launch", err);
    return ok();
}

EP_API ep_status ep_combine_backward(const ep_handle* h, const void* grad_out, const void* y, int32_t H,
                                     const float* topk_weights, void* grad_y, float* grad_weights,
                                     ep_stream_t stream) {
    ep_status st = check_handle(h);
    if (st != EP_OK) return st;
    if (H < 1 || H % 8 != 0) return invalid("hidden %d must be a positive multiple of 8", H);
    if (h->num_tokens > 0 && (grad_out == nullptr || !aligned(grad_out, 16)))
        return invalid("grad_out must be non-NULL and 16-byte aligned");
    if (y == nullptr || !aligned(y, 16)) return invalid("y must be non-NULL and 16-byte aligned");
    if (grad_y == nullptr || !aligned(grad_y, 16)) return invalid("grad_y must be non-NULL and 16-byte aligned");
    if (h->num_tokens > 0 && (grad_weights == nullptr || !aligned(grad_weights, 4)))
        return invalid("grad_weights must be non-NULL and 4-byte aligned");
    if (topk_weights && !aligned(topk_weights, 4)) return invalid("topk_weights misaligned");
    ep::CombineBackwardArgs a;
    a.grad_out = grad_out;
    a.y = y;
    a.topk_weights = topk_weights;
    a.grad_y = grad_y;
    a.grad_weights = grad_weights;
    a.slot_map = h->slot_map;
    a.pad_rows = h->pad_rows;
    a.num_pad_rows = h->num_pad_rows;
    a.error_word = h->error_word;
    a.T = h->num_tokens;
    a.k = h->num_topk;
    a.H = H;
    a.max_rows = h->max_recv_rows;
    a.max_pad_rows = h->num_experts * (h->expert_alignment - 1);
    cudaError_t err = ep::launch_combine_backward(a, (cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("combine backward launch", err);
    return ok();
}

EP_API ep_status ep_read_total_rows(const ep_handle* h, int32_t* total_rows, ep_stream_t stream) {
    ep_status st = check_handle(h);
    if (st != EP_OK) return st;
    if (total_rows == nullptr) return invalid("total_rows is NULL");
    int32_t v = 0;
    cudaError_t err = cudaMemcpyAsync(&v, h->offsets + h->num_experts, sizeof v, cudaMemcpyDeviceToHost,
                                      (cudaStream_t)stream);
    if (err == cudaSuccess) err = cudaStreamSynchronize((cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("reading total rows", err);
    *total_rows = v;
    return ok();
}

EP_API ep_status ep_read_recv_counts(const ep_handle* h, int32_t* host_counts, ep_stream_t stream) {
    ep_status st = check_handle(h);
    if (st != EP_OK) return st;
    if (host_counts == nullptr) return invalid("host_counts is NULL");
    cudaError_t err = cudaMemcpyAsync(host_counts, h->recv_counts, sizeof(int32_t) * h->num_experts,
                                      cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (err == cudaSuccess) err = cudaStreamSynchronize((cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("reading the per-expert rows", err);
    return ok();
}

EP_API ep_status ep_check_error(const ep_handle* h, uint32_t* bits, ep_stream_t stream) {
    ep_status st = check_handle(h);
    if (st != EP_OK) return st;
    uint32_t v = 0;
    cudaError_t err = cudaMemcpyAsync(&v, h->error_word, sizeof v, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (err == cudaSuccess) err = cudaMemsetAsync(h->error_word, 0, sizeof v, (cudaStream_t)stream);
    if (err == cudaSuccess) err = cudaStreamSynchronize((cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("reading the error word", err);
    if (bits) *bits = v;
    if (v != 0) {
        char buf[48];
        snprintf(buf, sizeof buf, "device error word 0x%x:", v);
        g_last_error = buf;
        if (v & EP_DEVERR_BAD_TOPK_IDX) g_last_error += " topk_idx outside [-1, num_experts)";
        if (v & EP_DEVERR_CAPACITY) g_last_error += " receive row beyond max_recv_rows";
        if (v & EP_DEVERR_TIMEOUT) g_last_error += " bounded wait timed out";
        return EP_ERR_DEVICE;
    }
    return ok();
}

}  // extern "C"
