// C-ABI front end of the multi-GPU entry points (include/ep_multi.h):
// rank-block geometry, the block's allocation and CUDA IPC, host-side
// argument checks, launches.
#include <cuda_runtime.h>

#include <climits>
#include <cstring>

#include "ep_internal.h"

namespace {

constexpr int32_t kMaxExpertsPerRank = 1024;

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }
int64_t round256(int64_t n) { return (n + 255) & ~(int64_t)255; }

template <class... Args>
ep_status invalid(const char* fmt, Args... args) {
    return ep::fail(EP_ERR_INVALID_ARG, fmt, args...);
}

ep_status cuda_failed(const char* what, cudaError_t err) {
    return ep::fail(EP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(err));
}

ep_status ok() {
    ep::fail(EP_OK, "%s", "");
    return EP_OK;
}

// Received-row format of a mode: 0 bf16, 1 e4m3 + f32 scales, 3 NVFP4.
int format_of(int mode) { return mode == EP_X_BF16_TO_FP8 ? EP_X_FP8 : mode; }

int hidden_multiple(int mode) {
    switch (mode) {
        case EP_X_BF16: return 8;
        case EP_X_FP8:
        case EP_X_BF16_TO_FP8: return 128;
        case EP_X_BF16_TO_NVFP4: return 32;
    }
    return 0;
}

ep_status check_geometry(const ep_mgpu_geometry* g) {
    if (g == nullptr) return invalid("geometry is NULL");
    ep_mgpu_geometry ref;
    ep_status st = ep_mgpu_geometry_init(&ref, g->rank, g->world, g->max_tokens, g->num_topk, g->num_experts,
                                         g->expert_alignment, g->hidden, (ep_x_mode)g->x_mode);
    if (st != EP_OK) return st;
    if (std::memcmp(&ref, g, sizeof ref) != 0)
        return invalid("geometry was modified after ep_mgpu_geometry_init");
    return EP_OK;
}

ep_status check_local(const ep_mgpu_geometry* g, const ep_handle* h, void* local_block, void* const* peers) {
    ep_status st = check_geometry(g);
    if (st != EP_OK) return st;
    if (h == nullptr) return invalid("local handle is NULL");
    if (h->num_segments != g->world || h->expert_alignment != 1)
        return invalid("local handle needs num_segments = world (%d) and expert_alignment = 1", g->world);
    if (h->num_topk != g->num_topk || h->num_experts != g->num_experts)
        return invalid("local handle's num_topk / num_experts differ from the geometry's");
    if (h->num_tokens < 0 || h->num_tokens > g->max_tokens)
        return invalid("local handle has %d tokens, more than max_tokens %d", h->num_tokens, g->max_tokens);
    if (h->slot_map == nullptr || h->offsets == nullptr) return invalid("local handle has NULL arrays");
    if (local_block == nullptr || !aligned(local_block, 256))
        return invalid("local_block must be non-NULL and 256-byte aligned");
    if (peers == nullptr || !aligned(peers, 8)) return invalid("peer_blocks must be non-NULL and 8-byte aligned");
    return EP_OK;
}

ep::MgpuArgs make_args(const ep_mgpu_geometry* g, const ep_handle* h, void* local_block, void* const* peers) {
    ep::MgpuArgs a;
    std::memset(&a, 0, sizeof a);
    a.g = *g;
    a.src.H = g->hidden;
    a.src.T = h->num_tokens;
    a.src.k = g->num_topk;
    a.T = h->num_tokens;
    a.slot_map = h->slot_map;
    a.offsets = h->offsets;
    a.local_block = (char*)local_block;
    a.peer_blocks = (char* const*)peers;
    return a;
}

}  // namespace

extern "C" {

EP_API ep_status ep_mgpu_geometry_init(ep_mgpu_geometry* g, int32_t rank, int32_t world, int32_t max_tokens,
                                       int32_t k, int32_t E, int32_t a, int32_t H, ep_x_mode mode) {
    if (g == nullptr) return invalid("geometry is NULL");
    if (world < 1 || world > ep::kMaxWorld) return invalid("world must be in [1, %d] (got %d)", ep::kMaxWorld, world);
    if (rank < 0 || rank >= world) return invalid("rank %d outside [0, world %d)", rank, world);
    if (E < 1 || E > ep::kMaxExperts || E % world != 0)
        return invalid("num_experts must be in [1, %d] and divisible by world (got %d for world %d)",
                       ep::kMaxExperts, E, world);
    if (E / world > kMaxExpertsPerRank) return invalid("too many experts per rank (%d)", E / world);
    if (max_tokens < 0) return invalid("max_tokens must be >= 0 (got %d)", max_tokens);
    if (k < 1 || k > ep::kMaxTopk) return invalid("num_topk must be in [1, %d] (got %d)", ep::kMaxTopk, k);
    if (a < 1) return invalid("expert_alignment must be >= 1 (got %d)", a);
    const int hm = hidden_multiple(mode);
    if (hm == 0) return invalid("unknown x mode %d", (int)mode);
    if (H < 1 || H % hm != 0) return invalid("hidden %d must be a positive multiple of %d in this mode", H, hm);
    const int64_t rows = (int64_t)world * max_tokens * k + (int64_t)(E / world) * (a - 1);
    if (rows > INT32_MAX) return invalid("world*max_tokens*k + (E/world)*(alignment-1) = %lld exceeds int32", (long long)rows);

    std::memset(g, 0, sizeof *g);
    g->rank = rank;
    g->world = world;
    g->max_tokens = max_tokens;
    g->num_topk = k;
    g->num_experts = E;
    g->expert_alignment = a;
    g->hidden = H;
    g->x_mode = format_of(mode);
    g->experts_per_rank = E / world;
    g->max_recv_rows = (int32_t)rows;
    const int fmt = format_of(mode);
    g->row_bytes = fmt == EP_X_BF16 ? 2 * H : fmt == EP_X_FP8 ? H : H / 2;
    g->scale_bytes = fmt == EP_X_BF16 ? 0 : fmt == EP_X_FP8 ? (H / 128) * 4 : H / 16;
    if (ep::mgpu_dispatch_smem_bytes(*g) > ep::kMaxDispatchSmem)
        return invalid("hidden %d needs more shared memory than a CTA has", H);

    int64_t at = 0;
    auto take = [&](int64_t bytes) {
        const int64_t here = at;
        at += round256(bytes > 0 ? bytes : 1);
        return here;
    };
    const int64_t R = rows > 0 ? rows : 1;
    g->off_recv_x = take(R * g->row_bytes);
    g->off_recv_scales = take(R * g->scale_bytes);
    g->off_recv_src = take(R * 4);
    g->off_recv_topk_idx = take(R * 4);
    g->off_recv_topk_weights = take(R * 4);
    g->off_y = take(R * (int64_t)H * 2);
    g->off_all_counts = take((int64_t)world * E * 4);
    g->off_dest = take((int64_t)max_tokens * k * 8);
    g->off_raw_counts = take((int64_t)(E / world) * 4);
    g->off_recv_counts = take((int64_t)(E / world) * 4);
    g->off_recv_offsets = take((int64_t)(E / world + 1) * 4);
    g->off_num_pad_rows = take(4);
    g->off_error_word = take(4);
    g->block_bytes = at;
    return ok();
}

EP_API ep_status ep_mgpu_block_alloc(size_t bytes, void** block) {
    if (block == nullptr || bytes == 0) return invalid("block must be non-NULL and bytes > 0");
    *block = nullptr;
    cudaError_t err = cudaMalloc(block, bytes);
    if (err != cudaSuccess) return cuda_failed("cudaMalloc", err);
    return ok();
}

EP_API ep_status ep_mgpu_block_free(void* block) {
    if (block == nullptr) return ok();
    cudaError_t err = cudaFree(block);
    if (err != cudaSuccess) return cuda_failed("cudaFree", err);
    return ok();
}

EP_API ep_status ep_ipc_export(const void* block, void* handle_out) {
    static_assert(sizeof(cudaIpcMemHandle_t) == EP_IPC_HANDLE_BYTES, "IPC handle size");
    if (block == nullptr || handle_out == nullptr) return invalid("block and handle_out must be non-NULL");
    cudaIpcMemHandle_t h;
    cudaError_t err = cudaIpcGetMemHandle(&h, const_cast<void*>(block));
    if (err != cudaSuccess) return cuda_failed("cudaIpcGetMemHandle", err);
    std::memcpy(handle_out, &h, sizeof h);
    return ok();
}

EP_API ep_status ep_ipc_import(const void* handle, void** block) {
    if (handle == nullptr || block == nullptr) return invalid("handle and block must be non-NULL");
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof h);
    *block = nullptr;
    cudaError_t err = cudaIpcOpenMemHandle(block, h, cudaIpcMemLazyEnablePeerAccess);
    if (err != cudaSuccess) return cuda_failed("cudaIpcOpenMemHandle", err);
    return ok();
}

EP_API ep_status ep_ipc_close(void* block) {
    if (block == nullptr) return invalid("block is NULL");
    cudaError_t err = cudaIpcCloseMemHandle(block);
    if (err != cudaSuccess) return cuda_failed("cudaIpcCloseMemHandle", err);
    return ok();
}

EP_API ep_status ep_mgpu_dispatch(const ep_mgpu_geometry* g, const ep_handle* h, const void* topk_idx,
                                  int32_t idx_is_int64, const float* topk_weights, ep_x_mode mode, const void* x,
                                  const float* x_scales, void* local_block, void* const* peers,
                                  ep_stream_t stream) {
    ep_status st = check_local(g, h, local_block, peers);
    if (st != EP_OK) return st;
    if (hidden_multiple(mode) == 0) return invalid("unknown x mode %d", (int)mode);
    if (format_of(mode) != g->x_mode)
        return invalid("x mode %d does not store the geometry's receive format", (int)mode);
    const int T = h->num_tokens;
    if (T > 0) {
        if (topk_idx == nullptr || !aligned(topk_idx, idx_is_int64 ? 8 : 4))
            return invalid("topk_idx must be non-NULL and aligned");
        if (x == nullptr || !aligned(x, 16)) return invalid("x must be non-NULL and 16-byte aligned");
        if (mode == EP_X_FP8 && (x_scales == nullptr || !aligned(x_scales, 4)))
            return invalid("x_scales must be non-NULL in EP_X_FP8 mode");
        if (topk_weights != nullptr && !aligned(topk_weights, 4)) return invalid("topk_weights must be 4-byte aligned");
    }
    ep::MgpuArgs a = make_args(g, h, local_block, peers);
    a.src.x = x;
    a.src.x_scales = x_scales;
    a.topk_idx = topk_idx;
    a.idx_is_int64 = idx_is_int64 ? 1 : 0;
    a.topk_weights = topk_weights;
    cudaError_t err = ep::launch_mgpu_dispatch(a, mode, (cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("mgpu dispatch launch", err);
    return ok();
}

EP_API ep_status ep_mgpu_combine(const ep_mgpu_geometry* g, const ep_handle* h, const float* topk_weights,
                                 void* local_block, void* const* peers, void* out, ep_stream_t stream) {
    ep_status st = check_local(g, h, local_block, peers);
    if (st != EP_OK) return st;
    if (h->num_tokens > 0 && (out == nullptr || !aligned(out, 16)))
        return invalid("out must be non-NULL and 16-byte aligned");
    if (topk_weights != nullptr && !aligned(topk_weights, 4)) return invalid("topk_weights must be 4-byte aligned");
    if (h->num_tokens == 0) return ok();
    ep::MgpuArgs a = make_args(g, h, local_block, peers);
    a.topk_weights = topk_weights;
    a.out = out;
    cudaError_t err = ep::launch_mgpu_combine(a, (cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("mgpu combine launch", err);
    return ok();
}

EP_API ep_status ep_mgpu_read_total_rows(const ep_mgpu_geometry* g, const void* local_block, int32_t* total_rows,
                                         ep_stream_t stream) {
    ep_status st = check_geometry(g);
    if (st != EP_OK) return st;
    if (local_block == nullptr || total_rows == nullptr) return invalid("local_block and total_rows must be non-NULL");
    const char* p = (const char*)local_block + g->off_recv_offsets + (int64_t)g->experts_per_rank * 4;
    cudaError_t err = cudaMemcpyAsync(total_rows, p, 4, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (err == cudaSuccess) err = cudaStreamSynchronize((cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("read total rows", err);
    return ok();
}

EP_API ep_status ep_mgpu_check_error(const ep_mgpu_geometry* g, void* local_block, uint32_t* bits,
                                     ep_stream_t stream) {
    ep_status st = check_geometry(g);
    if (st != EP_OK) return st;
    if (local_block == nullptr) return invalid("local_block is NULL");
    char* p = (char*)local_block + g->off_error_word;
    uint32_t v = 0;
    cudaError_t err = cudaMemcpyAsync(&v, p, 4, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (err == cudaSuccess) err = cudaMemsetAsync(p, 0, 4, (cudaStream_t)stream);
    if (err == cudaSuccess) err = cudaStreamSynchronize((cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_failed("check error", err);
    if (bits != nullptr) *bits = v;
    if (v != 0) return ep::fail(EP_ERR_DEVICE, "device error word 0x%x", v);
    return ok();
}

}  // extern "C"
