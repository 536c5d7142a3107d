// ep_get_layout_static: the layout step with scratch memory that belongs to
// the library, for callers that cannot give it a workspace buffer.
//
// Some callers have no way to allocate device memory at the point where
// they route tokens: for example a plugin inside a host program that owns
// every device allocation (a serving engine that plans all of its memory
// up front and refuses allocations behind its back), or plain C code that
// has no device allocator at hand.  For them the per-chunk histograms the
// layout needs live in a fixed array in this library instead.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds EP_STATIC_LAYOUT_SCRATCH_BYTES of it until the process
// exits.  Host code cannot pass the variable's name to a kernel (on the
// host it only stands for the symbol), so the first call on each device
// looks up its device address with cudaGetSymbolAddress, with that device
// current, and keeps it; that first call should therefore come before any
// stream capture.  The address is kept for the life of the process: a
// cudaDeviceReset of that device after the first call makes it stale, and
// is not supported.  All calls share the one array: calls whose layouts
// overlap on the GPU (other streams, or other threads on the same device)
// race on it.  Nothing in it needs to start at zero: every entry the
// layout reads is written earlier by the same call.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "ep_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_layout_scratch[EP_STATIC_LAYOUT_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_setup_mutex;
std::atomic<void*> g_scratch_ptr[kMaxDevices];  // device address of g_layout_scratch, per device

// The device address of the scratch array on the current device: looked up
// once per device (under a lock), then read without one.
cudaError_t scratch_on_current_device(void** out) {
    int dev = -1;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
        std::lock_guard<std::mutex> lock(g_setup_mutex);
        p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
        if (p == nullptr) {
            err = cudaGetSymbolAddress(&p, g_layout_scratch);
            if (err != cudaSuccess) return err;
            g_scratch_ptr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return cudaSuccess;
}

}  // namespace

extern "C" EP_API ep_status ep_get_layout_static(ep_handle* handle, const void* topk_idx,
                                                 int32_t idx_is_int64, const float* topk_weights,
                                                 int32_t* recv_topk_idx, float* recv_topk_weights,
                                                 ep_stream_t stream) {
    const size_t need = ep_layout_workspace_bytes(handle);  // 0 when the handle is bad
    if (need == 0) return ep::fail(EP_ERR_INVALID_ARG, "handle is NULL or invalid; use ep_handle_init");
    if (need > EP_STATIC_LAYOUT_SCRATCH_BYTES)
        return ep::fail(EP_ERR_INVALID_ARG,
                        "this layout needs %zu bytes of scratch, more than the %zu bytes the library "
                        "holds; use ep_get_layout with a caller-owned workspace",
                        need, (size_t)EP_STATIC_LAYOUT_SCRATCH_BYTES);
    void* scratch = nullptr;
    const cudaError_t err = scratch_on_current_device(&scratch);
    if (err != cudaSuccess)
        return ep::fail(EP_ERR_CUDA, "looking up the library's layout scratch: %s", cudaGetErrorString(err));
    return ep_get_layout(handle, topk_idx, idx_is_int64, topk_weights, recv_topk_idx, recv_topk_weights,
                         scratch, EP_STATIC_LAYOUT_SCRATCH_BYTES, stream);
}
