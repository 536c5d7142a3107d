// Internal interface between the C-ABI front end (ep_api.cpp) and the
// kernels (layout.cu, dispatch.cu, combine.cu).  Not installed.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "ep.h"
#include "ep_multi.h"

namespace ep {

// Layout: one thread per slot; slots are processed in chunks of whole
// tokens of at most kLayoutChunkSlots slots, one CTA per chunk.
constexpr int kLayoutThreads = 1024;
constexpr int kLayoutChunkSlots = kLayoutThreads;
constexpr int kMaxExperts = 1024;
constexpr int kMaxTopk = 32;

struct LayoutArgs {
    const void* topk_idx;
    const float* topk_weights;
    int32_t* recv_topk_idx;
    float* recv_topk_weights;
    ep_handle h;            // by value: pointers into the caller's block
    int32_t chunk_tokens;   // tokens per chunk
    int32_t num_chunks;
    int32_t* ws_hist;       // [num_chunks][E]
    int32_t* ws_seg;        // [num_chunks][S]
};

inline int layout_chunk_tokens(int k) { return kLayoutChunkSlots / k > 0 ? kLayoutChunkSlots / k : 1; }
inline int layout_num_chunks(int T, int k) {
    int ct = layout_chunk_tokens(k);
    int c = (T + ct - 1) / ct;
    return c > 0 ? c : 1;
}

cudaError_t launch_layout(const LayoutArgs& a, bool idx_is_int64, cudaStream_t stream);

struct DispatchArgs {
    const void* x;
    const float* x_scales;
    void* recv_x;
    void* recv_scales;    // f32 (FP8 modes) or e4m3 bytes (NVFP4)
    const int32_t* slot_map;
    const int32_t* pad_rows;
    const int32_t* num_pad_rows;
    uint32_t* error_word;
    int32_t T, k, H, max_rows;
    int32_t max_pad_rows;  // E*(alignment-1): bound on the padding rows
    int32_t bulk_scales;  // scale rows are a multiple of 16 bytes and recv_scales is 16-byte aligned
    int32_t x_ready;      // 1: x was complete before the previous grid let this one launch, so it
                          // may be read before waiting on that grid (only right after the layout)
    int32_t scales_ld;    // 0: scales row-major [rows][B]; > 0: MN-major [B][scales_ld]
};

// Shared memory one dispatch CTA needs for this mode and hidden size.
size_t dispatch_smem_bytes(ep_x_mode mode, int H);
constexpr size_t kMaxDispatchSmem = 200 * 1024;

cudaError_t launch_dispatch(const DispatchArgs& a, ep_x_mode mode, cudaStream_t stream);

// Layout and dispatch in one grid (every CTA computing the layout it needs)
// when the slots fit one layout chunk and the row path applies;
// cudaErrorNotSupported otherwise, with nothing launched.
cudaError_t launch_layout_dispatch_fused(const LayoutArgs& la, const DispatchArgs& a, ep_x_mode mode,
                                         bool idx_is_int64, cudaStream_t stream);

struct CombineArgs {
    const void* y;
    const float* topk_weights;       // nullable: unweighted
    const float* recv_weights_in;    // nullable
    float* out_weights;              // nullable
    void* out;
    const int32_t* slot_map;
    uint32_t* error_word;
    int32_t T, k, H, max_rows;
};

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t stream);

struct CombineFp8Args {
    const void* y_q;                 // [max_rows,H] e4m3 codes
    const float* y_scales;           // [max_rows,H/128]
    const float* topk_weights;       // nullable: unweighted
    void* out;                       // [T,H] bf16
    const int32_t* slot_map;
    uint32_t* error_word;
    int32_t T, k, H, max_rows;
};

cudaError_t launch_combine_fp8(const CombineFp8Args& a, cudaStream_t stream);

struct CombineBackwardArgs {
    const void* grad_out;            // [T,H] bf16
    const void* y;                   // [max_rows,H] bf16
    const float* topk_weights;       // [T,k] or nullable (all 1)
    void* grad_y;                    // [max_rows,H] bf16
    float* grad_weights;             // [T,k]
    const int32_t* slot_map;
    const int32_t* pad_rows;
    const int32_t* num_pad_rows;
    uint32_t* error_word;
    int32_t T, k, H, max_rows, max_pad_rows;
};

cudaError_t launch_combine_backward(const CombineBackwardArgs& a, cudaStream_t stream);

// Number of SMs of the current device (cached per device).
// Multi-GPU expert parallelism (include/ep_multi.h).
constexpr int kMaxWorld = 128;

struct MgpuArgs {
    ep_mgpu_geometry g;       // by value
    DispatchArgs src;         // x, x_scales, H (read by the dispatch item helpers)
    int32_t T;                // this rank's tokens
    const int32_t* slot_map;  // local handle (alignment 1): row among this rank's slots
    const int32_t* offsets;   // local handle: first local row of each expert
    const void* topk_idx;
    int32_t idx_is_int64;
    const float* topk_weights;
    char* local_block;
    char* const* peer_blocks; // device array [world]
    void* out;                // combine output [T,H] bf16
};

size_t mgpu_dispatch_smem_bytes(const ep_mgpu_geometry& g);
cudaError_t launch_mgpu_dispatch(const MgpuArgs& a, ep_x_mode mode, cudaStream_t stream);
cudaError_t launch_mgpu_combine(const MgpuArgs& a, cudaStream_t stream);

int device_sm_count();

// SM budget of this host thread (ep_set_num_sms): 0 = no budget, else the
// most SMs the dispatch and combine grids may occupy (at most the device's).
int sm_budget();

// With EP_DEBUG=1 in the environment (read once), prints a launch's kernel,
// variant, grid, block, dynamic shared memory and stream to stderr.
void debug_launch(const char* kernel, int variant, dim3 grid, dim3 block, size_t smem, cudaStream_t stream);
inline void debug_launch(const char* kernel, int variant, const cudaLaunchConfig_t& c) {
    debug_launch(kernel, variant, c.gridDim, c.blockDim, c.dynamicSmemBytes, c.stream);
}

// Records a printf-style message for ep_last_error() and returns status.
ep_status fail(ep_status status, const char* fmt, ...);

}  // namespace ep
