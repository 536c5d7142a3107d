/*
 * ep.h -- C ABI of a B200 (sm_100a) library for MoE expert-parallel
 * dispatch and combine on one GPU.
 *
 * What it computes is the dispatch / combine pair of the DeepEP V2 README,
 * section "Interfaces and examples" (dispatch_forward, dispatch_backward,
 * combine_forward, combine_backward and the decode example with a cached
 * handle), with the FP8 dispatch / BF16 combine workload of its section
 * "Performance".  Expert "ranks" are logical segments of this GPU's memory:
 * segment s owns experts [s*E/S, (s+1)*E/S), and no data leaves the device.
 *
 * Notation: T tokens, k = num_topk, E = num_experts, S = num_segments,
 * a = expert_alignment, H = hidden, B = H/128 FP8 scale blocks per row.
 * c_e = number of slots routed to expert e; A(c) = ceil(c/a)*a rows per
 * expert (A(0) = 0); R = sum_e A(c_e) receive rows; the worst case is
 * ep_max_recv_rows() = T*k + E*(a-1).
 *
 * Receive layout (expert-major, alignment-padded): expert e owns rows
 * [offsets[e], offsets[e+1]).  Its first c_e rows hold its slots in
 * ascending flat slot order s = t*k + j; the rest are padding rows (zero
 * data, zero scales, recv_src = recv_topk_idx = -1, weight 0).  Rows >= R
 * are never written.
 *
 * Conventions for every call:
 *   - All array pointers are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or synchronises, except where a call
 *     says "synchronises".  Row-major, densely packed.
 *   - Pointers that are read or written as vectors must be 16-byte
 *     aligned (x, recv_x, y, out); every array pointer must be 4-byte
 *     aligned.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream) and is stream-ordered.  Calls that do not
 *     synchronise may be captured in a CUDA graph.
 *   - Argument errors are found on the host before anything is launched:
 *     the call returns EP_ERR_INVALID_ARG, writes nothing, and
 *     ep_last_error() tells why.  A failed launch returns EP_ERR_CUDA.
 *   - Errors found on the device never trap: they set bits of the handle's
 *     error word (EP_DEVERR_*), which ep_check_error() reads and clears.
 */
#ifndef EP_B200_EP_H
#define EP_B200_EP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define EP_API __attribute__((visibility("default")))
#else
#define EP_API
#endif

#define EP_ABI_VERSION 1

typedef struct CUstream_st* ep_stream_t; /* same object as cudaStream_t */

typedef enum {
    EP_OK = 0,
    EP_ERR_INVALID_ARG = 1, /* host-side argument check failed; nothing launched */
    EP_ERR_DEVICE = 2,      /* ep_check_error: the device error word was non-zero */
    EP_ERR_CUDA = 3         /* a CUDA runtime call or launch failed */
} ep_status;

/* Device error word bits (sticky until ep_check_error). */
#define EP_DEVERR_BAD_TOPK_IDX 1u /* a topk_idx value outside [-1, E): slot treated as dropped */
#define EP_DEVERR_CAPACITY 2u     /* a row index >= max_recv_rows: write skipped */
#define EP_DEVERR_TIMEOUT 4u      /* a bounded wait gave up */
#define EP_DEVERR_CHECK 8u        /* a checked build (EP_CHECKED) found a broken invariant: access skipped */

/* Form of the x passed to ep_dispatch (DeepEP V2 README, "Interfaces and
 * examples": x is a bf16 tensor or an FP8 (data, scale_factors) tuple). */
typedef enum {
    EP_X_BF16 = 0,        /* x bf16 [T,H] -> recv_x bf16 [rows,H]; H % 8 == 0 */
    EP_X_FP8 = 1,         /* x e4m3 [T,H] + x_scales f32 [T,B] copied as they are; H % 128 == 0 */
    EP_X_BF16_TO_FP8 = 2, /* x bf16 [T,H] quantised per 1x128 block: amax = max|x| floored at
                             1e-4, scale = amax/448, q = e4m3_rn_satfinite(x * (448/amax));
                             -> recv_x e4m3 [rows,H] + recv_scales f32 [rows,B]; H % 128 == 0 */
    EP_X_BF16_TO_NVFP4 = 3 /* x bf16 [T,H] quantised to NVFP4 (the Hybrid-EP branch's NVFP4
                             type): per 1x16 block amax = max|x| floored at 6*2^-9, scale =
                             e4m3_rn_satfinite(amax/6), q = e2m1_rn_satfinite(x * (1/scale));
                             -> recv_x [rows,H/2] bytes (two E2M1 codes each, the even element
                             in the low nibble) + recv_scales [rows,H/16] e4m3 bytes; H % 32 == 0 */
} ep_x_mode;

/* Routing metadata of one layout (the pages' EPHandle).  A plain struct of
 * device pointers carved from one caller-owned device block by
 * ep_handle_init; reusable for any number of dispatch / combine calls with
 * the same routing (decode with a cached handle; combine_backward =
 * dispatch and dispatch_backward = combine with the forward's handle). */
typedef struct ep_handle {
    int32_t num_tokens, num_topk, num_experts, num_segments, expert_alignment, max_recv_rows;
    int32_t* counts;          /* [E]   c_e, slots routed to expert e */
    int32_t* recv_counts;     /* [E]   A(c_e): rows per expert (num_recv_tokens_per_expert_list) */
    int32_t* offsets;         /* [E+1] first row of expert e; offsets[E] = R */
    int32_t* seg_tokens;      /* [S]   tokens with at least one valid slot in segment s */
    int32_t* slot_map;        /* [T*k] row of slot t*k+j, or -1 when dropped */
    int32_t* recv_src;        /* [max_recv_rows] slot t*k+j held by each row; -1 on padding */
    int32_t* pad_rows;        /* [max(1, E*(a-1))] rows that are padding, in ascending order */
    int32_t* num_pad_rows;    /* [1]   number of padding rows, R - sum_e c_e */
    uint32_t* error_word;     /* [1]   EP_DEVERR_* bits */
} ep_handle;

/* Version of this ABI (EP_ABI_VERSION).  The pages have no counterpart:
 * this and the two calls below are the C ABI's own error reporting. */
EP_API int32_t ep_abi_version(void);

/* Human-readable name of a status code; never NULL. */
EP_API const char* ep_status_string(ep_status status);

/* Why the last call on this host thread returned an error ("" if none). */
EP_API const char* ep_last_error(void);

/* SM budget (DeepEP V2 README, "Interfaces and examples": num_sms, the
 * SMs the communication kernels may take, so that the expert GEMMs keep
 * the rest; "Performance": throughput at a given #SMs).  After
 * ep_set_num_sms(n) with n > 0, the dispatch and combine kernels that this
 * host thread launches (ep_dispatch, ep_dispatch_mn_scales,
 * ep_layout_dispatch's dispatch, ep_combine) use at most n CTAs, each
 * sized to fill one SM, so they occupy at most n SMs and leave the others
 * to a kernel running beside them on another stream.  n = 0 (the default)
 * lets them take every SM.  Budgets above the device's SM count are
 * clipped.  The layout kernels (one CTA per 1024 slots, a few
 * microseconds) do not follow it.  The setting belongs to the calling host
 * thread and is read when a call launches its kernels (a captured graph
 * keeps the grid it was captured with).  EP_ERR_INVALID_ARG for n < 0. */
EP_API ep_status ep_set_num_sms(int32_t num_sms);

/* The calling host thread's SM budget (0 = none). */
EP_API int32_t ep_get_num_sms(void);

/* Worst-case receive rows T*k + E*(a-1): the size to give recv_x, recv_src,
 * recv_topk_idx / weights and y so that any routing fits.  -1 on bad
 * arguments or int32 overflow.  Stands for the buffer sizing of the DeepEP
 * V2 README, "Interfaces and examples" (get_buffer_size_hint from
 * num_max_tokens_per_rank, hidden and top-k), here for caller-owned
 * receive tensors instead of a library-owned communication buffer. */
EP_API int32_t ep_max_recv_rows(int32_t num_tokens, int32_t num_topk, int32_t num_experts,
                                int32_t expert_alignment);

/* Bytes of the device block that ep_handle_init carves up (0 on bad
 * arguments): the storage of the handle (EPHandle, DeepEP V2 README,
 * "Interfaces and examples") that dispatch returns and combine reuses.  Limits: T >= 0, 1 <= k <= 32, 1 <= E <= 1024, S >= 1 and
 * S divides E, a >= 1, max_recv_rows >= ep_max_recv_rows(T, k, E, a). */
EP_API size_t ep_handle_bytes(int32_t num_tokens, int32_t num_topk, int32_t num_experts,
                              int32_t num_segments, int32_t expert_alignment,
                              int32_t max_recv_rows);

/* The handle (EPHandle, DeepEP V2 README, "Interfaces and examples") as a
 * plain struct of device pointers.  Fills *handle with pointers into
 * `device_block` (at least
 * ep_handle_bytes() bytes, 256-byte aligned, owned by the caller and kept
 * alive as long as the handle is used) and zeroes nothing: the layout
 * writes every field before use.  Host only; launches nothing. */
EP_API ep_status ep_handle_init(ep_handle* handle, int32_t num_tokens, int32_t num_topk,
                                int32_t num_experts, int32_t num_segments,
                                int32_t expert_alignment, int32_t max_recv_rows,
                                void* device_block, size_t block_bytes);

/* Bytes of device scratch that ep_get_layout needs for this handle's
 * shape (per-chunk expert histograms).  Always > 0. */
EP_API size_t ep_layout_workspace_bytes(const ep_handle* handle);

/* The layout step behind dispatch (DeepEP V2 README, "Interfaces and
 * examples": dispatch returns recv_topk_idx, recv_topk_weights and a handle
 * whose per-expert counts feed the expert GEMM; expert_alignment pads them).
 *
 *   topk_idx      [T,k] int64 (idx_is_int64 = 1) or int32 (0); -1 = dropped
 *                 slot; other values outside [0, E) set EP_DEVERR_BAD_TOPK_IDX
 *                 and are treated as dropped.
 *   topk_weights  [T,k] f32, or NULL (then recv_topk_weights gets 0s).
 *   recv_topk_idx [max_recv_rows] i32 out, or NULL: expert of each row, -1 on padding.
 *   recv_topk_weights [max_recv_rows] f32 out, or NULL: topk_weights of
 *                 each row's slot, 0 on padding.
 *   workspace     device scratch of ep_layout_workspace_bytes() bytes,
 *                 256-byte aligned; contents on entry do not matter.
 * Writes every handle array (rows < R of recv_src).  Never synchronises:
 * R stays on the device (see ep_read_total_rows). */
EP_API ep_status ep_get_layout(ep_handle* handle, const void* topk_idx, int32_t idx_is_int64,
                               const float* topk_weights, int32_t* recv_topk_idx,
                               float* recv_topk_weights, void* workspace,
                               size_t workspace_bytes, ep_stream_t stream);

/* Scratch held by the library for ep_get_layout_static (per GPU). */
#define EP_STATIC_LAYOUT_SCRATCH_BYTES ((size_t)1 << 20)

/* ep_get_layout without a workspace argument.  The paper has no
 * counterpart: this entry exists for callers that cannot allocate device
 * memory themselves -- code running inside a host program that owns every
 * device allocation (a serving engine with a fixed memory plan), or plain C
 * code without a device allocator -- and so cannot hand ep_get_layout a
 * workspace.  The per-chunk histograms go to a fixed array inside this
 * library instead: EP_STATIC_LAYOUT_SCRATCH_BYTES on every GPU that loads
 * it, kept until the process exits.  Same arguments (minus the workspace),
 * results and errors as ep_get_layout, plus EP_ERR_INVALID_ARG when
 * ep_layout_workspace_bytes(handle) exceeds EP_STATIC_LAYOUT_SCRATCH_BYTES
 * (for E = 256 experts about a million slots fit).  Allocates and frees
 * nothing.  The first call on each device looks up the array's device
 * address (cudaGetSymbolAddress) with that device current, so make that
 * first call before any stream capture.  That address is kept until the
 * process exits: a cudaDeviceReset of the device after the first call is
 * not supported (the kept address would be stale).  All calls share the
 * array: calls that overlap on the GPU race on it. */
EP_API ep_status ep_get_layout_static(ep_handle* handle, const void* topk_idx, int32_t idx_is_int64,
                                      const float* topk_weights, int32_t* recv_topk_idx,
                                      float* recv_topk_weights, ep_stream_t stream);

/* Dispatch (dispatch_forward; with a bf16 gradient and the forward's
 * handle it is combine_backward): row t of x goes to rows slot_map[t*k+j]
 * of recv_x for every valid j, padding rows are zeroed, rows >= R are not
 * touched.
 *   x          [T,H] bf16 (EP_X_BF16, EP_X_BF16_TO_FP8) or e4m3 bytes (EP_X_FP8)
 *   x_scales   [T,B] f32 for EP_X_FP8, else ignored (may be NULL)
 *   recv_x     [max_recv_rows,H] bf16 (EP_X_BF16) or e4m3 bytes, or [max_recv_rows,H/2]
 *              packed E2M1 (EP_X_BF16_TO_NVFP4)
 *   recv_scales [max_recv_rows,B] f32 for the FP8 modes, [max_recv_rows,H/16] e4m3 bytes
 *              for NVFP4, else ignored
 * The FP8 quantisation rounds to nearest-even with saturation at +-448. */
EP_API ep_status ep_dispatch(const ep_handle* handle, ep_x_mode mode, const void* x,
                             const float* x_scales, int32_t hidden, void* recv_x,
                             void* recv_scales, ep_stream_t stream);

/* Layout and dispatch in one call: the dispatch(x, topk_idx, topk_weights,
 * num_experts, expert_alignment) call of the DeepEP V2 README ("Interfaces
 * and examples"), which routes and sends in one step.  Arguments, results
 * and errors are those of ep_get_layout followed by ep_dispatch with the
 * same handle.  With more than one layout chunk of slots (T*k > 1024) it
 * launches the same kernels, but because it knows that the dispatch
 * directly follows the layout, the dispatch reads its x rows while the
 * layout still runs (the two calls cannot assume that).  With at most one
 * chunk (e.g. decode, T*k <= 1024) and no SM budget, one kernel does both:
 * every token CTA computes in shared memory the part of the layout its row
 * needs, and a few CTAs without a token write the handle's totals.  The
 * workspace is then checked but not written.  The outputs are the same
 * either way. */
EP_API ep_status ep_layout_dispatch(ep_handle* handle, const void* topk_idx, int32_t idx_is_int64,
                                    const float* topk_weights, int32_t* recv_topk_idx,
                                    float* recv_topk_weights, void* workspace,
                                    size_t workspace_bytes, ep_x_mode mode, const void* x,
                                    const float* x_scales, int32_t hidden, void* recv_x,
                                    void* recv_scales, ep_stream_t stream);

/* Dispatch with the FP8 block scales laid out the way a grouped FP8 GEMM
 * reads them (DeepEP V2 README, "News": V2 adopts a new GEMM layout;
 * "Interfaces and examples": the per-expert counts feed the GEMM).  The same
 * as ep_dispatch in the two FP8 modes (not NVFP4), except that the scale of block b of
 * receive row r goes to recv_scales_mn[b * scales_ld + r] (MN-major: one
 * column of rows per block).  scales_ld >= max_recv_rows and a multiple of
 * 4, so that every column starts 16-byte aligned for TMA; entries for rows
 * >= R and the column tails past max_recv_rows are not written. */
EP_API ep_status ep_dispatch_mn_scales(const ep_handle* handle, ep_x_mode mode, const void* x,
                                       const float* x_scales, int32_t hidden, void* recv_x,
                                       float* recv_scales_mn, int32_t scales_ld, ep_stream_t stream);

/* Copies A(c_e), the rows of each expert (the pages'
 * num_recv_tokens_per_expert_list), to host_counts[E].  Synchronises `stream`. */
EP_API ep_status ep_read_recv_counts(const ep_handle* handle, int32_t* host_counts, ep_stream_t stream);

/* Combine (combine_forward; unweighted it is dispatch_backward):
 *   out[t,:] = bf16( sum_j w[t,j] * y[slot_map[t*k+j],:] ) over valid slots,
 *   accumulated in fp32 as acc = fma(w, y, acc) from +0 in ascending j and
 *   rounded to bf16 (nearest-even) once.  A token with no valid slot gets +0.
 *   y            [max_recv_rows,H] bf16 expert outputs (only rows of valid slots are read)
 *   topk_weights [T,k] f32, or NULL: every w = 1 (dispatch_backward's sum)
 *   recv_weights_in [max_recv_rows] f32 or NULL; out_weights [T,k] f32 or
 *                NULL: when both are given, out_weights[t,j] =
 *                recv_weights_in[slot_map[t*k+j]] (0 for a dropped slot),
 *                the weight gradient of dispatch_backward.
 *   out          [T,H] bf16.  H % 8 == 0. */
EP_API ep_status ep_combine(const ep_handle* handle, const void* y, int32_t hidden,
                            const float* topk_weights, const float* recv_weights_in,
                            float* out_weights, void* out, ep_stream_t stream);

/* Combine of FP8 expert outputs: the low-precision combine (the DeepEP V2
 * README's introduction says its kernels support low precision, FP8
 * included; it fixes no arithmetic, so this is the plainest reading).  The
 * expert outputs come in the layout of the FP8 dispatch's output:
 *   y_q      [max_recv_rows,H] e4m3 codes (16-byte aligned)
 *   y_scales [max_recv_rows,H/128] f32, one scale per 1x128 block
 * Each value is v = decode(q) * scale in binary32 (one rounding), and
 *   out[t,:] = bf16( sum_j w[t,j] * v[slot_map[t*k+j],:] )
 * with the accumulation of ep_combine (fp32 FMA from +0 in ascending j, one
 * bf16 rounding).  topk_weights [T,k] f32 or NULL (every w = 1); out [T,H]
 * bf16.  H % 128 == 0.  Only rows of valid slots are read. */
EP_API ep_status ep_combine_fp8(const ep_handle* handle, const void* y_q, const float* y_scales,
                                int32_t hidden, const float* topk_weights, void* out,
                                ep_stream_t stream);

/* Backward of the weighted combine (combine_backward of the DeepEP V2
 * README, "Interfaces and examples", which runs as a dispatch of the output
 * gradient; with weights in the forward each row is also scaled):
 *   grad_y[slot_map[t*k+j], :] = bf16(w[t,j] * grad_out[t, :])   (binary32 product,
 *                                 one bf16 rounding); padding rows zeroed; rows >= R untouched
 *   grad_weights[t, j] = sum_h grad_out[t,h] * y[slot_map[t*k+j], h]   (binary32
 *                                 accumulation, fixed order; 0 for a dropped slot)
 *   grad_out     [T,H] bf16;  y [max_recv_rows,H] bf16 (the forward's expert outputs)
 *   topk_weights [T,k] f32, or NULL (every w = 1)
 *   grad_y       [max_recv_rows,H] bf16 out;  grad_weights [T,k] f32 out.  H % 8 == 0. */
EP_API ep_status ep_combine_backward(const ep_handle* handle, const void* grad_out, const void* y,
                                     int32_t hidden, const float* topk_weights, void* grad_y,
                                     float* grad_weights, ep_stream_t stream);

/* Copies R = offsets[E] to *total_rows on the host.  Synchronises `stream`.
 * This is the host read that the README's decode example ("Interfaces and
 * examples": a cached handle avoids a redundant CPU sync) keeps off the hot
 * path; every other call leaves R on the device. */
EP_API ep_status ep_read_total_rows(const ep_handle* handle, int32_t* total_rows,
                                    ep_stream_t stream);

/* Reads the device error word into *bits (may be NULL) and clears it.
 * Synchronises `stream`.  Returns EP_ERR_DEVICE if any bit was set.  The
 * pages have no counterpart (their kernels assert); this is the sync the
 * README's decode example avoids, taken only when the caller asks. */
EP_API ep_status ep_check_error(const ep_handle* handle, uint32_t* bits, ep_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EP_B200_EP_H */
