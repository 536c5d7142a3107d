/*
 * ep_multi.h -- expert parallelism across the GPUs of one NVLink domain.
 *
 * The DeepEP V2 README ("Performance": EP over the GPUs of an NVLink
 * domain, SM100 included; "Interfaces and examples": dispatch and combine
 * with a handle) runs dispatch and combine as an all-to-all between ranks.
 * Here the segments of ep.h become ranks: rank d of W owns experts
 * [d*E/W, (d+1)*E/W).  Each rank holds one device "rank block" whose
 * sections have the same offsets on every rank (ep_mgpu_geometry).  Every
 * rank maps every other rank's block (CUDA IPC over NVLink / NVSwitch), and
 * the kernels store received rows straight into the owner's block (TMA bulk
 * copies from shared memory, one destination each; plain 16-byte stores
 * where a destination is not 16-byte aligned) and load expert outputs
 * straight from it with plain 16-byte loads.
 *
 * One step on rank r, with T_r <= max_tokens tokens:
 *   1. ep_get_layout on a local handle (num_segments = W, alignment 1):
 *      this rank's per-expert counts and each slot's place among them.
 *   2. The caller's all-gather of handle.counts [E] over the W ranks, in
 *      rank order, into the block's all_counts [W][E] (e.g. NCCL).  This is
 *      the one exchange the layout needs.  It also orders this step's
 *      stores after every rank's use of its block in the previous step.
 *   3. ep_mgpu_dispatch: the row stores to the owners' blocks.
 *   4. A barrier across the W ranks, ordered on the stream (e.g. an NCCL
 *      all-reduce of one word).  After it every block holds its rows.
 *   5. The expert GEMMs: rank d reads recv_x / recv_scales and writes y,
 *      all in its own block.
 *   6. A barrier, so that every y is complete.
 *   7. ep_mgpu_combine: the weighted sum of each token's k rows, loaded
 *      from the owners' y.
 *
 * Receive layout on rank d.  Take the layout of ep.h over the W ranks'
 * batches concatenated in rank order (num_segments = W, alignment a), and
 * keep the rows of d's experts, renumbered from 0.  So local expert i
 * (global e = d*E/W + i) owns rows [recv_offsets[i], recv_offsets[i+1]).
 * Its first C_e rows hold its slots, ordered by source rank, then by flat
 * slot t*k+j.  They are followed by A(C_e) - C_e padding rows (zero data,
 * zero scales, recv_src = recv_topk_idx = -1, weight 0).  Here
 * C_e = sum over ranks of counts[e] and A(c) = ceil(c/a)*a.
 * recv_src[row] = r*max_tokens*k + t*k + j names the source rank r and
 * its slot.  Rows >= R_d = recv_offsets[E/W] are never written.
 *
 * Conventions are those of ep.h.  In addition, peer_blocks is a DEVICE
 * array [W] of the W blocks' addresses as mapped in this process
 * (peer_blocks[rank] == local_block).  No call here synchronises or waits
 * on another GPU: the ordering across ranks comes from the caller's
 * collectives in steps 2, 4 and 6.  Nothing in this file has been run
 * across several GPUs.  Its kernels were checked with all W blocks on one
 * GPU, and the whole path (CUDA IPC included) with two and four processes
 * sharing one GPU.  The stores over NVLink have not run.
 */
#ifndef EP_B200_EP_MULTI_H
#define EP_B200_EP_MULTI_H

#include "ep.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Shape of one rank block.  Section offsets are bytes from the block's
 * start, 256-byte aligned.  ep_mgpu_geometry_init fills every field. */
typedef struct ep_mgpu_geometry {
    int32_t rank, world, max_tokens, num_topk, num_experts, expert_alignment, hidden;
    int32_t x_mode;            /* receive format: EP_X_BF16, EP_X_FP8 / EP_X_BF16_TO_FP8
                                  (both store e4m3 + f32 scales) or EP_X_BF16_TO_NVFP4 */
    int32_t experts_per_rank;  /* E/W */
    int32_t max_recv_rows;     /* W*max_tokens*k + (E/W)*(a-1) */
    int32_t row_bytes;         /* bytes of one received row */
    int32_t scale_bytes;       /* bytes of one row of scales (0 for bf16) */
    int64_t off_recv_x;        /* [max_recv_rows][row_bytes]  written by every rank */
    int64_t off_recv_scales;   /* [max_recv_rows][scale_bytes]  written by every rank */
    int64_t off_recv_src;      /* [max_recv_rows] i32  written by every rank */
    int64_t off_recv_topk_idx; /* [max_recv_rows] i32: global expert id, -1 on padding */
    int64_t off_recv_topk_weights; /* [max_recv_rows] f32: the slot's weight, 0 on padding */
    int64_t off_y;             /* [max_recv_rows][H] bf16: expert outputs (the caller's GEMM) */
    int64_t off_all_counts;    /* [W][E] i32: the all-gather's target (step 2) */
    int64_t off_dest;          /* [max_tokens*k][2] i32: (rank, row) of each of this rank's
                                  slots, (-1, -1) when dropped; written by dispatch, read by combine */
    int64_t off_raw_counts;    /* [E/W] i32: C_e of each local expert */
    int64_t off_recv_counts;   /* [E/W] i32: A(C_e), rows per local expert (for the GEMM) */
    int64_t off_recv_offsets;  /* [E/W+1] i32: first row of each local expert; last = R_d */
    int64_t off_num_pad_rows;  /* [1] i32 */
    int64_t off_error_word;    /* [1] u32: EP_DEVERR_* bits of the multi-GPU kernels */
    int64_t block_bytes;       /* total size of a rank block */
} ep_mgpu_geometry;

/* Fills *g.  Limits: 0 <= rank < world, world >= 1 and divides E,
 * 1 <= E <= 1024, world <= 128, max_tokens >= 0, 1 <= k <= 32,
 * a >= 1, hidden as ep_dispatch requires for x_mode, and W*max_tokens*k
 * + (E/W)*(a-1) < 2^31.  Host only. */
EP_API ep_status ep_mgpu_geometry_init(ep_mgpu_geometry* g, int32_t rank, int32_t world,
                                       int32_t max_tokens, int32_t num_topk, int32_t num_experts,
                                       int32_t expert_alignment, int32_t hidden, ep_x_mode x_mode);

/* Allocates a rank block of `bytes` with cudaMalloc on the current device,
 * so that CUDA IPC can export it whole.  This is the one call in the
 * library that allocates.  Contents are undefined. */
EP_API ep_status ep_mgpu_block_alloc(size_t bytes, void** block);
EP_API ep_status ep_mgpu_block_free(void* block);

/* CUDA IPC of a rank block: ep_ipc_export writes
 * EP_IPC_HANDLE_BYTES bytes that another process, on this GPU or another
 * one of the node, passes to ep_ipc_import, which maps the block into that
 * process (peer access enabled lazily) and returns its address there.
 * ep_ipc_close unmaps an imported block.  A block cannot be imported by
 * the process that allocated it: use its own address there. */
#define EP_IPC_HANDLE_BYTES 64
EP_API ep_status ep_ipc_export(const void* block, void* handle_out);
EP_API ep_status ep_ipc_import(const void* handle, void** block);
EP_API ep_status ep_ipc_close(void* block);

/* Step 3: the multi-GPU dispatch (dispatch_forward across ranks).
 *   local         this rank's handle, after ep_get_layout (step 1) on the same
 *                 topk_idx: num_tokens = T_r <= max_tokens, num_segments = W,
 *                 expert_alignment = 1, same k and E as g.
 *   topk_idx      [T_r,k] int64 (idx_is_int64 = 1) or int32, as given to ep_get_layout.
 *   topk_weights  [T_r,k] f32 or NULL (received weights are then 0).
 *   mode, x, x_scales  as in ep_dispatch; mode must store g->x_mode's format.
 *   local_block   this rank's block;  peer_blocks  device array [W] of block addresses.
 * Quantises each token once (FP8 and NVFP4 as in ep_dispatch). Writes its valid rows,
 * and their recv_src / recv_topk_idx / recv_topk_weights, into the owners' blocks.
 * Writes this rank's dest and, from all_counts, its own receive totals
 * (raw_counts, recv_counts, recv_offsets, num_pad_rows) and its own padding rows.
 * A computed row >= max_recv_rows (all_counts not from this step's all-gather)
 * sets EP_DEVERR_CAPACITY in the block's error word and is skipped; a
 * topk_idx value outside [0, E) on a slot the layout kept (a topk_idx that
 * is not the layout's) sets EP_DEVERR_BAD_TOPK_IDX and drops the slot. */
EP_API ep_status ep_mgpu_dispatch(const ep_mgpu_geometry* g, const ep_handle* local,
                                  const void* topk_idx, int32_t idx_is_int64,
                                  const float* topk_weights, ep_x_mode mode, const void* x,
                                  const float* x_scales, void* local_block,
                                  void* const* peer_blocks, ep_stream_t stream);

/* Step 7: the multi-GPU combine (combine_forward across ranks):
 *   out[t,:] = bf16( sum_j w[t,j] * y_d[row,:] ), where (d, row) = dest[t*k+j] over valid
 * slots, with the arithmetic of ep_combine (fp32 FMA from +0 in ascending j, one
 * bf16 rounding).  topk_weights [T_r,k] f32 or NULL (every w = 1); out [T_r,H] bf16. */
EP_API ep_status ep_mgpu_combine(const ep_mgpu_geometry* g, const ep_handle* local,
                                 const float* topk_weights, void* local_block,
                                 void* const* peer_blocks, void* out, ep_stream_t stream);

/* Copies R_d = recv_offsets[E/W] of this rank's block to the host.  Synchronises. */
EP_API ep_status ep_mgpu_read_total_rows(const ep_mgpu_geometry* g, const void* local_block,
                                         int32_t* total_rows, ep_stream_t stream);

/* Reads the block's error word into *bits (may be NULL) and clears it.
 * Synchronises; EP_ERR_DEVICE if any bit was set. */
EP_API ep_status ep_mgpu_check_error(const ep_mgpu_geometry* g, void* local_block, uint32_t* bits,
                                     ep_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EP_B200_EP_MULTI_H */
