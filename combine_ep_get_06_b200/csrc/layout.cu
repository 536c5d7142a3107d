// Layout step of MoE dispatch: per-expert counts, the aligned expert-major
// receive layout and the deterministic slot map (DeepEP V2 README,
// "Interfaces and examples": the dispatch handle carries the routing
// metadata and the per-expert counts that feed the expert GEMM;
// expert_alignment pads each expert's block).  The building blocks are in
// layout_device.cuh.
//
//   one chunk  (T*k <= 1024, e.g. decode): a single CTA does everything.
//   many chunks (one CTA per <= 1024 slots of whole tokens):
//     count  - per-chunk expert histograms and segment token counts into
//              the workspace;
//     assign - launched with programmatic dependent launch: ranks its own
//              chunk while count still runs, then waits, reduces the
//              histograms of all chunks, scans the aligned expert sizes and
//              writes its slots and its share of the padding rows.
// Every layout kernel is launched with programmatic dependent launch and
// touches global memory only after waiting for the grid before it.
#include "layout_device.cuh"

namespace ep {
namespace {

using namespace layout_dev;

template <typename IdxT>
__global__ void __launch_bounds__(kThreads) layout_single_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) int smem_raw[];
    const int E = a.h.num_experts, S = a.h.num_segments;
    Smem m(smem_raw, E, S);
    const int64_t s = threadIdx.x;
    const bool has_slot = s < (int64_t)a.h.num_tokens * a.h.num_topk;
    // Launched with programmatic dependent launch: nothing global is read
    // or written before the previous grid (which may produce topk_idx or
    // still read the handle) has finished.
    pdl_wait();
    bool bad = false;
    int e = -1;
    float wv = 0.0f;
    if (has_slot) {
        e = read_expert((const IdxT*)a.topk_idx, s, E, bad);
        if (a.topk_weights) wv = __ldg(a.topk_weights + s);
    }
    pdl_launch_dependents();
    const int row = small_layout<IdxT>(a, m, e, bad, wv);
    if (has_slot) a.h.slot_map[s] = row;
    write_rows(a, m, 0, m.lcoff[E]);
    write_totals(a, m, E, S);
    write_padding(a, m, E, 0, m.padoff[E]);
}

template <typename IdxT>
__global__ void __launch_bounds__(kThreads) layout_count_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) int smem_raw[];
    const int E = a.h.num_experts, S = a.h.num_segments, k = a.h.num_topk;
    int* hist = smem_raw;
    int* seg = smem_raw + E;
    unsigned* tmask = reinterpret_cast<unsigned*>(seg + S);  // [2*kThreads]
    const int c = blockIdx.x, tid = threadIdx.x;
    const int t0 = c * a.chunk_tokens;
    const int t1 = min(a.h.num_tokens, t0 + a.chunk_tokens);
    const int64_t s = (int64_t)t0 * k + tid;
    const IdxT* idx = (const IdxT*)a.topk_idx;

    // The chunk's indices are asked into L2 while the previous grid still
    // runs: a prefetch returns no value and L2 is where every write lands,
    // so it cannot observe a stale index (the loads come after the wait).
    // Only the 16-byte aligned interior of the chunk, never past its ends.
    if (tid == 0) prefetch_interior_l2(idx + (int64_t)t0 * k, idx + (int64_t)t1 * k);
    // Programmatic dependent launch: wait for the previous grid before any
    // global load or store; only then let the assign pass start (it reads
    // topk_idx before waiting on this grid).
    pdl_wait();
    pdl_launch_dependents();
    bool bad = false;
    int e = -1;
    if (s < (int64_t)t1 * k) e = read_expert(idx, s, E, bad);
    for (int i = tid; i < E + S; i += blockDim.x) smem_raw[i] = 0;
    tmask[2 * tid] = 0;
    tmask[2 * tid + 1] = 0;
    if (bad) atomicOr(a.h.error_word, EP_DEVERR_BAD_TOPK_IDX);
    __syncthreads();
    if (e >= 0) atomicAdd(&hist[e], 1);
    if (S <= 64) mark_segment(tmask, tid / k, e, E, S, k);
    else count_segments_walk(idx, t0, t1, k, E, S, seg);
    __syncthreads();
    if (S <= 64) {
        count_segments_masks(tmask, t1 - t0, S, seg);
        __syncthreads();
    }
    for (int i = tid; i < E; i += blockDim.x) a.ws_hist[(int64_t)c * E + i] = hist[i];
    for (int i = tid; i < S; i += blockDim.x) a.ws_seg[(int64_t)c * S + i] = seg[i];
}

template <typename IdxT>
__global__ void __launch_bounds__(kThreads) layout_assign_kernel(LayoutArgs a) {
    extern __shared__ __align__(16) int smem_raw[];
    const int E = a.h.num_experts, S = a.h.num_segments, k = a.h.num_topk;
    Smem m(smem_raw, E, S);
    const int c = blockIdx.x, C = gridDim.x, tid = threadIdx.x;
    const int t0 = c * a.chunk_tokens;
    const int t1 = min(a.h.num_tokens, t0 + a.chunk_tokens);
    const int64_t s = (int64_t)t0 * k + tid;
    const bool has_slot = s < (int64_t)t1 * k;

    // Local work, independent of the count pass (topk_idx is an input).
    bool ignore = false;
    int e = -1;
    float wv = 0.0f;
    if (has_slot) {
        e = read_expert((const IdxT*)a.topk_idx, s, E, ignore);
        if (a.topk_weights) wv = __ldg(a.topk_weights + s);
    }
    zero_tab(m.tab, E);
    for (int i = tid; i < E; i += blockDim.x) {
        m.cnt[i] = 0;
        m.base[i] = 0;
    }
    for (int i = tid; i < S; i += blockDim.x) m.seg[i] = 0;
    __syncthreads();
    mark_slot(e, m.tab, E);
    __syncthreads();
    const int wrank = rank_in_warp(e, m.tab, E);
    __syncthreads();
    if (tid < E) m.lc[tid] = column_scan(m.tab, E);

    // Histograms of every chunk: totals, and the part from earlier chunks.
    pdl_wait();
    pdl_launch_dependents();
    reduce_columns(a.ws_hist, a.num_chunks, E, c, m.cnt, m.base);
    if (c == 0) reduce_columns(a.ws_seg, a.num_chunks, S, 0, m.seg, nullptr);
    __syncthreads();
    expert_offsets(m, E, a.h.expert_alignment);
    if (tid < E) m.base[tid] += m.off[tid];
    __syncthreads();

    const int crank = chunk_rank(m, e, wrank, E);
    stage_slot(m, s, e, crank, wv);
    const int row = slot_row(a, m, e, crank);
    if (has_slot) a.h.slot_map[s] = row;
    __syncthreads();
    write_rows(a, m, 0, m.lcoff[E]);
    if (c == 0) write_totals(a, m, E, S);
    const int P = m.padoff[E];
    write_padding(a, m, E, (int)((int64_t)P * c / C), (int)((int64_t)P * (c + 1) / C));
}

template <typename K>
cudaError_t launch(K kernel, const char* name, int grid, size_t smem, cudaStream_t stream, bool pdl,
                   const LayoutArgs& a) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    debug_launch(name, a.h.num_experts, cfg);
    return cudaLaunchKernelEx(&cfg, kernel, a);
}

template <typename IdxT>
cudaError_t launch_layout_t(const LayoutArgs& a, cudaStream_t stream) {
    const int E = a.h.num_experts, S = a.h.num_segments;
    const size_t smem = layout_dev::smem_bytes(E, S);
    auto single = layout_single_kernel<IdxT>;
    auto assign = layout_assign_kernel<IdxT>;
    cudaError_t err;
    if (smem > 48 * 1024) {
        if ((err = cudaFuncSetAttribute(single, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
            return err;
        if ((err = cudaFuncSetAttribute(assign, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
            return err;
    }
    if (a.num_chunks == 1) return launch(single, "layout_single_kernel", 1, smem, stream, true, a);
    const size_t smem_count = sizeof(int) * (E + S) + sizeof(unsigned) * 2 * kThreads;
    err = launch(layout_count_kernel<IdxT>, "layout_count_kernel", a.num_chunks, smem_count, stream, true, a);
    if (err != cudaSuccess) return err;
    return launch(assign, "layout_assign_kernel", a.num_chunks, smem, stream, true, a);
}

}  // namespace

cudaError_t launch_layout(const LayoutArgs& a, bool idx_is_int64, cudaStream_t stream) {
    return idx_is_int64 ? launch_layout_t<long long>(a, stream) : launch_layout_t<int>(a, stream);
}

}  // namespace ep
