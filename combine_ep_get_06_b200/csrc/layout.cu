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
#include "layout_device.cuh"

namespace ep {
namespace {

using namespace layout_dev;

template <typename IdxT>
__global__ void __launch_bounds__(kThreads) layout_single_kernel(LayoutArgs a) {
    extern __shared__ int smem_raw[];
    const int E = a.h.num_experts, S = a.h.num_segments;
    Smem m(smem_raw, E, S);
    const int tid = threadIdx.x;
    const int64_t s = tid;
    const bool has_slot = s < (int64_t)a.h.num_tokens * a.h.num_topk;
    bool bad = false;
    int e = -1;
    float wv = 0.0f;
    if (has_slot) {
        e = read_expert((const IdxT*)a.topk_idx, s, E, bad);
        if (a.topk_weights) wv = __ldg(a.topk_weights + s);
    }
    pdl_launch_dependents();
    const SlotRank r = small_layout<IdxT>(a, m, e, bad);
    if (has_slot) write_slot(a, s, slot_row(m, r, E), e, wv);
    write_totals(a, m, E);
    for (int g = tid; g < S; g += blockDim.x) a.h.seg_tokens[g] = m.seg[g];
    write_padding(a, m, E, 0, m.padoff[E]);
}

template <typename IdxT>
__global__ void __launch_bounds__(kThreads) layout_count_kernel(LayoutArgs a) {
    extern __shared__ int smem_raw[];
    const int E = a.h.num_experts, S = a.h.num_segments, k = a.h.num_topk;
    int* hist = smem_raw;
    int* seg = smem_raw + E;
    const int c = blockIdx.x, tid = threadIdx.x;
    const int t0 = c * a.chunk_tokens;
    const int t1 = min(a.h.num_tokens, t0 + a.chunk_tokens);
    const int64_t s = (int64_t)t0 * k + tid;
    const IdxT* idx = (const IdxT*)a.topk_idx;

    bool bad = false;
    int e = -1;
    if (s < (int64_t)t1 * k) e = read_expert(idx, s, E, bad);
    pdl_launch_dependents();
    for (int i = tid; i < E + S; i += blockDim.x) smem_raw[i] = 0;
    if (bad) atomicOr(a.h.error_word, EP_DEVERR_BAD_TOPK_IDX);
    __syncthreads();
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (peers & lanemask_lt()) == 0) atomicAdd(&hist[e], __popc(peers));
    count_segments(idx, t0, t1, k, E, S, e, seg);
    __syncthreads();
    for (int i = tid; i < E; i += blockDim.x) a.ws_hist[(int64_t)c * E + i] = hist[i];
    for (int i = tid; i < S; i += blockDim.x) a.ws_seg[(int64_t)c * S + i] = seg[i];
}

template <typename IdxT>
__global__ void __launch_bounds__(kThreads) layout_assign_kernel(LayoutArgs a) {
    extern __shared__ int smem_raw[];
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
    for (int i = tid; i < kWarps * E; i += blockDim.x) m.tab[i] = 0;
    for (int i = tid; i < E; i += blockDim.x) {
        m.cnt[i] = 0;
        m.base[i] = 0;
    }
    for (int i = tid; i < S; i += blockDim.x) m.seg[i] = 0;
    __syncthreads();
    const SlotRank r = rank_in_warp(e, m.tab, E);
    __syncthreads();
    if (tid < E) column_scan(m.tab, E);

    // Histograms of every chunk: totals, and the part from earlier chunks.
    pdl_wait();
    pdl_launch_dependents();
    reduce_columns(a.ws_hist, a.num_chunks, E, c, m.cnt, m.base);
    if (c == 0) reduce_columns(a.ws_seg, a.num_chunks, S, 0, m.seg, nullptr);
    __syncthreads();
    aligned_offsets(m, E, a.h.expert_alignment);
    if (tid < E) m.base[tid] += m.off[tid];
    __syncthreads();

    if (has_slot) write_slot(a, s, slot_row(m, r, E), e, wv);
    if (c == 0) {
        write_totals(a, m, E);
        for (int g = tid; g < S; g += blockDim.x) a.h.seg_tokens[g] = m.seg[g];
    }
    const int P = m.padoff[E];
    write_padding(a, m, E, (int)((int64_t)P * c / C), (int)((int64_t)P * (c + 1) / C));
}

template <typename K>
cudaError_t launch(K kernel, int grid, size_t smem, cudaStream_t stream, bool pdl, const LayoutArgs& a) {
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
    if (a.num_chunks == 1) return launch(single, 1, smem, stream, false, a);
    err = launch(layout_count_kernel<IdxT>, a.num_chunks, sizeof(int) * (E + S), stream, false, a);
    if (err != cudaSuccess) return err;
    return launch(assign, a.num_chunks, smem, stream, true, a);
}

}  // namespace

cudaError_t launch_layout(const LayoutArgs& a, bool idx_is_int64, cudaStream_t stream) {
    return idx_is_int64 ? launch_layout_t<long long>(a, stream) : launch_layout_t<int>(a, stream);
}

}  // namespace ep
