// MoE dispatch on one device (DeepEP V2 README, "Interfaces and examples",
// dispatch_forward; FP8 dispatching as in its section "Performance").
//
// Warp-granular: the unit of work is one warp's, and warps never wait on
// one another (no CTA barrier after the start).  A unit is either
//   - a token slice: 1024 consecutive elements of one token row.  The warp
//     loads them (16 bytes a lane per load, a warp load covers 512
//     contiguous bytes), converts them (FP8: amax over the 1x128 block, 16
//     lanes, by xor shuffles; scale and inverse by IEEE division; e4m3
//     conversion) into a per-warp shared-memory stage, and lanes j < k
//     copy the stage to the slice of receive row slot_map[t*k+j] with TMA
//     bulk copies (cp.async.bulk shared->global, one destination each); or
//   - a padding row: lanes copy a zeroed buffer over the row's slices.
// Units are numbered token-major (t, slice), then padding rows, and dealt
// to the warps grid-stride, so every warp gets the same mix of small units
// and the grid has no long tail.  Each warp keeps its next unit's loads
// and routing in flight while it converts and copies the current one, and
// cycles kStages stages: a stage is refilled only once the copies issued
// from it kStages units ago have read it.
//
// Three launch shapes share the per-unit code (dispatch_warp.cuh):
//   - warp units, 8-warp CTAs, 2 to an SM (the default);
//   - under an SM budget of n (ep_set_num_sms), warp units in n CTAs of 24
//     warps, each CTA filling an SM;
//   - batches of at most one layout chunk of slots (e.g. decode): the row
//     path, a CTA per token row with one bulk copy per destination row (see
//     the row path below).
//
// Launched with programmatic dependent launch: the first unit's x loads
// may be issued before waiting for the previous grid (only directly after
// the layout, which leaves x untouched), everything the layout writes is
// read after the wait, and the next grid may start launching once all
// copies are issued.
#include "dispatch_warp.cuh"
#include "layout_device.cuh"

namespace ep {
namespace {

using namespace warp_units;

constexpr int kWarps = 8;         // warps per CTA; two CTAs to an SM
constexpr int kBudgetWarps = 24;  // warps per CTA under an SM budget: one CTA fills an SM
constexpr int kStages = 4;
constexpr int kPrefetchUnits = 3;  // units after the first whose x is brought into L2 during the layout

__host__ __device__ inline size_t smem_bytes(const SliceGeo& g, int warps) {
    return (size_t)g.stage_bytes * (1 + warps * kStages);  // zero buffer + the warps' stages
}

// The routing of unit u, read from the handle (which the previous grid,
// the layout, may have written).
template <int kMode>
__device__ __forceinline__ Meta load_meta(const DispatchArgs& a, const SliceGeo& g, int64_t u,
                                          int64_t n_tok_units, int64_t n_units, int lane) {
    Meta m;
    m.row = -1;
    m.xs = 0.0f;
    if (u >= n_units) return m;
    if (u >= n_tok_units) {
        m.row = ld_cg(a.pad_rows + (u - n_tok_units));
        return m;
    }
    const int t = (int)(u / g.ns), s = (int)(u - (int64_t)t * g.ns);
    if (lane < a.k) m.row = ld_cg(a.slot_map + (size_t)t * a.k + lane);
    if (kMode == EP_X_FP8) {
        const int nb = min(kSliceElems, a.H - s * kSliceElems) / 128;
        if (lane < nb) m.xs = ld_cg(a.x_scales + (size_t)t * (a.H / 128) + s * (kSliceElems / 128) + lane);
    }
    return m;
}

// Stores scale b of receive row `row`: f32 row-major or MN-major (the
// latter under an L2 evict-last policy: each token's scales land in B
// different columns, 4 bytes per 32-byte sector, and the whole array fits
// in L2, so its sectors fill up there before write-back), or an e4m3 byte
// for NVFP4.
template <int kMode>
__device__ __forceinline__ void store_scale(const DispatchArgs& a, int row, int b, const unsigned char* sst,
                                            int bi, uint64_t keep) {
    if (kMode == EP_X_BF16_TO_NVFP4) {
        reinterpret_cast<unsigned char*>(a.recv_scales)[(size_t)row * (a.H / 16) + b] = sst ? sst[bi] : 0;
    } else {
        const float v = sst ? reinterpret_cast<const float*>(sst)[bi] : 0.0f;
        if (a.scales_ld > 0)
            st_f32_hint(reinterpret_cast<float*>(a.recv_scales) + (size_t)b * a.scales_ld + row, v, keep);
        else
            reinterpret_cast<float*>(a.recv_scales)[(size_t)row * (a.H / 128) + b] = v;
    }
}

// Whether the scales of a slice of ne elements go out as one bulk copy:
// scale rows a multiple of 16 bytes in a 16-byte aligned array (the host
// sets bulk_scales; never for MN-major scales), and the slice's scale
// bytes a multiple of 16.
template <int kMode>
__device__ __forceinline__ bool bulk_scales_ok(const DispatchArgs& a, int ne) {
    return a.bulk_scales && (ne / Mode<kMode>::kScaleBlock * Mode<kMode>::kScaleBytes) % 16 == 0;
}

// Zeroes the zero buffer at the start of `smem` (a barrier follows in the caller).
template <int kW>
__device__ __forceinline__ void zero_buffer(unsigned char* zeros, int bytes) {
    for (int i = threadIdx.x; i < bytes / 16; i += 32 * kW) reinterpret_cast<uint4*>(zeros)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
}

// The unit loop of one warp, from unit u on (its x loads already in nxt),
// then the end of the grid's work.  `smem` holds the zero buffer and then
// kStages stages per warp.
template <int kMode, int kW>
__device__ __forceinline__ void run_units(const DispatchArgs& a, const SliceGeo& g, unsigned char* smem,
                                          int64_t u, Loads<kMode> nxt, int64_t n_pad) {
    using M = Mode<kMode>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned char* const zeros = smem;  // [stage_bytes] of zeros
    unsigned char* const stages = smem + (size_t)g.stage_bytes * (1 + warp * kStages);
    char* const recv = (char*)a.recv_x;
    char* const rscl = (char*)a.recv_scales;
    const int k = a.k;
    const uint64_t keep = a.scales_ld > 0 ? l2_evict_last_policy() : 0;
    const int64_t n_tok_units = (int64_t)a.T * g.ns;
    const int64_t stride = (int64_t)gridDim.x * kW;
    const int64_t n_units = n_tok_units + n_pad;
    Meta nmeta = load_meta<kMode>(a, g, u, n_tok_units, n_units, lane);

    int it = 0;  // token units of this warp (selects the stage)
    for (; u < n_units; u += stride) {
        const Loads<kMode> cur = nxt;
        const Meta m = nmeta;
        {
            const int64_t un = u + stride;
            nxt = load_x<kMode>(a, g, un, n_tok_units, lane);
            nmeta = load_meta<kMode>(a, g, un, n_tok_units, n_units, lane);
        }

        if (u >= n_tok_units) {
            // A padding row: zero data and scales.
            const int row = m.row;
            if (row < 0 || row >= a.max_rows) {
                if (row >= a.max_rows && lane == 0) atomicOr(a.error_word, EP_DEVERR_CAPACITY);
                continue;
            }
            if (!EP_CHECK(u - n_tok_units < n_pad, a.error_word)) continue;
            for (int s = lane; s < g.ns; s += 32) {
                const int ne = min(kSliceElems, a.H - s * kSliceElems);
                bulk_s2g(recv + (size_t)row * g.row_bytes + (size_t)s * g.out_bytes, zeros,
                         ne * g.out_bytes / kSliceElems);
                if (M::kScales && bulk_scales_ok<kMode>(a, ne))
                    bulk_s2g(rscl + (size_t)row * g.srow_bytes + (size_t)s * g.sout_bytes, zeros,
                             ne / M::kScaleBlock * M::kScaleBytes);
            }
            bulk_commit();
            if (M::kScales) {
                constexpr int kPerSlice = kSliceElems / M::kScaleBlock;
                const int B = a.H / M::kScaleBlock;
                for (int b = lane; b < B; b += 32) {
                    const int s = b / kPerSlice;
                    if (!bulk_scales_ok<kMode>(a, min(kSliceElems, a.H - s * kSliceElems)))
                        store_scale<kMode>(a, row, b, nullptr, 0, keep);
                }
            }
            continue;
        }

        // A token slice.
        const int t = (int)(u / g.ns), s = (int)(u - (int64_t)t * g.ns);
        const int ne = min(kSliceElems, a.H - s * kSliceElems);
        unsigned char* const st = stages + (size_t)(it % kStages) * g.stage_bytes;
        unsigned char* const sst = st + g.out_bytes;
        ++it;
        // The copies issued from this stage kStages units ago must have read it.
        if (lane < k) bulk_wait_read<kStages - 1>();
        __syncwarp();
        fill_stage<kMode>(cur, m, ne, lane, st, sst);
        fence_proxy_async_smem();
        __syncwarp();

        const int sb = M::kScales ? ne / M::kScaleBlock * M::kScaleBytes : 0;
        const bool bulk_scl = M::kScales && bulk_scales_ok<kMode>(a, ne);
        if (lane < k) {
            const int row = m.row;
            const int db = ne * g.out_bytes / kSliceElems;
            if (row >= 0 && row < a.max_rows &&
                EP_CHECK(t < a.T && (size_t)s * g.out_bytes + db <= (size_t)g.row_bytes &&
                             (size_t)s * g.sout_bytes + sb <= (size_t)g.srow_bytes,
                         a.error_word)) {
                bulk_s2g(recv + (size_t)row * g.row_bytes + (size_t)s * g.out_bytes, st, db);
                if (bulk_scl) bulk_s2g(rscl + (size_t)row * g.srow_bytes + (size_t)s * g.sout_bytes, sst, sb);
            } else if (row >= a.max_rows) {
                atomicOr(a.error_word, EP_DEVERR_CAPACITY);
            }
            bulk_commit();
        }
        if (M::kScales && !bulk_scl) {
            // MN-major scales, or scale rows that are not a multiple of 16 bytes: plain stores.
            const int nb = ne / M::kScaleBlock, b0 = s * (kSliceElems / M::kScaleBlock);
            for (int j = 0; j < k; ++j) {
                const int row = __shfl_sync(0xffffffffu, m.row, j);
                if (row < 0 || row >= a.max_rows) continue;
                for (int b = lane; b < nb; b += 32) store_scale<kMode>(a, row, b0 + b, sst, b, keep);
            }
        }
    }
    // Let the next grid start launching while the copies drain.
    pdl_launch_dependents();
    bulk_wait_all();
}

template <int kMode, int kW>
__global__ void __launch_bounds__(32 * kW, kW == kWarps ? 2 : 1) dispatch_kernel(DispatchArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    const SliceGeo g = slice_geo(kMode, a.H);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    zero_buffer<kW>(smem, g.stage_bytes);
    __syncthreads();

    const int64_t n_tok_units = (int64_t)a.T * g.ns;
    const int64_t stride = (int64_t)gridDim.x * kW;
    const int64_t u = (int64_t)blockIdx.x * kW + warp;

    Loads<kMode> nxt;
    if (!a.x_ready) {
        // x may still be written by the previous grid: only ask L2 for the
        // first units (a prefetch returns no value, and L2 is where every
        // write lands), and load them after the wait.
        const int64_t up = u + (int64_t)lane * stride;
        if (lane <= kPrefetchUnits && up < n_tok_units) {
            const int t = (int)(up / g.ns), s = (int)(up - (int64_t)t * g.ns);
            const int ne = min(kSliceElems, a.H - s * kSliceElems);
            const size_t eb = kMode == EP_X_FP8 ? 1 : 2;  // input bytes per element
            bulk_prefetch_l2((const char*)a.x + ((size_t)t * a.H + (size_t)s * kSliceElems) * eb,
                             (uint32_t)(ne * eb));
        }
    } else {
        // x is complete: load the first unit and ask L2 for the next few
        // while the layout finishes.
        nxt = load_x<kMode>(a, g, u, n_tok_units, lane);
        const int64_t up = u + (int64_t)(lane + 1) * stride;
        if (lane < kPrefetchUnits && up < n_tok_units) {
            const int t = (int)(up / g.ns), s = (int)(up - (int64_t)t * g.ns);
            const int ne = min(kSliceElems, a.H - s * kSliceElems);
            const size_t eb = kMode == EP_X_FP8 ? 1 : 2;  // input bytes per element
            bulk_prefetch_l2((const char*)a.x + ((size_t)t * a.H + (size_t)s * kSliceElems) * eb,
                             (uint32_t)(ne * eb));
        }
    }
    pdl_wait();
    if (!a.x_ready) nxt = load_x<kMode>(a, g, u, n_tok_units, lane);
    run_units<kMode, kW>(a, g, smem, u, nxt, ld_cg(a.num_pad_rows));
}

// --------------------------------------------------------------- row path
//
// Small batches (at most one layout chunk of slots, e.g. decode): a CTA
// takes whole token rows.  Each lane converts items of 16 consecutive
// elements (8 in bf16) into one shared row buffer -- a 1x128 block is 8
// lanes (3 shuffles), an NVFP4 block one lane -- so a row of hidden 7168
// takes two rounds of the CTA's threads (one in the 16-warp CTAs of the
// one-kernel layout path).  After a barrier lane 0 of warp j copies the
// whole row, and its scale row, to the receive row of slot j (j, j + the
// CTA's warps, ...) with one bulk copy each.  A decode launch (T=128, hidden
// 7168, FP8) took 4.19 us in warp units, whose copies are seven times as
// many and a seventh of the size.  Padding rows go one thread per row,
// slice by slice from a zeroed buffer.
constexpr int kRowWarps = 8;
// The one-kernel layout + dispatch takes 16-warp CTAs (one to an SM): a
// decode row converts in one round and the layout steps spread over twice
// the threads (the cached-handle launch measured faster with 8 warps).
constexpr int kLayoutWarps = 16;
constexpr int kLayoutThreads = 32 * kLayoutWarps;
static_assert(kLayoutChunkSlots % kLayoutThreads == 0, "a one-chunk layout spreads evenly over a CTA");

template <bool kLayout>
struct RowShape {
    static constexpr int kWarps = kLayout ? kLayoutWarps : kRowWarps;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kMinBlocks = kLayout ? 1 : 2;  // CTAs per SM the registers allow for
};
constexpr size_t kRowSmemMax = 96 * 1024;

template <int kMode>
struct RowItem {
    static constexpr int kElems = kMode == EP_X_BF16 ? 8 : 16;  // elements of an item
    static constexpr bool kTwoLoads = kMode == EP_X_BF16_TO_FP8 || kMode == EP_X_BF16_TO_NVFP4;  // 32 B of bf16
};

struct Item2 {
    uint4 v0, v1;
};

template <int kMode>
__device__ __forceinline__ Item2 row_load(const DispatchArgs& a, int t, int c, bool active) {
    Item2 it;
    it.v0 = it.v1 = make_uint4(0, 0, 0, 0);
    if (!active) return it;
    const size_t eb = kMode == EP_X_FP8 ? 1 : 2;  // input bytes per element
    const char* src = (const char*)a.x + ((size_t)t * a.H + (size_t)c * RowItem<kMode>::kElems) * eb;
    it.v0 = ld_stream(src);
    if (RowItem<kMode>::kTwoLoads) it.v1 = ld_stream(src + 16);
    return it;
}

// Converts item c of token t into the row buffer (and its block's scale
// into the scale buffer).  All 32 lanes of a warp call it together.
template <int kMode>
__device__ __forceinline__ void row_fill(const DispatchArgs& a, int t, int c, bool active, const Item2& it,
                                         unsigned char* rowbuf, unsigned char* sclbuf) {
    if (kMode == EP_X_BF16 || kMode == EP_X_FP8) {
        if (active) {
            reinterpret_cast<uint4*>(rowbuf)[c] = it.v0;
            if (kMode == EP_X_FP8 && (c & 7) == 0)
                reinterpret_cast<float*>(sclbuf)[c >> 3] = ld_cg(a.x_scales + (size_t)t * (a.H / 128) + (c >> 3));
        }
        return;
    }
    float f[16];
    unpack8(it.v0, f);
    unpack8(it.v1, f + 8);
    float amax = fmaxf(amax8(f), amax8(f + 8));
    if (kMode == EP_X_BF16_TO_FP8) {
        // a 1x128 block is 8 lanes (all active or all inactive: H % 128 == 0)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
        float scale, inv;
        fp8_scale(amax, scale, inv);
        const uint4 q = make_uint4(e4m3x4(f, inv), e4m3x4(f + 4, inv), e4m3x4(f + 8, inv), e4m3x4(f + 12, inv));
        if (active) {
            reinterpret_cast<uint4*>(rowbuf)[c] = q;
            if ((c & 7) == 0) reinterpret_cast<float*>(sclbuf)[c >> 3] = scale;
        }
    } else {
        float inv;
        const __nv_fp8_storage_t code = nvfp4_scale(amax, inv);  // the item is one 1x16 block
        const uint2 q = make_uint2(e2m1x8(f, inv), e2m1x8(f + 8, inv));
        if (active) {
            reinterpret_cast<uint2*>(rowbuf)[c] = q;
            sclbuf[c] = code;
        }
    }
}

__host__ __device__ inline size_t row_smem_bytes(const SliceGeo& g) {
    return (size_t)g.ns * g.out_bytes + (size_t)g.ns * g.sout_bytes + g.stage_bytes;  // row, scales, zeros
}

// ---- the layout inside every CTA (one-chunk batches through ep_layout_dispatch)
//
// With at most kLayoutChunkSlots slots there is no layout grid.  Every CTA
// reads all T*k expert indices into shared memory and computes what it
// needs: the per-expert counts and the counts before its first token
// (shared atomics), the aligned expert offsets (a scan over the experts),
// and, for each slot of its tokens, the number of earlier slots with the
// same expert (for its first token the prefix counts plus the token's own
// earlier slots; for later ones ballot counts over the index array), which
// gives the slot's row.  It writes the handle entries of its own slots and
// of the padding rows it zeroes.  The handle totals (per-expert arrays,
// tokens per segment) are written in slices by the CTAs without a token
// row, or by all CTAs when every CTA has one.  No CTA waits for another.

// Shared memory of the in-CTA layout, after the row buffers.
struct RowLayout {
    int* eidx;    // [T*k] expert of each slot, -1 when dropped
    int* cnt;     // [E]   slots of each expert
    int* pre;     // [E]   slots of each expert before the CTA's first token
    int* off;     // [E+1] first row of each expert
    int* padoff;  // [E+1] first padding index of each expert
    int* wsum;    // [2*kLayoutWarps] scan of the warps' sums
    float* w0;    // [kMaxTopk] weights of the CTA's first token's slots
    __device__ RowLayout(int* p, int n, int E) {
        eidx = p;
        cnt = eidx + n;
        pre = cnt + E;
        off = pre + E;
        padoff = off + E + 1;
        wsum = padoff + E + 1;
        w0 = reinterpret_cast<float*>(wsum + 2 * kLayoutWarps);
    }
};

__host__ __device__ inline size_t row_layout_bytes(int n, int E) {
    return sizeof(int) * ((size_t)n + 2 * (size_t)E + 2 * ((size_t)E + 1) + 2 * kLayoutWarps + kMaxTopk);
}

// off / padoff from cnt: aligned rows A(c) = ceil(c/a)*a and padding rows
// A(c) - c, scanned over the experts by kLayoutThreads threads, each taking a
// run of consecutive experts.  Barriers inside; ends with one.
__device__ __forceinline__ void row_expert_offsets(const RowLayout& L, int E, int align) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (E + kLayoutThreads - 1) / kLayoutThreads;
    const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
    int r = 0, p = 0;
    for (int e = e0; e < e1; ++e) {
        const int c = L.cnt[e], re = align == 1 ? c : (c + align - 1) / align * align;
        r += re;
        p += re - c;
    }
    int ri = r, pi = p;  // inclusive scan within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int ro = __shfl_up_sync(0xffffffffu, ri, o), po = __shfl_up_sync(0xffffffffu, pi, o);
        if (lane >= o) {
            ri += ro;
            pi += po;
        }
    }
    if (lane == 31) {
        L.wsum[warp] = ri;
        L.wsum[kLayoutWarps + warp] = pi;
    }
    __syncthreads();
    int rb = ri - r, pb = pi - p;
    for (int w = 0; w < warp; ++w) {
        rb += L.wsum[w];
        pb += L.wsum[kLayoutWarps + w];
    }
    for (int e = e0; e < e1; ++e) {
        const int c = L.cnt[e], re = align == 1 ? c : (c + align - 1) / align * align;
        L.off[e] = rb;
        L.padoff[e] = pb;
        rb += re;
        pb += re - c;
    }
    if (tid == kLayoutThreads - 1) {
        L.off[E] = rb;
        L.padoff[E] = pb;
    }
    __syncthreads();
}

// Row of padding index p: the expert by binary search on padoff.
__device__ __forceinline__ int row_pad_row(const RowLayout& L, int E, int p) {
    int lo = 0, hi = E;  // padoff[lo] <= p < padoff[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (L.padoff[mid] <= p) lo = mid;
        else hi = mid;
    }
    return L.off[lo] + L.cnt[lo] + (p - L.padoff[lo]);
}

// The in-CTA layout in two parts, so that the row conversion runs while
// the index loads are in flight.  row_layout_load issues the loads of the
// T*k expert indices (a thread takes kSlotsPerThread consecutive slots)
// and of the weights of the CTA's first token, and zeroes the counts;
// row_layout_count then (after a barrier) stores the indices, counts them
// per expert (and before the CTA's first token), and scans the offsets.
constexpr int kSlotsPerThread = kLayoutChunkSlots / kLayoutThreads;

// An index load issued where it stands (a volatile asm is not moved past
// the other volatile loads), so that it is in flight during the conversion.
template <typename IdxT>
__device__ __forceinline__ long long ld_idx(const IdxT* p) {
    static_assert(sizeof(IdxT) == 8 || sizeof(IdxT) == 4, "int32 or int64 indices");
    if constexpr (sizeof(IdxT) == 8) {
        long long v;
        asm volatile("ld.global.nc.s64 %0, [%1];" : "=l"(v) : "l"(p));
        return v;
    } else {
        int v;
        asm volatile("ld.global.nc.s32 %0, [%1];" : "=r"(v) : "l"(p));
        return v;
    }
}
// The two consecutive indices of a thread in one vector load (p aligned to
// the pair: 16 bytes for int64, 8 for int32): fewer load instructions and
// L2 requests for the same bytes, which every CTA of the grid reads.
template <typename IdxT>
__device__ __forceinline__ void ld_idx2(const IdxT* p, long long (&v)[2]) {
    if constexpr (sizeof(IdxT) == 8) {
        asm volatile("ld.global.nc.v2.s64 {%0, %1}, [%2];" : "=l"(v[0]), "=l"(v[1]) : "l"(p));
    } else {
        int a, b;
        asm volatile("ld.global.nc.v2.s32 {%0, %1}, [%2];" : "=r"(a), "=r"(b) : "l"(p));
        v[0] = a;
        v[1] = b;
    }
}
__device__ __forceinline__ float ld_weight(const float* p) {
    float v;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// Raw values (checked in row_layout_count) and, for threads below k, the
// weight of the CTA's first token's slot tid, kept in registers until then.
template <typename IdxT>
__device__ __forceinline__ void row_layout_load(const LayoutArgs& la, const RowLayout& L,
                                                long long (&ev)[kSlotsPerThread], float& w0) {
    const int E = la.h.num_experts, n = la.h.num_tokens * la.h.num_topk;
    const int tid = threadIdx.x;
    static_assert(kSlotsPerThread == 2, "ld_idx2 loads two slots");
    const int i0 = tid * kSlotsPerThread;
    if (i0 + kSlotsPerThread <= n && (reinterpret_cast<uintptr_t>(la.topk_idx) % (2 * sizeof(IdxT))) == 0) {
        ld_idx2((const IdxT*)la.topk_idx + i0, ev);
    } else {
#pragma unroll
        for (int r = 0; r < kSlotsPerThread; ++r) {
            const int i = i0 + r;
            ev[r] = i < n ? ld_idx((const IdxT*)la.topk_idx + i) : -1;
        }
    }
    w0 = 0.0f;
    if (tid < la.h.num_topk && la.topk_weights && (int)blockIdx.x < la.h.num_tokens)
        w0 = ld_weight(la.topk_weights + (size_t)blockIdx.x * la.h.num_topk + tid);
    for (int e = tid; e < E; e += kLayoutThreads) {
        L.cnt[e] = 0;
        L.pre[e] = 0;
    }
}

__device__ __forceinline__ void row_layout_count(const LayoutArgs& la, const RowLayout& L,
                                                 const long long (&ev)[kSlotsPerThread], float w0) {
    const int E = la.h.num_experts, n = la.h.num_tokens * la.h.num_topk;
    const int tid = threadIdx.x;
    if (tid < la.h.num_topk) L.w0[tid] = w0;
    __syncthreads();  // the counts are zero
    const int first = blockIdx.x * la.h.num_topk;  // the CTA's first slot
    const bool has_token = (int)blockIdx.x < la.h.num_tokens;
    bool bad = false;
#pragma unroll
    for (int r = 0; r < kSlotsPerThread; ++r) {
        const int i = tid * kSlotsPerThread + r;
        if (i < n) {
            // a value outside [-1, E) flags the error word and drops the slot
            const bool ok = ev[r] >= -1 && ev[r] < E;
            bad |= !ok;
            const int e = ok ? (int)ev[r] : -1;
            L.eidx[i] = e;
            if (e >= 0) {
                atomicAdd(&L.cnt[e], 1);
                if (has_token && i < first) atomicAdd(&L.pre[e], 1);
            }
        }
    }
    if (bad) atomicOr(la.h.error_word, EP_DEVERR_BAD_TOPK_IDX);
    __syncthreads();
    row_expert_offsets(L, E, la.h.expert_alignment);
}

// The rows of token t's slots into rows_s, and their handle entries.  Slot
// j is warp j % kLayoutWarps's: its row is off[e] plus the number of earlier
// slots (flat order) with expert e.  For the CTA's first token that is
// pre[e] plus the token's own earlier slots; for later ones (several tokens
// to a CTA) the slots are counted 128 at a time by ballots.
__device__ __forceinline__ void row_slots(const LayoutArgs& la, const RowLayout& L, int t, int* rows_s) {
    const int k = la.h.num_topk, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int j = warp; j < k; j += kLayoutWarps) {
        const int s = t * k + j;
        const int e = L.eidx[s];
        int row = -1;
        if (e >= 0) {
            int before = 0;
            if (t == (int)blockIdx.x) {  // the CTA's first token: pre counts the slots before it
                before = L.pre[e];
                for (int jj = 0; jj < j; ++jj) before += L.eidx[t * k + jj] == e;
            } else {
                for (int c = 0; c < s; c += 128) {
                    bool hit[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int i = c + 32 * q + lane;
                        hit[q] = i < s && L.eidx[i] == e;
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) before += __popc(__ballot_sync(0xffffffffu, hit[q]));
                }
            }
            row = L.off[e] + before;
            if (row >= la.h.max_recv_rows) {
                if (lane == 0) atomicOr(la.h.error_word, EP_DEVERR_CAPACITY);
                row = -1;
            } else if (!EP_CHECK(before < L.cnt[e], la.h.error_word)) {
                row = -1;  // the rank must fall inside the expert's slots (checked builds only)
            } else if (lane == 0) {
                la.h.recv_src[row] = s;
                if (la.recv_topk_idx) la.recv_topk_idx[row] = e;
                if (la.recv_topk_weights)
                    la.recv_topk_weights[row] =
                        !la.topk_weights ? 0.0f : t == (int)blockIdx.x ? L.w0[j] : __ldg(la.topk_weights + s);
            }
        }
        if (lane == 0) {
            la.h.slot_map[s] = row;
            rows_s[j] = row;
        }
    }
}

// The handle totals, in shares.  When the grid has CTAs without a token row
// (blockIdx.x >= T), those alone take the shares, so that the token CTAs
// end with their row copies; otherwise every CTA takes one.  Share b of G:
// the per-expert arrays of experts [E*b/G, E*(b+1)/G), and the token
// counts of segments g = b, b+G, ... (a token counts once in each segment
// one of its valid slots reaches; block sum of the threads' counts).
// Share 0 also writes offsets[E] and the padding count.
__device__ __forceinline__ void row_totals(const LayoutArgs& la, const RowLayout& L) {
    const int E = la.h.num_experts, S = la.h.num_segments, k = la.h.num_topk, T = la.h.num_tokens;
    const int tb = (int)gridDim.x > T ? T : 0;  // the first CTA with a share
    if ((int)blockIdx.x < tb) return;          // CTA-uniform
    const int b = blockIdx.x - tb, G = gridDim.x - tb, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int e0 = (int)((int64_t)E * b / G), e1 = (int)((int64_t)E * (b + 1) / G);
    for (int e = e0 + tid; e < e1; e += kLayoutThreads) {
        la.h.counts[e] = L.cnt[e];
        la.h.recv_counts[e] = L.off[e + 1] - L.off[e];
        la.h.offsets[e] = L.off[e];
    }
    if (b == 0 && tid == 0) {
        la.h.offsets[E] = L.off[E];
        *la.h.num_pad_rows = L.padoff[E];
    }
    const int per_seg = E / S;
    for (int gs = b; gs < S; gs += G) {
        const int lo = gs * per_seg, hi = lo + per_seg;  // the segment's experts
        int c = 0;
        for (int t = tid; t < T; t += kLayoutThreads) {
            bool has = false;
            for (int j = 0; j < k; ++j) {
                const int e = L.eidx[t * k + j];
                has |= e >= lo && e < hi;
            }
            c += has;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        __syncthreads();  // wsum is free
        if (lane == 0) L.wsum[warp] = c;
        __syncthreads();
        if (tid == 0) {
            int sum = 0;
            for (int w = 0; w < kLayoutWarps; ++w) sum += L.wsum[w];
            la.h.seg_tokens[gs] = sum;
        }
    }
}

// The row path.  kLayout: the in-CTA layout above (launched as the first
// grid of ep_layout_dispatch, so x too is read only after the wait);
// otherwise the routing comes from the handle the layout grid wrote.
template <int kMode, bool kLayout, typename IdxT>
__global__ void __launch_bounds__(RowShape<kLayout>::kThreads, RowShape<kLayout>::kMinBlocks)
    dispatch_row_kernel(DispatchArgs a, LayoutArgs la) {
    constexpr int kW = RowShape<kLayout>::kWarps, kT = RowShape<kLayout>::kThreads;
    using M = Mode<kMode>;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ int rows_s[kMaxTopk];
    const SliceGeo g = slice_geo(kMode, a.H);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    unsigned char* const rowbuf = smem;                                   // [ns][out_bytes]
    unsigned char* const sclbuf = smem + (size_t)g.ns * g.out_bytes;      // [ns][sout_bytes]
    unsigned char* const zeros = sclbuf + (size_t)g.ns * g.sout_bytes;    // [stage_bytes]
    const RowLayout L(reinterpret_cast<int*>(zeros + g.stage_bytes), kLayout ? a.T * a.k : 0,
                      kLayout ? la.h.num_experts : 0);
    char* const recv = (char*)a.recv_x;
    char* const rscl = (char*)a.recv_scales;
    const int k = a.k, T = a.T;
    const uint64_t keep = a.scales_ld > 0 ? l2_evict_last_policy() : 0;
    zero_buffer<kW>(zeros, g.stage_bytes);
    __syncthreads();

    // The thread's items of a row are c = warp*32 + lane + j*kT,
    // taken two at a time with both loads issued first.  The first pair of
    // the CTA's first row is loaded before the wait when x is already
    // complete (directly after the layout grid).
    const int ipr = a.H / RowItem<kMode>::kElems;
    const int c0 = warp * 32;
    Item2 fa, fb;
    const bool first_ok = blockIdx.x < (unsigned)T;
    if (a.x_ready && first_ok) {
        fa = row_load<kMode>(a, blockIdx.x, c0 + lane, c0 + lane < ipr);
        fb = row_load<kMode>(a, blockIdx.x, c0 + kT + lane, c0 + kT + lane < ipr);
    }
    pdl_wait();
    if (!a.x_ready && first_ok) {
        fa = row_load<kMode>(a, blockIdx.x, c0 + lane, c0 + lane < ipr);
        fb = row_load<kMode>(a, blockIdx.x, c0 + kT + lane, c0 + kT + lane < ipr);
    }
    bool have_first = first_ok && c0 < ipr;  // used by the first pass of the loop below
    long long ev[kSlotsPerThread];
    float w0 = 0.0f;
    if (kLayout) row_layout_load<IdxT>(la, L, ev, w0);
    bool laid_out = !kLayout;  // CTA-uniform

    const bool bulk_scl = M::kScales && a.bulk_scales;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        if (!kLayout && tid < k) rows_s[tid] = ld_cg(a.slot_map + (size_t)t * k + tid);
        for (int c = c0; c < ipr; c += 2 * kT) {
            const int ca = c + lane, cb = c + kT + lane;
            Item2 ia, ib;
            if (have_first) {
                ia = fa;
                ib = fb;
                have_first = false;
            } else {
                ia = row_load<kMode>(a, t, ca, ca < ipr);
                ib = row_load<kMode>(a, t, cb, cb < ipr);
            }
            row_fill<kMode>(a, t, ca, ca < ipr, ia, rowbuf, sclbuf);
            if (c + kT < ipr) row_fill<kMode>(a, t, cb, cb < ipr, ib, rowbuf, sclbuf);
        }
        if (kLayout) {
            if (!laid_out) {
                row_layout_count(la, L, ev, w0);
                laid_out = true;
            }
            row_slots(la, L, t, rows_s);
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (lane == 0) {  // warp j issues the copies of slots j, j + kW, ...
            for (int j = warp; j < k; j += kW) {
                const int row = rows_s[j];
                if (row >= 0 && row < a.max_rows) {
                    bulk_s2g(recv + (size_t)row * g.row_bytes, rowbuf, g.row_bytes);
                    if (bulk_scl) bulk_s2g(rscl + (size_t)row * g.srow_bytes, sclbuf, g.srow_bytes);
                } else if (row >= a.max_rows) {
                    atomicOr(a.error_word, EP_DEVERR_CAPACITY);
                }
            }
            bulk_commit();
            if (t + (int)gridDim.x < T) bulk_wait_read<0>();  // the buffer is refilled for the next token
        }
        if (M::kScales && !bulk_scl) {
            // MN-major scales, or scale rows that are not a multiple of 16 bytes: plain stores.
            const int B = a.H / M::kScaleBlock;
            for (int i = tid; i < k * B; i += blockDim.x) {
                const int row = rows_s[i / B];
                if (row >= 0 && row < a.max_rows) store_scale<kMode>(a, row, i % B, sclbuf, i % B, keep);
            }
        }
        __syncthreads();
    }

    if (!laid_out) row_layout_count(la, L, ev, w0);  // a CTA with no token (padding rows only)

    // Padding rows, one thread per row, slice by slice from the zero buffer.
    const int n_pad = kLayout ? L.padoff[la.h.num_experts] : ld_cg(a.num_pad_rows);
    for (int p = blockIdx.x * blockDim.x + tid; p < n_pad; p += gridDim.x * blockDim.x) {
        int row;
        if (kLayout) {
            row = row_pad_row(L, la.h.num_experts, p);
            la.h.pad_rows[p] = row;
            if (row < a.max_rows) {
                la.h.recv_src[row] = -1;
                if (la.recv_topk_idx) la.recv_topk_idx[row] = -1;
                if (la.recv_topk_weights) la.recv_topk_weights[row] = 0.0f;
            }
        } else {
            row = ld_cg(a.pad_rows + p);
        }
        if (row < 0 || row >= a.max_rows) {
            if (row >= a.max_rows) atomicOr(a.error_word, EP_DEVERR_CAPACITY);
            continue;
        }
        for (int s = 0; s < g.ns; ++s) {
            const int ne = min(kSliceElems, a.H - s * kSliceElems);
            bulk_s2g(recv + (size_t)row * g.row_bytes + (size_t)s * g.out_bytes, zeros, ne * g.out_bytes / kSliceElems);
            if (M::kScales && bulk_scales_ok<kMode>(a, ne))
                bulk_s2g(rscl + (size_t)row * g.srow_bytes + (size_t)s * g.sout_bytes, zeros,
                         ne / M::kScaleBlock * M::kScaleBytes);
        }
        bulk_commit();
        if (M::kScales) {
            constexpr int kPerSlice = kSliceElems / M::kScaleBlock;
            const int B = a.H / M::kScaleBlock;
            for (int b = 0; b < B; ++b)
                if (!bulk_scales_ok<kMode>(a, min(kSliceElems, a.H - (b / kPerSlice) * kSliceElems)))
                    store_scale<kMode>(a, row, b, nullptr, 0, keep);
        }
    }
    if (kLayout) row_totals(la, L);
    pdl_launch_dependents();
    bulk_wait_all();
}

constexpr int kTotalsCtas = 8;

template <int kMode, bool kLayout, typename IdxT>
cudaError_t launch_row_t(const DispatchArgs& a, const LayoutArgs& la, cudaStream_t stream) {
    const SliceGeo g = slice_geo(kMode, a.H);
    const size_t smem =
        row_smem_bytes(g) + (kLayout ? row_layout_bytes(a.T * a.k, la.h.num_experts) : 0);
    auto kernel = dispatch_row_kernel<kMode, kLayout, IdxT>;
    cudaError_t err;
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, RowShape<kLayout>::kThreads, smem);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t cap = (int64_t)device_sm_count() * per_sm;
    // With the layout: up to kTotalsCtas more CTAs than tokens take the
    // handle totals (row_totals), on SMs the token CTAs leave free.
    int64_t want = a.T + (kLayout ? std::min(la.h.num_segments, kTotalsCtas) : 0);
    const int64_t pad_ctas = ((int64_t)a.max_pad_rows + RowShape<kLayout>::kThreads - 1) / RowShape<kLayout>::kThreads;
    if (pad_ctas > want) want = pad_ctas;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(want < 1 ? 1 : (want < cap ? want : cap)));
    cfg.blockDim = dim3(RowShape<kLayout>::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    debug_launch(kLayout ? "dispatch_row_kernel(layout)" : "dispatch_row_kernel", kMode, cfg);
    return cudaLaunchKernelEx(&cfg, kernel, a, la);
}

// Whether a dispatch of this shape takes the row path: at most one layout
// chunk of slots, no SM budget, and a row buffer that fits.
bool row_path(const DispatchArgs& a, int mode) {
    return (int64_t)a.T * a.k <= kLayoutChunkSlots && sm_budget() == 0 &&
           row_smem_bytes(slice_geo(mode, a.H)) <= kRowSmemMax;
}

template <int kMode, int kW>
cudaError_t launch_w(const DispatchArgs& a, int max_ctas, cudaStream_t stream) {
    const SliceGeo g = slice_geo(kMode, a.H);
    const size_t smem = smem_bytes(g, kW);
    auto kernel = dispatch_kernel<kMode, kW>;
    cudaError_t err;
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 32 * kW, smem);
    if (err != cudaSuccess) return err;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    // Persistent grid, no larger than the work: the number of padding rows
    // is only known on the device, E*(alignment-1) bounds it.
    const int64_t cap = max_ctas > 0 ? max_ctas : (int64_t)device_sm_count() * per_sm;
    const int64_t units = (int64_t)a.T * g.ns + a.max_pad_rows;
    const int64_t want = (units + kW - 1) / kW;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(want < 1 ? 1 : (want < cap ? want : cap)));
    cfg.blockDim = dim3(32 * kW);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    debug_launch(kW == kWarps ? "dispatch_kernel" : "dispatch_kernel(budget)", kMode, cfg);
    return cudaLaunchKernelEx(&cfg, kernel, a);
}

// Under an SM budget of n: n CTAs of kBudgetWarps warps, each the size of
// an SM, so the grid holds at most n SMs.  Without one, batches of at most
// one layout chunk of slots take the row path.
template <int kMode>
cudaError_t launch_t(const DispatchArgs& a, cudaStream_t stream) {
    const int budget = sm_budget();
    if (budget > 0) return launch_w<kMode, kBudgetWarps>(a, budget, stream);
    if (row_path(a, kMode)) return launch_row_t<kMode, false, int>(a, LayoutArgs{}, stream);
    return launch_w<kMode, kWarps>(a, 0, stream);
}

template <int kMode>
cudaError_t launch_fused_m(const LayoutArgs& la, const DispatchArgs& a, bool idx_is_int64, cudaStream_t stream) {
    return idx_is_int64 ? launch_row_t<kMode, true, long long>(a, la, stream)
                        : launch_row_t<kMode, true, int>(a, la, stream);
}

}  // namespace

size_t dispatch_smem_bytes(ep_x_mode mode, int H) { return smem_bytes(slice_geo(mode, H), kBudgetWarps); }

cudaError_t launch_layout_dispatch_fused(const LayoutArgs& la, const DispatchArgs& a, ep_x_mode mode,
                                         bool idx_is_int64, cudaStream_t stream) {
    if (la.num_chunks != 1 || !row_path(a, mode) ||
        row_smem_bytes(slice_geo(mode, a.H)) + row_layout_bytes(a.T * a.k, la.h.num_experts) >
            kRowSmemMax)
        return cudaErrorNotSupported;
    switch (mode) {
        case EP_X_BF16: return launch_fused_m<EP_X_BF16>(la, a, idx_is_int64, stream);
        case EP_X_FP8: return launch_fused_m<EP_X_FP8>(la, a, idx_is_int64, stream);
        case EP_X_BF16_TO_FP8: return launch_fused_m<EP_X_BF16_TO_FP8>(la, a, idx_is_int64, stream);
        case EP_X_BF16_TO_NVFP4: return launch_fused_m<EP_X_BF16_TO_NVFP4>(la, a, idx_is_int64, stream);
    }
    return cudaErrorInvalidValue;
}

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
