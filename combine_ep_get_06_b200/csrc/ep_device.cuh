// Device helpers shared by the kernels: vector loads / stores with cache
// hints, bf16 / e4m3 conversions, TMA bulk copies and programmatic
// dependent launch.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ep.h"

namespace ep {

// Checked builds (EP_CHECKED defined): EP_CHECK(cond, word) evaluates an
// invariant that the kernels' own logic already guarantees; when it fails
// it sets EP_DEVERR_CHECK in the error word and yields false, so that the
// caller skips the access.  Never traps.  Production builds compile it to
// `true`.
#ifdef EP_CHECKED
#define EP_CHECK(cond, word) ((cond) ? true : (atomicOr((word), EP_DEVERR_CHECK), false))
#else
#define EP_CHECK(cond, word) true
#endif

// 16-byte load of streamed data that does not allocate in L1 (every byte
// is read once).  Not the non-coherent path: with programmatic dependent
// launch the data may come from the grid that ran just before.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 16-byte store of output that this kernel does not read again.
__device__ __forceinline__ void st_stream(void* p, const uint4& v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// Coherent (L2) scalar loads, for data the previous grid may have written.
__device__ __forceinline__ int ld_cg(const int* p) { return __ldcg(p); }
__device__ __forceinline__ float ld_cg(const float* p) { return __ldcg(p); }

// Two packed bf16 (low half first) -> two floats, exactly.
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Two floats -> two bf16, round to nearest-even, a in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Two floats -> two e4m3 bytes (a in the low byte), round to nearest-even,
// saturating finite values to +-448.
__device__ __forceinline__ uint32_t pack_e4m3x2(float a, float b) {
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// ---- programmatic dependent launch (no-ops when launched without it)

// Blocks until the grids this one depends on have completed and their
// memory is visible.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next grid in the stream begin launching.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- TMA bulk copies shared -> global (one destination each)

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Makes this thread's generic-proxy shared-memory writes visible to the
// async proxy (the TMA engine) before a bulk copy reads them.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Orders this thread's completed bulk-copy writes to global memory (async
// proxy) with its later generic-proxy accesses and fences.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// bytes: multiple of 16; both addresses 16-byte aligned.
__device__ __forceinline__ void bulk_s2g(void* gdst, const void* ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
                 "r"(smem_addr(ssrc)), "r"(bytes)
                 : "memory");
}

// Asks the TMA engine to bring [p, p + bytes) into L2 (no shared memory,
// no completion to wait for).  p 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
// An L2 prefetch of the 16-byte aligned part of [lo, hi): it never reaches
// past either end of the range.
__device__ __forceinline__ void prefetch_interior_l2(const void* lo, const void* hi) {
    const uintptr_t a = ((uintptr_t)lo + 15) & ~(uintptr_t)15, b = (uintptr_t)hi & ~(uintptr_t)15;
    if (b > a) bulk_prefetch_l2((const void*)a, (uint32_t)(b - a));
}

// An L2 evict-last policy (createpolicy) and a store that takes one.
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void st_f32_hint(float* p, float v, uint64_t policy) {
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(policy) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until at most N committed groups of this thread still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Waits until all committed groups of this thread have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

}  // namespace ep
