// Device helpers shared by the layout, dispatch and combine kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "cgl.h"

namespace cgl {

constexpr uint32_t kErrRange = 1u << CGL_ERANGE;
constexpr uint32_t kErrCapacity = 1u << CGL_ECAPACITY;

constexpr int kMaxTopk = 32;
constexpr int kMaxExperts = 1024;

// OR an error bit into the caller's status word (error paths only).
__device__ __forceinline__ void report(uint32_t *status, uint32_t bit) {
    if (status != nullptr) atomicOr(status, bit);
}

// 16-byte global load through the non-coherent path, not kept in L1: every
// byte the copy kernels read is read once.
__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// 16-byte global load through the non-coherent path, allocated in L1: for
// reads whose other half of the 32-byte sector the next instruction reads.
__device__ __forceinline__ uint4 ld_nc_l1_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// 16-byte global store with the streaming (evict-first) cache hint.
__device__ __forceinline__ void st_cs_v4(void *p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// Two floats -> two E4M3 bytes, round to nearest even, finite values past 448
// clamp to +-448 (PTX cvt ... satfinite).  `lo` lands in bits 7:0.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two floats -> two BF16 values, round to nearest even.  `lo` lands in bits 15:0.
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Programmatic dependent launch (sm_90+).  The copy kernels are launched with
// programmatic stream serialisation: they may start while the kernel before
// them is still finishing, so they must griddep_wait() before reading anything
// it (or an earlier kernel) wrote.  No kernel here triggers its dependents
// early: each block's exit is its trigger, so the next kernel's blocks launch
// as this kernel's blocks finish instead of taking SM resources that this
// kernel's own blocks still need (measured: an early trigger cost 15% of the
// BF16 step).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Bulk asynchronous copy (TMA engine, no tensor map) of `bytes` from shared to
// global memory, tracked in the issuing thread's bulk group.  Both addresses
// 16-byte aligned, bytes a multiple of 16.  The shared data must have been
// made visible to the async proxy (fence_proxy_async) before the call.  Every
// bulk copy here writes receive rows that this kernel never reads again, so
// their L2 lines are marked evict-first: they drain to HBM during the copy
// kernel instead of during the next one (prefill step 151.9 -> 150.5 us: the
// combine no longer pays for the dispatch's dirty lines).
__device__ __forceinline__ void bulk_store(void *gdst, const void *ssrc, uint32_t bytes) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(ssrc);
    uint64_t policy;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;" ::"l"(gdst),
                 "r"(s), "r"(bytes), "l"(policy)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N committed bulk groups of this thread still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until every committed bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Order this thread's generic-proxy shared-memory writes before later async-proxy reads.
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Ask the TMA engine to bring `bytes` of global memory at `src` into L2 (no
// data lands in the SM; completion is not tracked).  src 16-byte aligned,
// bytes a multiple of 16.
__device__ __forceinline__ void prefetch_l2_bulk(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// 2^e as a float, for e in [-126, 127].
__device__ __forceinline__ float exp2_int(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// The block's scale and reciprocal.  IEEE: scale = amax_c / 448, inv = 448 /
// amax_c (correctly rounded divisions).  Power of two (UE8M0): scale = 2^e for
// the smallest integer e with 448 * 2^e >= amax_c, inv = 2^-e.  e starts from
// the exponent of the rounded quotient amax_c / 448, rounded up unless that
// quotient is a power of two; the rounding can leave it one off on either side
// of a power of two, so two comparisons of 448 * 2^e (exact in binary32) with
// amax_c settle it.  amax_c in [1e-4, FLT_MAX] keeps e in [-22, 120].
__device__ __forceinline__ void block_scale(float amax_c, bool pow2, float &scale, float &inv) {
    if (!pow2) {
        scale = __fdiv_rn(amax_c, 448.0f);
        inv = __fdiv_rn(448.0f, amax_c);
        return;
    }
    const uint32_t s = __float_as_uint(__fdiv_rn(amax_c, 448.0f));
    int e = (int)((s >> 23) & 0xFFu) - 127;
    if (s & 0x7FFFFFu) ++e;
    if (__fmul_rn(448.0f, exp2_int(e - 1)) >= amax_c) --e;
    if (__fmul_rn(448.0f, exp2_int(e)) < amax_c) ++e;
    scale = exp2_int(e);
    inv = exp2_int(-e);
}

// Widen the low / high BF16 of a 32-bit word to float (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Largest |value| among the 16 BF16 values in (a, b), as a float (exact: a
// maximum does not round).  The sign bits are cleared and the maximum taken on
// BF16 pairs (max.bf16x2), then between the two halves; NaN inputs are outside
// the contract (the pairwise maximum, like fmaxf, prefers the number).
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t p, uint32_t q) {
    uint32_t r;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(p), "r"(q));
    return r;
}
__device__ __forceinline__ float absmax16(const uint4 a, const uint4 b) {
    constexpr uint32_t kAbs = 0x7FFF7FFFu;
    const uint32_t m01 = bf16x2_max(a.x & kAbs, a.y & kAbs), m23 = bf16x2_max(a.z & kAbs, a.w & kAbs);
    const uint32_t m45 = bf16x2_max(b.x & kAbs, b.y & kAbs), m67 = bf16x2_max(b.z & kAbs, b.w & kAbs);
    const uint32_t m = bf16x2_max(bf16x2_max(m01, m23), bf16x2_max(m45, m67));
    return fmaxf(bf16_lo(m), bf16_hi(m));
}

// E4M3 codes of the 16 BF16 values in (a, b), each multiplied by inv first.
__device__ __forceinline__ uint4 quant16(const uint4 a, const uint4 b, float inv) {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = cvt_e4m3x2(__fmul_rn(bf16_lo(w[2 * i]), inv), __fmul_rn(bf16_hi(w[2 * i]), inv));
        const uint32_t hi =
            cvt_e4m3x2(__fmul_rn(bf16_lo(w[2 * i + 1]), inv), __fmul_rn(bf16_hi(w[2 * i + 1]), inv));
        q[i] = lo | (hi << 16);
    }
    return make_uint4(q[0], q[1], q[2], q[3]);
}

}  // namespace cgl
