// Device-side helpers shared by the kernels: element types, mbarriers and TMA
// tile loads written as inline PTX for sm_100a, and the error word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pa.h"

namespace pa {

// ------------------------------------------------------------------ element types

struct F16Tag {
    using T = __half;
    static constexpr int kBytes = 2;
    static constexpr bool kIsBF16 = false;
    // widen two packed 16-bit values (low half first) to fp32
    static __device__ __forceinline__ float2 widen2(uint32_t w) {
        return __half22float2(*reinterpret_cast<const __half2*>(&w));
    }
    static __device__ __forceinline__ uint16_t round1(float x) {
        __half h = __float2half_rn(x);
        return *reinterpret_cast<uint16_t*>(&h);
    }
};

struct BF16Tag {
    using T = __nv_bfloat16;
    static constexpr int kBytes = 2;
    static constexpr bool kIsBF16 = true;
    static __device__ __forceinline__ float2 widen2(uint32_t w) {
        // a bfloat16 is the top half of a binary32: widening is a shift
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    static __device__ __forceinline__ uint16_t round1(float x) {
        __nv_bfloat16 h = __float2bfloat16_rn(x);
        return *reinterpret_cast<uint16_t*>(&h);
    }
};

// 2^x by the hardware's approximate base-2 exponential (MUFU), subnormal
// results flushed to zero; exp2(-inf) = 0.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// OCP FP8 E4M3 cache elements (1 byte).  Widening goes through the hardware's exact
// e4m3x2 -> f16x2 conversion, then f16 -> f32 (both exact).
struct E4M3Tag {
    static constexpr int kBytes = 1;
    // widen two packed codes (low byte first) to fp32
    static __device__ __forceinline__ float2 widen2(uint32_t pair16) {
        uint32_t h;
        const unsigned short in = (unsigned short)pair16;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(in));
        return __half22float2(*reinterpret_cast<const __half2*>(&h));
    }
    // two packed codes (low byte first) as an exact f16x2 pair (low half first)
    static __device__ __forceinline__ uint32_t to_f16x2(uint32_t pair16) {
        uint32_t h;
        const unsigned short in = (unsigned short)pair16;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(in));
        return h;
    }
    // nearest codes of two floats (round to nearest even, saturating at +-448), lo in the low byte
    static __device__ __forceinline__ uint32_t encode2(float lo, float hi) {
        unsigned short d;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
        return d;
    }
};

// Power-of-two scale that enters 16-bit values of a wider range (bf16) into f16
// arithmetic: given their largest magnitude mx, s = 2^k brings it to [2^14, 2^15)
// (k clamped so that s and 1/s are normal floats).  x * s is then exact in f16
// for every |x| >= 2^-31 mx; smaller ones round to f16's subnormal grid.
__device__ __forceinline__ void f16_entry_scale(float mx, float& s, float& s_inv) {
    const int ebits = (int)((__float_as_uint(mx) >> 23) & 0xffu);
    const int k = ebits == 0 ? 0 : max(-114, min(126, 141 - ebits));
    s = __uint_as_float((uint32_t)(127 + k) << 23);
    s_inv = __uint_as_float((uint32_t)(127 - k) << 23);
}

// (lo, hi) -> f16x2, lo in the low half
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// ------------------------------------------------------------------- error word

__device__ __forceinline__ void report(int32_t* err_word, int bits) {
    if (err_word) atomicOr(err_word, bits);
}

// --------------------------------------------------------------------- mbarrier

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// One poll of an mbarrier phase.  The thread may be suspended by the hardware for
// up to `hint_ns` while the phase is still open (it resumes as soon as the phase
// completes), so a waiting warp sleeps instead of spinning on issue slots.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Every wait in the library is bounded: after kWaitPolls polls of at most
// kWaitHintNs each (about 2 s in all) the caller gives up, reports
// PA_DEVERR_TIMEOUT and unwinds.
#ifndef PA_WAIT_HINT_NS
#define PA_WAIT_HINT_NS 20000
#endif
constexpr uint32_t kWaitHintNs = PA_WAIT_HINT_NS;
constexpr uint32_t kWaitPolls = 2000000000u / kWaitHintNs;

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitPolls; ++i)
        if (mbar_try_wait(bar, parity, kWaitHintNs)) return true;
    return false;
}

// ------------------------------------------------------------------------- TMA

// One tiled tensor copy global -> shared, completion counted in bytes on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// Same, with an L2 eviction-priority hint (a createpolicy value).
__device__ __forceinline__ void tma_load_3d_hint(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                                 uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Orders this thread's earlier shared-memory accesses (generic proxy) before
// later bulk-copy (async proxy) accesses to the same shared memory.
__device__ __forceinline__ void fence_proxy_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Named barrier over `count` threads (a multiple of 32), id 1..15.
__device__ __forceinline__ void named_barrier(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

}  // namespace pa
