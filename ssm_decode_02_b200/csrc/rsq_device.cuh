// rsq_device.cuh -- device helpers of the quantized recurrent-state decode kernels.
//
// Inline PTX for sm_100a: mbarriers and bulk asynchronous copies (the TMA
// engine's 1-D form) that stage contiguous state tiles into shared memory,
// packed two-wide binary32 arithmetic (fma/mul/add .f32x2), byte permutes for
// code packing, and a Philox4x32-10 block function written from its published
// definition (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as
// 1, 2, 3", SC'11).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace rsq {

// ---------------------------------------------------------------------------
// Shared-memory addresses, mbarriers, bulk copies
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Arrive once on `bar` and add `bytes` to its expected transaction count.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// Arrive once on `bar` (release: this thread's earlier shared-memory writes
// are visible to threads that observe the phase complete).
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Bounded wait for the phase with the given parity to complete.  Returns false
// when the iteration limit is reached (the caller reports a timeout).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t max_iters) {
    for (uint32_t it = 0; it < max_iters; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// Shared-memory add with acquire-release semantics at CTA scope: the caller's
// earlier accesses (and, through a preceding __syncwarp, its warp's) happen
// before those of any thread that later reads the value it wrote.
__device__ __forceinline__ uint32_t atom_add_acq_rel_cta(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(smem_u32(p)), "r"(v)
                 : "memory");
    return old;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses 16-byte
// aligned) completing as a transaction on `bar`.  No multicast.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// ---------------------------------------------------------------------------
// Packed two-wide binary32 arithmetic (one instruction, two IEEE operations)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t pk(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void upk(uint64_t r, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
// d = a*b + c, rounded to nearest, per lane of the pair
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// rounding toward minus infinity
__device__ __forceinline__ uint64_t add2_rm(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rm.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// d = a*b + c rounded toward plus / minus infinity (exact product, one rounding)
__device__ __forceinline__ uint64_t fma2_rp(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rp.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fma2_rm(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rm.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// FP8 E4M3: two codes from two floats (round to nearest even, saturating to
// +-448); `hi` lands in the upper byte of the 16-bit result.
__device__ __forceinline__ uint32_t e4m3x2_from_f32(float hi, float lo) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}
// Two E4M3 codes (low byte first) to two floats (exact, through f16).
__device__ __forceinline__ void e4m3x2_to_f32(uint32_t two, float& lo, float& hi) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(two)));
    asm("{ .reg .f16 a, b; mov.b32 {a, b}, %2; cvt.f32.f16 %0, a; cvt.f32.f16 %1, b; }"
        : "=f"(lo), "=f"(hi) : "r"(h2));
}

// hi(a * b) + c (32-bit unsigned)
__device__ __forceinline__ uint32_t umulhi_add(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// (a & MASK) | bits in one logic operation (the mask an immediate, `bits` a register)
template <uint32_t MASK>
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t bits) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "n"(MASK), "r"(bits));
    return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// max over three values; a NaN in any input gives NaN
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
    float d;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float max_nan(float a, float b) {
    float d;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) {
    return __uint_as_float(bits16 << 16);
}

// ---------------------------------------------------------------------------
// Philox4x32-10 block function (SC'11): ten rounds; each round multiplies
// words 0 and 2 by the two Philox multipliers, xors the high halves into words
// 1 and 3 with the round key, and the key advances by the two Weyl increments.
// ---------------------------------------------------------------------------
struct U4 {
    uint32_t x, y, z, w;
};

// Round keys rk0[r], rk1[r] are the key advanced r times by the Weyl increments.
__device__ __forceinline__ U4 philox4x32_10(U4 c, const uint32_t (&rk0)[10], const uint32_t (&rk1)[10]) {
    constexpr uint32_t kMulA = 0xD2511F53u, kMulB = 0xCD9E8D57u;
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint32_t hiA = __umulhi(kMulA, c.x), loA = kMulA * c.x;
        const uint32_t hiB = __umulhi(kMulB, c.z), loB = kMulB * c.z;
        c = U4{hiB ^ c.y ^ rk0[round], loB, hiA ^ c.w ^ rk1[round], loA};
    }
    return c;
}

}  // namespace rsq
