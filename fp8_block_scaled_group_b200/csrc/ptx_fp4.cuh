// Inline-PTX building blocks for the NVFP4 kernels on sm_100a: the e4m3
// value of a code, the packed E2M1 conversion, the scale-factor copy into
// TMEM and the block-scaled MMA (kind::mxf4nvf4).
#pragma once

#include "ptx.cuh"

namespace fp8q {

// Exact value of an e4m3 code (1 sign, 4 exponent bits with bias 7, 3
// mantissa bits; exponent field 0 holds m * 2^-9). The NaN codes are not
// expected.
__device__ __forceinline__ float e4m3_value(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u;
    const uint32_t m = c & 7u;
    const float mag = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : static_cast<float>(m) * 0x1p-9f;
    return (c & 0x80u) ? -mag : mag;
}

// --------------------------------------------------------------- e2m1 --

// Eight fp32 -> eight E2M1 codes (round to nearest even, saturate to +-6)
// packed two to a byte, element 2j in the low nibble of byte j.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// ------------------------------------------- block-scaled NVFP4 (MMA) --

// Shared-memory descriptor of one scale-factor atom: 32 rows of 16 bytes,
// contiguous, read as four 8-row core matrices 128 bytes apart (stride
// offset), no swizzle, descriptor version 1. One core matrix spans the row,
// so the leading offset is unused.
__device__ __forceinline__ uint64_t smem_desc_sf_atom(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(128u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    return d;
}

// Copy one scale-factor atom (32 rows x 128 bits) from shared memory into
// TMEM columns taddr .. taddr+3 of every 32-lane quarter (the same 32 rows
// in each quarter). Ordered with this thread's later tcgen05.mma.
__device__ __forceinline__ void tmem_copy_sf_atom(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[tmem] (+)= (A . sfa) * (B . sfb)^T with packed E2M1 operands and one
// E4M3 scale per 16 elements of K (kind::mxf4nvf4, block16), one CTA,
// K = 64 per instruction. sfa/sfb are TMEM addresses of the scale columns.
__device__ __forceinline__ void mma_mxf4nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}

// Instruction descriptor of the block-scaled MMA above: A = B = E2M1
// (format 1 in bits 7-9 and 10-12), both K-major, N / 8 in bits 17-22,
// scale format E4M3 (bit 23 = 0), M / 16 in bits 24-28, scale-factor ids 0,
// dense K = 64.
__host__ __device__ constexpr uint32_t idesc_e2m1_ue4m3(uint32_t M, uint32_t N) {
    return (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

}  // namespace fp8q
