// Per-128-group quantization arithmetic shared by the kernels that emit FP8
// activations (the activation quantizers, and SiLU(gate)*up for the FFN's
// down projection): streaming loads and stores, bf16 widening, the group
// amax, the scale max(amax, 1e-10)/448 and the codes e4m3_rne_satfinite(x/s)
// (pages "spark_model/layers/ops/dispatch_proj.rs", `cublas_fp8_proj`, and
// "spark_model/layers/ops/fp8_act_quant_floor.rs", module header).
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace fp8q {

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_stream8(void* p, uint2 v) {
    asm volatile("st.global.cs.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

// 8 packed bf16 -> 8 fp32 (exact widening).
__device__ __forceinline__ void widen8(const uint4 v, float (&f)[8]) {
    f[0] = __uint_as_float(v.x << 16);
    f[1] = __uint_as_float(v.x & 0xFFFF0000u);
    f[2] = __uint_as_float(v.y << 16);
    f[3] = __uint_as_float(v.y & 0xFFFF0000u);
    f[4] = __uint_as_float(v.z << 16);
    f[5] = __uint_as_float(v.z & 0xFFFF0000u);
    f[6] = __uint_as_float(v.w << 16);
    f[7] = __uint_as_float(v.w & 0xFFFF0000u);
}

// |x| maximum of 8 packed bf16, as fp32. With the sign bits cleared, finite
// non-negative IEEE values order like their bit patterns, so the maximum is
// taken on the integers, two 16-bit lanes at a time.
__device__ __forceinline__ float absmax8_bits(const uint4 v) {
    const uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
    const uint32_t hi = m >> 16, lo = m & 0xFFFFu;
    return __uint_as_float((hi > lo ? hi : lo) << 16);
}

// The scale of a group with absolute maximum `amax`: RN(max(amax, 1e-10)/448),
// the correctly rounded fp32 quotient, formed with Markstein's correction
// (P. Markstein, IBM J. Res. Dev. 34(1), 1990) from c = RN(1/448):
//   q0 = RN(a c),  e = RN(a - 448 q0) (exact with a fused multiply-add),
//   s  = RN(q0 + e c).
// amax is the largest |x| of a group of bf16 values, so a takes at most
// 20645 distinct values (1e-10 and the bf16 values above it);
// fp8q_check_division compares this with IEEE division on every one of them.
constexpr float kInv448 = 0x1.24924ap-9f;  // RN(1/448)
__device__ __forceinline__ float group_scale(float amax) {
    const float a = fmaxf(amax, 1e-10f);
    const float q0 = __fmul_rn(a, kInv448);
    const float e = __fmaf_rn(-q0, 448.0f, a);
    return __fmaf_rn(e, kInv448, q0);
}

// -RN(1/s) for a group scale s: the hardware reciprocal approximation
// (rcp.approx, within an ulp) refined by one Newton-Raphson step with a
// fused multiply-add, r = r0 + r0 (1 - s r0), then negated. Group scales
// take at most 20645 values (see group_scale), and fp8q_check_division
// compares this with the correctly rounded reciprocal on every one of them.
__device__ __forceinline__ float neg_recip(float s) {
    float r0;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(s));
    const float e = __fmaf_rn(-s, r0, 1.0f);
    return -__fmaf_rn(r0, e, r0);
}

// The negated quotient -(x / s) for a pair of values, rounded to nearest
// even, from nr = -RN(1/s) and one remainder correction (Markstein's
// division scheme, P. Markstein, IBM J. Res. Dev. 34(1), 1990):
//   q0 = RN(x * nr) = -RN(x / s approx.),
//   e  = RN(q0 * s + x)   (the exact remainder, with a fused multiply-add),
//   q  = RN(e * nr + q0).
// Every step is the negation of the scheme run on +r, because rounding to
// nearest is symmetric, so q is exactly -(the scheme's quotient) for x != 0.
// For x = +-0 the zeros come out with the sign of -x (-0 + +0 = +0 in round
// to nearest), so negating the result's code gives the code of a zero with
// the sign of x, with no per-element sign repair. For every pair (x, amax) of
// bf16 values with |x| <= amax, the code this gives, sign-flipped, equals the
// code of the IEEE quotient x / s: fp8q_check_division verifies it
// exhaustively on the device.
__device__ __forceinline__ float2 neg_div2_by_scale(float2 x, float s, float nr) {
    const float2 q0 = __fmul2_rn(x, make_float2(nr, nr));
    const float2 e = __ffma2_rn(q0, make_float2(s, s), x);
    return __ffma2_rn(e, make_float2(nr, nr), q0);
}

// e4m3 codes of -v are those of v with the sign bit flipped (round to
// nearest even and saturation to +-448 are symmetric); four codes per word.
constexpr uint32_t kCodeSignBits = 0x80808080u;

// 8 values / s -> 8 codes packed little-endian, given nr = -RN(1/s).
__device__ __forceinline__ uint2 encode8_nr(const float (&f)[8], float s, float nr) {
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 q = neg_div2_by_scale(make_float2(f[2 * i], f[2 * i + 1]), s, nr);
        c[i] = cvt_e4m3x2(q.x, q.y);
    }
    return make_uint2((c[0] | (c[1] << 16)) ^ kCodeSignBits, (c[2] | (c[3] << 16)) ^ kCodeSignBits);
}

__device__ __forceinline__ uint2 encode8(const float (&f)[8], float s) {
    return encode8_nr(f, s, neg_recip(s));
}

// max(|a|, |b|) of two pairs of packed bf16 per half (the sign bit of each
// result half is the xor of the inputs' signs: clear it before use).
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Let a dependent kernel (the GEMM of a fused linear, launched with
// programmatic stream serialization) start its set-up while this grid runs.
// The dependent may launch once every CTA has either triggered or exited.
// Measured on B200: when every CTA triggers, the GEMM launches as soon as
// the last quantizer CTA has started, which takes ~0.7 us off a
// decode-width linear; but on grids of about 2000 or more of these small
// CTAs, triggering from all of them slows the quantizer itself by ~0.6 us.
// So the single-group kernel triggers only on grids of at most 1024 CTAs,
// and the multi-group kernel only from its last 2048 CTAs.
constexpr uint32_t kSingleTriggerMaxGrid = 1024;
constexpr uint32_t kMultiTriggerTail = 2048;

__device__ __forceinline__ void trigger_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Zero the pad rows m..mp-1 of the K-major scales, spread over the grid.
__device__ __forceinline__ void zero_kmajor_pad(float* __restrict__ s_k, uint32_t m, uint32_t mp, uint32_t G) {
    const uint32_t pad = mp - m;
    if (pad == 0) return;
    const uint32_t nblk = gridDim.x * gridDim.y;
    const uint32_t bid = blockIdx.y * gridDim.x + blockIdx.x;
    const uint32_t total = pad * G;
    for (uint32_t p = bid * blockDim.x + threadIdx.x; p < total; p += nblk * blockDim.x) {
        const uint32_t g = p / pad;
        s_k[static_cast<size_t>(g) * mp + m + (p - g * pad)] = 0.0f;
    }
}

}  // namespace fp8q
