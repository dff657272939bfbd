// The dense FFN's activation step: h = bf16(silu(gate) * up), then the
// per-token, per-128-group FP8 quantization of h for the down projection.
//
// Page "spark_model/layers/ops/dispatch_proj.rs", doc of
// `cublas_fp8_proj_prequant`: the FFN quantizes its input once for the gate
// and up projections and quantizes "the post-SiLU intermediate" once more
// for the down projection. The pages do not print the activation; this
// library defines h as the real value silu(g) * u = g * u / (1 + e^-g)
// rounded once to bf16 (nearest, ties to even), g and u being the bf16
// outputs of the gate and up projections.
//
// Evaluation. Fast path, fp32: p = g*u (exact: two 8-bit significands),
// v = p / (1 + e^-g) with the hardware exponential and reciprocal. v is
// within a few fp32 ulps of the real value, so rounding v to bf16 gives the
// right answer unless v lies near a bf16 rounding tie (bits 15..0 of v close
// to 0x8000). Such values, and results outside the range where the fp32
// evaluation is accurate (|v| below 2^-126 or from 2^126 up), take the slow
// path in fp64, which rounds exactly; for g > 32 the factor 1/(1+e^-g) is
// within 2^-46 of 1, p is either exactly a bf16 tie or at least 2^-17 |p|
// from one, and a tie goes toward zero because silu(g) < g.
// fp8q_check_silu_mul runs both paths on every pair of finite bf16 inputs
// and counts the pairs where the fast path is taken and disagrees with the
// slow one (zero on B200).
//
// Kernel: like the multi-group activation quantizer, 8 lanes own one
// 128-element group (16 elements per lane: two 16-byte loads of gate and two
// of up), 8 groups x 4 tokens per 64-thread CTA. h is packed back into bf16
// pairs and goes through exactly the quantizer's group arithmetic.
#include <cuda_bf16.h>

#include "group_quant.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace fp8q {

namespace {


// bf16 magnitude bits of a > 0 (finite double), nearest; ties to even, or
// toward zero when tie_down. Overflow gives +inf (0x7F80).
__device__ uint32_t bf16_magnitude_from_double(double a, bool tie_down) {
    if (a < 0x1p-126) {
        // subnormal bf16: multiples of 2^-133; a * 2^133 is exact
        const double x = a * 0x1p133;
        const double fl = floor(x);
        const double fr = x - fl;
        double n = fl;
        if (fr > 0.5 || (fr == 0.5 && !tie_down && fmod(fl, 2.0) != 0.0)) n = fl + 1.0;
        return static_cast<uint32_t>(n);  // 128 is the smallest normal, 0x0080
    }
    const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(a));
    const unsigned long long rem = b & ((1ull << 45) - 1ull);  // below bf16's 7 fraction bits
    unsigned long long t = b >> 45;                            // exponent(11) | fraction(7)
    const unsigned long long half = 1ull << 44;
    if (rem > half || (rem == half && !tie_down && (t & 1ull))) t += 1ull;
    // rebias 1023 -> 127; a carry out of the fraction bumps the exponent
    const unsigned long long h = t - (896ull << 7);
    return h >= 0x7F80ull ? 0x7F80u : static_cast<uint32_t>(h);
}

__device__ __noinline__ uint32_t silu_mul_slow(float g, float u) {
    const uint32_t sign = ((__float_as_uint(g) ^ __float_as_uint(u)) >> 16) & 0x8000u;
    const double p = static_cast<double>(g) * static_cast<double>(u);  // exact
    if (p == 0.0) return sign;
    if (g > 32.0f) return sign | bf16_magnitude_from_double(fabs(p), true);
    const double v = fabs(p / (1.0 + exp(-static_cast<double>(g))));
    if (v == 0.0) return sign;
    return sign | bf16_magnitude_from_double(v, false);
}

// log2(e) split as kLog2eHi + kLog2eLo (kLog2eHi = log2(e) rounded to
// fp32), and ln(2), for the exponential below.
constexpr float kLog2eHi = 1.44269502162933349609375f;
constexpr float kLog2eLo = 1.925963e-08f;
constexpr float kLn2 = 0.6931472f;
// Relative half-width of the interval around v that must round to one bf16
// value for the fast result to stand: 2^-20, i.e. 8 to 16 fp32 ulps of v.
constexpr float kTieBand = 0x1p-20f;

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Minimum and maximum that return NaN when either input is NaN.
__device__ __forceinline__ float min_nan(float a, float b) {
    float r;
    asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ float max_nan(float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ uint32_t bf16x2_rn(float2 v) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(v.y), "f"(v.x));
    return r;
}

// The fast fp32 evaluation of two elements: v = g*u / (1 + e^-g), returned
// in *v. The exponential is 2^y, y = -g*log2(e), with y carried as a
// rounded product plus its exact error (fma) and the product with the low
// part of log2(e) (Cody and Waite's argument splitting): 2^(yh + yl) =
// 2^yh * (1 + yl ln 2) to first order in the tiny yl. The quotient is the
// approximate reciprocal's product plus one remainder correction. The
// result is the packed bf16 rounding of v(1 + kTieBand); it stands (*ok)
// when v(1 - kTieBand) rounds to the same pair and both |v| lie in
// [2^-126, 2^126), where the evaluation is accurate. An overflowing g*u or
// e^-g shows up there as an infinite, zero or NaN v.
__device__ __forceinline__ uint32_t silu_mul_fast2(float2 g, float2 u, bool* ok, float2* v_out) {
    const float2 p = __fmul2_rn(g, u);  // exact for normal results: two 8-bit significands
    const float2 L = make_float2(kLog2eHi, kLog2eHi);
    const float2 yh = __fmul2_rn(g, L);                                   // g log2(e), rounded
    const float2 yerr = __ffma2_rn(g, L, make_float2(-yh.x, -yh.y));      // its exact error
    const float2 yl = __ffma2_rn(g, make_float2(kLog2eLo, kLog2eLo), yerr);
    const float2 t = make_float2(ex2_approx(-yh.x), ex2_approx(-yh.y));  // 2^-yh
    const float2 e = __ffma2_rn(t, __fmul2_rn(yl, make_float2(-kLn2, -kLn2)), t);
    const float2 d = __fadd2_rn(e, make_float2(1.0f, 1.0f));
    const float2 r = make_float2(rcp_approx(d.x), rcp_approx(d.y));
    const float2 v0 = __fmul2_rn(p, r);
    const float2 v = __ffma2_rn(__ffma2_rn(make_float2(-v0.x, -v0.y), d, p), r, v0);
    const uint32_t hi = bf16x2_rn(__fmul2_rn(v, make_float2(1.0f + kTieBand, 1.0f + kTieBand)));
    const uint32_t lo = bf16x2_rn(__fmul2_rn(v, make_float2(1.0f - kTieBand, 1.0f - kTieBand)));
    // NaN-propagating, so a NaN v (overflowed g*u or e^-g) fails both tests
    const float vmin = min_nan(fabsf(v.x), fabsf(v.y));
    const float vmax = max_nan(fabsf(v.x), fabsf(v.y));
    *ok = hi == lo && vmin >= 0x1p-126f && vmax < 0x1p126f;
    *v_out = v;
    return hi;
}

// 8 packed bf16 gates and ups -> 8 packed bf16 h. Pairs the fast path
// cannot settle (rare) go through the fp64 path, in a branch the whole warp
// takes only when some lane needs it.
__device__ __forceinline__ uint4 silu_mul8(const uint4 g, const uint4 u) {
    float gf[8], uf[8];
    widen8(g, gf);
    widen8(u, uf);
    uint32_t h[4];
    uint32_t ok = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        bool okj;
        float2 v;
        h[j] = silu_mul_fast2(make_float2(gf[2 * j], gf[2 * j + 1]), make_float2(uf[2 * j], uf[2 * j + 1]), &okj, &v);
        ok |= (okj ? 1u : 0u) << j;
    }
    if (__any_sync(0xFFFFFFFFu, ok != 0xFu)) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (!(ok & (1u << j)))
                h[j] = silu_mul_slow(gf[2 * j], uf[2 * j]) | (silu_mul_slow(gf[2 * j + 1], uf[2 * j + 1]) << 16);
    }
    return make_uint4(h[0], h[1], h[2], h[3]);
}

// 1-D grid of ceil(G/8) * m CTAs of 64 threads: CTA t * ceil(G/8) + bx
// handles token t, and its octet o owns group 8*bx + o. Row t of gate
// starts at gate + t*ld, likewise up.
// Waits on the grid it depends on (the gate/up projection, when launched as
// its programmatic dependent) before loading.
__global__ void __launch_bounds__(64) silu_mul_quant_kernel(const uint16_t* __restrict__ gate,
                                                           const uint16_t* __restrict__ up, uint32_t ld,
                                                           uint8_t* __restrict__ q, float* __restrict__ s_row,
                                                           float* __restrict__ s_k, uint32_t m, uint32_t i,
                                                           uint32_t mp) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (blockIdx.x + kMultiTriggerTail >= gridDim.x) trigger_dependents();
    const uint32_t G = i >> 7;
    const uint32_t gx = (G + 7) >> 3;
    const uint32_t t = blockIdx.x / gx;
    const uint32_t lane = threadIdx.x & 7;
    const uint32_t g = (blockIdx.x - t * gx) * 8 + (threadIdx.x >> 3);
    const bool g_ok = g < G;
    uint4 a0, a1, b0, b1;
    if (g_ok) {
        const size_t off = static_cast<size_t>(t) * ld + static_cast<size_t>(g) * 128 + lane * 8;
        a0 = ld_stream16(gate + off);
        a1 = ld_stream16(gate + off + 64);
        b0 = ld_stream16(up + off);
        b1 = ld_stream16(up + off + 64);
    } else {
        a0 = a1 = b0 = b1 = make_uint4(0u, 0u, 0u, 0u);
    }
    const uint4 h0 = silu_mul8(a0, b0);
    const uint4 h1 = silu_mul8(a1, b1);
    float amax = fmaxf(absmax8_bits(h0), absmax8_bits(h1));
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    const float s = group_scale(amax);
    float f0[8], f1[8];
    widen8(h0, f0);
    widen8(h1, f1);
    const uint2 c0 = encode8(f0, s);
    const uint2 c1 = encode8(f1, s);
    if (g_ok) {
        uint8_t* dst = q + static_cast<size_t>(t) * i + static_cast<size_t>(g) * 128 + lane * 8;
        st_stream8(dst, c0);
        st_stream8(dst + 64, c1);
        if (lane == 0) {
            if (s_row) s_row[static_cast<size_t>(t) * G + g] = s;
            s_k[static_cast<size_t>(g) * mp + t] = s;
        }
    }
    zero_kmajor_pad(s_k, m, mp, G);
}

// Exhaustive check of the fast path: CTA b takes the gate with bf16 bits b
// (non-finite patterns skipped) and runs every finite bf16 up through both
// paths. counts[0] += pairs, counts[1] += pairs where the fast path is taken,
// counts[2] += pairs where it is taken and differs from the slow path.
// max_err_bits: the largest |v - v64| in fp32 ulps of v over the taken
// pairs, v the fast fp32 value and v64 the fp64 evaluation (as an fp32 bit
// pattern, atomicMax).
__global__ void __launch_bounds__(256) check_silu_mul_kernel(unsigned long long* __restrict__ counts,
                                                             uint32_t* __restrict__ max_err_bits) {
    const uint32_t gb = blockIdx.x;
    unsigned long long pairs = 0, taken = 0, bad = 0;
    float worst = 0.0f;
    if ((gb & 0x7F80u) != 0x7F80u) {
        const float g = __uint_as_float(gb << 16);
        for (uint32_t ub = threadIdx.x; ub < 0x10000u; ub += blockDim.x) {
            if ((ub & 0x7F80u) == 0x7F80u) continue;
            const float u = __uint_as_float(ub << 16);
            bool ok;
            float2 v;
            const uint32_t hf = silu_mul_fast2(make_float2(g, g), make_float2(u, u), &ok, &v) & 0xFFFFu;
            ++pairs;
            if (!ok) continue;
            ++taken;
            bad += hf != silu_mul_slow(g, u);
            const double vd = static_cast<double>(g) * static_cast<double>(u) / (1.0 + exp(-static_cast<double>(g)));
            const int e = static_cast<int>((__float_as_uint(v.x) >> 23) & 0xFF) - 127 - 23;  // ulp of v = 2^e
            worst = fmaxf(worst, static_cast<float>(ldexp(fabs(static_cast<double>(v.x) - vd), -e)));
        }
    }
    for (int o = 16; o > 0; o >>= 1) {
        pairs += __shfl_xor_sync(0xFFFFFFFFu, pairs, o);
        taken += __shfl_xor_sync(0xFFFFFFFFu, taken, o);
        bad += __shfl_xor_sync(0xFFFFFFFFu, bad, o);
        worst = fmaxf(worst, __shfl_xor_sync(0xFFFFFFFFu, worst, o));
    }
    if ((threadIdx.x & 31) == 0) {
        atomicAdd(&counts[0], pairs);
        atomicAdd(&counts[1], taken);
        atomicAdd(&counts[2], bad);
        atomicMax(max_err_bits, __float_as_uint(worst));
    }
}

}  // namespace

cudaError_t launch_silu_mul_quant(const SiluLaunch& L, bool pdl, cudaStream_t stream) {
    const uint32_t G = L.i >> 7;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(((G + 7) / 8) * L.m, 1, 1);
    cfg.blockDim = dim3(64, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, silu_mul_quant_kernel, static_cast<const uint16_t*>(L.gate),
                                       static_cast<const uint16_t*>(L.up), L.ld, static_cast<uint8_t*>(L.q),
                                       L.s_row, L.s_k, L.m, L.i, L.mp);
    note_launch();
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_check_silu_mul(unsigned long long* counts, uint32_t* max_err_bits, cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(counts, 0, 3 * sizeof(unsigned long long), stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(max_err_bits, 0, sizeof(uint32_t), stream);
    if (e != cudaSuccess) return e;
    check_silu_mul_kernel<<<0x10000, 256, 0, stream>>>(counts, max_err_bits);
    note_launch();
    return cudaGetLastError();
}

}  // namespace fp8q
