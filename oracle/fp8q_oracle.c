/*
 * fp8q oracle — TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct CPU restatement of the W8A8 FP8
 * block-scaled linear projection described on the pages
 * "spark_model/layers/ops/dispatch_proj.rs" (doc comments of
 * `cublas_fp8_proj`, `cublas_fp8_proj_prequant`, `fp8_act_scale_to_kmajor`,
 * `cublas_fp8_m_pad`, `dequant_fp8_bf16_into`) and
 * "spark_model/layers/ops/fp8_act_quant_floor.rs" (module header).
 *
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * may load this library. The product path (libfp8q.so) never links, loads or
 * calls it, and the two share no code, header, table or helper.
 *
 * The pages name the activation quantizer (`per_token_group_quant_fp8`,
 * "FP8 + per-[token,128-of-K] scales", "FP32 activation scales", "FP8 E4M3")
 * but never print its body. The arithmetic here is the method's standard
 * definition, written out step by step:
 *   amax  = max_j |x_j|                       over one 128-wide K group
 *   s     = max(amax, 1e-10f) / 448.0f        one IEEE fp32 division
 *   q_j   = e4m3_rne_satfinite(x_j / s)       IEEE fp32 division, then
 *                                             round-to-nearest-even into
 *                                             OCP E4M3FN, saturating at 448
 * Precision: the scale and the quotients are fp32 (the pages fix FP32
 * scales); the code decision is taken on that fp32 quotient. The encoder
 * works in double, where every step below is exact.
 *
 * Beyond the FP8 linear it restates the dense FFN's SiLU(gate) * up step,
 * the per-row weight format, the FP8-to-bf16 weight dequantizer and the
 * NVFP4 projection arms (E2M1 elements with E4M3 scales per 16 along K);
 * each section states its own reading of the pages.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared (no -ffast-math, no -ffp-contract
 * beyond "off": fp32 results must be IEEE single-rounded).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#if !defined(FLT_EVAL_METHOD) || FLT_EVAL_METHOD != 0
#error "the oracle needs fp32 expressions evaluated in fp32 (FLT_EVAL_METHOD == 0)"
#endif

#define GROUP 128            /* K-group width and weight block edge */
#define E4M3_MAX 448.0       /* largest finite OCP E4M3FN magnitude */

/* ---------------------------------------------------------------- bf16 -- */

/* bf16 is the top half of an IEEE binary32: widening is a 16-bit shift. */
float oracle_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ---------------------------------------------------------------- e4m3 -- */

/*
 * Decode one OCP E4M3FN code ("FP8 E4M3", dispatch_proj.rs,
 * `dequant_fp8_bf16_into` doc: every such value is exactly a bf16).
 * Layout: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
 * Exponent field 0 holds subnormals m/8 * 2^-6. The only NaNs are
 * S.1111.111; there is no infinity.
 */
double oracle_e4m3_decode(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* Round a non-negative double to the nearest integer, ties to even. */
static double round_half_even(double v)
{
    double f = floor(v);
    double frac = v - f; /* exact for the values used here */
    if (frac > 0.5)
        return f + 1.0;
    if (frac < 0.5)
        return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/*
 * Encode one finite fp32 value into E4M3FN with round-to-nearest-even and
 * saturation to the largest finite value (448), keeping the sign of zero.
 *   |t| >= 448           -> 0x7E | sign (values in (448,464) round to 448
 *                           anyway; larger ones would round to 480, which the
 *                           format cannot hold, so saturation clamps them)
 *   |t| <  2^-6          -> subnormal: mantissa = RNE(|t| / 2^-9); a result
 *                           of 8 is the smallest normal, code 0x08
 *   otherwise            -> e = floor(log2 |t|), mantissa = RNE((|t|/2^e - 1)*8);
 *                           a mantissa of 8 carries into the exponent
 */
uint8_t oracle_e4m3_encode(float t)
{
    uint8_t sign = signbit(t) ? 0x80 : 0x00;
    double a = fabs((double)t);
    int e;
    double r;
    if (a >= E4M3_MAX)
        return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {
        r = round_half_even(a * 512.0); /* a / 2^-9, exact */
        return (uint8_t)(sign | (uint8_t)r); /* r in 0..8; 8 == code 0x08 */
    }
    e = (int)floor(log2(a));
    /* log2 of a double can be off by one ulp near powers of two: fix e so
       that 2^e <= a < 2^(e+1) holds exactly. */
    while (ldexp(1.0, e) > a)
        e--;
    while (ldexp(1.0, e + 1) <= a)
        e++;
    r = round_half_even((ldexp(a, -e) - 1.0) * 8.0);
    if (r == 8.0) {
        r = 0.0;
        e += 1;
    }
    return (uint8_t)(sign | (uint8_t)(((e + 7) << 3) | (int)r));
}

/* ------------------------------------------------- group quantization -- */

/*
 * Quantize one group of `len` values (given as fp32, each exactly a bf16)
 * with the shared scale: steps a1 (amax), a2 (scale) and a3 (codes).
 * Returns the fp32 scale.
 */
static float quantize_group(const float *x, size_t stride, size_t len, uint8_t *q, size_t qstride)
{
    float amax = 0.0f;
    float s;
    size_t j;
    for (j = 0; j < len; j++) {
        float v = fabsf(x[j * stride]);
        if (v > amax)
            amax = v;
    }
    s = (amax > 1e-10f ? amax : 1e-10f) / 448.0f; /* one fp32 division */
    for (j = 0; j < len; j++) {
        float t = x[j * stride] / s;              /* one fp32 division */
        q[j * qstride] = oracle_e4m3_encode(t);
    }
    return s;
}

/* ceil16(M): the padded token extent of the K-major scales
   (dispatch_proj.rs, `cublas_fp8_m_pad`). */
uint32_t oracle_m_pad(uint32_t m)
{
    return (m + 15u) / 16u * 16u;
}

/*
 * Per-token, per-128-K-group activation quantization with both scale
 * layouts (dispatch_proj.rs: `cublas_fp8_proj` quantizes "the real M
 * tokens"; `fp8_act_scale_to_kmajor` rewrites `[M, K/128]` into
 * `[K/128, M_pad]` and zero-fills rows M..M_pad).
 *   x        bf16 bits, [m, k] row-major
 *   q        e4m3 codes, [m, k] row-major
 *   s_row    fp32, [m, k/128] row-major            (may be NULL)
 *   s_kmaj   fp32, [k/128, ceil16(m)]; s_kmaj[g][t] = s_row[t][g] for t < m,
 *            +0.0f for m <= t < ceil16(m)          (may be NULL)
 * Returns 0, or -1 if k is not a multiple of 128.
 */
int oracle_quant_act(const uint16_t *x, uint32_t m, uint32_t k,
                     uint8_t *q, float *s_row, float *s_kmaj)
{
    uint32_t G, mp, t, g, j;
    float buf[GROUP];
    if (k % GROUP != 0)
        return -1;
    G = k / GROUP;
    mp = oracle_m_pad(m);
    for (t = 0; t < m; t++) {
        for (g = 0; g < G; g++) {
            const uint16_t *xg = x + (size_t)t * k + (size_t)g * GROUP;
            float s;
            for (j = 0; j < GROUP; j++)
                buf[j] = oracle_bf16_to_f32(xg[j]);
            s = quantize_group(buf, 1, GROUP, q + (size_t)t * k + (size_t)g * GROUP, 1);
            if (s_row)
                s_row[(size_t)t * G + g] = s;
            if (s_kmaj)
                s_kmaj[(size_t)g * mp + t] = s;
        }
    }
    if (s_kmaj)
        for (g = 0; g < G; g++)
            for (t = m; t < mp; t++)
                s_kmaj[(size_t)g * mp + t] = 0.0f;
    return 0;
}

/*
 * Weight pre-quantization per 128x128 block: the same amax / scale / code
 * steps taken over a whole block. Layout follows the block-scaled
 * `Fp8Weight` of dispatch_proj.rs (`dequant_fp8_bf16_into` doc):
 *   w        bf16 bits [n, k] row-major
 *   wq       e4m3 codes [n, k] row-major
 *   w_scale  fp32 [n/128, k/128] row-major, read as scale[(r/128)*(k/128) + c/128]
 * Returns 0, or -1 unless n and k are multiples of 128.
 */
int oracle_quant_weight(const uint16_t *w, uint32_t n, uint32_t k,
                        uint8_t *wq, float *w_scale)
{
    uint32_t NB, G, bn, bg, r, c;
    float blk[GROUP * GROUP];
    uint8_t qb[GROUP * GROUP];
    if (n % GROUP != 0 || k % GROUP != 0)
        return -1;
    NB = n / GROUP;
    G = k / GROUP;
    for (bn = 0; bn < NB; bn++) {
        for (bg = 0; bg < G; bg++) {
            float s;
            for (r = 0; r < GROUP; r++)
                for (c = 0; c < GROUP; c++)
                    blk[r * GROUP + c] = oracle_bf16_to_f32(
                        w[(size_t)(bn * GROUP + r) * k + (size_t)bg * GROUP + c]);
            s = quantize_group(blk, 1, (size_t)GROUP * GROUP, qb, 1);
            w_scale[(size_t)bn * G + bg] = s;
            for (r = 0; r < GROUP; r++)
                for (c = 0; c < GROUP; c++)
                    wq[(size_t)(bn * GROUP + r) * k + (size_t)bg * GROUP + c] = qb[r * GROUP + c];
        }
    }
    return 0;
}

/* ------------------------------------------------------- GEMM reference -- */

/*
 * Float64 dequantized reference of the block-scaled GEMM
 * (dispatch_proj.rs, `cublas_fp8_proj` / `cublas_fp8_proj_prequant`:
 * out[M,N] = act[M,K] @ weight^T, activation scales per [token, 128 of K]),
 * for a weight whose scales follow the block geometry of
 * `dequant_fp8_bf16_into`: the scale of weight element [col][kk] is
 *   w_s[(col / block_n) * (k / block_k) + kk / block_k]
 * (block_n = block_k = 128 for the block-scaled format; block_n = 1,
 * block_k = k for the per-row format, one multiplier per weight row):
 *   ref[i][col] = sum_kk  deq(q[r_i][kk]) * a_s[r_i][kk/128]
 *                       * deq(wq[col][kk]) * w_s[...]
 * for each requested row r_i (rows == NULL means rows 0..n_rows-1).
 *   q      e4m3 [m, k];  a_s  fp32 [m, k/128] row-major (the definition's
 *          own indexing; the K-major copy is a layout of the same numbers)
 *   wq     e4m3 [n, k];  w_s  fp32, indexed as above
 *   ref    float64 [n_rows, n]
 * Rows are independent; `first`/`count` select a slice of the requested
 * rows so a caller may split the work over threads.
 */
void oracle_gemm_ref_rows_geom(const uint8_t *q, const float *a_s,
                               const uint8_t *wq, const float *w_s,
                               uint32_t n, uint32_t k, uint32_t block_n, uint32_t block_k,
                               const int64_t *rows, size_t first, size_t count,
                               double *ref)
{
    double lut[256];
    uint32_t G = k / GROUP;
    uint32_t sk = k / block_k;
    size_t i;
    uint32_t col, kk;
    for (i = 0; i < 256; i++)
        lut[i] = oracle_e4m3_decode((uint8_t)i);
    for (i = first; i < first + count; i++) {
        int64_t r = rows ? rows[i] : (int64_t)i;
        const uint8_t *qa = q + (size_t)r * k;
        const float *sa = a_s + (size_t)r * G;
        for (col = 0; col < n; col++) {
            const uint8_t *qw = wq + (size_t)col * k;
            const float *sw = w_s + (size_t)(col / block_n) * sk;
            double acc = 0.0;
            for (kk = 0; kk < k; kk++)
                acc += lut[qa[kk]] * (double)sa[kk / GROUP] * lut[qw[kk]] * (double)sw[kk / block_k];
            ref[i * n + col] = acc;
        }
    }
}

/* The block-scaled case: 128 x 128 weight-scale blocks. */
void oracle_gemm_ref_rows(const uint8_t *q, const float *a_s,
                          const uint8_t *wq, const float *w_s,
                          uint32_t n, uint32_t k,
                          const int64_t *rows, size_t first, size_t count,
                          double *ref)
{
    oracle_gemm_ref_rows_geom(q, a_s, wq, w_s, n, k, GROUP, GROUP, rows, first, count, ref);
}

/*
 * Per-row FP8 weight (dispatch_proj.rs, `dequant_fp8_bf16_into`: the
 * per-row format has block_n = 1, block_k = K, one multiplier per row).
 * The pages take such weights from a checkpoint and do not say how they
 * were quantized; the reading taken is the same amax / scale / code steps
 * as every other block, over the whole row:
 *   w        bf16 bits [n, k] row-major
 *   wq       e4m3 codes [n, k] row-major
 *   w_scale  fp32 [n]: max(max_j |w[r][j]|, 1e-10) / 448
 * Returns 0, or -1 if k is 0.
 */
int oracle_quant_weight_rowwise(const uint16_t *w, uint32_t n, uint32_t k,
                                uint8_t *wq, float *w_scale)
{
    uint32_t r, c;
    float *row;
    if (k == 0)
        return -1;
    row = (float *)malloc((size_t)k * sizeof(float));
    if (!row)
        return -1;
    for (r = 0; r < n; r++) {
        for (c = 0; c < k; c++)
            row[c] = oracle_bf16_to_f32(w[(size_t)r * k + c]);
        w_scale[r] = quantize_group(row, 1, k, wq + (size_t)r * k, 1);
    }
    free(row);
    return 0;
}

/*
 * The acceptance test of a computed output against the reference:
 *   |y - ref| <= 8e-3 * |ref| + 1e-3 * rms(ref)   for every element,
 * rms taken over all `count` reference values given. `y` is bf16 bits.
 * Returns the number of elements that fail; writes the worst ratio
 * |y-ref| / (8e-3|ref| + 1e-3 rms) to *worst.
 */
size_t oracle_check_tolerance(const uint16_t *y, const double *ref, size_t count, double *worst)
{
    double ss = 0.0, rms, w = 0.0;
    size_t i, bad = 0;
    for (i = 0; i < count; i++)
        ss += ref[i] * ref[i];
    rms = count ? sqrt(ss / (double)count) : 0.0;
    for (i = 0; i < count; i++) {
        double yv = (double)oracle_bf16_to_f32(y[i]);
        double err = fabs(yv - ref[i]);
        double bound = 8e-3 * fabs(ref[i]) + 1e-3 * rms;
        double ratio = bound > 0.0 ? err / bound : (err > 0.0 ? INFINITY : 0.0);
        if (!(err <= bound))
            bad++;
        if (ratio > w || ratio != ratio)
            w = ratio;
    }
    if (worst)
        *worst = w;
    return bad;
}

/* Encode `count` fp32 values one by one with oracle_e4m3_encode (sweeps). */
void oracle_e4m3_encode_array(const float *t, size_t count, uint8_t *out)
{
    size_t i;
    for (i = 0; i < count; i++)
        out[i] = oracle_e4m3_encode(t[i]);
}

/* ------------------------------------------- dense FFN: SiLU(gate) * up -- */

/*
 * The dense FFN of dispatch_proj.rs (doc of `cublas_fp8_proj_prequant`)
 * quantizes its input once for the gate and up projections, then quantizes
 * "the post-SiLU intermediate" once more for the down projection. The pages
 * print neither that activation nor its precision; the reading taken here:
 *   gate, up  the bf16 outputs of the two projections
 *   h         = bf16_rne( silu(gate) * up ),  silu(z) = z / (1 + e^-z),
 *             the real value rounded once to bf16 (the quantizer's input
 *             type), so that the definition does not depend on how an
 *             exponential is approximated.
 * Zero results keep the sign of gate*up (silu(z) has the sign of z).
 */

#if !defined(LDBL_MANT_DIG) || LDBL_MANT_DIG < 64
#error "the SiLU oracle needs an extended long double (64-bit significand)"
#endif

/* bf16 bits of a finite, nonzero long double magnitude a, rounded to the
   nearest bf16 (8-bit significand, binary32 exponent range), ties to even
   unless tie_down is set, in which case a tie goes to the smaller value.
   Overflow gives infinity (0x7F80). */
static uint16_t bf16_magnitude_bits(long double a, int tie_down)
{
    int e;
    long double q, fl, frac, n;
    long double quantum;
    uint32_t code;
    if (a < ldexpl(1.0L, -126)) {
        quantum = ldexpl(1.0L, -133);        /* subnormal spacing */
    } else {
        (void)frexpl(a, &e);                 /* a = f * 2^e, f in [0.5, 1) */
        quantum = ldexpl(1.0L, e - 1 - 7);   /* 7 fraction bits below the leading one */
    }
    q = a / quantum;                         /* exact: scaling by a power of two */
    fl = floorl(q);
    frac = q - fl;
    if (frac > 0.5L)
        n = fl + 1.0L;
    else if (frac < 0.5L)
        n = fl;
    else if (tie_down)
        n = fl;
    else
        n = (fmodl(fl, 2.0L) == 0.0L) ? fl : fl + 1.0L;
    a = n * quantum;                         /* the rounded magnitude, exact */
    if (a >= ldexpl(1.0L, 128))
        return 0x7F80;
    {
        float f = (float)a;                  /* exact: a is a bf16 value */
        uint32_t u;
        memcpy(&u, &f, sizeof u);
        code = u >> 16;
    }
    return (uint16_t)code;
}

/*
 * h = bf16_rne(silu(g) * u) for bf16 inputs g, u (bit patterns).
 * P = g*u is exact in long double (two 8-bit significands). For g <= 32
 * the value P / (1 + e^-g) is formed in long double (64-bit significand):
 * its relative error is a few 2^-64, far below the bf16 rounding step, and
 * since e^-g is transcendental for g != 0 the real value is never exactly a
 * rounding tie. For g > 32 the factor 1/(1+e^-g) differs from 1 by less
 * than 2^-46, while P (16 significant bits) either sits exactly on a bf16
 * tie or lies at least 2^-17 |P| away from one; so the result is P rounded
 * to bf16, except that an exact tie goes toward zero, because
 * silu(g) < g for every g > 0.
 */
uint16_t oracle_silu_mul_bf16(uint16_t g_bits, uint16_t u_bits)
{
    float gf = oracle_bf16_to_f32(g_bits);
    float uf = oracle_bf16_to_f32(u_bits);
    long double g = (long double)gf, u = (long double)uf;
    long double p = g * u;
    uint16_t sign = (uint16_t)((g_bits ^ u_bits) & 0x8000u);
    long double v;
    if (p == 0.0L)
        return sign;
    if (g > 32.0L)
        return (uint16_t)(sign | bf16_magnitude_bits(fabsl(p), 1));
    v = p / (1.0L + expl(-g));
    return (uint16_t)(sign | bf16_magnitude_bits(fabsl(v), 0));
}

/* Round each float64 value to bf16 bits, nearest, ties to even (the
   projections' bf16 outputs in the FFN reference). Signed zeros kept. */
void oracle_round_bf16_array(const double *v, size_t count, uint16_t *out)
{
    size_t i;
    for (i = 0; i < count; i++) {
        uint16_t sign = signbit(v[i]) ? 0x8000u : 0u;
        out[i] = v[i] == 0.0 ? sign : (uint16_t)(sign | bf16_magnitude_bits(fabsl((long double)v[i]), 0));
    }
}

/*
 * SiLU-and-multiply followed by the per-token group quantization of the
 * result, as the FFN feeds its down projection:
 *   gate, up  bf16 bits; row t of gate starts at gate + t*ld, likewise up
 *   h[t][j]   = oracle_silu_mul_bf16(gate[t][j], up[t][j]),  j < i
 *   q, s_row, s_kmaj exactly as oracle_quant_act over h ([m, i])
 * Returns 0, or -1 if i is not a multiple of 128.
 */
int oracle_silu_mul_quant(const uint16_t *gate, const uint16_t *up, size_t ld,
                          uint32_t m, uint32_t i, uint8_t *q, float *s_row, float *s_kmaj)
{
    uint32_t G, mp, t, g, j;
    float buf[GROUP];
    if (i % GROUP != 0)
        return -1;
    G = i / GROUP;
    mp = oracle_m_pad(m);
    for (t = 0; t < m; t++) {
        for (g = 0; g < G; g++) {
            float s;
            for (j = 0; j < GROUP; j++) {
                size_t c = (size_t)g * GROUP + j;
                buf[j] = oracle_bf16_to_f32(oracle_silu_mul_bf16(gate[(size_t)t * ld + c], up[(size_t)t * ld + c]));
            }
            s = quantize_group(buf, 1, GROUP, q + (size_t)t * i + (size_t)g * GROUP, 1);
            if (s_row)
                s_row[(size_t)t * G + g] = s;
            if (s_kmaj)
                s_kmaj[(size_t)g * mp + t] = s;
        }
    }
    if (s_kmaj)
        for (g = 0; g < G; g++)
            for (t = m; t < mp; t++)
                s_kmaj[(size_t)g * mp + t] = 0.0f;
    return 0;
}

/* h for `count` (gate, up) pairs (sweeps). */
void oracle_silu_mul_bf16_array(const uint16_t *g, const uint16_t *u, size_t count, uint16_t *h)
{
    size_t i;
    for (i = 0; i < count; i++)
        h[i] = oracle_silu_mul_bf16(g[i], u[i]);
}

/* --------------------------------------------- FP8 weight back to bf16 -- */

/*
 * Dequantize an FP8 weight to bf16 (dispatch_proj.rs, `dequant_fp8_bf16_into`:
 * an [N,K] bf16 result, block (128,128) or, for the per-row format,
 * (1,K)). The pages do not print the kernel; the reading taken is the plain
 * one: each element is the bf16 nearest to the exact product
 *   deq(wq[r][c]) * w_s[(r/block_n) * (k/block_k) + c/block_k]
 * (ties to even, sign of zero kept). The product of a 4-bit and a 24-bit
 * significand is exact in double, so there is one rounding.
 * Returns 0, or -1 if the blocks do not tile [n, k].
 */
int oracle_dequant_fp8_bf16(const uint8_t *wq, const float *w_s, uint32_t n, uint32_t k,
                            uint32_t block_n, uint32_t block_k, uint16_t *out)
{
    uint32_t r, c, sk;
    if (block_n == 0 || block_k == 0 || n % block_n || k % block_k)
        return -1;
    sk = k / block_k;
    for (r = 0; r < n; r++) {
        for (c = 0; c < k; c++) {
            double v = oracle_e4m3_decode(wq[(size_t)r * k + c]) *
                       (double)w_s[(size_t)(r / block_n) * sk + c / block_k];
            uint16_t sign = signbit(v) ? 0x8000u : 0u;
            out[(size_t)r * k + c] =
                v == 0.0 ? sign : (uint16_t)(sign | bf16_magnitude_bits(fabsl((long double)v), 0));
        }
    }
    return 0;
}

/* --------------------------------------------------------------- NVFP4 -- */

/*
 * The NVFP4 projection arms (dispatch_proj.rs, doc comments of
 * `cutlass_nvfp4_proj`, `cutlass_nvfp4_weight_transposed_cached` and
 * `cutlass_nvfp4_proj_from_fp8`). The pages fix the geometry: two 4-bit
 * elements per byte along K ([K/2, N] data), one scale per 16 elements along
 * K ([K/16, N] scales) and one fp32 second-level scale per weight
 * (`weight_scale_2`; 1.0 for a weight packed from an FP8 checkpoint). They
 * print neither the element format nor the packer. The readings taken:
 *   - elements are NVFP4's E2M1 (1 sign bit, 2 exponent bits with bias 1,
 *     1 mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; no Inf, no NaN)
 *     and block scales are E4M3 codes, the format's own definition;
 *   - within a byte the element with the even K index sits in the low nibble;
 *   - the packer follows the format's plain recipe, one fp32 operation a step:
 *       amax = max_j |x_j|                    over 16 consecutive K elements
 *       sf   = e4m3_rne_satfinite(amax / (6 * s2))
 *       s    = deq(sf) * s2                   the block's effective scale
 *       q_j  = e2m1_rne_satfinite(x_j / s)    (s == 0: every q_j is a zero
 *                                              carrying the sign of x_j)
 *     with s2 the second-level scale of the operand.
 */

#define NVFP4_BLOCK 16       /* K elements that share one block scale */
#define E2M1_MAX 6.0         /* largest E2M1 magnitude */

/* Decode one E2M1 code (low 4 bits of `code`). Exponent field 0 holds the
   subnormals m * 0.5; otherwise the value is 2^(e-1) * (1 + m/2). */
double oracle_e2m1_decode(uint8_t code)
{
    int sign = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, e - 1);
    return sign ? -mag : mag;
}

/*
 * Encode one fp32 value into E2M1, round to nearest with ties to the even
 * code, saturating at 6 and keeping the sign of zero. Inside a binade the
 * representable magnitudes are evenly spaced (0.5 below 2, 1 in [2, 4),
 * 2 in [4, 6]); a/spacing is then an integer whose parity is the parity of
 * the code, so rounding that quotient half-to-even rounds the code
 * half-to-even. NaN input is outside the contract.
 */
uint8_t oracle_e2m1_encode(float t)
{
    uint8_t sign = signbit(t) ? 0x8 : 0x0;
    double a = fabs((double)t);
    double spacing, r;
    uint8_t c;
    if (a >= E2M1_MAX)
        return (uint8_t)(sign | 0x7);
    spacing = a < 2.0 ? 0.5 : (a < 4.0 ? 1.0 : 2.0);
    r = round_half_even(a / spacing) * spacing;   /* exact: spacing is a power of two */
    for (c = 0; c < 8; c++)
        if (oracle_e2m1_decode(c) == r)
            return (uint8_t)(sign | c);
    return 0xFF; /* unreachable: r is always one of the eight magnitudes */
}

/* Encode `count` fp32 values one by one with oracle_e2m1_encode (sweeps). */
void oracle_e2m1_encode_array(const float *t, size_t count, uint8_t *out)
{
    size_t i;
    for (i = 0; i < count; i++)
        out[i] = oracle_e2m1_encode(t[i]);
}

/*
 * Pack a bf16 matrix into NVFP4 along K with second-level scale s2:
 *   x   bf16 bits [r, k] row-major
 *   q   [r, k/2] bytes: element 2j of a row in the low nibble of byte j,
 *       element 2j+1 in the high nibble
 *   sf  E4M3 codes [r, k/16] row-major, one per 16-element block
 * Returns 0, or -1 if k is not a multiple of 16 or s2 is not a positive,
 * finite fp32 value.
 */
int oracle_nvfp4_quant(const uint16_t *x, uint32_t r, uint32_t k, float s2, uint8_t *q, uint8_t *sf)
{
    uint32_t row, b, j, nb;
    if (k % NVFP4_BLOCK != 0 || !(s2 > 0.0f) || isinf(s2))
        return -1;
    nb = k / NVFP4_BLOCK;
    for (row = 0; row < r; row++) {
        for (b = 0; b < nb; b++) {
            float v[NVFP4_BLOCK];
            float amax = 0.0f, t, s;
            uint8_t code;
            for (j = 0; j < NVFP4_BLOCK; j++) {
                v[j] = oracle_bf16_to_f32(x[(size_t)row * k + (size_t)b * NVFP4_BLOCK + j]);
                if (fabsf(v[j]) > amax)
                    amax = fabsf(v[j]);
            }
            t = amax / (6.0f * s2);                       /* fp32 product, then fp32 division */
            code = oracle_e4m3_encode(t);
            s = (float)oracle_e4m3_decode(code) * s2;     /* one fp32 product */
            sf[(size_t)row * nb + b] = code;
            for (j = 0; j < NVFP4_BLOCK; j += 2) {
                uint8_t lo, hi;
                if (s == 0.0f) {
                    lo = signbit(v[j]) ? 0x8 : 0x0;
                    hi = signbit(v[j + 1]) ? 0x8 : 0x0;
                } else {
                    lo = oracle_e2m1_encode(v[j] / s);    /* one fp32 division */
                    hi = oracle_e2m1_encode(v[j + 1] / s);
                }
                q[((size_t)row * k + (size_t)b * NVFP4_BLOCK + j) / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
    return 0;
}

/*
 * The second-level scale of a synthetic NVFP4 checkpoint weight: the pages
 * take `weight_scale_2` from the checkpoint and never say how it was made.
 * The reading taken is the format's usual choice, which lets the largest
 * block scale reach E4M3's 448:
 *   s2 = max(amax over the whole tensor, 1e-10) / (6 * 448)
 * (one fp32 division; 2688 is exact).
 */
float oracle_nvfp4_global_scale(const uint16_t *x, size_t count)
{
    float amax = 0.0f;
    size_t i;
    for (i = 0; i < count; i++) {
        float v = fabsf(oracle_bf16_to_f32(x[i]));
        if (v > amax)
            amax = v;
    }
    return (amax > 1e-10f ? amax : 1e-10f) / 2688.0f;
}

/*
 * Float64 reference of the NVFP4 projection for the requested rows:
 *   ref[i][col] = s2a * s2w * sum_kk deq(qa[r_i][kk]) * deq(sfa[r_i][kk/16])
 *                                  * deq(qw[col][kk]) * deq(sfw[col][kk/16])
 *   qa, sfa  packed activation [m, k/2] and its E4M3 scales [m, k/16]
 *   qw, sfw  packed weight [n, k/2] and its E4M3 scales [n, k/16]
 * (layouts as oracle_nvfp4_quant writes them); ref float64 [rows, n].
 * Every product and every 16-element partial sum is exact in double.
 */
void oracle_nvfp4_gemm_ref_rows(const uint8_t *qa, const uint8_t *sfa, float s2a,
                                const uint8_t *qw, const uint8_t *sfw, float s2w,
                                uint32_t n, uint32_t k, const int64_t *rows,
                                size_t first, size_t count, double *ref)
{
    double e2m1[16], e4m3[256];
    uint32_t nb = k / NVFP4_BLOCK, col, b, j;
    size_t i;
    for (i = 0; i < 16; i++)
        e2m1[i] = oracle_e2m1_decode((uint8_t)i);
    for (i = 0; i < 256; i++)
        e4m3[i] = oracle_e4m3_decode((uint8_t)i);
    for (i = first; i < first + count; i++) {
        int64_t r = rows ? rows[i] : (int64_t)i;
        for (col = 0; col < n; col++) {
            double acc = 0.0;
            for (b = 0; b < nb; b++) {
                double part = 0.0;
                for (j = 0; j < NVFP4_BLOCK; j++) {
                    size_t kk = (size_t)b * NVFP4_BLOCK + j;
                    uint8_t ba = qa[((size_t)r * k + kk) / 2];
                    uint8_t bw = qw[((size_t)col * k + kk) / 2];
                    uint8_t ca = (kk & 1) ? (uint8_t)(ba >> 4) : (uint8_t)(ba & 0xF);
                    uint8_t cw = (kk & 1) ? (uint8_t)(bw >> 4) : (uint8_t)(bw & 0xF);
                    part += e2m1[ca] * e2m1[cw];
                }
                acc += part * e4m3[sfa[(size_t)r * nb + b]] * e4m3[sfw[(size_t)col * nb + b]];
            }
            ref[i * n + col] = acc * (double)s2a * (double)s2w;
        }
    }
}
