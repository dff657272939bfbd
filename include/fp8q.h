/*
 * fp8q — W8A8 FP8 block-scaled linear projection for NVIDIA B200 (sm_100a).
 *
 * C ABI of libfp8q.so. The operations follow the pages
 *   "spark_model/layers/ops/dispatch_proj.rs"      (P-DP below) and
 *   "spark_model/layers/ops/fp8_act_quant_floor.rs" (P-FL below):
 *   - per-token, per-128-K-group FP8 E4M3 activation quantization with FP32
 *     scales (P-DP, `cublas_fp8_proj`: "FP8 + per-[token,128-of-K] scales"),
 *     with the scales stored both row-major [M, K/128] and K-major
 *     [K/128, ceil16(M)] with zeroed pad rows (P-DP, `fp8_act_scale_to_kmajor`
 *     and the ⚠ SCALE LAYOUT note of `cublas_fp8_proj_prequant`);
 *   - a GEMM out[M,N] = act[M,K] @ weight^T over FP8 weights carrying FP32
 *     per-128x128-block scales, bf16 out (P-DP, `cublas_fp8_proj_prequant`,
 *     `dequant_fp8_bf16_into` for the weight-scale indexing);
 *   - the fused linear that runs both in one call (P-DP, `cublas_fp8_proj`);
 *   - the choice between the one-group-per-CTA and the multi-group-per-CTA
 *     quantizer by a CTA-count floor (P-FL, module header and
 *     `fp8_act_quant_hopper_reject`), re-derived for the device's SM count;
 *   - the dense FFN that quantizes its input once for the gate and up
 *     projections and quantizes the post-SiLU intermediate once for the down
 *     projection (P-DP, doc of `cublas_fp8_proj_prequant`);
 *   - the NVFP4 projection arms: E2M1 operands with E4M3 scales per 16
 *     elements of K on the block-scaled tensor cores, and the FP8-to-bf16
 *     weight dequantizer the from-FP8 arm starts with (P-DP,
 *     `cutlass_nvfp4_proj`, `cutlass_nvfp4_proj_from_fp8`,
 *     `dequant_fp8_bf16_into`).
 *
 * Conventions shared by every call:
 *   - Data pointers are DEVICE pointers owned by the caller, 16-byte aligned.
 *     The library allocates no device memory.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls
 *     only enqueue work; nothing synchronizes.
 *   - bf16 is IEEE bfloat16; e4m3 is OCP FP8 E4M3FN (bias 7, max 448, NaN
 *     only at S.1111.111). Matrices are row-major.
 *   - K and N must be multiples of 128 (the NVFP4 calls state their own K
 *     rule). M == 0 is accepted and launches
 *     nothing (pointers may then be NULL). M*K, N*K and M*N must stay
 *     below 2^31.
 *   - Every argument is checked before anything is enqueued; a failed check
 *     returns its status and leaves all buffers untouched.
 *   - A device other than compute capability 10.0 returns
 *     FP8Q_ERR_UNSUPPORTED_DEVICE; there is no fallback path.
 *   - NaN or Inf in the inputs is outside the contract (results undefined).
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP8Q_OK = 0,
    FP8Q_ERR_NULL = 1,               /* a required pointer is NULL                 */
    FP8Q_ERR_SHAPE = 2,              /* K or N not a multiple of 128, or too large */
    FP8Q_ERR_ALIGN = 3,              /* a pointer is not 16-byte aligned           */
    FP8Q_ERR_WORKSPACE = 4,          /* workspace smaller than required            */
    FP8Q_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed          */
    FP8Q_ERR_DEVICE_TIMEOUT = 6,     /* a kernel's bounded wait ran out            */
    FP8Q_ERR_UNSUPPORTED_DEVICE = 7, /* current device is not sm_100               */
    FP8Q_ERR_ARG = 8                 /* any other invalid argument                 */
} fp8q_status;

/* Human-readable name of a status code; never NULL. */
const char *fp8q_status_string(int status);

/* Library version string. */
const char *fp8q_version(void);

/* ceil16(m): the token extent of the K-major scales (P-DP, `cublas_fp8_m_pad`). */
uint32_t fp8q_m_pad(uint32_t m);

/* ------------------------------------------------------ variant pick ---- */

/* Quantizer variants. SINGLE quantizes one 128-wide group per CTA; MULTI
   quantizes 8 consecutive groups of a few consecutive tokens per CTA
   (fp8q_quant_pick_t.groups_per_cta). Both emit the same bytes (P-FL: the
   two quantizers of the pages emit identical bytes, so the choice is one of
   speed only). */
enum { FP8Q_QUANT_AUTO = 0, FP8Q_QUANT_SINGLE = 1, FP8Q_QUANT_MULTI = 2 };

typedef struct {
    int32_t variant;          /* FP8Q_QUANT_SINGLE or FP8Q_QUANT_MULTI       */
    uint32_t grid_x;          /* CTAs launched                               */
    uint32_t block_x;         /* threads per CTA                             */
    uint32_t groups_per_cta;  /* 128-wide K groups one CTA quantizes         */
    uint32_t multi_ctas;      /* CTAs the MULTI variant would launch         */
    uint32_t floor_ctas;      /* the CTA floor MULTI must reach              */
    int32_t forced;           /* 1 when `requested` overrode the floor       */
} fp8q_quant_pick_t;

/*
 * The smallest M at which a multi-group quantizer whose CTA covers
 * `groups_per_cta` K-groups of `rows_per_cta` tokens reaches the CTA floor
 * ceil(min_ctas_per_sm * sm_count) at this K. Its grid is
 * ceil((K/128)/groups_per_cta) x ceil(M/rows_per_cta) CTAs; with
 * rows_per_cta = 1 this is the pages' formula ceil(floor / grid_y)
 * (P-FL, `fp8_quant_hopper_min_m` and the per-K table of the module header:
 * 132 SMs, 8 groups, 2 CTAs/SM gives 53/44/16 at K = 5120/6144/17408).
 * fp8q_quant_pick applies exactly this function, with the floor measured for
 * B200 (2/3 of a CTA per SM for this library's multi-group kernel). Pure host
 * function. Returns 0 when k < 128, groups_per_cta or rows_per_cta is 0, or
 * min_ctas_per_sm is negative or NaN.
 */
uint32_t fp8q_quant_floor_min_m(uint32_t k, uint32_t sm_count, uint32_t groups_per_cta, uint32_t rows_per_cta,
                                float min_ctas_per_sm);

/*
 * Which quantizer variant runs for (m, k) on a device with `sm_count` SMs,
 * and on what grid (P-FL, `Fp8QuantPick`: the kernel and its grid travel
 * together). `requested` is FP8Q_QUANT_AUTO (apply the floor) or a variant
 * to force. Pure host function; no device is touched.
 * Errors: FP8Q_ERR_NULL (out), FP8Q_ERR_SHAPE (k % 128), FP8Q_ERR_ARG
 * (unknown variant or sm_count == 0).
 */
fp8q_status fp8q_quant_pick(uint32_t m, uint32_t k, uint32_t sm_count, int32_t requested,
                            fp8q_quant_pick_t *out);

/* ---------------------------------------------------------- kernels ---- */

/*
 * Per-token-group activation quantization (P-DP, `cublas_fp8_proj`, first
 * step; P-FL for the variant). For each token t < m and group g < k/128:
 *   amax = max_j |x[t][128g+j]|,  s = max(amax, 1e-10f) / 448.0f  (fp32),
 *   q[t][128g+j] = e4m3_rne_satfinite(x[t][128g+j] / s)            (fp32 div)
 *   x         bf16 [m, k]                                  (input)
 *   q         e4m3 [m, k]                                  (output)
 *   s_row     fp32 [m, k/128] row-major; may be NULL to skip this layout
 *   s_kmajor  fp32 [k/128, ceil16(m)]: s_kmajor[g][t] = s for t < m and
 *             +0.0f for m <= t < ceil16(m)                 (output, required)
 * The variant follows fp8q_quant_pick(m, k, <device SMs>, FP8Q_QUANT_AUTO)
 * unless the environment variable FP8Q_QUANT_VARIANT=single|multi forces it.
 * Errors: NULL, ALIGN, SHAPE, UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_quant_act(const void *x, void *q, float *s_row, float *s_kmajor,
                           uint32_t m, uint32_t k, void *stream);

/* fp8q_quant_act with the variant chosen by the caller (FP8Q_QUANT_AUTO,
   FP8Q_QUANT_SINGLE or FP8Q_QUANT_MULTI); the bytes written are identical. */
fp8q_status fp8q_quant_act_variant(const void *x, void *q, float *s_row, float *s_kmajor,
                                   uint32_t m, uint32_t k, int32_t variant, void *stream);

/*
 * Weight pre-quantization per 128x128 block (the block-scaled `Fp8Weight`
 * of P-DP; scale indexing of `dequant_fp8_bf16_into`): for each block
 * (bn, bg) the same amax / scale / RNE-satfinite steps as above, taken over
 * the block's 128x128 values.
 *   w        bf16 [n, k]              (input)
 *   wq       e4m3 [n, k]              (output)
 *   w_scale  fp32 [n/128, k/128]      (output), scale of element (r, c) at
 *            w_scale[(r/128)*(k/128) + c/128]
 * Errors: NULL, ALIGN, SHAPE, UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_quant_weight(const void *w, void *wq, float *w_scale,
                              uint32_t n, uint32_t k, void *stream);

/*
 * Block-scaled FP8 GEMM (P-DP, `cublas_fp8_proj_prequant`):
 *   y[t][c] = bf16_rn( sum_g s_kmajor[g][t] * w_scale[c/128][g]
 *                      * sum_{j<128} q[t][128g+j] * wq[c][128g+j] )
 * with the inner sums from FP8 tensor-core MMA in fp32 and the scaled
 * promotion in fp32.
 *   q         e4m3 [m, k]               (input; rows >= m are never read)
 *   s_kmajor  fp32 [k/128, ceil16(m)]   (input, as written by fp8q_quant_act)
 *   wq        e4m3 [n, k], w_scale fp32 [n/128, k/128]        (inputs)
 *   y         bf16 [m, n]               (output; exactly m rows are written)
 * Errors: NULL, ALIGN, SHAPE, UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_gemm_blockscaled(const void *q, const float *s_kmajor, const void *wq,
                                  const float *w_scale, void *y,
                                  uint32_t m, uint32_t n, uint32_t k, void *stream);

/*
 * Weight formats: the geometry of the weight scales (P-DP,
 * `dequant_fp8_bf16_into`: one rule, scale[(n/block_n)*(K/block_k) + k/block_k],
 * serves both layouts):
 *   FP8Q_WEIGHT_BLOCK128  block_n = block_k = 128: w_scale fp32 [n/128, k/128]
 *   FP8Q_WEIGHT_PER_ROW   block_n = 1, block_k = K: w_scale fp32 [n], one
 *                         multiplier per weight row (the compressed-tensors
 *                         per-row checkpoint format the pages name)
 */
enum { FP8Q_WEIGHT_BLOCK128 = 0, FP8Q_WEIGHT_PER_ROW = 1 };

/*
 * Per-row weight quantization: for each row r of w bf16 [n, k],
 *   w_scale[r] = max(max_j |w[r][j]|, 1e-10f) / 448.0f,
 *   wq[r][j]   = e4m3_rne_satfinite(w[r][j] / w_scale[r]),
 * the activation quantizer's arithmetic over a 1 x k block. (The pages load
 * such weights from a checkpoint; the quantizer is this library's.)
 * k a multiple of 128; n*k below 2^31.
 * Errors: NULL, ALIGN, SHAPE, UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_quant_weight_rowwise(const void *w, void *wq, float *w_scale,
                                      uint32_t n, uint32_t k, void *stream);

/*
 * fp8q_gemm_blockscaled for either weight format:
 *   y[t][c] = bf16_rn( sum_g s_kmajor[g][t] * ws(c, g)
 *                      * sum_{j<128} q[t][128g+j] * wq[c][128g+j] )
 * with ws(c, g) = w_scale[c/128][g] (FP8Q_WEIGHT_BLOCK128) or w_scale[c]
 * (FP8Q_WEIGHT_PER_ROW; applied once per output after the sum over g).
 * Errors: as fp8q_gemm_blockscaled, plus ARG for an unknown format.
 */
fp8q_status fp8q_gemm_ex(const void *q, const float *s_kmajor, const void *wq,
                         const float *w_scale, int32_t weight_format, void *y,
                         uint32_t m, uint32_t n, uint32_t k, void *stream);

/*
 * Workspace bytes fp8q_linear needs for (m, k): the FP8 activation
 * [m, k] at offset 0, then the K-major scales [k/128, ceil16(m)] fp32 at
 * offset fp8q_linear_scale_offset(m, k).
 */
size_t fp8q_linear_workspace_bytes(uint32_t m, uint32_t k);
size_t fp8q_linear_scale_offset(uint32_t m, uint32_t k);

/*
 * Fused W8A8 linear (P-DP, `cublas_fp8_proj`): quantize x exactly as
 * fp8q_quant_act does (same bytes, same K-major scales, left in the
 * workspace), then run fp8q_gemm_blockscaled into y. One call; the kernels
 * are chained on `stream`.
 *   x bf16 [m, k]; wq e4m3 [n, k]; w_scale fp32 [n/128, k/128]; y bf16 [m, n]
 *   workspace: device memory of at least fp8q_linear_workspace_bytes(m, k),
 *              256-byte aligned, owned by the caller.
 * Errors: NULL, ALIGN, SHAPE, WORKSPACE, UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_linear(const void *x, const void *wq, const float *w_scale, void *y,
                        void *workspace, size_t workspace_bytes,
                        uint32_t m, uint32_t n, uint32_t k, void *stream);

/*
 * fp8q_linear_ex at decode widths (m <= 32) in ONE launch: the decode GEMM
 * quantizes x itself, K block by K block, straight into its shared-memory
 * operand tiles (page P-DP's decode path quantizes in a separate launch).
 * Results are bit-identical to fp8q_linear_ex, including the FP8 bytes and
 * K-major scales it leaves in the workspace. Every weight slice of the GEMM
 * quantizes the same activation blocks, so this path does more arithmetic:
 * on B200 it measured slower than the two-launch fp8q_linear_ex (21.0 vs
 * 12.4 us at m=25, n=6144, k=5120), which therefore remains the default.
 * Errors: as fp8q_linear_ex; SHAPE also when m > 32.
 */
fp8q_status fp8q_linear_decode_fused(const void *x, const void *wq, const float *w_scale,
                                     int32_t weight_format, void *y,
                                     void *workspace, size_t workspace_bytes,
                                     uint32_t m, uint32_t n, uint32_t k, void *stream);

/* fp8q_linear for either weight format (see fp8q_gemm_ex). */
fp8q_status fp8q_linear_ex(const void *x, const void *wq, const float *w_scale,
                           int32_t weight_format, void *y,
                           void *workspace, size_t workspace_bytes,
                           uint32_t m, uint32_t n, uint32_t k, void *stream);

/*
 * fp8q_linear for callers that cannot allocate device memory. The paper has
 * no counterpart to this call; it exists for callers that are handed inputs
 * and outputs but cannot obtain a device buffer for the workspace: a plugin
 * inside a runtime that owns the whole device-memory budget, or a
 * latency-critical loop where a cudaMalloc could synchronize the device.
 *
 * Same arguments, results and kernels as fp8q_linear, minus the workspace:
 * the FP8 activation and its K-major scales go to a fixed 16 MiB device
 * array inside the library (every GPU that loads the library holds it until
 * the process exits). The call allocates nothing and calls no allocating
 * routine.
 *   - Limit: fp8q_linear_workspace_bytes(m, k) must be at most 16 MiB
 *     (about m*k <= 16.2 million, e.g. m = 1168 at k = 5120); larger calls
 *     return FP8Q_ERR_WORKSPACE without enqueuing anything.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture. The address is cached with the ID of the
 *     CUDA context it was found in, and looked up again when a call finds
 *     another context current (after cudaDeviceReset, say).
 *   - Every call on a device shares the one array and it keeps the last
 *     call's contents; nothing in it needs clearing, because each call
 *     overwrites all of it that it reads. Calls that overlap on the GPU
 *     (different streams, or different host threads, on one device) race on
 *     the array: serialize them.
 * Errors: NULL, ALIGN, SHAPE, WORKSPACE (too large), UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_linear_noalloc(const void *x, const void *wq, const float *w_scale, void *y,
                                uint32_t m, uint32_t n, uint32_t k, void *stream);

/* --------------------------------------------------------- dense FFN ---- */

/*
 * SiLU(gate) * up, then the activation quantization of the result, as the
 * dense FFN feeds its down projection (P-DP, doc of
 * `cublas_fp8_proj_prequant`: "quantizes the post-SiLU intermediate once for
 * `down`"). The pages do not print the activation; this library defines
 *   h[t][j] = bf16_rne( silu(gate[t][j]) * up[t][j] ),
 *   silu(z) = z / (1 + e^-z),
 * the real value rounded once to bf16 (ties to even; a zero result carries
 * the sign of gate*up), and then quantizes h exactly as fp8q_quant_act
 * quantizes x: same group arithmetic, same codes, same two scale layouts.
 *   gate, up   bf16, m rows of i values; row t starts at gate + t*ld
 *              (likewise up), ld >= i and a multiple of 8 (inputs)
 *   q          e4m3 [m, i]                       (output)
 *   s_rowmajor fp32 [m, i/128] or NULL           (output)
 *   s_kmajor   fp32 [i/128, ceil16(m)], pad rows zeroed (output, required)
 * i must be a multiple of 128; m*ld below 2^31.
 * Errors: NULL, ALIGN, SHAPE, UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_silu_mul_quant(const void *gate, const void *up, uint32_t ld, void *q,
                                float *s_rowmajor, float *s_kmajor,
                                uint32_t m, uint32_t i, void *stream);

/*
 * Workspace of fp8q_ffn for (m, d, i): offsets[0..4] are the byte offsets
 * of q_x e4m3 [m, d], s_x fp32 [d/128, ceil16(m)], gate|up bf16 [m, 2i]
 * (row t: i gate values, then i up values), q_h e4m3 [m, i] and
 * s_h fp32 [i/128, ceil16(m)], each 256-byte aligned; offsets[5] is the
 * total size. Errors: NULL, SHAPE (d or i not a positive multiple of 128).
 */
fp8q_status fp8q_ffn_workspace_layout(uint32_t m, uint32_t d, uint32_t i, size_t *offsets);
size_t fp8q_ffn_workspace_bytes(uint32_t m, uint32_t d, uint32_t i);

/*
 * Dense FFN with FP8 weights (P-DP, doc of `cublas_fp8_proj_prequant`):
 *   q_x, s_x   = quant(x)                        once, for gate and up
 *   [gate|up]  = gemm(q_x, w_gate_up)            one GEMM, N = 2i, bf16 out
 *   q_h, s_h   = fp8q_silu_mul_quant(gate, up)
 *   y          = gemm(q_h, w_down)               bf16 out
 * Every intermediate stays in the workspace for inspection.
 *   x               bf16 [m, d]                                  (input)
 *   w_gate_up       e4m3 [2i, d]: rows 0..i-1 gate, i..2i-1 up    (input)
 *   w_gate_up_scale fp32 [2i/128, d/128]                         (input)
 *   w_down          e4m3 [d, i], w_down_scale fp32 [d/128, i/128] (inputs)
 *   y               bf16 [m, d]                                  (output)
 *   workspace       >= fp8q_ffn_workspace_bytes(m, d, i), 256-byte aligned
 * d and i must be multiples of 128. The four kernels are chained on
 * `stream`, each a programmatic dependent of the one before it.
 * Errors: NULL, ALIGN, SHAPE, WORKSPACE, UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_ffn(const void *x, const void *w_gate_up, const float *w_gate_up_scale,
                     const void *w_down, const float *w_down_scale, void *y,
                     void *workspace, size_t workspace_bytes,
                     uint32_t m, uint32_t d, uint32_t i, void *stream);

/* ------------------------------------------------------------ NVFP4 ---- */

/*
 * NVFP4 projection arms (P-DP, `cutlass_nvfp4_proj`,
 * `cutlass_nvfp4_weight_transposed_cached`, `cutlass_nvfp4_proj_from_fp8`).
 * An NVFP4 operand of R rows and K columns is
 *   q       [R, K/2] bytes of E2M1 codes (1 sign bit, 2 exponent bits with
 *           bias 1, 1 mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6),
 *           two to a byte along K, element 2j in the low nibble of byte j.
 *           This is the [N, K/2] layout the pages' GEMM consumes; their
 *           [K/2, N] checkpoint layout is its byte transpose.
 *   scales  one E4M3 code per 16 elements of K, row-major [R, K/16] and in
 *           the MMA layout the GEMM reads: one 512-byte atom per 128 rows
 *           (R padded up to a multiple of 128, pad scales zero) and 64
 *           elements of K, atoms ordered K-fastest within a 128-row block,
 *           byte (r%32)*16 + ((r%128)/32)*4 + (k/16)%4 inside an atom.
 *   s2      one fp32 second-level scale (the pages' `weight_scale_2`).
 * Element (r, k) is worth s2 * e4m3(scale[r][k/16]) * e2m1(q[r][k]).
 */

/* Bytes of the MMA-layout scales of a rows x k operand: ceil128(rows) * k/16. */
size_t fp8q_nvfp4_sf_mma_bytes(uint32_t rows, uint32_t k);

/*
 * Pack bf16 x [rows, k] into NVFP4 with second-level scale s2. Per
 * 16-element block along K, in fp32:
 *   sf = e4m3_rne_satfinite(amax / (6 * s2))
 *   s  = e4m3(sf) * s2
 *   q  = e2m1_rne_satfinite(x / s)   (IEEE division; a zero s gives zeros
 *                                     carrying the sign of x)
 * Writes q [rows, k/2], sf_rowmajor [rows, k/16] (may be NULL) and sf_mma
 * (fp8q_nvfp4_sf_mma_bytes(rows, k) bytes, pad rows zeroed).
 * k a multiple of 64; rows*k below 2^31; s2 positive and finite; x, q and
 * sf_mma 16-byte aligned. rows == 0 returns FP8Q_OK and launches nothing.
 * Errors: NULL, ALIGN, SHAPE, ARG (s2), UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_nvfp4_quant(const void *x, void *q, void *sf_rowmajor, void *sf_mma,
                             float s2, uint32_t rows, uint32_t k, void *stream);

/*
 * NVFP4 GEMM on the block-scaled tensor cores:
 *   y[t][c] = bf16_rn( s2a * s2w * sum_k e2m1(qa[t][k]) * e4m3(sfa[t][k/16])
 *                                        * e2m1(qw[c][k]) * e4m3(sfw[c][k/16]) )
 * qa [m, k/2] with its MMA-layout scales sfa_mma, qw [n, k/2] with sfw_mma,
 * y bf16 [m, n] row-major. k a multiple of 256, n of 128; m*k, n*k and m*n
 * below 2^31; s2a, s2w positive and finite; every pointer 16-byte aligned.
 * m == 0 returns FP8Q_OK and launches nothing.
 * Errors: NULL, ALIGN, SHAPE, ARG, UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_nvfp4_gemm(const void *qa, const void *sfa_mma, float s2a,
                            const void *qw, const void *sfw_mma, float s2w,
                            void *y, uint32_t m, uint32_t n, uint32_t k, void *stream);

/* Workspace of fp8q_nvfp4_linear: the packed activation at offset 0 (m*k/2
   bytes, rounded up to 256), then its MMA-layout scales (rounded up to 256). */
size_t fp8q_nvfp4_linear_workspace_bytes(uint32_t m, uint32_t k);

/*
 * NVFP4 projection of a bf16 activation x [m, k], packed inside the call as
 * the pages' projection does: fp8q_nvfp4_quant(x, s2a) into `workspace`
 * (256-byte aligned, fp8q_nvfp4_linear_workspace_bytes(m, k) bytes), then
 * fp8q_nvfp4_gemm as its programmatic dependent on `stream`. The pages' call
 * takes no activation scale: s2a = 1 reproduces it.
 * Errors: as the two calls, plus WORKSPACE.
 */
fp8q_status fp8q_nvfp4_linear(const void *x, float s2a, const void *qw, const void *sfw_mma,
                              float s2w, void *y, void *workspace, size_t workspace_bytes,
                              uint32_t m, uint32_t n, uint32_t k, void *stream);

/*
 * FP8 weight back to bf16 (P-DP, `dequant_fp8_bf16_into`, the first step of
 * `cutlass_nvfp4_proj_from_fp8`): y[r][c] is the bf16 nearest to the exact
 * product e4m3(wq[r][c]) * ws(r, c) (ties to even, one rounding), with ws
 * the weight-format geometry above. k a multiple of 128 (n too for
 * FP8Q_WEIGHT_BLOCK128); n*k below 2^31; pointers 16-byte aligned.
 * Packing the result with fp8q_nvfp4_quant(s2 = 1) gives the pages' NVFP4
 * weight from an FP8 checkpoint.
 * Errors: NULL, ALIGN, SHAPE, ARG (format), UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_dequant_fp8_bf16(const void *wq, const float *w_scale, int32_t weight_format,
                                  void *y, uint32_t n, uint32_t k, void *stream);

/* ------------------------------------------------------- diagnostics ---- */

/*
 * Environment overrides, read once per process, for sweeps:
 *   FP8Q_QUANT_VARIANT=single|multi  the activation quantizer's variant (the
 *                                    bytes are the same either way)
 *   FP8Q_DECODE_SPLIT=<n>            K split of the FP8 GEMM at m <= 64
 *                                    (CTAs per cluster, at most 8 and k/128)
 *   FP8Q_NVFP4_SPLIT=<n>             K split of the NVFP4 GEMM when one row of
 *                                    128-column tiles is used (at most 8 and
 *                                    k/256)
 *   FP8Q_LOG=1                       one line on stderr the first time each
 *                                    quantizer choice is taken
 * The two splits group the fp32 partial sums differently, so y can change in
 * its last bits with them; a given split always gives the same y.
 */

/*
 * Convert `count` fp32 values to E2M1 codes (one per byte, low nibble) with
 * the conversion fp8q_nvfp4_quant uses (round-to-nearest-even, saturating
 * at 6). Used to check the conversion exhaustively. Device pointers.
 * Errors: NULL, UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_convert_e2m1(const float *in, uint8_t *out, size_t count, void *stream);

/*
 * Convert `count` fp32 values to e4m3 codes with the same device routine
 * the quantizers use (round-to-nearest-even, saturating at 448). Used to
 * check the conversion exhaustively. Device pointers.
 * Errors: NULL, UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_convert_e4m3(const float *in, uint8_t *out, size_t count, void *stream);

/*
 * Exhaustive device check of the quantizers' division. The quantizers form
 * the scale s = max(amax, 1e-10f)/448 and its reciprocal with a remainder
 * correction each, and x / s from that reciprocal and one more remainder
 * correction, instead of IEEE divisions. This call runs, for every finite
 * non-negative bf16 amax and every bf16 x with |x| <= amax (both signs),
 * those steps and the IEEE ones, and compares the scales, reciprocals, e4m3
 * codes and fp32 quotients.
 *   counts  device pointer to 4 uint64: [0] pairs checked (1065402240),
 *           [1] code mismatches, [2] fp32 quotient mismatches, [3] amax
 *           values whose scale or reciprocal differs from the IEEE one.
 * Errors: NULL, UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_check_division(unsigned long long *counts, void *stream);

/*
 * Exhaustive device check of SiLU(gate) * up. fp8q_silu_mul_quant forms h
 * in fp32 with the hardware exponential and reciprocal and falls back to an
 * exact fp64 evaluation near bf16 rounding ties and outside the fp32 path's
 * accurate range. This call runs both evaluations on every pair of finite
 * bf16 (gate, up).
 *   counts        device pointer to 3 uint64: [0] pairs (4261478400),
 *                 [1] pairs where the fp32 path is taken, [2] of those, the
 *                 pairs whose bf16 result differs from the fp64 path's
 *   max_err_bits  device pointer to 1 uint32: the largest error of the fp32
 *                 value, in fp32 ulps, as the bit pattern of an fp32 number
 * Errors: NULL, UNSUPPORTED_DEVICE, CUDA.
 */
fp8q_status fp8q_check_silu_mul(unsigned long long *counts, uint32_t *max_err_bits, void *stream);

/*
 * Diagnostic of the bounded waits (not part of the method): runs the two
 * kernels of fp8q_linear on the same arguments (the multi-group quantizer,
 * forced, then the GEMM that m selects) with every copy of their producers
 * suppressed and every wait bounded by `wait_budget_cycles` SM clocks, so
 * that each kernel's waits run out. Each kernel then raises its bit in the
 * device error word (fp8q_device_error: bit 2 the quantizer, bit 0 the GEMM),
 * lets nothing in flight outlive it, frees its tensor memory and returns; y
 * and the workspace are left unspecified. The call returns FP8Q_OK once both
 * kernels are enqueued; the context stays usable afterwards.
 * wait_budget_cycles: 1 .. 2e9 (about one second at B200 clocks; tests pass
 * about a millisecond). Errors: ARG, and those of fp8q_linear.
 */
fp8q_status fp8q_diag_stalled_linear(const void *x, const void *wq, const float *w_scale, void *y,
                                     void *workspace, size_t workspace_bytes,
                                     uint32_t m, uint32_t n, uint32_t k,
                                     uint64_t wait_budget_cycles, void *stream);

/* Number of kernels this library has launched in this process. */
uint64_t fp8q_launch_count(void);

/*
 * Read and clear the device error words of the current device: non-zero when
 * a kernel's bounded wait ran out (the kernel then stopped early and its
 * outputs are incomplete). Bit 0: an FP8 GEMM; bit 1: the NVFP4 GEMM; bit 2:
 * the multi-group activation quantizer. Synchronizes `stream` first. Returns FP8Q_OK or
 * FP8Q_ERR_DEVICE_TIMEOUT (with *code set), or FP8Q_ERR_CUDA.
 */
fp8q_status fp8q_device_error(void *stream, uint32_t *code);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H */
