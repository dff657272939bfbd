// Activation and weight quantizers: bf16 -> OCP FP8 E4M3 with fp32 scales.
//
// Method (pages "spark_model/layers/ops/dispatch_proj.rs", `cublas_fp8_proj`,
// and "spark_model/layers/ops/fp8_act_quant_floor.rs", module header):
// per token and per 128-wide K group, amax = max |x|, s = max(amax, 1e-10)/448
// (IEEE fp32 division), q = e4m3 RNE-satfinite of x/s (IEEE fp32 division).
//
// Both activation variants are one HBM stream. In SINGLE a 128-element group
// is owned by 16 lanes holding 8 bf16 each (one 16-byte load), in MULTI by 8
// lanes holding 16; amax is reduced with xor-shuffles inside those lanes and
// each lane stores its codes as 8-byte stores, so a group's 128 codes leave
// as contiguous runs.
// The scale goes to the row-major [M, K/128] buffer and, in the same kernel,
// to the K-major [K/128, ceil16(M)] buffer, whose pad rows the same launch
// zero-fills; the pages spend a separate transpose launch on that layout
// (`fp8_act_scale_to_kmajor`).
//
//   SINGLE: one group per CTA (16 threads), grid (K/128, M).
//   MULTI : 8 consecutive groups of RPC consecutive tokens per CTA
//           (64 threads, 8 lanes per group), grid (ceil((K/128)/8),
//           ceil(M/RPC)). Each lane keeps 2*RPC independent 16-byte loads
//           in flight.
#include <cuda_bf16.h>

#include "group_quant.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace fp8q {

// SINGLE: blockDim 16, grid (G, M): CTA (g, t) quantizes group g of token t.
__global__ void __launch_bounds__(16) quant_act_single_kernel(const uint16_t* __restrict__ x,
                                                             uint8_t* __restrict__ q, float* __restrict__ s_row,
                                                             float* __restrict__ s_k, uint32_t m, uint32_t k,
                                                             uint32_t mp) {
    if (gridDim.x * gridDim.y <= kSingleTriggerMaxGrid) trigger_dependents();
    const uint32_t G = gridDim.x;
    const uint32_t g = blockIdx.x, t = blockIdx.y;
    const uint32_t lane = threadIdx.x;
    const size_t off = static_cast<size_t>(t) * k + static_cast<size_t>(g) * 128 + lane * 8;
    const uint4 v = ld_stream16(x + off);
    float f[8];
    widen8(v, f);
    float amax = absmax8_bits(v);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0x0000FFFFu, amax, o));
    const float s = group_scale(amax);
    st_stream8(q + off, encode8(f, s));
    if (lane == 0) {
        if (s_row) s_row[static_cast<size_t>(t) * G + g] = s;
        s_k[static_cast<size_t>(g) * mp + t] = s;
    }
    zero_kmajor_pad(s_k, m, mp, G);
}

// MULTI: blockDim 64, grid (ceil(G/8), ceil(m/RPC)). Eight lanes own one
// group: lane l holds elements 8l..8l+7 and 64+8l..64+8l+7 of it (two 16-byte
// loads, each instruction covering the group's 128 contiguous bytes), so the
// per-group work (scale, reciprocal, shuffles, scale stores) is shared by 16
// elements per lane. Octet o of CTA (bx, by) owns group g = 8*bx + o for
// tokens RPC*by .. RPC*by + RPC - 1; every load of the CTA is issued before
// any arithmetic. Token validity is the same for the whole CTA, so rows past
// m are skipped outright; a group past G (K/128 not a multiple of 8) computes
// on zeros, so the shuffles still see their full warp, and stores nothing.
template <int RPC>
__global__ void __launch_bounds__(64) quant_act_multi_kernel(const uint16_t* __restrict__ x,
                                                            uint8_t* __restrict__ q, float* __restrict__ s_row,
                                                            float* __restrict__ s_k, uint32_t m, uint32_t k,
                                                            uint32_t mp) {
    if ((blockIdx.y * gridDim.x + blockIdx.x) + kMultiTriggerTail >= gridDim.x * gridDim.y) trigger_dependents();
    const uint32_t G = k >> 7;
    const uint32_t lane = threadIdx.x & 7;
    const uint32_t g = blockIdx.x * 8 + (threadIdx.x >> 3);
    const uint32_t t0 = blockIdx.y * RPC;
    const bool g_ok = g < G;
    const uint32_t rows = m - t0 < static_cast<uint32_t>(RPC) ? m - t0 : static_cast<uint32_t>(RPC);
    uint4 v[RPC][2];
#pragma unroll
    for (int r = 0; r < RPC; ++r) {
        if (g_ok && static_cast<uint32_t>(r) < rows) {
            const uint16_t* src = x + static_cast<size_t>(t0 + r) * k + static_cast<size_t>(g) * 128 + lane * 8;
            v[r][0] = ld_stream16(src);
            v[r][1] = ld_stream16(src + 64);
        } else {
            v[r][0] = make_uint4(0u, 0u, 0u, 0u);
            v[r][1] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
#pragma unroll
    for (int r = 0; r < RPC; ++r) {
        if (static_cast<uint32_t>(r) >= rows) break;
        const uint32_t t = t0 + r;
        float amax = fmaxf(absmax8_bits(v[r][0]), absmax8_bits(v[r][1]));
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        const float s = group_scale(amax);
        float f0[8], f1[8];
        widen8(v[r][0], f0);
        widen8(v[r][1], f1);
        const uint2 c0 = encode8(f0, s);
        const uint2 c1 = encode8(f1, s);
        if (g_ok) {
            uint8_t* dst = q + static_cast<size_t>(t) * k + static_cast<size_t>(g) * 128 + lane * 8;
            st_stream8(dst, c0);
            st_stream8(dst + 64, c1);
            if (lane == 0) {
                if (s_row) s_row[static_cast<size_t>(t) * G + g] = s;
                s_k[static_cast<size_t>(g) * mp + t] = s;
            }
        }
    }
    zero_kmajor_pad(s_k, m, mp, G);
}

// Weight blocks: grid (K/128, N/128), 256 threads. The block's 128 rows x
// 256 bytes are 2048 16-byte chunks; thread i owns chunks i + 256 j.
__global__ void __launch_bounds__(256) quant_weight_kernel(const uint16_t* __restrict__ w, uint8_t* __restrict__ wq,
                                                           float* __restrict__ w_scale, uint32_t k) {
    __shared__ float red[8];
    const uint32_t G = gridDim.x;
    const uint32_t bg = blockIdx.x, bn = blockIdx.y;
    float f[8][8];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t c = threadIdx.x + 256u * j;
        const size_t off = static_cast<size_t>(bn * 128u + (c >> 4)) * k + bg * 128u + (c & 15u) * 8u;
        const uint4 v = ld_stream16(w + off);
        widen8(v, f[j]);
        amax = fmaxf(amax, absmax8_bits(v));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
    const float s = group_scale(amax);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t c = threadIdx.x + 256u * j;
        const size_t off = static_cast<size_t>(bn * 128u + (c >> 4)) * k + bg * 128u + (c & 15u) * 8u;
        *reinterpret_cast<uint2*>(wq + off) = encode8(f[j], s);
    }
    if (threadIdx.x == 0) w_scale[static_cast<size_t>(bn) * G + bg] = s;
}

// Per-row weights (scale block 1 x K): one CTA of 256 threads per row. The
// row's amax is reduced over the whole row, then the row is read again and
// encoded with that one scale.
__global__ void __launch_bounds__(256) quant_weight_rowwise_kernel(const uint16_t* __restrict__ w,
                                                                   uint8_t* __restrict__ wq,
                                                                   float* __restrict__ w_scale, uint32_t k) {
    __shared__ float red[8];
    const size_t base = static_cast<size_t>(blockIdx.x) * k;
    float amax = 0.0f;
    for (uint32_t c = threadIdx.x * 8u; c < k; c += 256u * 8u) amax = fmaxf(amax, absmax8_bits(ld_stream16(w + base + c)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
    const float s = group_scale(amax);
    for (uint32_t c = threadIdx.x * 8u; c < k; c += 256u * 8u) {
        float f[8];
        widen8(*reinterpret_cast<const uint4*>(w + base + c), f);
        *reinterpret_cast<uint2*>(wq + base + c) = encode8(f, s);
    }
    if (threadIdx.x == 0) w_scale[blockIdx.x] = s;
}

// Element-wise fp32 -> e4m3 with the conversion the quantizers use.
__global__ void convert_e4m3_kernel(const float* __restrict__ in, uint8_t* __restrict__ out, size_t n) {
    const size_t pairs = (n + 1) / 2;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < pairs;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const size_t e = 2 * i;
        const bool two = e + 1 < n;
        const uint16_t c = cvt_e4m3x2(in[e], two ? in[e + 1] : 0.0f);
        out[e] = static_cast<uint8_t>(c & 0xFF);
        if (two) out[e + 1] = static_cast<uint8_t>(c >> 8);
    }
}

// Exhaustive check of the quantizers' division against IEEE division. CTA b
// takes amax = the non-negative bf16 with bit pattern b (0 .. 0x7F7F, every
// finite value), forms s = group_scale(amax) and, for every bf16 x with
// |x| <= amax and both signs, compares the e4m3 code of div2_by_scale with
// the code of __fdiv_rn(x, s), and the fp32 quotients themselves.
// counts[0] += pairs checked, counts[1] += code mismatches,
// counts[2] += fp32 quotient mismatches.
__global__ void __launch_bounds__(256) check_division_kernel(unsigned long long* __restrict__ counts) {
    const uint32_t a_bits = blockIdx.x;
    const float amax = __uint_as_float(a_bits << 16);
    const float s = group_scale(amax);
    const float r = __frcp_rn(s);
    unsigned long long pairs = 0, code_bad = 0, quot_bad = 0;
    for (uint32_t xb = threadIdx.x; xb <= a_bits; xb += blockDim.x) {
        const float xp = __uint_as_float(xb << 16);
        const float2 xv = make_float2(xp, -xp);
        const float2 qf = div2_by_scale(xv, s, r);
        const float qa = __fdiv_rn(xv.x, s), qb = __fdiv_rn(xv.y, s);
        const uint16_t c_fast = cvt_e4m3x2(qf.x, qf.y);
        const uint16_t c_ieee = cvt_e4m3x2(qa, qb);
        pairs += 2;
        code_bad += ((c_fast & 0xFF) != (c_ieee & 0xFF)) + ((c_fast >> 8) != (c_ieee >> 8));
        quot_bad += (__float_as_uint(qf.x) != __float_as_uint(qa)) + (__float_as_uint(qf.y) != __float_as_uint(qb));
    }
    for (int o = 16; o > 0; o >>= 1) {
        pairs += __shfl_xor_sync(0xFFFFFFFFu, pairs, o);
        code_bad += __shfl_xor_sync(0xFFFFFFFFu, code_bad, o);
        quot_bad += __shfl_xor_sync(0xFFFFFFFFu, quot_bad, o);
    }
    if ((threadIdx.x & 31) == 0) {
        atomicAdd(&counts[0], pairs);
        atomicAdd(&counts[1], code_bad);
        atomicAdd(&counts[2], quot_bad);
    }
}

// ------------------------------------------------------------ launchers --

cudaError_t launch_quant_act(const QuantLaunch& L, cudaStream_t stream) {
    const uint32_t G = L.k >> 7;
    if (L.variant == kVariantSingle) {
        dim3 grid(G, L.m);
        quant_act_single_kernel<<<grid, 16, 0, stream>>>(static_cast<const uint16_t*>(L.x), static_cast<uint8_t*>(L.q),
                                                         L.s_row, L.s_k, L.m, L.k, L.mp);
    } else {
        dim3 grid((G + 7) / 8, (L.m + kMultiRowsPerCta - 1) / kMultiRowsPerCta);
        quant_act_multi_kernel<kMultiRowsPerCta><<<grid, 64, 0, stream>>>(
            static_cast<const uint16_t*>(L.x), static_cast<uint8_t*>(L.q), L.s_row, L.s_k, L.m, L.k, L.mp);
    }
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_quant_weight(const void* w, void* wq, float* w_scale, uint32_t n, uint32_t k,
                                cudaStream_t stream) {
    dim3 grid(k / 128, n / 128);
    quant_weight_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint16_t*>(w), static_cast<uint8_t*>(wq),
                                                  w_scale, k);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_quant_weight_rowwise(const void* w, void* wq, float* w_scale, uint32_t n, uint32_t k,
                                        cudaStream_t stream) {
    quant_weight_rowwise_kernel<<<n, 256, 0, stream>>>(static_cast<const uint16_t*>(w), static_cast<uint8_t*>(wq),
                                                       w_scale, k);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_check_division(unsigned long long* counts, cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(counts, 0, 3 * sizeof(unsigned long long), stream);
    if (e != cudaSuccess) return e;
    check_division_kernel<<<0x7F80, 256, 0, stream>>>(counts);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_convert_e4m3(const float* in, uint8_t* out, size_t n, cudaStream_t stream) {
    const size_t pairs = (n + 1) / 2;
    size_t blocks = (pairs + 255) / 256;
    if (blocks > 148u * 64u) blocks = 148u * 64u;
    if (blocks == 0) blocks = 1;
    convert_e4m3_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(in, out, n);
    note_launch();
    return cudaGetLastError();
}

}  // namespace fp8q
