// Activation and weight quantizers: bf16 -> OCP FP8 E4M3 with fp32 scales.
//
// Method (pages "spark_model/layers/ops/dispatch_proj.rs", `cublas_fp8_proj`,
// and "spark_model/layers/ops/fp8_act_quant_floor.rs", module header):
// per token and per 128-wide K group, amax = max |x|, s = max(amax, 1e-10)/448
// (IEEE fp32 division), q = e4m3 RNE-satfinite of x/s (IEEE fp32 division).
//
// Both activation variants are one HBM stream. A 128-element group is owned
// by 16 lanes holding 8 bf16 each (one 16-byte load); amax is reduced with
// four xor-shuffles inside the 16 lanes; each lane stores its 8 codes as one
// 8-byte store, so a group's 128 codes leave as one contiguous 128-byte run.
// The scale goes to the row-major [M, K/128] buffer and, in the same kernel,
// to the K-major [K/128, ceil16(M)] buffer, whose pad rows the same launch
// zero-fills; the pages spend a separate transpose launch on that layout
// (`fp8_act_scale_to_kmajor`).
//
//   SINGLE: one group per CTA (16 threads), grid (K/128, M).
//   MULTI : 8 consecutive groups of RPC consecutive tokens per CTA
//           (128 threads), grid (ceil((K/128)/8), ceil(M/RPC)). Each lane
//           keeps RPC independent 16-byte loads in flight.
#include <cuda_bf16.h>

#include "internal.h"
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

__device__ __forceinline__ float absmax8(const float (&f)[8]) {
    float a = fabsf(f[0]);
#pragma unroll
    for (int i = 1; i < 8; ++i) a = fmaxf(a, fabsf(f[i]));
    return a;
}

// The scale of a group with absolute maximum `amax`: one fp32 division.
__device__ __forceinline__ float group_scale(float amax) {
    return __fdiv_rn(fmaxf(amax, 1e-10f), 448.0f);
}

// 8 values / s (IEEE division each) -> 8 codes packed little-endian.
__device__ __forceinline__ uint2 encode8(const float (&f)[8], float s) {
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint16_t p = cvt_e4m3x2(__fdiv_rn(f[2 * i], s), __fdiv_rn(f[2 * i + 1], s));
        c[i] = p;
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
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

// SINGLE: blockDim 16, grid (G, M): CTA (g, t) quantizes group g of token t.
__global__ void __launch_bounds__(16) quant_act_single_kernel(const uint16_t* __restrict__ x,
                                                             uint8_t* __restrict__ q, float* __restrict__ s_row,
                                                             float* __restrict__ s_k, uint32_t m, uint32_t k,
                                                             uint32_t mp) {
    const uint32_t G = gridDim.x;
    const uint32_t g = blockIdx.x, t = blockIdx.y;
    const uint32_t lane = threadIdx.x;
    const size_t off = static_cast<size_t>(t) * k + static_cast<size_t>(g) * 128 + lane * 8;
    float f[8];
    widen8(ld_stream16(x + off), f);
    float amax = absmax8(f);
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

// MULTI: blockDim 128 (8 half-warps), grid (ceil(G/8), ceil(m/RPC)).
// Half-warp h of CTA (bx, by) owns group g = 8*bx + h for tokens
// RPC*by .. RPC*by + RPC - 1. Out-of-range groups/tokens compute on zeros
// (so every shuffle sees its full warp) and store nothing.
template <int RPC>
__global__ void __launch_bounds__(128) quant_act_multi_kernel(const uint16_t* __restrict__ x,
                                                             uint8_t* __restrict__ q, float* __restrict__ s_row,
                                                             float* __restrict__ s_k, uint32_t m, uint32_t k,
                                                             uint32_t mp) {
    const uint32_t G = k >> 7;
    const uint32_t lane = threadIdx.x & 15;
    const uint32_t g = blockIdx.x * 8 + (threadIdx.x >> 4);
    const uint32_t t0 = blockIdx.y * RPC;
    const bool g_ok = g < G;
    uint4 v[RPC];
#pragma unroll
    for (int r = 0; r < RPC; ++r) {
        const uint32_t t = t0 + r;
        if (g_ok && t < m)
            v[r] = ld_stream16(x + static_cast<size_t>(t) * k + static_cast<size_t>(g) * 128 + lane * 8);
        else
            v[r] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int r = 0; r < RPC; ++r) {
        const uint32_t t = t0 + r;
        float f[8];
        widen8(v[r], f);
        float amax = absmax8(f);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        const float s = group_scale(amax);
        const uint2 codes = encode8(f, s);
        if (g_ok && t < m) {
            st_stream8(q + static_cast<size_t>(t) * k + static_cast<size_t>(g) * 128 + lane * 8, codes);
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
        widen8(ld_stream16(w + off), f[j]);
        amax = fmaxf(amax, absmax8(f[j]));
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

// ------------------------------------------------------------ launchers --

cudaError_t launch_quant_act(const QuantLaunch& L, cudaStream_t stream) {
    const uint32_t G = L.k >> 7;
    if (L.variant == kVariantSingle) {
        dim3 grid(G, L.m);
        quant_act_single_kernel<<<grid, 16, 0, stream>>>(static_cast<const uint16_t*>(L.x), static_cast<uint8_t*>(L.q),
                                                         L.s_row, L.s_k, L.m, L.k, L.mp);
    } else {
        dim3 grid((G + 7) / 8, (L.m + kMultiRowsPerCta - 1) / kMultiRowsPerCta);
        quant_act_multi_kernel<kMultiRowsPerCta><<<grid, 128, 0, stream>>>(
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
