// Activation and weight quantizers: bf16 -> OCP FP8 E4M3 with fp32 scales.
//
// Method (pages "spark_model/layers/ops/dispatch_proj.rs", `cublas_fp8_proj`,
// and "spark_model/layers/ops/fp8_act_quant_floor.rs", module header):
// per token and per 128-wide K group, amax = max |x|, s = max(amax, 1e-10)/448
// (IEEE fp32 division), q = e4m3 RNE-satfinite of x/s (IEEE fp32 division).
//
// The scale goes to the row-major [M, K/128] buffer and, in the same kernel,
// to the K-major [K/128, ceil16(M)] buffer, whose pad rows the same launch
// zero-fills; the pages spend a separate transpose launch on that layout
// (`fp8_act_scale_to_kmajor`).
//
//   SINGLE: one group per CTA (16 threads, 16 bytes each), 1-D grid of M*G
//           CTAs: many small CTAs, the lowest latency for decode widths.
//   MULTI : a persistent streaming kernel. X [M, K] row-major is one
//           contiguous run of M*G groups of 256 bytes, in (token, group)
//           order, and so are the codes (128 bytes a group) and the
//           row-major scales. The run is cut into stages of 32 groups (8 KB
//           of X); CTA c takes stages c, c + C, c + 2C, ... A producer thread
//           streams each stage into a shared-memory ring with one bulk copy
//           (cp.async.bulk, completion counted on an mbarrier), up to
//           kStreamSlots stages ahead, so an SM keeps up to 4 x 48 KB of X in
//           flight from the kernel's first cycles. Eight consumer warps each
//           quantize 4 groups of every stage (8 lanes per group, 16 elements
//           a lane) and store codes and scales directly.
#include <cuda_bf16.h>

#include "group_quant.cuh"
#include "internal.h"
#include "ptx.cuh"

#include <mutex>

namespace fp8q {

// Device error word of the activation quantizer (bit 2 of fp8q_device_error):
// a streaming CTA gave up on a bounded wait.
__device__ uint32_t g_quant_error = 0;
constexpr uint32_t kQuantErrorBit = 4u;

// SINGLE: blockDim 16, 1-D grid of G*M CTAs: CTA b quantizes group b % G of
// token b / G.
__global__ void __launch_bounds__(16) quant_act_single_kernel(const uint16_t* __restrict__ x,
                                                             uint8_t* __restrict__ q, float* __restrict__ s_row,
                                                             float* __restrict__ s_k, uint32_t m, uint32_t k,
                                                             uint32_t mp) {
    const uint32_t G = k >> 7;
    const uint32_t t = blockIdx.x / G, g = blockIdx.x - t * G;
    const uint32_t lane = threadIdx.x;
    const size_t off = static_cast<size_t>(t) * k + static_cast<size_t>(g) * 128 + lane * 8;
    // Nothing is read or written in global memory before the grid this
    // launch may depend on has completed; only then may the dependent (the
    // GEMM of a fused linear) launch, so that everything before this kernel
    // in the stream has completed when it starts.
    grid_dependency_wait();
    if (gridDim.x <= kSingleTriggerMaxGrid) trigger_dependents();
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

// MULTI (streaming). Every warp is an independent stream: its lane 0
// bulk-copies chunks of kStreamChunkGroups groups (4 KB of X) into the
// warp's own ring of kStreamSlots shared-memory slots, each completion
// counted on the slot's own mbarrier, and the warp quantizes each chunk as
// it lands, two lanes per group (64 elements a lane). The chunk's codes (2 KB,
// contiguous in Q) are gathered in a shared-memory staging buffer and leave
// with one bulk store, so every 128-byte line of Q is written whole. No warp
// waits for another. Chunk c goes to CTA c % gridDim.x, warp
// (c / gridDim.x) % kStreamWarps, so consecutive chunks are in flight on
// different SMs.
constexpr uint32_t kStreamChunkBytes = kStreamChunkGroups * 256;
constexpr uint32_t kStreamCodeBytes = kStreamChunkGroups * 128;
constexpr uint32_t kStreamWarpBytes = kStreamSlots * kStreamChunkBytes + kStreamCodeBytes;
constexpr uint32_t kStreamSmemBytes = kStreamWarps * (kStreamWarpBytes + kStreamSlots * 8);
static_assert(kStreamChunkGroups == 16, "two lanes per group, 32 lanes a chunk");

// Bounded wait on one of this warp's barriers; false when the budget ran out.
__device__ __forceinline__ bool warp_slot_wait(uint64_t* bar, uint32_t parity, long long budget) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > budget) return false;
    return true;
}

__global__ void __launch_bounds__(kStreamThreads, kStreamCtasPerSm)
    quant_act_stream_kernel(const uint16_t* __restrict__ x, uint8_t* __restrict__ q, float* __restrict__ s_row,
                            float* __restrict__ s_k, uint32_t m, uint32_t k, uint32_t mp, long long budget,
                            uint32_t no_copies) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* ring = smem + warp * kStreamWarpBytes;
    uint8_t* codes = ring + kStreamSlots * kStreamChunkBytes;  // this warp's staging buffer
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStreamWarps * kStreamWarpBytes) + warp * kStreamSlots;
    const uint32_t G = k >> 7;
    const uint32_t total = m * G;  // groups; m*k < 2^31 keeps this below 2^24
    const uint32_t chunks = (total + kStreamChunkGroups - 1) / kStreamChunkGroups;
    const uint32_t first = blockIdx.x + gridDim.x * warp;
    const uint32_t stride = gridDim.x * kStreamWarps;
    const uint32_t mine = first < chunks ? (chunks - 1 - first) / stride + 1 : 0;

    if (lane == 0) {
        for (uint32_t i = 0; i < kStreamSlots; ++i) mbar_init(&full[i], 1);
        fence_mbar_init();
    }
    __syncwarp();
    // Nothing is read or written in global memory before the grid this
    // launch may depend on has completed; only then may the dependent (the
    // GEMM of a fused linear) launch, so that everything before this kernel
    // in the stream has completed when it starts.
    grid_dependency_wait();
    trigger_dependents();
    zero_kmajor_pad(s_k, m, mp, G);

    auto issue = [&](uint32_t i) {
        const uint32_t slot = i % kStreamSlots;
        const uint32_t g0 = (first + i * stride) * kStreamChunkGroups;
        const uint32_t n = total - g0 < kStreamChunkGroups ? total - g0 : kStreamChunkGroups;
        mbar_arrive_expect_tx(&full[slot], n * 256u);
        bulk_load(ring + slot * kStreamChunkBytes, x + static_cast<size_t>(g0) * 128, n * 256u, &full[slot]);
    };
    uint32_t issued = 0;
    if (lane == 0 && !no_copies) {
        for (; issued < kStreamSlots && issued < mine; ++issued) issue(issued);
    }

    // Lane 2*gl + p owns half p of group gl of each chunk: 16-byte pieces
    // c = 2j + p, j = 0..7 (elements 8c..8c+7), read in the order
    // j = (i + gl) % 8 so that the eight lanes of every shared-memory phase
    // touch eight different 16-byte columns of a 128-byte row.
    const uint32_t gl = lane >> 1, p = lane & 1u;
    bool ok = true;
    uint32_t done = 0;
    for (; done < mine; ++done) {
        const uint32_t slot = done % kStreamSlots;
        if (!__all_sync(0xFFFFFFFFu, warp_slot_wait(&full[slot], (done / kStreamSlots) & 1u, budget))) {
            ok = false;
            break;
        }
        const uint32_t g0 = (first + done * stride) * kStreamChunkGroups;
        const uint32_t gf = g0 + gl;
        const bool valid = gf < total;
        uint4 v[8];
        const uint8_t* src = ring + slot * kStreamChunkBytes + gl * 256u + p * 16u;
#pragma unroll
        for (uint32_t i = 0; i < 8; ++i)
            v[i] = valid ? *reinterpret_cast<const uint4*>(src + ((i + gl) & 7u) * 32u) : make_uint4(0u, 0u, 0u, 0u);
        // group amax: pairwise max of |bf16| over the 32 words, then the two
        // halves, then the partner lane
        uint32_t w[16];
#pragma unroll
        for (uint32_t i = 0; i < 4; ++i) {
            w[4 * i + 0] = absmax_bf16x2(v[2 * i].x, v[2 * i + 1].x);
            w[4 * i + 1] = absmax_bf16x2(v[2 * i].y, v[2 * i + 1].y);
            w[4 * i + 2] = absmax_bf16x2(v[2 * i].z, v[2 * i + 1].z);
            w[4 * i + 3] = absmax_bf16x2(v[2 * i].w, v[2 * i + 1].w);
        }
#pragma unroll
        for (uint32_t n = 8; n > 0; n >>= 1)
#pragma unroll
            for (uint32_t i = 0; i < n; ++i) w[i] = absmax_bf16x2(w[i], w[i + n]);
        const uint32_t hi = (w[0] >> 16) & 0x7FFFu, lo = w[0] & 0x7FFFu;
        float amax = __uint_as_float((hi > lo ? hi : lo) << 16);
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        // Every lane has read its pieces (the maximum used them all): the
        // slot may be refilled with the chunk kStreamSlots ahead.
        __syncwarp();
        if (lane == 0 && issued < mine) {
            fence_proxy_async_smem();
            issue(issued++);
        }
        const float sc = group_scale(amax);
        const float nr = neg_recip(sc);
        uint2 c[8];
#pragma unroll
        for (uint32_t i = 0; i < 8; ++i) {
            float f[8];
            widen8(v[i], f);
            c[i] = encode8_nr(f, sc, nr);
        }
        // The staging buffer is free once the previous chunk's bulk store
        // has read it.
        if (lane == 0) bulk_store_wait_read();
        __syncwarp();
        uint8_t* row = codes + gl * 128u + p * 8u;
#pragma unroll
        for (uint32_t i = 0; i < 8; ++i) *reinterpret_cast<uint2*>(row + ((i + gl) & 7u) * 16u) = c[i];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            const uint32_t n = total - g0 < kStreamChunkGroups ? total - g0 : kStreamChunkGroups;
            bulk_store(q + static_cast<size_t>(g0) * 128, codes, n * 128u);
        }
        if (valid && p == 0) {
            if (s_row) s_row[gf] = sc;
            const uint32_t t = gf / G;
            s_k[static_cast<size_t>(gf - t * G) * mp + t] = sc;
        }
    }
    if (!ok) {
        // A wait ran out: report it, and let this warp's copies still in
        // flight land (bounded) before the warp exits.
        if (lane == 0) {
            atomicOr(&g_quant_error, kQuantErrorBit);
            for (uint32_t i = done; i < issued; ++i)
                warp_slot_wait(&full[i % kStreamSlots], (i / kStreamSlots) & 1u, kWaitBudgetCycles);
        }
    }
    // The codes are in global memory before the warp (and its CTA's shared
    // memory) goes away.
    if (lane == 0) bulk_store_wait_all();
    __syncwarp();
}

// Weight blocks: a 1-D grid of (N/128) * (K/128) CTAs of 256 threads, CTA
// bn * (K/128) + bg quantizing block (bn, bg). The block's 128 rows x 256
// bytes are 2048 16-byte chunks; thread i owns chunks i + 256 j.
__global__ void __launch_bounds__(256) quant_weight_kernel(const uint16_t* __restrict__ w, uint8_t* __restrict__ wq,
                                                           float* __restrict__ w_scale, uint32_t k) {
    __shared__ float red[8];
    const uint32_t G = k >> 7;
    const uint32_t bn = blockIdx.x / G, bg = blockIdx.x - bn * G;
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
// finite value). It checks the group scale and its negated reciprocal
// against __fdiv_rn and __frcp_rn, then, for every bf16 x with |x| <= amax
// and both signs, compares the sign-flipped e4m3 code of neg_div2_by_scale
// with the code of the IEEE quotient __fdiv_rn(x, s), and the negated fp32
// quotients with __fdiv_rn's.
// counts[0] += pairs checked, counts[1] += code mismatches,
// counts[2] += fp32 quotient mismatches, counts[3] += amax values whose
// scale or reciprocal differs from the IEEE one.
__global__ void __launch_bounds__(256) check_division_kernel(unsigned long long* __restrict__ counts) {
    const uint32_t a_bits = blockIdx.x;
    const float amax = __uint_as_float(a_bits << 16);
    const float s = group_scale(amax);
    const float nr = neg_recip(s);
    const float s_ieee = __fdiv_rn(fmaxf(amax, 1e-10f), 448.0f);
    if (threadIdx.x == 0)
        atomicAdd(&counts[3], static_cast<unsigned long long>((__float_as_uint(s) != __float_as_uint(s_ieee)) +
                                                              (__float_as_uint(-nr) != __float_as_uint(__frcp_rn(s_ieee)))));
    unsigned long long pairs = 0, code_bad = 0, quot_bad = 0;
    for (uint32_t xb = threadIdx.x; xb <= a_bits; xb += blockDim.x) {
        const float xp = __uint_as_float(xb << 16);
        const float2 xv = make_float2(xp, -xp);
        const float2 qn = neg_div2_by_scale(xv, s, nr);
        const float qa = __fdiv_rn(xv.x, s_ieee), qb = __fdiv_rn(xv.y, s_ieee);
        const uint16_t c_fast = cvt_e4m3x2(qn.x, qn.y) ^ static_cast<uint16_t>(kCodeSignBits & 0xFFFFu);
        const uint16_t c_ieee = cvt_e4m3x2(qa, qb);
        pairs += 2;
        code_bad += ((c_fast & 0xFF) != (c_ieee & 0xFF)) + ((c_fast >> 8) != (c_ieee >> 8));
        quot_bad += ((__float_as_uint(qn.x) ^ 0x80000000u) != __float_as_uint(qa)) +
                    ((__float_as_uint(qn.y) ^ 0x80000000u) != __float_as_uint(qb));
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

uint32_t stream_grid(uint32_t m, uint32_t k, uint32_t sms) {
    const uint32_t total = m * (k >> 7);
    const uint32_t chunks = (total + kStreamChunkGroups - 1) / kStreamChunkGroups;
    const uint32_t cap = sms * kStreamCtasPerSm;
    return chunks < cap ? chunks : cap;
}

cudaError_t launch_quant_act(const QuantLaunch& L, cudaStream_t stream) {
    const uint32_t G = L.k >> 7;
    // Both kernels wait for the grid before them (griddepcontrol.wait) before
    // touching global memory, so they may launch as soon as that grid allows.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    if (L.variant == kVariantSingle) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(G * L.m, 1, 1);
        cfg.blockDim = dim3(16, 1, 1);
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, quant_act_single_kernel, static_cast<const uint16_t*>(L.x),
                                                 static_cast<uint8_t*>(L.q), L.s_row, L.s_k, L.m, L.k, L.mp);
        note_launch();
        return e != cudaSuccess ? e : cudaGetLastError();
    }
    static std::once_flag once[64];
    static cudaError_t optin[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [dev] {
        optin[dev] = cudaFuncSetAttribute(quant_act_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(kStreamSmemBytes));
    });
    if (optin[dev] != cudaSuccess) return optin[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(stream_grid(L.m, L.k, L.sms), 1, 1);
    cfg.blockDim = dim3(kStreamThreads, 1, 1);
    cfg.dynamicSmemBytes = kStreamSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, quant_act_stream_kernel, static_cast<const uint16_t*>(L.x),
                           static_cast<uint8_t*>(L.q), L.s_row, L.s_k, L.m, L.k, L.mp,
                           L.diag_budget != 0 ? L.diag_budget : kWaitBudgetCycles,
                           L.diag_budget != 0 ? 1u : 0u);
    note_launch();
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t read_clear_quant_error(uint32_t* code, cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    uint32_t zero = 0;
    e = cudaMemcpyFromSymbol(code, g_quant_error, sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    if (*code) e = cudaMemcpyToSymbol(g_quant_error, &zero, sizeof(uint32_t));
    return e;
}

cudaError_t launch_quant_weight(const void* w, void* wq, float* w_scale, uint32_t n, uint32_t k,
                                cudaStream_t stream) {
    quant_weight_kernel<<<(k / 128) * (n / 128), 256, 0, stream>>>(static_cast<const uint16_t*>(w), static_cast<uint8_t*>(wq),
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
    cudaError_t e = cudaMemsetAsync(counts, 0, 4 * sizeof(unsigned long long), stream);
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
