// Block-scaled FP8 GEMM on the 5th-generation tensor cores.
//
//   y[t][c] = bf16( sum_g  a_s[t][g] * w_s[c/128][g] * P_g[t][c] ),
//   P_g[t][c] = sum_{j<128} q[t][128g+j] * wq[c][128g+j]
//
// (pages "spark_model/layers/ops/dispatch_proj.rs", `cublas_fp8_proj_prequant`:
// FP8 activation with per-[token,128-of-K] scales times an FP8 weight with
// per-128x128-block scales, bf16 out.)
//
// The scales are arbitrary fp32 values, so each 128-wide K block's partial
// product P_g is formed on its own by tcgen05 MMA (kind::f8f6f4, fp32 in
// TMEM) and promoted into an fp32 register accumulator by the epilogue warps
// with one scalar per row: a_s[t][g] * w_s[nb][g] (a 128-wide N tile lies in
// one weight block row, so the weight scale is one number per tile and K
// block). TMEM holds two partial buffers, so MMA of block g+1 overlaps the
// promotion of block g.
//
// CTA = 6 warps, tile 128 (tokens) x 128 (n), two CTAs per SM:
//   warp 0     TMA producer: A tile [128 x 128 B] and B tile [128 x 128 B]
//              per K block into a 3-stage ring (128-byte swizzle)
//   warp 1     TMEM allocator and MMA issuer (one thread)
//   warps 2-5  promotion + epilogue; warp w reads TMEM lanes 32*(w%4)..+31,
//              i.e. tile rows 32*(w%4)..+31, one row per thread
// Rows past M are zero-filled by TMA and never stored.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace fp8q {

// Device error word of this library, read and cleared by fp8q_device_error():
// bit 0 = a GEMM CTA gave up on a bounded wait.
__device__ uint32_t g_device_error = 0;

namespace {

constexpr uint32_t BM = 128;
constexpr uint32_t BN = 128;
constexpr uint32_t BK = 128;
constexpr uint32_t kStages = 3;
constexpr uint32_t kThreads = 192;
constexpr uint32_t kTileBytesA = BM * BK;
constexpr uint32_t kTileBytesB = BN * BK;
constexpr uint32_t kTmemCols = 2 * BN;

struct __align__(1024) GemmSmem {
    uint8_t a[kStages][kTileBytesA];
    uint8_t b[kStages][kTileBytesB];
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    uint32_t abort;
    uint32_t consumed;  // K blocks whose TMA data the MMA thread has seen land
};

constexpr size_t kSmemBytes = sizeof(GemmSmem) + 1024;  // + alignment slack

__global__ void __launch_bounds__(kThreads, 2)
    gemm_blockscaled_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const float* __restrict__ s_k, const float* __restrict__ w_s, uint16_t* __restrict__ y,
                            uint32_t M, uint32_t N, uint32_t G, uint32_t Mp) {
    extern __shared__ uint8_t smem_raw[];
    GemmSmem& sm = *reinterpret_cast<GemmSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t warp = threadIdx.x >> 5;
    const uint32_t lane = threadIdx.x & 31;
    const uint32_t nb = blockIdx.x;
    const uint32_t n0 = nb * BN;
    const uint32_t m0 = blockIdx.y * BM;
    volatile uint32_t* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (uint32_t s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (uint32_t b = 0; b < 2; ++b) {
            mbar_init(&sm.tfull[b], 1);
            mbar_init(&sm.tempty[b], 4);
        }
        mbar_init(&sm.mma_done, 1);
        sm.abort = 0;
        sm.consumed = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    uint32_t issued = 0;  // producer: K blocks whose loads were issued

    if (warp == 0) {
        if (lane == 0) {
            for (uint32_t kb = 0; kb < G; ++kb) {
                const uint32_t s = kb % kStages;
                const uint32_t ph = (kb / kStages) & 1u;
                if (!mbar_wait(&sm.empty[s], ph ^ 1u, abort)) break;
                mbar_arrive_expect_tx(&sm.full[s], kTileBytesA + kTileBytesB);
                tma_load_2d(sm.a[s], &tmA, &sm.full[s], static_cast<int32_t>(kb * BK), static_cast<int32_t>(m0));
                tma_load_2d(sm.b[s], &tmB, &sm.full[s], static_cast<int32_t>(kb * BK), static_cast<int32_t>(n0));
                issued = kb + 1;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_e4m3_f32(BM, BN);
            for (uint32_t kb = 0; kb < G; ++kb) {
                const uint32_t s = kb % kStages;
                const uint32_t ph = (kb / kStages) & 1u;
                if (!mbar_wait(&sm.full[s], ph, abort)) break;
                sm.consumed = kb + 1;
                const uint32_t b = kb & 1u;
                const uint32_t tph = (kb >> 1) & 1u;
                if (!mbar_wait(&sm.tempty[b], tph ^ 1u, abort)) break;
                tc_fence_after();
                const uint32_t d = tmem + b * BN;
                const uint64_t ad = smem_desc_k_sw128(smem_addr(sm.a[s]));
                const uint64_t bd = smem_desc_k_sw128(smem_addr(sm.b[s]));
#pragma unroll
                for (uint32_t kk = 0; kk < BK / 32; ++kk)  // K = 32 bytes per MMA; +32 B = +2 in the address field
                    mma_f8f6f4(d, ad + 2u * kk, bd + 2u * kk, idesc, kk > 0 ? 1u : 0u);
                mma_commit(&sm.empty[s]);
                mma_commit(&sm.tfull[b]);
            }
            // Every MMA this thread issued has completed once mma_done fires.
            mma_commit(&sm.mma_done);
            volatile uint32_t never = 0;
            mbar_wait(&sm.mma_done, 0, &never);
        }
    } else {
        const uint32_t quad = warp & 3u;
        const uint32_t row = m0 + quad * 32u + lane;
        const bool row_ok = row < M;
        float acc[BN];
#pragma unroll
        for (uint32_t i = 0; i < BN; ++i) acc[i] = 0.0f;
        float a_next = row_ok ? s_k[row] : 0.0f;
        bool ok = true;
        for (uint32_t kb = 0; kb < G; ++kb) {
            const uint32_t b = kb & 1u;
            const uint32_t tph = (kb >> 1) & 1u;
            const float a_cur = a_next;
            const float w_cur = __ldg(w_s + static_cast<size_t>(nb) * G + kb);
            if (row_ok && kb + 1 < G) a_next = s_k[static_cast<size_t>(kb + 1) * Mp + row];
            ok = mbar_wait(&sm.tfull[b], tph, abort);
            if (!__all_sync(0xFFFFFFFFu, ok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float c = a_cur * w_cur;
            const uint32_t taddr = tmem + ((quad * 32u) << 16) + b * BN;
#pragma unroll
            for (uint32_t ch = 0; ch < BN / 16; ++ch) {
                float v[16];
                tmem_load16(taddr + ch * 16u, v);
#pragma unroll
                for (uint32_t i = 0; i < 16; ++i) acc[ch * 16 + i] = fmaf(c, v[i], acc[ch * 16 + i]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.tempty[b]);
        }
        if (ok && row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(y + static_cast<size_t>(row) * N + n0);
#pragma unroll
            for (uint32_t j = 0; j < BN / 8; ++j) {
                uint32_t p[4];
#pragma unroll
                for (uint32_t e = 0; e < 4; ++e) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(acc[8 * j + 2 * e], acc[8 * j + 2 * e + 1]);
                    p[e] = *reinterpret_cast<uint32_t*>(&h);
                }
                dst[j] = make_uint4(p[0], p[1], p[2], p[3]);
            }
        }
    }

    // Teardown. On the normal path every TMA load was consumed and every MMA
    // was waited for by the epilogue. After a timed-out wait, first let the
    // copies and MMAs this CTA started finish (bounded), then free TMEM.
    tc_fence_before();
    __syncthreads();
    if (*abort) {
        volatile uint32_t never = 0;
        if (threadIdx.x == 0) atomicOr(&g_device_error, 1u);
        if (warp == 0 && lane == 0) {
            for (uint32_t kb = sm.consumed; kb < issued; ++kb)
                mbar_wait(&sm.full[kb % kStages], (kb / kStages) & 1u, &never);
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------ host side --

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A [rows, inner] uint8 matrix (row stride = inner bytes) read in
// [box_rows, 128-byte] tiles with the 128-byte swizzle.
bool make_map_u8(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t read_clear_device_error(uint32_t* code, cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    uint32_t zero = 0;
    e = cudaMemcpyFromSymbol(code, g_device_error, sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    if (*code) e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(uint32_t));
    return e;
}

cudaError_t launch_gemm(const GemmLaunch& L, cudaStream_t stream) {
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(gemm_blockscaled_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(kSmemBytes));
    });
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap ta, tb;
    if (!make_map_u8(&ta, L.q, L.k, L.m, BM) || !make_map_u8(&tb, L.wq, L.k, L.n, BN))
        return cudaErrorInvalidValue;
    dim3 grid(L.n / BN, (L.m + BM - 1) / BM);
    gemm_blockscaled_kernel<<<grid, kThreads, kSmemBytes, stream>>>(ta, tb, L.s_k, L.w_scale,
                                                                    static_cast<uint16_t*>(L.y), L.m, L.n, L.k / BK,
                                                                    L.mp);
    note_launch();
    return cudaGetLastError();
}

}  // namespace fp8q
