// Block-scaled FP8 GEMM on the 5th-generation tensor cores.
//
//   y[t][c] = bf16( sum_g  a_s[t][g] * w_s[c/128][g] * P_g[t][c] ),
//   P_g[t][c] = sum_{j<128} q[t][128g+j] * wq[c][128g+j]
//
// (page "spark_model/layers/ops/dispatch_proj.rs", `cublas_fp8_proj_prequant`:
// an FP8 activation with per-[token,128-of-K] scales times an FP8 weight with
// per-128x128-block scales, bf16 out; weight-scale indexing as in
// `dequant_fp8_bf16_into`.)
//
// The scales are arbitrary fp32 values, so each 128-wide K block's partial
// product P_g is formed on its own by tcgen05 MMA (kind::f8f6f4, fp32 in
// TMEM) and promoted into fp32 register accumulators by the epilogue warps,
// one scalar per row and weight block: a_s[t][g] * w_s[c/128][g]. TMEM holds
// two partial buffers, so the MMA of block g+1 overlaps the promotion of g.
//
// Persistent kernel on CTA pairs (clusters of 2, one CTA per SM). A pair
// owns a 256 x 256 output tile and issues M=256 N=256 MMAs across both SMs
// (cta_group::2): each CTA stages its own 128 rows of A and its own 128 of
// the 256 rows of B, so each SM's shared memory carries a third less traffic
// per flop than a single-SM 128 x 256 tile. Per CTA, 12 warps:
//   warp 0      TMA producer: A [128 x 128 B] and B [128 x 128 B] per K block
//               into a 6-stage ring (128-byte swizzle), completion counted on
//               the even CTA's barrier; plus the block's 128 activation
//               scales (one K-major row slice) into an 8-slot local ring
//   warp 1      TMEM allocation for the pair; in the even CTA, the MMA issuer
//   warps 2-3   idle after set-up
//   warps 4-11  promotion + epilogue. Warp w reads TMEM lanes 32*(w%4)..+31
//               of its own CTA (its tile rows) and column half (w-4)/4 (128
//               columns, one weight block), one row per thread
// Tiles are visited M-fastest so the pairs running at one time share weight
// tiles through L2. Rows past M and columns past N are zero-filled by TMA
// and never stored.
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

constexpr uint32_t BM = 128;       // rows per CTA
constexpr uint32_t BM_PAIR = 256;  // rows per CTA pair (one MMA)
constexpr uint32_t BN = 256;       // output columns per tile
constexpr uint32_t BN_CTA = 128;   // rows of B staged by each CTA
constexpr uint32_t BK = 128;
constexpr uint32_t kStages = 6;
constexpr uint32_t kScaleStages = 8;
constexpr uint32_t kThreads = 384;
constexpr uint32_t kEpiWarps = 8;
constexpr uint32_t kTileBytesA = BM * BK;
constexpr uint32_t kTileBytesB = BN_CTA * BK;
constexpr uint32_t kScaleBytes = BM * 4;
constexpr uint32_t kTmemCols = 2 * BN;  // two partial buffers of BN fp32 columns
// Register split: warpgroup 0 (producer, MMA, idle) gives registers to the
// two promotion warpgroups. 128*40 + 256*232 = 64512 = 384 * 168, the
// launch allocation; the host checks the compiled count before launching.
constexpr uint32_t kRegsLow = 40;
constexpr uint32_t kRegsHigh = 232;
constexpr uint32_t kLaunchRegsNeeded = (128 * kRegsLow + 256 * kRegsHigh) / kThreads;

struct __align__(1024) GemmSmem {
    uint8_t a[kStages][kTileBytesA];
    uint8_t b[kStages][kTileBytesB];
    float a_scale[kScaleStages][BM];
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t sfull[kScaleStages];
    uint64_t sempty[kScaleStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    uint32_t _pad;
    uint32_t abort;
    uint32_t consumed;  // K blocks whose TMA data the MMA thread has seen land
};

constexpr size_t kSmemBytes = sizeof(GemmSmem) + 1024;  // + alignment slack

struct Shape {
    uint32_t M, N, G, Mp;
    uint32_t num_m, num_tiles;
};

__device__ __forceinline__ void tile_coords(const Shape& sh, uint32_t tile, uint32_t& m0, uint32_t& n0) {
    const uint32_t tm = tile % sh.num_m;
    const uint32_t tn = tile / sh.num_m;
    m0 = tm * BM_PAIR;
    n0 = tn * BN;
}

// Spin for about `cycles` SM clocks (bounded by construction).
__device__ __forceinline__ void spin_cycles(long long cycles) {
    const long long t0 = clock64();
    while (clock64() - t0 < cycles) {
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_blockscaled_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmS, const float* __restrict__ w_s,
                            uint16_t* __restrict__ y, const Shape sh) {
    extern __shared__ uint8_t smem_raw[];
    GemmSmem& sm = *reinterpret_cast<GemmSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t warp = threadIdx.x >> 5;
    const uint32_t lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const uint32_t pair = blockIdx.x >> 1;
    const uint32_t num_pairs = gridDim.x >> 1;
    volatile uint32_t* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (uint32_t s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 2);  // one expect-tx arrival from each CTA of the pair
            mbar_init(&sm.empty[s], 1);
        }
        for (uint32_t s = 0; s < kScaleStages; ++s) {
            mbar_init(&sm.sfull[s], 1);
            mbar_init(&sm.sempty[s], kEpiWarps);
        }
        for (uint32_t b = 0; b < 2; ++b) {
            mbar_init(&sm.tfull[b], 1);
            mbar_init(&sm.tempty[b], 2 * kEpiWarps);  // promotion warps of both CTAs
        }
        mbar_init(&sm.mma_done, 1);
        sm.abort = 0;
        sm.consumed = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmS);
    }
    if (warp == 1) {
        tmem_alloc_pair(&sm.tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // barriers of both CTAs initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t G = sh.G;

    uint32_t issued = 0;  // producer: K blocks whose loads were issued (all tiles)

    if (warp < 4) {
        regs_dec<kRegsLow>();
        if (warp == 0 && lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (uint32_t tile = pair; ok && tile < sh.num_tiles; tile += num_pairs) {
                uint32_t m0, n0;
                tile_coords(sh, tile, m0, n0);
                const int32_t my_m = static_cast<int32_t>(m0 + rank * BM);
                const int32_t my_n = static_cast<int32_t>(n0 + rank * BN_CTA);
                for (uint32_t kb = 0; kb < G; ++kb, ++it) {
                    const uint32_t s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    const uint32_t ss = it % kScaleStages;
                    const uint32_t sph = (it / kScaleStages) & 1u;
                    if (!mbar_wait(&sm.empty[s], ph ^ 1u, abort) || !mbar_wait(&sm.sempty[ss], sph ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.sfull[ss], kScaleBytes);
                    tma_load_2d(sm.a_scale[ss], &tmS, &sm.sfull[ss], my_m, static_cast<int32_t>(kb));
                    const uint32_t full_even = mapa_shared(smem_addr(&sm.full[s]), 0);
                    mbar_arrive_expect_tx_cluster(full_even, kTileBytesA + kTileBytesB);
                    tma_load_2d_pair(sm.a[s], &tmA, full_even, static_cast<int32_t>(kb * BK), my_m);
                    tma_load_2d_pair(sm.b[s], &tmB, full_even, static_cast<int32_t>(kb * BK), my_n);
                    issued = it + 1;
                }
            }
        } else if (warp == 1 && lane == 0 && rank == 0) {
            constexpr uint32_t idesc = idesc_e4m3_f32(BM_PAIR, BN);
            uint32_t it = 0;
            bool ok = true;
            for (uint32_t tile = pair; ok && tile < sh.num_tiles; tile += num_pairs) {
                for (uint32_t kb = 0; kb < G; ++kb, ++it) {
                    const uint32_t s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    const uint32_t b = it & 1u;
                    const uint32_t tph = (it >> 1) & 1u;
                    if (!mbar_wait(&sm.full[s], ph, abort)) {
                        ok = false;
                        break;
                    }
                    sm.consumed = it + 1;
                    if (!mbar_wait(&sm.tempty[b], tph ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d = tmem + b * BN;
                    const uint64_t ad = smem_desc_k_sw128(smem_addr(sm.a[s]));
                    const uint64_t bd = smem_desc_k_sw128(smem_addr(sm.b[s]));
#pragma unroll
                    for (uint32_t kk = 0; kk < BK / 32; ++kk)  // K = 32 bytes per MMA: +2 in the address field
                        mma_f8f6f4_pair(d, ad + 2u * kk, bd + 2u * kk, idesc, kk > 0 ? 1u : 0u);
                    mma_commit_pair_multicast(&sm.empty[s], 0x3);
                    mma_commit_pair_multicast(&sm.tfull[b], 0x3);
                }
            }
            // Every MMA this thread issued has completed once mma_done fires.
            mma_commit_pair(&sm.mma_done);
            volatile uint32_t never = 0;
            mbar_wait(&sm.mma_done, 0, &never);
        }
    } else {
        regs_inc<kRegsHigh>();
        const uint32_t quad = warp & 3u;
        const uint32_t half = (warp - 4u) >> 2;
        const uint32_t lane_off = (quad * 32u) << 16;
        const uint32_t r_local = quad * 32u + lane;
        const uint32_t tempty_even[2] = {mapa_shared(smem_addr(&sm.tempty[0]), 0),
                                         mapa_shared(smem_addr(&sm.tempty[1]), 0)};
        uint32_t it = 0;
        bool ok = true;
        for (uint32_t tile = pair; ok && tile < sh.num_tiles; tile += num_pairs) {
            uint32_t m0, n0;
            tile_coords(sh, tile, m0, n0);
            const uint32_t row = m0 + rank * BM + r_local;
            const bool row_ok = row < sh.M;
            const uint32_t col0 = n0 + half * 128u;
            const bool col_ok = col0 < sh.N;
            // One weight block row per warp: its G scales are one short
            // contiguous run that stays in L1 after the first K block.
            const float* ws_row = w_s + static_cast<size_t>(col_ok ? col0 / 128u : 0u) * G;
            float2 acc[64];
#pragma unroll
            for (uint32_t i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
            float w_next = __ldg(ws_row);
            for (uint32_t kb = 0; kb < G; ++kb, ++it) {
                const uint32_t b = it & 1u;
                const uint32_t tph = (it >> 1) & 1u;
                const uint32_t ss = it % kScaleStages;
                const uint32_t sph = (it / kScaleStages) & 1u;
                const float w_cur = w_next;
                if (kb + 1 < G) w_next = __ldg(ws_row + kb + 1);
                const bool got = mbar_wait(&sm.sfull[ss], sph, abort) && mbar_wait(&sm.tfull[b], tph, abort);
                if (!__all_sync(0xFFFFFFFFu, got)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float c = sm.a_scale[ss][r_local] * w_cur;
                const float2 c2 = make_float2(c, c);
                const uint32_t taddr = tmem + lane_off + b * BN + half * 128u;
#pragma unroll
                for (uint32_t ch = 0; ch < 2; ++ch) {
                    uint32_t v[64];
                    tmem_load64(taddr + ch * 64u, v);
#pragma unroll
                    for (uint32_t i = 0; i < 32; ++i)
                        acc[ch * 32 + i] = __ffma2_rn(
                            c2, make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])),
                            acc[ch * 32 + i]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_cluster(tempty_even[b]);
                    mbar_arrive(&sm.sempty[ss]);
                }
            }
            if (ok && row_ok && col_ok) {
                uint4* dst = reinterpret_cast<uint4*>(y + static_cast<size_t>(row) * sh.N + col0);
#pragma unroll
                for (uint32_t j = 0; j < 16; ++j) {
                    uint32_t p[4];
#pragma unroll
                    for (uint32_t e = 0; e < 4; ++e) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(acc[4 * j + e].x, acc[4 * j + e].y);
                        p[e] = *reinterpret_cast<uint32_t*>(&h);
                    }
                    dst[j] = make_uint4(p[0], p[1], p[2], p[3]);
                }
            }
        }
    }

    // Teardown. On the normal path every TMA load was consumed and every MMA
    // completed before the promotion warps finished. After a timed-out wait
    // (in either CTA) the loads this pair started may still be landing:
    // the even CTA waits for the ones it can see, and both CTAs then give
    // in-flight copies a bounded grace period before the pair synchronises
    // and frees TMEM.
    tc_fence_before();
    __syncthreads();
    if (*abort) {
        volatile uint32_t never = 0;
        if (threadIdx.x == 0) atomicOr(&g_device_error, 1u);
        if (warp == 0 && lane == 0) {
            if (rank == 0)
                for (uint32_t it = sm.consumed; it < issued; ++it)
                    mbar_wait(&sm.full[it % kStages], (it / kStages) & 1u, &never);
            const uint32_t first = issued > kScaleStages ? issued - kScaleStages : 0u;
            for (uint32_t it = first; it < issued; ++it)
                mbar_wait(&sm.sfull[it % kScaleStages], (it / kScaleStages) & 1u, &never);
            spin_cycles(200000);
        }
        __syncthreads();
    }
    cluster_sync_all();  // no remote arrive or pair MMA can still target this CTA
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
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

// The K-major activation scales [G, Mp] fp32 read as [1 x 128] row slices
// (128 tokens of one K group); tokens past Mp read as zero.
bool make_map_scales(CUtensorMap* map, const float* base, uint64_t mp, uint64_t g) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {mp, g};
    cuuint64_t strides[1] = {mp * sizeof(float)};
    cuuint32_t box[2] = {BM, 1};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

struct KernelSetup {
    cudaError_t err = cudaSuccess;
    int sms = 0;
};

// Once per device ordinal: shared-memory opt-in, the register split check
// and the SM count.
const KernelSetup& setup_for_device() {
    static std::mutex mu;
    static KernelSetup table[64];
    static bool done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    std::lock_guard<std::mutex> lock(mu);
    KernelSetup& k = table[dev];
    if (!done[dev]) {
        done[dev] = true;
        k.err = cudaFuncSetAttribute(gemm_blockscaled_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(kSmemBytes));
        cudaFuncAttributes attr;
        if (k.err == cudaSuccess) k.err = cudaFuncGetAttributes(&attr, gemm_blockscaled_kernel);
        // setmaxnreg.inc waits until the registers it asks for are free in
        // the CTA's allocation: refuse to launch a build whose allocation
        // cannot cover the split.
        if (k.err == cudaSuccess && static_cast<uint32_t>(attr.numRegs) < kLaunchRegsNeeded)
            k.err = cudaErrorInvalidConfiguration;
        if (k.err == cudaSuccess) k.err = cudaDeviceGetAttribute(&k.sms, cudaDevAttrMultiProcessorCount, dev);
    }
    return k;
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
    const KernelSetup& ks = setup_for_device();
    if (ks.err != cudaSuccess) return ks.err;
    CUtensorMap ta, tb, ts;
    if (!make_map_u8(&ta, L.q, L.k, L.m, BM) || !make_map_u8(&tb, L.wq, L.k, L.n, BN_CTA) ||
        !make_map_scales(&ts, L.s_k, L.mp, L.k / BK))
        return cudaErrorInvalidValue;
    Shape sh;
    sh.M = L.m;
    sh.N = L.n;
    sh.G = L.k / BK;
    sh.Mp = L.mp;
    sh.num_m = (L.m + BM_PAIR - 1) / BM_PAIR;
    sh.num_tiles = sh.num_m * ((L.n + BN - 1) / BN);
    const uint32_t max_pairs = static_cast<uint32_t>(ks.sms) / 2;
    const uint32_t grid = 2 * (sh.num_tiles < max_pairs ? sh.num_tiles : max_pairs);
    gemm_blockscaled_kernel<<<grid, kThreads, kSmemBytes, stream>>>(ta, tb, ts, L.w_scale,
                                                                    static_cast<uint16_t*>(L.y), sh);
    note_launch();
    return cudaGetLastError();
}

}  // namespace fp8q
