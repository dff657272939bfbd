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
//               the even CTA's barrier; for long K also the block's 128
//               activation scales (one K-major row slice) into an 8-slot
//               local ring (otherwise the promotion warps load them, see
//               kDirect below)
//   warp 1      TMEM allocation for the pair; in the even CTA, the MMA issuer
//               of the even K blocks (TMEM buffer 0)
//   warp 2      in the even CTA, the MMA issuer of the odd K blocks (buffer 1)
//   warp 3      idle after set-up
//   warps 4-11  promotion + epilogue. Warp w reads TMEM lanes 32*(w%4)..+31
//               of its own CTA (its tile rows) and column half (w-4)/4 (128
//               columns, one weight block), one row per thread; at the end of
//               a tile it writes its 32 x 128 bf16 outputs through a 2 KB
//               shared-memory buffer with TMA stores
// Tiles are visited M-fastest so the pairs running at one time share weight
// tiles through L2. Rows past M and columns past N are zero-filled by TMA
// and never stored (the output map clips them). With per-row weight scales (one per weight row, the
// scale block 1 x K of `dequant_fp8_bf16_into`'s per-row layout) the
// promotion folds in a_s[t][g] only and the epilogue multiplies each output
// column by its row's scale once.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <mutex>

#include "group_quant.cuh"
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
static_assert(kStages % 2 == 0, "each stage must always be consumed by the same MMA issuer");
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

// Output staging: per promotion warp, one 32-row x 32-column bf16 block
// (64-byte rows, 64-byte swizzle) that a TMA store writes to y.
constexpr uint32_t kOutCols = 32;
constexpr uint32_t kOutStageBytes = 32 * kOutCols * 2;

struct __align__(1024) GemmSmem {
    uint8_t a[kStages][kTileBytesA];
    uint8_t b[kStages][kTileBytesB];
    uint8_t out[kEpiWarps][kOutStageBytes];
    float a_scale[kScaleStages][BM];
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t sfull[kScaleStages];
    uint64_t sempty[kScaleStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t mma_done[2];
    uint32_t tmem_base;
    uint32_t _pad;
    uint32_t abort;
    uint32_t consumed[2];  // per MMA issuer: 1 + its last K block whose TMA data it has seen land
};

constexpr size_t kSmemBytes = sizeof(GemmSmem) + 1024;  // + alignment slack

struct Shape {
    uint32_t M, N, G, Mp;
    uint32_t num_m, num_tiles;
    uint32_t w_per_row;  // weight scales: 0 = [N/128, K/128] blocks, 1 = one per weight row [N]
    uint32_t no_copies;  // timeout diagnostics: the producer issues no copies
    long long budget;    // clock budget of every wait
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

// kDirect: where the promotion warps get the activation scales.
//   true   each thread loads its row's scale of each K block from the
//          K-major array in global memory (L2), four K blocks ahead; the
//          TMA producer then issues only the A and B copies of a K block
//   false  the TMA producer also copies the block's 128 scales of this
//          CTA's rows into an 8-slot shared-memory ring
// Measured on B200: with the producer doing one wait and two copies per K
// block, M=1168 N=17408 K=5120 runs 6 % faster (137.5 -> 129.7 us); at
// K=17408 the streaming operands evict the scales from L2 and the ring is
// 10 % faster (488 vs 535 us). The host picks direct loads up to
// kDirectScalesMaxG K blocks.
constexpr uint32_t kDirectScalesMaxG = 64;

template <bool kDirect>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_blockscaled_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmY,
                            const float* __restrict__ s_k, const float* __restrict__ w_s, const Shape sh) {
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
        mbar_init(&sm.mma_done[0], 1);
        mbar_init(&sm.mma_done[1], 1);
        sm.abort = 0;
        sm.consumed[0] = sm.consumed[1] = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (!kDirect) tma_prefetch_desc(&tmS);
        tma_prefetch_desc(&tmY);
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
        if (warp == 0 && lane == 0 && !sh.no_copies) {
            // Set-up above overlaps the producing kernel (quantizer) when
            // launched as its dependent; its outputs are read from here on.
            grid_dependency_wait();
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
                    if (!mbar_wait(&sm.empty[s], ph ^ 1u, abort, sh.budget)) {
                        ok = false;
                        break;
                    }
                    if constexpr (!kDirect) {
                        const uint32_t ss = it % kScaleStages;
                        const uint32_t sph = (it / kScaleStages) & 1u;
                        if (!mbar_wait(&sm.sempty[ss], sph ^ 1u, abort, sh.budget)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&sm.sfull[ss], kScaleBytes);
                        tma_load_2d(sm.a_scale[ss], &tmS, &sm.sfull[ss], my_m, static_cast<int32_t>(kb));
                    }
                    const uint32_t full_even = mapa_shared(smem_addr(&sm.full[s]), 0);
                    mbar_arrive_expect_tx_cluster(full_even, kTileBytesA + kTileBytesB);
                    tma_load_2d_pair(sm.a[s], &tmA, full_even, static_cast<int32_t>(kb * BK), my_m);
                    tma_load_2d_pair(sm.b[s], &tmB, full_even, static_cast<int32_t>(kb * BK), my_n);
                    issued = it + 1;
                }
            }
        } else if ((warp == 1 || warp == 2) && lane == 0 && rank == 0) {
            // Two MMA issuers, one per TMEM buffer: warp 1 issues the K
            // blocks of even index (buffer 0), warp 2 those of odd index
            // (buffer 1). Four back-to-back tcgen05.mma hold their warp's SM
            // sub-partition for about three MMA durations, which delays the
            // promotion warps sharing it; alternating issuers halves that
            // stall on each sub-partition. The two buffers' MMAs are
            // independent, reuse of a buffer is ordered by its tempty
            // barrier, and with an even stage count every stage is always
            // consumed (and committed) by the same issuer.
            constexpr uint32_t idesc = idesc_e4m3_f32(BM_PAIR, BN);
            const uint32_t par = warp - 1u;
            uint32_t it = 0;
            bool ok = true;
            for (uint32_t tile = pair; ok && tile < sh.num_tiles; tile += num_pairs) {
                for (uint32_t kb = 0; kb < G; ++kb, ++it) {
                    if ((it & 1u) != par) continue;
                    const uint32_t s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    const uint32_t b = it & 1u;
                    const uint32_t tph = (it >> 1) & 1u;
                    if (!mbar_wait(&sm.full[s], ph, abort, sh.budget)) {
                        ok = false;
                        break;
                    }
                    sm.consumed[par] = it + 1;
                    if (!mbar_wait(&sm.tempty[b], tph ^ 1u, abort, sh.budget)) {
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
            mma_commit_pair(&sm.mma_done[par]);
            volatile uint32_t never = 0;
            mbar_wait(&sm.mma_done[par], 0, &never);
        }
    } else {
        regs_inc<kRegsHigh>();
        const uint32_t quad = warp & 3u;
        const uint32_t half = (warp - 4u) >> 2;
        const uint32_t lane_off = (quad * 32u) << 16;
        const uint32_t r_local = quad * 32u + lane;
        const uint32_t tempty_even[2] = {mapa_shared(smem_addr(&sm.tempty[0]), 0),
                                         mapa_shared(smem_addr(&sm.tempty[1]), 0)};
        // The activation scales come from the quantizer's K-major output,
        // and nothing else in global memory is touched before the grid this
        // launch depends on has completed either.
        grid_dependency_wait();
        uint32_t it = 0;
        bool ok = true;
        for (uint32_t tile = pair; ok && tile < sh.num_tiles; tile += num_pairs) {
            uint32_t m0, n0;
            tile_coords(sh, tile, m0, n0);
            const uint32_t row = m0 + rank * BM + r_local;
            const bool row_ok = row < sh.M;
            const uint32_t col0 = n0 + half * 128u;
            const bool col_ok = col0 < sh.N;
            // Block-scaled weights: one weight block row per warp, whose G
            // scales are one short contiguous run that stays in L1 after the
            // first K block. Per-row weights: the promotion folds in the
            // activation scale only and the epilogue applies each column's
            // weight scale.
            const bool per_row = sh.w_per_row != 0;
            const float* ws_row = w_s + static_cast<size_t>(col_ok && !per_row ? col0 / 128u : 0u) * G;
            float2 acc[64];
#pragma unroll
            for (uint32_t i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
            float w_next = per_row ? 1.0f : __ldg(ws_row);
            // This row's activation scale of each K block, loaded four
            // blocks ahead through a small register queue, so an L2 miss
            // (the operands streaming through L2 can evict the scales at
            // large K) stays off the K-block cycle. Rows past M have no
            // scales and are never stored.
            const float* a_row = s_k + (row_ok ? row : 0u);
            float aq0 = 0.0f, aq1 = 0.0f, aq2 = 0.0f, aq3 = 0.0f;
            if constexpr (kDirect) {
                aq0 = row_ok && 0 < G ? __ldg(a_row) : 0.0f;
                aq1 = row_ok && 1 < G ? __ldg(a_row + static_cast<size_t>(1) * sh.Mp) : 0.0f;
                aq2 = row_ok && 2 < G ? __ldg(a_row + static_cast<size_t>(2) * sh.Mp) : 0.0f;
                aq3 = row_ok && 3 < G ? __ldg(a_row + static_cast<size_t>(3) * sh.Mp) : 0.0f;
            }
            for (uint32_t kb = 0; kb < G; ++kb, ++it) {
                const uint32_t b = it & 1u;
                const uint32_t tph = (it >> 1) & 1u;
                const uint32_t ss = it % kScaleStages;
                const uint32_t sph = (it / kScaleStages) & 1u;
                const float w_cur = w_next;
                float a_cur = aq0;
                if constexpr (kDirect) {
                    aq0 = aq1;
                    aq1 = aq2;
                    aq2 = aq3;
                    aq3 = row_ok && kb + 4 < G ? __ldg(a_row + static_cast<size_t>(kb + 4) * sh.Mp) : 0.0f;
                }
                if (!per_row && kb + 1 < G) w_next = __ldg(ws_row + kb + 1);
                const bool got = (kDirect || mbar_wait(&sm.sfull[ss], sph, abort, sh.budget)) && mbar_wait(&sm.tfull[b], tph, abort, sh.budget);
                if (!__all_sync(0xFFFFFFFFu, got)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if constexpr (!kDirect) a_cur = sm.a_scale[ss][r_local];
                const float c = a_cur * w_cur;
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
                    if constexpr (!kDirect) mbar_arrive(&sm.sempty[ss]);
                }
            }
            // Warps whose 32 rows all lie past M have nothing to store.
            if (ok && col_ok && m0 + rank * BM + quad * 32u < sh.M) {
                if (per_row) {
                    const float4* wv = reinterpret_cast<const float4*>(w_s + col0);
#pragma unroll
                    for (uint32_t j = 0; j < 32; ++j) {
                        const float4 v = __ldg(wv + j);
                        acc[2 * j] = __fmul2_rn(acc[2 * j], make_float2(v.x, v.y));
                        acc[2 * j + 1] = __fmul2_rn(acc[2 * j + 1], make_float2(v.z, v.w));
                    }
                }
                // The warp's 32 rows x 128 columns leave as four 32 x 32
                // bf16 blocks: each lane packs its row of a block into the
                // warp's staging buffer (16-byte chunk j of row r at chunk
                // j ^ ((r >> 1) & 3), the 64-byte swizzle of the output map),
                // and lane 0 stores the block with TMA, asynchronously, so the
                // warps go on to the next tile's promotion. Rows past M are
                // clipped by the map.
                uint8_t* stg = sm.out[warp - 4u];
                const int32_t y_row = static_cast<int32_t>(m0 + rank * BM + quad * 32u);
#pragma unroll
                for (uint32_t c = 0; c < 128u / kOutCols; ++c) {
                    if (lane == 0) bulk_store_wait_read();  // the block before has left the buffer
                    __syncwarp();
#pragma unroll
                    for (uint32_t j = 0; j < 4; ++j) {
                        uint32_t p[4];
#pragma unroll
                        for (uint32_t e = 0; e < 4; ++e) {
                            const float2 v = acc[16 * c + 4 * j + e];
                            __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
                            p[e] = *reinterpret_cast<uint32_t*>(&h);
                        }
                        *reinterpret_cast<uint4*>(stg + lane * 64u + ((j ^ ((lane >> 1) & 3u)) << 4)) =
                            make_uint4(p[0], p[1], p[2], p[3]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) tma_store_2d(&tmY, stg, static_cast<int32_t>(col0 + c * kOutCols), y_row);
                }
            }
        }
        // Every output block of this warp is in global memory before the CTA
        // (and its staging buffer) goes away.
        if (lane == 0) bulk_store_wait_all();
        __syncwarp();
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
            if (rank == 0) {
                const uint32_t from = sm.consumed[0] < sm.consumed[1] ? sm.consumed[0] : sm.consumed[1];
                for (uint32_t it = from; it < issued; ++it)
                    if (it >= sm.consumed[it & 1u]) mbar_wait(&sm.full[it % kStages], (it / kStages) & 1u, &never);
            }
            if constexpr (!kDirect) {
                const uint32_t first = issued > kScaleStages ? issued - kScaleStages : 0u;
                for (uint32_t it = first; it < issued; ++it)
                    mbar_wait(&sm.sfull[it % kScaleStages], (it / kScaleStages) & 1u, &never);
            }
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

// ------------------------------------------------------ decode widths --
//
// M <= 64 tokens: the weight is the big operand, so the MMA is swapped.
// Each CTA multiplies a 128-row slice of W (the MMA's M) by all the tokens
// (the MMA's N, NT = 32 or 64 wide) over one contiguous range of K blocks:
//   D[n][t] = sum_j wq[n][128g+j] * q[t][128g+j]          (tcgen05, fp32, TMEM)
//   acc[n][t] += (w_s[n/128][g] * a_s[t][g]) * D[n][t]     (promotion, fp32)
// One promotion thread owns one weight row and its NT token accumulators.
// With only N/128 weight slices (40-48 at the pages' decode shapes), K is
// split S ways and the S CTAs of a slice form a thread-block cluster; each
// parks its [NT x 128] fp32 partial in shared memory and the cluster sums
// the S partials through distributed shared memory in a fixed order (the
// result does not depend on timing), each CTA storing a share of the token
// rows as bf16. CTA = 6 warps: warp 0 TMA producer (W [128 x 128 B], tokens
// [NT x 128 B] and the block's NT token scales per stage, 4 stages, so two
// CTAs fit per SM and the clusters of a call fit the GPU at once), warp 1
// TMEM allocator and MMA issuer, warps 2-5 promotion (warp w reads TMEM
// lanes 32*(w%4)..+31). A stage is freed after five arrivals: the MMA's
// commit and the four promotion warps that read its token scales.
//
// FUSE (M <= 32): the activation quantizer runs inside this kernel. Four
// more warps (6-9) read each K block of the bf16 activation X [M, K] (from
// L2) and write its FP8 codes straight into the stage's token tile, in the
// 128-byte-swizzled K-major layout the MMA descriptor expects, and its
// per-token scales into the stage's scale slot, with the quantizer's own
// group arithmetic (the bytes equal fp8q_quant_act's). Every weight slice
// quantizes the same X blocks; the CTAs of slice 0 also store the codes and
// K-major scales (pad rows zeroed) to global memory, so the call leaves the
// same workspace as the unfused path. A stage then fills on five arrivals:
// the weight copy's expect-tx and the four quantizer warps, whose generic
// shared-memory writes are fenced to the async proxy first.

constexpr uint32_t kDecStages = 4;
constexpr uint32_t kDecBufs = 4;
constexpr uint32_t kDecThreads = 192;
constexpr uint32_t kDecEpiWarps = 4;
constexpr uint32_t kDecMaxSplit = 8;
constexpr uint32_t kDecMaxTokens = 64;
constexpr uint32_t kDecQuantWarps = 4;
constexpr uint32_t kDecFusedThreads = kDecThreads + 32 * kDecQuantWarps;
constexpr uint32_t kDecFusedMaxTokens = 32;

template <uint32_t NT>
struct __align__(1024) DecodeSmem {
    uint8_t w[kDecStages][BM * BK];
    uint8_t t[kDecStages][NT * BK];
    float t_scale[kDecStages][NT];
    uint64_t full[kDecStages];
    uint64_t empty[kDecStages];
    uint64_t tfull[kDecBufs];
    uint64_t tempty[kDecBufs];
    uint64_t mma_done;
    uint32_t tmem_base;
    uint32_t abort;
    uint32_t consumed;
};

template <uint32_t NT>
constexpr size_t decode_smem_bytes() {
    return sizeof(DecodeSmem<NT>) + 1024;
}

struct DecodeShape {
    uint32_t M, N, G, split, Mp;
    uint32_t w_per_row;  // weight scales: 0 = [N/128, K/128] blocks, 1 = one per weight row [N]
    uint32_t no_copies;  // timeout diagnostics: the producer issues no copies
    long long budget;    // clock budget of every wait
};

template <uint32_t NT>
__device__ __forceinline__ void tmem_load_nt(uint32_t taddr, uint32_t (&r)[NT]);

template <>
__device__ __forceinline__ void tmem_load_nt<64>(uint32_t taddr, uint32_t (&r)[64]) {
    tmem_load64(taddr, r);
}

template <>
__device__ __forceinline__ void tmem_load_nt<32>(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;"
        : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
          "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
          "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
          "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
        :
        : "memory");
}

template <uint32_t NT, bool FUSE>
__global__ void __launch_bounds__(FUSE ? kDecFusedThreads : kDecThreads, 2)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmT,
                       const __grid_constant__ CUtensorMap tmS, const float* __restrict__ w_s,
                       uint16_t* __restrict__ y, const DecodeShape sh, const uint16_t* __restrict__ x,
                       uint8_t* __restrict__ q_out, float* __restrict__ s_out) {
    static_assert(!FUSE || NT <= kDecFusedMaxTokens, "the fused quantizer serves at most 32 tokens");
    extern __shared__ uint8_t smem_raw[];
    using Smem = DecodeSmem<NT>;
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr uint32_t kCols = kDecBufs * NT;  // 128 or 256 TMEM columns
    const uint32_t warp = threadIdx.x >> 5;
    const uint32_t lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // clusters of `split` consecutive CTAs: rank == K split
    const uint32_t nb = blockIdx.x / sh.split;  // weight block row
    const uint32_t n0 = nb * BM;
    const uint32_t G = sh.G;
    const uint32_t kb0 = rank * G / sh.split;
    const uint32_t nk = (rank + 1) * G / sh.split - kb0;
    volatile uint32_t* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (uint32_t s = 0; s < kDecStages; ++s) {
            mbar_init(&sm.full[s], FUSE ? 1 + kDecQuantWarps : 1);
            mbar_init(&sm.empty[s], 1 + kDecEpiWarps);
        }
        for (uint32_t b = 0; b < kDecBufs; ++b) {
            mbar_init(&sm.tfull[b], 1);
            mbar_init(&sm.tempty[b], kDecEpiWarps);
        }
        mbar_init(&sm.mma_done, 1);
        sm.abort = 0;
        sm.consumed = 0;
        fence_mbar_init();
    }
    // The weight tiles of the first stages are requested at once, so their
    // DRAM latency overlaps the TMEM allocation and the block barrier (and,
    // launched as the quantizer's dependent, the quantizer itself: the weight
    // is not written by the preceding grid, and everything before that grid
    // had finished when it let this one launch). Each such stage's barrier
    // is armed here with all of the stage's bytes; the token tile and its
    // scales follow once the preceding grid has completed.
    const uint32_t pre = sh.no_copies ? 0u : (nk < kDecStages ? nk : kDecStages);
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW);
        for (uint32_t it = 0; it < pre; ++it) {
            mbar_arrive_expect_tx(&sm.full[it], FUSE ? BM * BK : BM * BK + NT * BK + NT * 4);
            tma_load_2d(sm.w[it], &tmW, &sm.full[it], static_cast<int32_t>((kb0 + it) * BK), static_cast<int32_t>(n0));
        }
        tma_prefetch_desc(&tmT);
        tma_prefetch_desc(&tmS);
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, kCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    uint32_t issued = 0;

    float acc[NT];
#pragma unroll
    for (uint32_t i = 0; i < NT; ++i) acc[i] = 0.0f;
    const uint32_t r_local = (warp & 3u) * 32u + lane;  // weight row within the slice

    if (warp == 0) {
        if (lane == 0 && !sh.no_copies) {
            issued = pre;  // the early weight copies are in flight
            grid_dependency_wait();
            for (uint32_t it = 0; it < nk; ++it) {
                const uint32_t kb = kb0 + it;
                const uint32_t s = it % kDecStages;
                const uint32_t ph = (it / kDecStages) & 1u;
                if (it < pre) {
                    if (!FUSE) {
                        tma_load_2d(sm.t[s], &tmT, &sm.full[s], static_cast<int32_t>(kb * BK), 0);
                        tma_load_2d(sm.t_scale[s], &tmS, &sm.full[s], 0, static_cast<int32_t>(kb));
                    }
                    continue;
                }
                if (!mbar_wait(&sm.empty[s], ph ^ 1u, abort, sh.budget)) break;
                if (FUSE) {
                    mbar_arrive_expect_tx(&sm.full[s], BM * BK);
                    tma_load_2d(sm.w[s], &tmW, &sm.full[s], static_cast<int32_t>(kb * BK), static_cast<int32_t>(n0));
                } else {
                    mbar_arrive_expect_tx(&sm.full[s], BM * BK + NT * BK + NT * 4);
                    tma_load_2d(sm.w[s], &tmW, &sm.full[s], static_cast<int32_t>(kb * BK), static_cast<int32_t>(n0));
                    tma_load_2d(sm.t[s], &tmT, &sm.full[s], static_cast<int32_t>(kb * BK), 0);
                    tma_load_2d(sm.t_scale[s], &tmS, &sm.full[s], 0, static_cast<int32_t>(kb));
                }
                issued = it + 1;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_e4m3_f32(BM, NT);
            for (uint32_t it = 0; it < nk; ++it) {
                const uint32_t s = it % kDecStages;
                const uint32_t ph = (it / kDecStages) & 1u;
                const uint32_t b = it % kDecBufs;
                const uint32_t tph = (it / kDecBufs) & 1u;
                if (!mbar_wait(&sm.full[s], ph, abort, sh.budget)) break;
                sm.consumed = it + 1;
                if (!mbar_wait(&sm.tempty[b], tph ^ 1u, abort, sh.budget)) break;
                tc_fence_after();
                const uint32_t d = tmem + b * NT;
                const uint64_t ad = smem_desc_k_sw128(smem_addr(sm.w[s]));
                const uint64_t bd = smem_desc_k_sw128(smem_addr(sm.t[s]));
#pragma unroll
                for (uint32_t kk = 0; kk < BK / 32; ++kk)
                    mma_f8f6f4(d, ad + 2u * kk, bd + 2u * kk, idesc, kk > 0 ? 1u : 0u);
                mma_commit(&sm.empty[s]);
                mma_commit(&sm.tfull[b]);
            }
            mma_commit(&sm.mma_done);
            volatile uint32_t never = 0;
            mbar_wait(&sm.mma_done, 0, &never);
        }
    } else if (warp < 2 + kDecEpiWarps) {
        // Per-row weights: the weight scale is applied once, after the
        // split-K reduction.
        const bool per_row = sh.w_per_row != 0;
        const float* ws_row = w_s + static_cast<size_t>(per_row ? 0u : nb) * G;
        const uint32_t lane_off = ((warp & 3u) * 32u) << 16;
        float w_next = per_row ? 1.0f : (nk > 0 ? __ldg(ws_row + kb0) : 0.0f);
        for (uint32_t it = 0; it < nk; ++it) {
            const uint32_t s = it % kDecStages;
            const uint32_t b = it % kDecBufs;
            const uint32_t tph = (it / kDecBufs) & 1u;
            const float wsc = w_next;
            if (!per_row && it + 1 < nk) w_next = __ldg(ws_row + kb0 + it + 1);
            const bool got = mbar_wait(&sm.tfull[b], tph, abort, sh.budget);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            tc_fence_after();
            uint32_t v[NT];
            tmem_load_nt<NT>(tmem + lane_off + b * NT, v);
#pragma unroll
            for (uint32_t i = 0; i < NT; ++i) acc[i] = fmaf(wsc * sm.t_scale[s][i], __uint_as_float(v[i]), acc[i]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.tempty[b]);
                mbar_arrive(&sm.empty[s]);  // this warp is done with the stage's token scales
            }
        }
    } else if (FUSE) {
        // Quantizer warps: sixteen threads own one token's 128-element group
        // (16 bytes of X each), eight tokens at a time.
        const uint32_t qt = threadIdx.x - kDecThreads;  // 0..127
        const uint32_t gi = qt >> 4;
        const uint32_t l = qt & 15u;
        const uint32_t half_mask = 0xFFFFu << (16u * (gi & 1u));
        const uint32_t K = G * BK;
        // Token rows past M stay zero (codes and scales) in every stage.
        for (uint32_t idx = qt; idx < kDecStages * (NT - sh.M) * 8u; idx += 32u * kDecQuantWarps) {
            const uint32_t st = idx / ((NT - sh.M) * 8u);
            const uint32_t r = idx % ((NT - sh.M) * 8u);
            *reinterpret_cast<uint4*>(&sm.t[st][(sh.M + r / 8u) * BK + (r % 8u) * 16u]) = make_uint4(0u, 0u, 0u, 0u);
        }
        for (uint32_t idx = qt; idx < kDecStages * NT; idx += 32u * kDecQuantWarps)
            if (idx % NT >= sh.M) sm.t_scale[idx / NT][idx % NT] = 0.0f;
        // Token t = gi + 8 r of round r. The X loads of the next K block are
        // issued before waiting for this one's stage, so their L2 latency
        // overlaps the wait and this block's arithmetic.
        constexpr uint32_t R = NT / 8u;
        uint4 cur[R], nxt[R];
        auto load_block = [&](uint32_t kb, uint4 (&v)[R]) {
#pragma unroll
            for (uint32_t r = 0; r < R; ++r) {
                const uint32_t t = gi + 8u * r;
                v[r] = t < sh.M ? ld_stream16(x + static_cast<size_t>(t) * K + static_cast<size_t>(kb) * BK + l * 8u)
                                : make_uint4(0u, 0u, 0u, 0u);
            }
        };
        if (nk > 0) load_block(kb0, cur);
        for (uint32_t it = 0; it < nk; ++it) {
            const uint32_t kb = kb0 + it;
            const uint32_t s = it % kDecStages;
            const uint32_t ph = (it / kDecStages) & 1u;
            if (it + 1 < nk) load_block(kb + 1, nxt);
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.empty[s], ph ^ 1u, abort, sh.budget))) break;
#pragma unroll
            for (uint32_t r = 0; r < R; ++r) {
                const uint32_t t = gi + 8u * r;
                if (t >= sh.M) continue;  // the same for the sixteen threads of a token
                const size_t src = static_cast<size_t>(t) * K + static_cast<size_t>(kb) * BK + l * 8u;
                float amax = absmax8_bits(cur[r]);
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(half_mask, amax, o));
                const float scale = group_scale(amax);
                float f[8];
                widen8(cur[r], f);
                const uint2 c = encode8(f, scale);
                // 128-byte swizzle: 16-byte chunk j of row t sits at chunk j ^ (t % 8)
                *reinterpret_cast<uint2*>(&sm.t[s][t * BK + ((((l >> 1) ^ (t & 7u)) << 4) | ((l & 1u) << 3))]) = c;
                if (l == 0) sm.t_scale[s][t] = scale;
                if (nb == 0) {
                    st_stream8(q_out + src, c);
                    if (l == 0) s_out[static_cast<size_t>(kb) * sh.Mp + t] = scale;
                }
            }
            if (nb == 0 && qt < sh.Mp - sh.M) s_out[static_cast<size_t>(kb) * sh.Mp + sh.M + qt] = 0.0f;
            // make the generic-proxy shared-memory writes visible to the MMA
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if ((threadIdx.x & 31u) == 0) mbar_arrive(&sm.full[s]);
#pragma unroll
            for (uint32_t r = 0; r < R; ++r) cur[r] = nxt[r];
        }
    }

    // After a timed-out wait, let the copies this CTA started land (bounded).
    tc_fence_before();
    __syncthreads();
    if (*abort) {
        volatile uint32_t never = 0;
        if (threadIdx.x == 0) atomicOr(&g_device_error, 1u);
        if (warp == 0 && lane == 0)
            for (uint32_t it = sm.consumed; it < issued; ++it)
                mbar_wait(&sm.full[it % kDecStages], (it / kDecStages) & 1u, &never);
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kCols);
    }

    // Split-K reduction across the cluster. The operand stages are idle now
    // (every MMA and copy of this CTA finished), so the weight stages hold
    // this CTA's partial, transposed: red[t][row] (consecutive threads write
    // consecutive words).
    float* red = reinterpret_cast<float*>(&sm.w[0][0]);
    if (warp >= 2 && warp < 2 + kDecEpiWarps) {
#pragma unroll
        for (uint32_t i = 0; i < NT; ++i) red[i * BM + r_local] = acc[i];
    }
    cluster_sync_all();
    // CTA `rank` owns tokens rank, rank + split, ... Thread (tq, jq) of its
    // first four warps sums rows 4jq .. 4jq+3 of every fourth owned token:
    // one 16-byte read per peer and token, and one 8-byte store.
    if (threadIdx.x < BM && !*abort) {
        const uint32_t jq = threadIdx.x & 31u;
        const uint32_t tq = threadIdx.x >> 5;
        const uint32_t j = 4u * jq;
        const uint32_t red_addr = smem_addr(red);
        const float4 w_row = sh.w_per_row ? __ldg(reinterpret_cast<const float4*>(w_s + n0 + j))
                                          : make_float4(1.0f, 1.0f, 1.0f, 1.0f);
        for (uint32_t t = rank + sh.split * tq; t < sh.M; t += 4u * sh.split) {
            // Issue every peer's load before adding (independent remote
            // reads in flight together), then sum in rank order.
            float4 part[kDecMaxSplit];
#pragma unroll
            for (uint32_t p = 0; p < kDecMaxSplit; ++p)
                part[p] = p < sh.split ? ld_shared_cluster_f32x4(mapa_shared(red_addr + (t * BM + j) * 4u, p))
                                       : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            float4 sum = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
            for (uint32_t p = 0; p < kDecMaxSplit; ++p) {
                sum.x += part[p].x;
                sum.y += part[p].y;
                sum.z += part[p].z;
                sum.w += part[p].w;
            }
            if (sh.w_per_row) {
                sum.x *= w_row.x;
                sum.y *= w_row.y;
                sum.z *= w_row.z;
                sum.w *= w_row.w;
            }
            const __nv_bfloat162 lo = __floats2bfloat162_rn(sum.x, sum.y);
            const __nv_bfloat162 hi = __floats2bfloat162_rn(sum.z, sum.w);
            *reinterpret_cast<uint2*>(y + static_cast<size_t>(t) * sh.N + n0 + j) =
                make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
        }
    }
    cluster_sync_all();  // peers' partials stay in place until every CTA has read them
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

// The bf16 output y [rows, cols] written in [32 x 32] blocks with the
// 64-byte swizzle (the GEMM epilogue's staging layout).
bool make_map_out_bf16(CUtensorMap* map, void* base, uint64_t cols, uint64_t rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {kOutCols, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The K-major activation scales [G, Mp] fp32 read as [1 x box] row slices
// (box tokens of one K group); tokens past Mp read as zero.
bool make_map_scales_box(CUtensorMap* map, const float* base, uint64_t mp, uint64_t g, uint32_t box_tokens) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {mp, g};
    cuuint64_t strides[1] = {mp * sizeof(float)};
    cuuint32_t box[2] = {box_tokens, 1};
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
        // setmaxnreg.inc waits until the registers it asks for are free in
        // the CTA's allocation: refuse to launch a build whose allocation
        // cannot cover the split.
        for (auto fn : {gemm_blockscaled_kernel<true>, gemm_blockscaled_kernel<false>}) {
            if (k.err == cudaSuccess)
                k.err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kSmemBytes));
            cudaFuncAttributes attr;
            if (k.err == cudaSuccess) k.err = cudaFuncGetAttributes(&attr, fn);
            if (k.err == cudaSuccess && static_cast<uint32_t>(attr.numRegs) < kLaunchRegsNeeded)
                k.err = cudaErrorInvalidConfiguration;
        }
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

template <uint32_t NT, bool FUSE>
cudaError_t decode_smem_optin() {
    static std::once_flag once;
    static cudaError_t err = cudaSuccess;
    std::call_once(once, [] {
        err = cudaFuncSetAttribute(gemm_decode_kernel<NT, FUSE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(decode_smem_bytes<NT>()));
    });
    return err;
}

// K split for `slices` weight slices of G K blocks: about 1.6 CTAs per SM
// in total (the B200 sweep of splits 1..8 at N = 6144 and 5120 found its
// best times there: 240 CTAs for 48 and for 40 slices), at most 8 and at
// most G. FP8Q_DECODE_SPLIT=<n> overrides it.
uint32_t decode_split(uint32_t slices, uint32_t G, int sms) {
    static const int forced = [] {
        const char* e = std::getenv("FP8Q_DECODE_SPLIT");
        return e ? std::atoi(e) : 0;
    }();
    const uint32_t limit = kDecMaxSplit < G ? kDecMaxSplit : G;
    if (forced > 0) return static_cast<uint32_t>(forced) < limit ? static_cast<uint32_t>(forced) : limit;
    const uint32_t target = static_cast<uint32_t>(sms) * 8u / 5u;
    uint32_t s = (target + slices / 2) / slices;
    if (s < 1) s = 1;
    return s < limit ? s : limit;
}

template <uint32_t NT, bool FUSE>
cudaError_t launch_decode(const GemmLaunch& L, int sms, cudaStream_t stream) {
    const cudaError_t attr_err = decode_smem_optin<NT, FUSE>();
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap tw, tt, ts;
    if (!make_map_u8(&tw, L.wq, L.k, L.n, BM) || !make_map_u8(&tt, L.q, L.k, L.m, NT) ||
        !make_map_scales_box(&ts, L.s_k, L.mp, L.k / BK, NT))
        return cudaErrorInvalidValue;
    DecodeShape sh;
    sh.M = L.m;
    sh.N = L.n;
    sh.G = L.k / BK;
    sh.Mp = L.mp;
    sh.w_per_row = L.w_per_row ? 1u : 0u;
    sh.no_copies = L.diag_budget != 0 ? 1u : 0u;
    sh.budget = L.diag_budget != 0 ? L.diag_budget : kWaitBudgetCycles;
    const uint32_t slices = L.n / BM;
    const uint32_t split = decode_split(slices, sh.G, sms);
    sh.split = split;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(split * slices, 1, 1);
    cfg.blockDim = dim3(FUSE ? kDecFusedThreads : kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = decode_smem_bytes<NT>();
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = L.pdl ? 2 : 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_decode_kernel<NT, FUSE>, tw, tt, ts, L.w_scale,
                                       static_cast<uint16_t*>(L.y), sh, static_cast<const uint16_t*>(L.x),
                                       static_cast<uint8_t*>(const_cast<void*>(L.q)), const_cast<float*>(L.s_k));
    note_launch();
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_gemm(const GemmLaunch& L, cudaStream_t stream) {
    const KernelSetup& ks = setup_for_device();
    if (ks.err != cudaSuccess) return ks.err;
    if (L.x) {
        // the quantizer runs inside the decode kernel (q and s_k are outputs)
        if (L.m > kDecFusedMaxTokens) return cudaErrorInvalidValue;
        return launch_decode<32, true>(L, ks.sms, stream);
    }
    if (L.m <= 32) return launch_decode<32, false>(L, ks.sms, stream);
    if (L.m <= kDecMaxTokens) return launch_decode<64, false>(L, ks.sms, stream);
    CUtensorMap ta, tb, ts, ty;
    if (!make_map_u8(&ta, L.q, L.k, L.m, BM) || !make_map_u8(&tb, L.wq, L.k, L.n, BN_CTA) ||
        !make_map_scales_box(&ts, L.s_k, L.mp, L.k / BK, BM) || !make_map_out_bf16(&ty, L.y, L.n, L.m))
        return cudaErrorInvalidValue;
    Shape sh;
    sh.M = L.m;
    sh.N = L.n;
    sh.G = L.k / BK;
    sh.Mp = L.mp;
    sh.num_m = (L.m + BM_PAIR - 1) / BM_PAIR;
    sh.num_tiles = sh.num_m * ((L.n + BN - 1) / BN);
    sh.w_per_row = L.w_per_row ? 1u : 0u;
    sh.no_copies = L.diag_budget != 0 ? 1u : 0u;
    sh.budget = L.diag_budget != 0 ? L.diag_budget : kWaitBudgetCycles;
    const uint32_t max_pairs = static_cast<uint32_t>(ks.sms) / 2;
    const uint32_t grid = 2 * (sh.num_tiles < max_pairs ? sh.num_tiles : max_pairs);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = L.pdl ? 1 : 0;
    const bool direct = sh.G <= kDirectScalesMaxG;
    cudaError_t e = direct ? cudaLaunchKernelEx(&cfg, gemm_blockscaled_kernel<true>, ta, tb, ts, ty, L.s_k, L.w_scale, sh)
                           : cudaLaunchKernelEx(&cfg, gemm_blockscaled_kernel<false>, ta, tb, ts, ty, L.s_k, L.w_scale, sh);
    note_launch();
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fp8q
