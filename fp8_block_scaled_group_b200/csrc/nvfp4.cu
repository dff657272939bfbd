// NVFP4 projection arms on sm_100a (page
// "spark_model/layers/ops/dispatch_proj.rs": `cutlass_nvfp4_proj`,
// `cutlass_nvfp4_weight_transposed_cached`, `cutlass_nvfp4_proj_from_fp8`,
// and `dequant_fp8_bf16_into` for the FP8 weight the last of them starts
// from).
//
// Formats. An NVFP4 operand is E2M1 elements packed two to a byte along K
// (element 2j in the low nibble of byte j), one E4M3 scale per 16 elements
// of K, and one fp32 second-level scale s2 for the whole operand. The packer
// writes the scales twice: row-major [rows, K/16], and in the layout the
// tensor cores read them from, here called the MMA layout: one 512-byte atom
// per 128 rows and 64 elements of K, atoms ordered K-fastest within a
// 128-row block, and inside an atom
//     byte (r % 32) * 16 + ((r % 128) / 32) * 4 + (k / 16) % 4
// for row r and element k. Rows past `rows` up to the next multiple of 128
// hold zero scales.
//
// Kernels:
//   nvfp4_quant_kernel       bf16 -> packed E2M1 + E4M3 scales, one thread
//                            per 16-element block:
//                              sf = e4m3_rne_satfinite(amax / (6 * s2))
//                              s  = e4m3_value(sf) * s2
//                              q  = e2m1_rne_satfinite(x / s)
//                            with IEEE fp32 division (a zero s gives signed
//                            zeros)
//   dequant_fp8_bf16_kernel  FP8 weight -> bf16, each element the bf16
//                            nearest to the exact product code * scale
//   nvfp4_gemm_kernel<BN>    y = bf16(alpha * sum_k a * sfa * w * sfw),
//                            alpha = s2a * s2w, on tcgen05.mma
//                            kind::mxf4nvf4 with the E4M3 scales applied by
//                            the tensor cores (block16)
//
// The GEMM is a persistent single-CTA kernel: a CTA owns a 128 x BN output
// tile (BN = 256, or 128 at decode widths so that more CTAs stream the
// weight), takes K in stages of 256 elements (128 bytes a row: one
// 128-byte swizzle atom) and issues four K = 64 MMAs per stage. When one
// row of 128-column tiles leaves SMs idle (decode widths), K is split over
// a cluster of up to 8 CTAs, one per SM, whose fp32 partials are summed
// through distributed shared memory in rank order. Per stage
// TMA brings A [128 x 128 B] and B [BN x 128 B]; two or three bulk copies
// bring the scale atoms of the stage (2 KB per 128 rows). The MMA thread
// copies the stage's atoms into TMEM (tcgen05.cp, 4 columns per atom, the
// same 32 rows broadcast to every lane quarter) right before the MMAs that
// read them; a copy and the MMAs issued after it by the same thread run in
// order, so one set of scale columns serves every stage. Warps:
//   warp 0     TMA / bulk-copy producer
//   warp 1     TMEM allocation; MMA issuer (one thread)
//   warps 2-5  epilogue: warp w reads TMEM lanes 32*(w%4)..+31 (tile rows),
//              scales by alpha, rounds to bf16 and stores its rows
// TMEM: accumulator buffers from column 0 (one of 256 columns for
// BN = 256, two of 128 for BN = 128, one of 128 for decode widths' 32-row A
// stages), then the A scales (4 columns per K = 64 step) and the B scales
// (4 columns per 128 rows per step); 512 columns allocated, or 256 at
// decode widths so that two CTAs share an SM.
// Every mbarrier wait is bounded; a CTA that gives up sets bit 1 of this
// file's error word and winds down.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <mutex>

#include "group_quant.cuh"
#include "internal.h"
#include "nvfp4.h"
#include "ptx_fp4.cuh"

namespace fp8q {

__device__ uint32_t g_nvfp4_error = 0;

namespace {

constexpr uint32_t kBlk = 16;           // K elements per E4M3 scale
constexpr uint32_t kSfAtomBytes = 512;  // 128 rows x 4 scales

// Byte offset of the scale of (row, K block b) in the MMA layout.
__device__ __forceinline__ size_t sf_mma_offset(uint32_t row, uint32_t b, uint32_t k) {
    const size_t atom = static_cast<size_t>(row >> 7) * (k >> 6) + (b >> 2);
    return atom * kSfAtomBytes + (row & 31u) * 16u + ((row >> 5) & 3u) * 4u + (b & 3u);
}

// ------------------------------------------------------------ packer --

__global__ void __launch_bounds__(256) nvfp4_quant_kernel(const uint16_t* __restrict__ x, uint8_t* __restrict__ q,
                                                          uint8_t* __restrict__ sf_row, uint8_t* __restrict__ sf_mma,
                                                          float s2, uint32_t rows, uint32_t rows_pad, uint32_t k) {
    const uint32_t nb = k / kBlk;
    const uint64_t total = static_cast<uint64_t>(rows_pad) * nb;
    const float denom = __fmul_rn(6.0f, s2);
    for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
        const uint32_t row = static_cast<uint32_t>(i / nb);
        const uint32_t b = static_cast<uint32_t>(i % nb);
        const size_t mma_off = sf_mma_offset(row, b, k);
        if (row >= rows) {
            sf_mma[mma_off] = 0;
            continue;
        }
        const uint16_t* src = x + static_cast<size_t>(row) * k + static_cast<size_t>(b) * kBlk;
        float lo[8], hi[8];
        widen8(ld_stream16(src), lo);
        widen8(ld_stream16(src + 8), hi);
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fmaxf(fabsf(lo[j]), fabsf(hi[j])));
        const uint32_t code = cvt_e4m3x2(__fdiv_rn(amax, denom), 0.0f) & 0xFFu;
        const float s = __fmul_rn(e4m3_value(code), s2);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            lo[j] = s == 0.0f ? copysignf(0.0f, lo[j]) : __fdiv_rn(lo[j], s);
            hi[j] = s == 0.0f ? copysignf(0.0f, hi[j]) : __fdiv_rn(hi[j], s);
        }
        const uint2 packed = make_uint2(cvt_e2m1x8(lo), cvt_e2m1x8(hi));
        *reinterpret_cast<uint2*>(q + static_cast<size_t>(row) * (k / 2) + static_cast<size_t>(b) * 8u) = packed;
        if (sf_row) sf_row[static_cast<size_t>(row) * nb + b] = static_cast<uint8_t>(code);
        sf_mma[mma_off] = static_cast<uint8_t>(code);
    }
}

// ------------------------------------------------ FP8 -> bf16 weight --

// bf16 bits of the exact product a * b, rounded once to nearest even: the
// fp32 product p and its exact remainder r = a*b - p decide the one case
// where rounding p again could differ, p lying exactly on a bf16 midpoint.
__device__ __forceinline__ uint32_t bf16_of_product(float a, float b) {
    const float p = __fmul_rn(a, b);
    const float r = __fmaf_rn(a, b, -p);
    const uint32_t bits = __float_as_uint(p);
    const uint32_t low = bits & 0xFFFFu;
    const uint32_t h = bits >> 16;
    bool up;
    if (low != 0x8000u)
        up = low > 0x8000u;
    else if (r != 0.0f)
        up = (r > 0.0f) == (p > 0.0f);  // the exact magnitude lies above |p|
    else
        up = (h & 1u) != 0u;
    return h + (up ? 1u : 0u);
}

__global__ void __launch_bounds__(256) dequant_fp8_bf16_kernel(const uint8_t* __restrict__ wq,
                                                               const float* __restrict__ w_s,
                                                               uint16_t* __restrict__ y, uint32_t n, uint32_t k,
                                                               uint32_t block_n, uint32_t block_k) {
    const uint32_t nc = k / 16u;
    const uint32_t sk = k / block_k;
    const uint64_t total = static_cast<uint64_t>(n) * nc;
    for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
        const uint32_t row = static_cast<uint32_t>(i / nc);
        const uint32_t c0 = static_cast<uint32_t>(i % nc) * 16u;
        const float s = __ldg(w_s + static_cast<size_t>(row / block_n) * sk + c0 / block_k);
        const uint4 codes = ld_stream16(wq + static_cast<size_t>(row) * k + c0);
        const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
        uint32_t o[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
            const uint32_t c_lo = (w[e / 4] >> (8 * (e % 4))) & 0xFFu;
            const uint32_t c_hi = (w[e / 4] >> (8 * (e % 4 + 1))) & 0xFFu;
            o[e / 2] = bf16_of_product(e4m3_value(c_lo), s) | (bf16_of_product(e4m3_value(c_hi), s) << 16);
        }
        uint4* dst = reinterpret_cast<uint4*>(y + static_cast<size_t>(row) * k + c0);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

// Element-wise fp32 -> E2M1 with the packer's conversion, one code per byte.
__global__ void convert_e2m1_kernel(const float* __restrict__ in, uint8_t* __restrict__ out, size_t n) {
    const size_t groups = (n + 7) / 8;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < groups;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = 8 * i + j < n ? in[8 * i + j] : 0.0f;
        const uint32_t c = cvt_e2m1x8(v);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (8 * i + j < n) out[8 * i + j] = static_cast<uint8_t>((c >> (4 * j)) & 0xFu);
    }
}

// -------------------------------------------------------------- GEMM --

constexpr uint32_t kBM = 128;
constexpr uint32_t kStageKBytes = 128;                       // 256 E2M1 elements per row
constexpr uint32_t kKSteps = 4;                              // K = 64 MMAs per stage
constexpr uint32_t kSfStageBytes = kKSteps * kSfAtomBytes;   // one 128-row block's scales per stage
constexpr uint32_t kThreads = 192;
constexpr uint32_t kEpiWarps = 4;

// AR: rows of A each stage holds. 128 in general; 32 when all of M fits in
// 32 rows (decode widths), so that a stage takes 24 KB and two CTAs fit an
// SM. The MMA still reads 128 rows of A: rows 32..127 come from whatever
// the shared memory after the stage holds, finite E2M1 codes whose scale
// factors are the zero pad rows of the A scales, and they only feed output
// rows that are never stored.
template <uint32_t BN, uint32_t AR>
struct Cfg {
    static constexpr uint32_t kStages = BN == 256 ? 4 : (AR == 32 ? 4 : 6);
    // One accumulator buffer at AR = 32, so that the allocation (256
    // columns) lets two CTAs share an SM's tensor memory.
    static constexpr uint32_t kAccBufs = BN == 256 || AR == 32 ? 1 : 2;
    static constexpr uint32_t kNBlk = BN / 128;  // 128-row scale blocks of B per tile
    static constexpr uint32_t kSfbBytes = kNBlk * kSfStageBytes;
    static constexpr uint32_t kStageTx = AR * kStageKBytes + BN * kStageKBytes + kSfStageBytes + kSfbBytes;
    static constexpr uint32_t kSfaCol = kAccBufs * BN;  // A scales: 4 columns per K = 64 step
    static constexpr uint32_t kSfbCol = kSfaCol + 4 * kKSteps;
    static constexpr uint32_t kTmemCols = kSfbCol + 4 * kNBlk * kKSteps <= 256 ? 256 : 512;
    static_assert(kSfbCol + 4 * kNBlk * kKSteps <= kTmemCols, "scale columns exceed the allocation");
};

// Output staging: per epilogue warp, one 32-row x 32-column bf16 block
// (64-byte rows, 64-byte swizzle) that a TMA store writes to y.
constexpr uint32_t kOutCols = 32;
constexpr uint32_t kOutStageBytes = 32 * kOutCols * 2;

template <uint32_t BN, uint32_t AR>
struct __align__(1024) Smem {
    uint8_t a[Cfg<BN, AR>::kStages][AR * kStageKBytes];
    uint8_t b[Cfg<BN, AR>::kStages][BN * kStageKBytes];
    uint8_t out[kEpiWarps][kOutStageBytes];
    uint8_t sfa[Cfg<BN, AR>::kStages][kSfStageBytes];
    uint8_t sfb[Cfg<BN, AR>::kStages][Cfg<BN, AR>::kSfbBytes];
    uint64_t full[Cfg<BN, AR>::kStages];
    uint64_t empty[Cfg<BN, AR>::kStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    uint32_t abort;
    uint32_t consumed;
};

template <uint32_t BN, uint32_t AR>
constexpr size_t smem_bytes() {
    return sizeof(Smem<BN, AR>) + 1024;  // + alignment slack
}
static_assert(smem_bytes<256, 128>() <= 227 * 1024 && smem_bytes<128, 128>() <= 227 * 1024,
              "shared memory exceeds the per-CTA limit");

struct Shape {
    uint32_t M, N, K;
    uint32_t num_m, num_tiles;
    float alpha;
    // K split (1: persistent over tiles). With split > 1 (one 128-row tile
    // of A, BN = 128) the grid is split x tiles CTAs in clusters of `split`:
    // CTA `rank` of a cluster takes K stages [rank, rank + 1) * stages / split
    // of its tile, parks its fp32 partial in shared memory, and the cluster
    // sums the partials through distributed shared memory in rank order.
    uint32_t split;
};

constexpr uint32_t kMaxSplit = 8;
constexpr uint32_t kRedStride = 132;  // floats per partial row (128 + 4: 16-byte rows, staggered banks)

template <uint32_t BN, uint32_t AR>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmY, const uint8_t* __restrict__ sfa,
                      const uint8_t* __restrict__ sfb, uint16_t* __restrict__ y, const Shape sh) {
    using C = Cfg<BN, AR>;
    extern __shared__ uint8_t smem_raw[];
    Smem<BN, AR>& sm =
        *reinterpret_cast<Smem<BN, AR>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t warp = threadIdx.x >> 5;
    const uint32_t lane = threadIdx.x & 31;
    const uint32_t kt_count = sh.K / (2 * kStageKBytes);
    const size_t sf_block_bytes = static_cast<size_t>(sh.K / 64) * kSfAtomBytes;  // one 128-row block
    volatile uint32_t* abort = &sm.abort;
    // Only the 128-column tiles split K; their B stages hold the partial
    // (at most AR rows).
    static_assert(BN != 128 || AR * kRedStride * sizeof(float) <= sizeof(sm.b), "the partial does not fit the B stages");
    const uint32_t split = BN == 128 ? sh.split : 1u;
    const uint32_t rank = cluster_ctarank();  // 0 without clusters
    const uint32_t tile0 = split > 1 ? blockIdx.x / split : blockIdx.x;
    const uint32_t tile_step = split > 1 ? sh.num_tiles : gridDim.x;  // split: one tile per CTA
    const uint32_t kt_begin = rank * kt_count / split;
    const uint32_t kt_end = (rank + 1) * kt_count / split;

    if (threadIdx.x == 0) {
        for (uint32_t s = 0; s < C::kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (uint32_t b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], kEpiWarps);
        }
        mbar_init(&sm.mma_done, 1);
        sm.abort = 0;
        sm.consumed = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmY);
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    uint32_t issued = 0;

    if (warp == 0) {
        if (lane == 0) {
            grid_dependency_wait();
            uint32_t it = 0;
            bool ok = true;
            for (uint32_t tile = tile0; ok && tile < sh.num_tiles; tile += tile_step) {
                const uint32_t m0 = (tile % sh.num_m) * kBM;
                const uint32_t n0 = (tile / sh.num_m) * BN;
                const uint8_t* sfa_blk = sfa + static_cast<size_t>(m0 / 128) * sf_block_bytes;
                const uint8_t* sfb_blk = sfb + static_cast<size_t>(n0 / 128) * sf_block_bytes;
                for (uint32_t kt = kt_begin; kt < kt_end; ++kt, ++it) {
                    const uint32_t s = it % C::kStages;
                    const uint32_t ph = (it / C::kStages) & 1u;
                    if (!mbar_wait(&sm.empty[s], ph ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.full[s], C::kStageTx);
                    const int32_t kx = static_cast<int32_t>(kt * kStageKBytes);
                    tma_load_2d(sm.a[s], &tmA, &sm.full[s], kx, static_cast<int32_t>(m0));
                    tma_load_2d(sm.b[s], &tmB, &sm.full[s], kx, static_cast<int32_t>(n0));
                    bulk_load(sm.sfa[s], sfa_blk + static_cast<size_t>(kt) * kSfStageBytes, kSfStageBytes,
                              &sm.full[s]);
#pragma unroll
                    for (uint32_t j = 0; j < C::kNBlk; ++j)
                        bulk_load(sm.sfb[s] + j * kSfStageBytes,
                                  sfb_blk + j * sf_block_bytes + static_cast<size_t>(kt) * kSfStageBytes,
                                  kSfStageBytes, &sm.full[s]);
                    issued = it + 1;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_e2m1_ue4m3(kBM, BN);
            uint32_t it = 0, local = 0;
            bool ok = true;
            for (uint32_t tile = tile0; ok && tile < sh.num_tiles; tile += tile_step, ++local) {
                const uint32_t buf = local % C::kAccBufs;
                const uint32_t bph = (local / C::kAccBufs) & 1u;
                if (!mbar_wait(&sm.acc_empty[buf], bph ^ 1u, abort)) break;
                tc_fence_after();
                const uint32_t d = tmem + buf * BN;
                for (uint32_t kt = kt_begin; kt < kt_end; ++kt, ++it) {
                    const uint32_t s = it % C::kStages;
                    const uint32_t ph = (it / C::kStages) & 1u;
                    if (!mbar_wait(&sm.full[s], ph, abort)) {
                        ok = false;
                        break;
                    }
                    sm.consumed = it + 1;
                    tc_fence_after();
                    const uint32_t sfa_s = smem_addr(sm.sfa[s]);
                    const uint32_t sfb_s = smem_addr(sm.sfb[s]);
#pragma unroll
                    for (uint32_t j = 0; j < kKSteps; ++j) {
                        tmem_copy_sf_atom(tmem + C::kSfaCol + 4u * j, smem_desc_sf_atom(sfa_s + j * kSfAtomBytes));
#pragma unroll
                        for (uint32_t nb = 0; nb < C::kNBlk; ++nb)
                            tmem_copy_sf_atom(tmem + C::kSfbCol + 4u * (j * C::kNBlk + nb),
                                              smem_desc_sf_atom(sfb_s + nb * kSfStageBytes + j * kSfAtomBytes));
                    }
                    const uint64_t ad = smem_desc_k_sw128(smem_addr(sm.a[s]));
                    const uint64_t bd = smem_desc_k_sw128(smem_addr(sm.b[s]));
#pragma unroll
                    for (uint32_t j = 0; j < kKSteps; ++j)
                        mma_mxf4nvf4(d, ad + 2u * j, bd + 2u * j, idesc, tmem + C::kSfaCol + 4u * j,
                                     tmem + C::kSfbCol + 4u * C::kNBlk * j, (kt != kt_begin || j != 0) ? 1u : 0u);
                    mma_commit(&sm.empty[s]);
                }
                if (!ok) break;
                mma_commit(&sm.acc_full[buf]);
            }
            // every MMA and scale copy of this CTA completes before TMEM is freed
            mma_commit(&sm.mma_done);
            volatile uint32_t never = 0;
            mbar_wait(&sm.mma_done, 0, &never);
        }
    } else {
        const uint32_t quarter = warp & 3u;
        const uint32_t lane_off = (quarter * 32u) << 16;
        uint32_t local = 0;
        for (uint32_t tile = tile0; tile < sh.num_tiles; tile += tile_step, ++local) {
            const uint32_t m0 = (tile % sh.num_m) * kBM;
            const uint32_t n0 = (tile / sh.num_m) * BN;
            const uint32_t buf = local % C::kAccBufs;
            const uint32_t bph = (local / C::kAccBufs) & 1u;
            const bool got = mbar_wait(&sm.acc_full[buf], bph, abort);
            if (!__all_sync(0xFFFFFFFFu, got)) break;
            tc_fence_after();
            const uint32_t row = m0 + quarter * 32u + lane;
            if (split > 1) {
                // The partial, fp32, into the idle B stages (every MMA of
                // this CTA has completed): red[row][column].
                float* red = reinterpret_cast<float*>(&sm.b[0][0]);
#pragma unroll 1
                for (uint32_t c = 0; c < BN / 64; ++c) {
                    uint32_t v[64];
                    tmem_load64(tmem + lane_off + buf * BN + c * 64u, v);
                    if (row < sh.M) {
                        float4* dst = reinterpret_cast<float4*>(red + row * kRedStride + c * 64u);
#pragma unroll
                        for (uint32_t j = 0; j < 16; ++j)
                            dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                 __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                    }
                }
                continue;
            }
            // The warp's 32 rows leave as 32 x 32 bf16 blocks through a 2 KB
            // shared-memory buffer (16-byte chunk j of row r at chunk
            // j ^ ((r >> 1) & 3), the 64-byte swizzle of the output map),
            // stored by one lane with TMA; rows past M are clipped by the map.
            // The accumulator is released as soon as its last columns are in
            // registers.
            const bool rows_live = m0 + quarter * 32u < sh.M;
            uint8_t* stg = sm.out[warp - 2u];
            const int32_t y_row = static_cast<int32_t>(m0 + quarter * 32u);
#pragma unroll 1
            for (uint32_t c = 0; c < BN / 64; ++c) {
                uint32_t v[64];
                tmem_load64(tmem + lane_off + buf * BN + c * 64u, v);
                if (c == BN / 64 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.acc_empty[buf]);
                }
                if (!rows_live) continue;
#pragma unroll
                for (uint32_t h2 = 0; h2 < 2; ++h2) {
                    if (lane == 0) bulk_store_wait_read();  // the block before has left the buffer
                    __syncwarp();
#pragma unroll
                    for (uint32_t j = 0; j < 4; ++j) {
                        uint32_t w[4];
#pragma unroll
                        for (uint32_t h = 0; h < 4; ++h) {
                            const uint32_t e = 32 * h2 + 8 * j + 2 * h;
                            const __nv_bfloat16 e0 = __float2bfloat16_rn(sh.alpha * __uint_as_float(v[e]));
                            const __nv_bfloat16 e1 = __float2bfloat16_rn(sh.alpha * __uint_as_float(v[e + 1]));
                            w[h] = static_cast<uint32_t>(__bfloat16_as_ushort(e0)) |
                                   (static_cast<uint32_t>(__bfloat16_as_ushort(e1)) << 16);
                        }
                        *reinterpret_cast<uint4*>(stg + lane * 64u + ((j ^ ((lane >> 1) & 3u)) << 4)) =
                            make_uint4(w[0], w[1], w[2], w[3]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0)
                        tma_store_2d(&tmY, stg, static_cast<int32_t>(n0 + c * 64u + h2 * kOutCols), y_row);
                }
            }
        }
        // Every output block of this warp is in global memory before the CTA
        // (and its staging buffer) goes away.
        if (lane == 0) bulk_store_wait_all();
        __syncwarp();
    }

    // After a timed-out wait, let the copies this CTA started land (bounded).
    tc_fence_before();
    __syncthreads();
    if (*abort) {
        volatile uint32_t never = 0;
        if (threadIdx.x == 0) atomicOr(&g_nvfp4_error, 2u);
        if (warp == 0 && lane == 0)
            for (uint32_t it = sm.consumed; it < issued; ++it)
                mbar_wait(&sm.full[it % C::kStages], (it / C::kStages) & 1u, &never);
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }

    if (split > 1) {
        // CTA `rank` owns tokens rank, rank + split, ...; thread (tq, jq) of
        // its first four warps sums columns 4jq .. 4jq+3 of every fourth
        // owned token over the cluster in rank order, one 16-byte read per
        // peer, scales by alpha and stores four bf16 outputs.
        cluster_sync_all();
        if (threadIdx.x < 128 && !*abort) {
            const uint32_t jq = threadIdx.x & 31u;
            const uint32_t tq = threadIdx.x >> 5;
            const uint32_t j = 4u * jq;
            const uint32_t n0 = tile0 * BN;
            const uint32_t red_addr = smem_addr(&sm.b[0][0]);
            for (uint32_t t = rank + split * tq; t < sh.M; t += 4u * split) {
                float4 part[kMaxSplit];
#pragma unroll
                for (uint32_t p = 0; p < kMaxSplit; ++p)
                    part[p] = p < split ? ld_shared_cluster_f32x4(mapa_shared(red_addr + (t * kRedStride + j) * 4u, p))
                                        : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                float4 sum = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
                for (uint32_t p = 0; p < kMaxSplit; ++p) {
                    sum.x += part[p].x;
                    sum.y += part[p].y;
                    sum.z += part[p].z;
                    sum.w += part[p].w;
                }
                const __nv_bfloat162 lo = __floats2bfloat162_rn(sh.alpha * sum.x, sh.alpha * sum.y);
                const __nv_bfloat162 hi = __floats2bfloat162_rn(sh.alpha * sum.z, sh.alpha * sum.w);
                *reinterpret_cast<uint2*>(y + static_cast<size_t>(t) * sh.N + n0 + j) =
                    make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
            }
        }
        cluster_sync_all();  // peers' partials stay in place until every CTA has read them
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

// A packed operand [rows, inner bytes] read in [box_rows, 128-byte] tiles
// with the 128-byte swizzle; rows past `rows` read as zero.
bool make_map_packed(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner};
    cuuint32_t box[2] = {kStageKBytes, box_rows};
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

struct Setup {
    cudaError_t err = cudaSuccess;
    int sms = 0;
};

const Setup& setup_for_device() {
    static std::mutex mu;
    static Setup table[64];
    static bool done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    std::lock_guard<std::mutex> lock(mu);
    Setup& s = table[dev];
    if (!done[dev]) {
        done[dev] = true;
        s.err = cudaFuncSetAttribute(nvfp4_gemm_kernel<256, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem_bytes<256, 128>()));
        if (s.err == cudaSuccess)
            s.err = cudaFuncSetAttribute(nvfp4_gemm_kernel<128, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem_bytes<128, 128>()));
        if (s.err == cudaSuccess)
            s.err = cudaFuncSetAttribute(nvfp4_gemm_kernel<128, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem_bytes<128, 32>()));
        if (s.err == cudaSuccess) s.err = cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev);
    }
    return s;
}

unsigned grid_for(uint64_t items, int sms) {
    uint64_t blocks = (items + 255) / 256;
    const uint64_t cap = static_cast<uint64_t>(sms > 0 ? sms : 148) * 16u;
    if (blocks > cap) blocks = cap;
    return static_cast<unsigned>(blocks ? blocks : 1);
}

template <uint32_t BN, uint32_t AR>
cudaError_t launch_gemm_bn(const Nvfp4GemmLaunch& L, int sms, cudaStream_t stream) {
    CUtensorMap ta, tb, ty;
    if (!make_map_packed(&ta, L.qa, L.k / 2, L.m, AR) || !make_map_packed(&tb, L.qw, L.k / 2, L.n, BN) ||
        !make_map_out_bf16(&ty, L.y, L.n, L.m))
        return cudaErrorInvalidValue;
    Shape sh;
    sh.M = L.m;
    sh.N = L.n;
    sh.K = L.k;
    sh.num_m = (L.m + kBM - 1) / kBM;
    sh.num_tiles = sh.num_m * (L.n / BN);
    sh.alpha = L.alpha;
    // One row of 128-column tiles with fewer tiles than SMs (decode
    // widths): split K so that more SMs stream the weight, aiming at 0.8
    // CTA per SM-slot in total (1.6 per SM with 32-row A stages, which fit
    // two to an SM; 0.8 otherwise), at most kMaxSplit per cluster and at
    // least one K stage each. Measured on B200 at M=25, N=6144, K=5120
    // (48 tiles): 32-row stages ran 11.4 / 10.3 / 9.9 / 9.6 / 14.3 us at
    // splits 2 / 3 / 4 / 5 / 6 (5 chosen); 128-row stages 15.5 / 11.7 /
    // 17.5 us at 1 / 2 / 3 (2 chosen). Larger splits no longer fit at once.
    const uint32_t kt_count = L.k / (2 * kStageKBytes);
    uint32_t split = 1;
    if (BN == 128 && sh.num_m == 1) {
        const float target = (AR == 32 ? 1.6f : 0.8f) * static_cast<float>(sms);
        uint32_t s = static_cast<uint32_t>(target / static_cast<float>(sh.num_tiles) + 0.5f);
        if (s > kMaxSplit) s = kMaxSplit;
        if (s > kt_count) s = kt_count;
        split = s < 1 ? 1 : s;
        // FP8Q_NVFP4_SPLIT=<n> overrides the choice (sweeps).
        static const int forced = [] {
            const char* e = std::getenv("FP8Q_NVFP4_SPLIT");
            return e ? std::atoi(e) : 0;
        }();
        if (forced > 0) {
            split = static_cast<uint32_t>(forced);
            if (split > kMaxSplit) split = kMaxSplit;
            if (split > kt_count) split = kt_count;
        }
    }
    sh.split = split;
    const uint32_t slots = (AR == 32 ? 2u : 1u) * static_cast<uint32_t>(sms);  // CTAs resident at once
    const uint32_t grid = split > 1 ? split * sh.num_tiles : (sh.num_tiles < slots ? sh.num_tiles : slots);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes<BN, AR>();
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    uint32_t na = 0;
    if (split > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = split;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (L.pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    cudaError_t e = cudaLaunchKernelEx(&cfg, nvfp4_gemm_kernel<BN, AR>, ta, tb, ty, static_cast<const uint8_t*>(L.sfa),
                                       static_cast<const uint8_t*>(L.sfw), static_cast<uint16_t*>(L.y), sh);
    note_launch();
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

cudaError_t launch_nvfp4_quant(const void* x, void* q, void* sf_row, void* sf_mma, float s2, uint32_t rows,
                               uint32_t k, cudaStream_t stream) {
    const Setup& s = setup_for_device();
    if (s.err != cudaSuccess) return s.err;
    const uint32_t rows_pad = (rows + 127u) / 128u * 128u;
    nvfp4_quant_kernel<<<grid_for(static_cast<uint64_t>(rows_pad) * (k / kBlk), s.sms), 256, 0, stream>>>(
        static_cast<const uint16_t*>(x), static_cast<uint8_t*>(q), static_cast<uint8_t*>(sf_row),
        static_cast<uint8_t*>(sf_mma), s2, rows, rows_pad, k);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_dequant_fp8_bf16(const void* wq, const float* w_scale, void* y, uint32_t n, uint32_t k,
                                    uint32_t block_n, uint32_t block_k, cudaStream_t stream) {
    const Setup& s = setup_for_device();
    if (s.err != cudaSuccess) return s.err;
    dequant_fp8_bf16_kernel<<<grid_for(static_cast<uint64_t>(n) * (k / 16u), s.sms), 256, 0, stream>>>(
        static_cast<const uint8_t*>(wq), w_scale, static_cast<uint16_t*>(y), n, k, block_n, block_k);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_nvfp4_gemm(const Nvfp4GemmLaunch& L, cudaStream_t stream) {
    const Setup& s = setup_for_device();
    if (s.err != cudaSuccess) return s.err;
    // One 128-row tile of A (decode widths): 128-column tiles, so that twice
    // as many CTAs stream the weight. Otherwise 256 columns where N allows.
    // Decode widths (M <= 32): 32-row A stages, two CTAs per SM.
    if (L.m <= 32) return launch_gemm_bn<128, 32>(L, s.sms, stream);
    if (L.m <= kBM || L.n % 256u != 0) return launch_gemm_bn<128, 128>(L, s.sms, stream);
    return launch_gemm_bn<256, 128>(L, s.sms, stream);
}

cudaError_t launch_convert_e2m1(const float* in, uint8_t* out, size_t n, cudaStream_t stream) {
    const Setup& s = setup_for_device();
    if (s.err != cudaSuccess) return s.err;
    convert_e2m1_kernel<<<grid_for((n + 7) / 8, s.sms), 256, 0, stream>>>(in, out, n);
    note_launch();
    return cudaGetLastError();
}

cudaError_t read_clear_nvfp4_error(uint32_t* code, cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    uint32_t zero = 0;
    e = cudaMemcpyFromSymbol(code, g_nvfp4_error, sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    if (*code) e = cudaMemcpyToSymbol(g_nvfp4_error, &zero, sizeof(uint32_t));
    return e;
}

}  // namespace fp8q
