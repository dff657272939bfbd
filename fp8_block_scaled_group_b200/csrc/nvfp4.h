// Host-side declarations of the NVFP4 kernels (nvfp4.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace fp8q {

// Bytes of the scale factors in the MMA's layout for `rows` rows of K
// elements: one 512-byte atom per 128 rows (padded) and 64 elements of K.
inline size_t nvfp4_sf_mma_bytes(uint32_t rows, uint32_t k) {
    return static_cast<size_t>((rows + 127u) / 128u) * 128u * (k / 16u);
}

// bf16 [rows, k] -> E2M1 pairs [rows, k/2], E4M3 block scales row-major
// [rows, k/16] (sf_row may be null) and in the MMA layout (sf_mma, pad rows
// zeroed), with second-level scale s2.
cudaError_t launch_nvfp4_quant(const void* x, void* q, void* sf_row, void* sf_mma, float s2, uint32_t rows,
                               uint32_t k, cudaStream_t stream);

// FP8 weight [n, k] with fp32 scales (block block_n x block_k) -> bf16 [n, k].
cudaError_t launch_dequant_fp8_bf16(const void* wq, const float* w_scale, void* y, uint32_t n, uint32_t k,
                                    uint32_t block_n, uint32_t block_k, cudaStream_t stream);

struct Nvfp4GemmLaunch {
    const void* qa;      // [m, k/2] packed E2M1
    const void* sfa;     // MMA-layout scales of qa
    const void* qw;      // [n, k/2] packed E2M1
    const void* sfw;     // MMA-layout scales of qw
    void* y;             // [m, n] bf16
    float alpha;         // s2a * s2w
    uint32_t m, n, k;
    bool pdl;            // launched as the programmatic dependent of the kernel before it
};

cudaError_t launch_nvfp4_gemm(const Nvfp4GemmLaunch& L, cudaStream_t stream);

// fp32 -> one E2M1 code per value (low nibble), for sweeps of the conversion.
cudaError_t launch_convert_e2m1(const float* in, uint8_t* out, size_t n, cudaStream_t stream);

// Error word of the NVFP4 GEMM (bit 1 = a CTA gave up on a bounded wait),
// read and cleared after synchronising `stream`.
cudaError_t read_clear_nvfp4_error(uint32_t* code, cudaStream_t stream);

}  // namespace fp8q
