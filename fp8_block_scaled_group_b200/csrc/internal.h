// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace fp8q {

// Quantizer variants (values match FP8Q_QUANT_SINGLE / FP8Q_QUANT_MULTI).
constexpr int kVariantSingle = 1;
constexpr int kVariantMulti = 2;

// MULTI geometry (the streaming quantizer): every warp streams chunks of 16
// groups (4 KB of X) through its own ring of 2 shared-memory slots and a
// 2 KB code staging buffer; 7 warps a CTA, up to 3 CTAs per SM.
constexpr uint32_t kStreamChunkGroups = 16;
constexpr uint32_t kStreamSlots = 2;
constexpr uint32_t kStreamWarps = 7;
constexpr uint32_t kStreamThreads = 32 * kStreamWarps;
constexpr uint32_t kStreamCtasPerSm = 3;
// MULTI runs when its grid (one CTA per chunk, at most kStreamCtasPerSm per
// SM) holds at least this many CTAs per SM; below it the one-group-per-CTA
// kernel's many small CTAs finish sooner. From a B200 sweep of both variants
// over M in 1..4576 at K = 5120, 6144, 17408: SINGLE was faster up to 68
// MULTI CTAs and MULTI from 72 on, so the floor is ceil(0.47 * 148) = 70.
constexpr float kMultiMinCtasPerSm = 0.47f;

// CTAs of the MULTI grid for (m, k) on `sms` SMs.
uint32_t stream_grid(uint32_t m, uint32_t k, uint32_t sms);

struct QuantLaunch {
    const void* x;
    void* q;
    float* s_row;
    float* s_k;
    uint32_t m, k, mp;
    int variant;
    uint32_t sms;  // SMs of the device (sizes the MULTI grid)
    // Timeout diagnostics only (0 in normal use): the MULTI kernel issues
    // no copies and bounds each wait by this many clocks.
    long long diag_budget = 0;
};

cudaError_t launch_quant_act(const QuantLaunch& L, cudaStream_t stream);
cudaError_t launch_quant_weight(const void* w, void* wq, float* w_scale, uint32_t n, uint32_t k,
                                cudaStream_t stream);
cudaError_t launch_quant_weight_rowwise(const void* w, void* wq, float* w_scale, uint32_t n, uint32_t k,
                                        cudaStream_t stream);
cudaError_t launch_convert_e4m3(const float* in, uint8_t* out, size_t n, cudaStream_t stream);
cudaError_t launch_check_division(unsigned long long* counts, cudaStream_t stream);

struct GemmLaunch {
    const void* q;
    const float* s_k;
    const void* wq;
    const float* w_scale;
    void* y;
    uint32_t m, n, k, mp;
    bool pdl;        // launched as the programmatic dependent of the kernel before it
    bool w_per_row;  // w_scale holds one scale per weight row [n] instead of [n/128, k/128] blocks
    // Non-null (m <= 32 only): the bf16 activation [m, k]; the decode kernel
    // quantizes it itself and writes q and the K-major s_k as outputs.
    const void* x = nullptr;
    // Timeout diagnostics only (0 in normal use): the kernel's producer
    // issues no copies and each wait is bounded by this many clocks.
    long long diag_budget = 0;
};

cudaError_t launch_gemm(const GemmLaunch& L, cudaStream_t stream);
constexpr uint32_t kFusedDecodeMaxTokens = 32;

// SiLU(gate) * up rounded to bf16, then quantized per 128-group of tokens.
struct SiluLaunch {
    const void* gate;
    const void* up;
    uint32_t ld;  // elements between consecutive rows of gate and of up
    void* q;
    float* s_row;
    float* s_k;
    uint32_t m, i, mp;
};

cudaError_t launch_silu_mul_quant(const SiluLaunch& L, bool pdl, cudaStream_t stream);
cudaError_t launch_check_silu_mul(unsigned long long* counts, uint32_t* max_err_bits, cudaStream_t stream);

cudaError_t read_clear_device_error(uint32_t* code, cudaStream_t stream);
cudaError_t read_clear_quant_error(uint32_t* code, cudaStream_t stream);

void note_launch();

}  // namespace fp8q
