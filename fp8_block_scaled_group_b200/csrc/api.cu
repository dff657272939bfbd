// C ABI of libfp8q.so: argument checks, the quantizer variant pick, and the
// launch sequence of each call. Declarations and contracts: include/fp8q.h.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "fp8q.h"
#include "internal.h"
#include "nvfp4.h"
#include "ptx.cuh"

namespace fp8q {

static std::atomic<uint64_t> g_launches{0};

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {

constexpr uint32_t kGroup = 128;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

uint32_t ceil_div(uint32_t a, uint32_t b) { return (a + b - 1) / b; }

// Per-device facts, queried once per device.
struct DeviceInfo {
    int major = -1, minor = -1, sms = 0;
};

fp8q_status current_device(DeviceInfo* out) {
    static std::mutex mu;
    static DeviceInfo cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return FP8Q_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(mu);
    DeviceInfo& d = cache[dev];
    if (d.major < 0) {
        if (cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            d = DeviceInfo{};
            cudaGetLastError();
            return FP8Q_ERR_CUDA;
        }
    }
    *out = d;
    if (d.major != 10 || d.minor != 0) return FP8Q_ERR_UNSUPPORTED_DEVICE;
    return FP8Q_OK;
}

// FP8Q_QUANT_VARIANT=single|multi forces a variant (read once).
int32_t env_variant() {
    static int32_t v = [] {
        const char* e = std::getenv("FP8Q_QUANT_VARIANT");
        if (!e) return static_cast<int32_t>(FP8Q_QUANT_AUTO);
        if (!std::strcmp(e, "single")) return static_cast<int32_t>(FP8Q_QUANT_SINGLE);
        if (!std::strcmp(e, "multi")) return static_cast<int32_t>(FP8Q_QUANT_MULTI);
        return static_cast<int32_t>(FP8Q_QUANT_AUTO);
    }();
    return v;
}

// FP8Q_LOG=1: one line per process per pick branch, so a run that sees both
// decode and prefill widths reports both variants once.
void log_pick(const fp8q_quant_pick_t& p, uint32_t m, uint32_t k) {
    static const bool on = [] {
        const char* e = std::getenv("FP8Q_LOG");
        return e && e[0] == '1';
    }();
    if (!on) return;
    static std::atomic<bool> said[4];
    const int slot = (p.variant == FP8Q_QUANT_MULTI ? 1 : 0) + (p.forced ? 2 : 0);
    if (said[slot].exchange(true)) return;
    std::fprintf(stderr,
                 "fp8q: act-quant variant %s at M=%u K=%u grid=%u block=%u (multi grid %u CTAs, floor %u)%s\n",
                 p.variant == FP8Q_QUANT_MULTI ? "multi" : "single", m, k, p.grid_x, p.block_x, p.multi_ctas,
                 p.floor_ctas, p.forced ? " [forced]" : "");
}

// Shapes first; with M == 0 there is nothing to read or write, so the
// pointers of empty buffers (possibly NULL) are accepted.
fp8q_status check_quant_args(const void* x, const void* q, const float* s_row, const float* s_k, uint32_t m,
                             uint32_t k) {
    if (k == 0 || k % kGroup) return FP8Q_ERR_SHAPE;
    if (m == 0) return FP8Q_OK;
    if (!x || !q || !s_k) return FP8Q_ERR_NULL;
    if (static_cast<uint64_t>(m) * k >= (1ull << 31)) return FP8Q_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(q) || !aligned16(s_k) || (s_row && !aligned16(s_row))) return FP8Q_ERR_ALIGN;
    return FP8Q_OK;
}

fp8q_status check_gemm_args(const void* q, const float* s_k, const void* wq, const float* w_s, const void* y,
                            uint32_t m, uint32_t n, uint32_t k) {
    if (k == 0 || k % kGroup || n == 0 || n % kGroup) return FP8Q_ERR_SHAPE;
    if (m == 0) return FP8Q_OK;
    if (!q || !s_k || !wq || !w_s || !y) return FP8Q_ERR_NULL;
    if (static_cast<uint64_t>(m) * k >= (1ull << 31) || static_cast<uint64_t>(n) * k >= (1ull << 31) ||
        static_cast<uint64_t>(m) * n >= (1ull << 31))
        return FP8Q_ERR_SHAPE;
    if (!aligned16(q) || !aligned16(s_k) || !aligned16(wq) || !aligned16(w_s) || !aligned16(y))
        return FP8Q_ERR_ALIGN;
    return FP8Q_OK;
}

fp8q_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return FP8Q_OK;
    cudaGetLastError();
    return FP8Q_ERR_CUDA;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ceil(min_ctas_per_sm * sm_count), at least 1.
uint64_t floor_cta_count(uint32_t sm_count, float min_ctas_per_sm) {
    const double f = std::ceil(static_cast<double>(min_ctas_per_sm) * (sm_count ? sm_count : 1u) - 1e-9);
    return f < 1.0 ? 1u : static_cast<uint64_t>(f);
}

}  // namespace
}  // namespace fp8q

using namespace fp8q;

extern "C" {

const char* fp8q_status_string(int status) {
    switch (status) {
        case FP8Q_OK: return "FP8Q_OK";
        case FP8Q_ERR_NULL: return "FP8Q_ERR_NULL: a required pointer is NULL";
        case FP8Q_ERR_SHAPE: return "FP8Q_ERR_SHAPE: K and N must be non-zero multiples of 128 and sizes below 2^31";
        case FP8Q_ERR_ALIGN: return "FP8Q_ERR_ALIGN: pointers must be 16-byte aligned";
        case FP8Q_ERR_WORKSPACE: return "FP8Q_ERR_WORKSPACE: workspace too small or misaligned";
        case FP8Q_ERR_CUDA: return "FP8Q_ERR_CUDA: a CUDA call failed";
        case FP8Q_ERR_DEVICE_TIMEOUT: return "FP8Q_ERR_DEVICE_TIMEOUT: a kernel gave up on a bounded wait";
        case FP8Q_ERR_UNSUPPORTED_DEVICE: return "FP8Q_ERR_UNSUPPORTED_DEVICE: needs compute capability 10.0 (B200)";
        case FP8Q_ERR_ARG: return "FP8Q_ERR_ARG: invalid argument";
        default: return "FP8Q_ERR_UNKNOWN";
    }
}

const char* fp8q_version(void) { return "fp8q 0.1.0 (sm_100a)"; }

uint32_t fp8q_m_pad(uint32_t m) { return (m + 15u) / 16u * 16u; }

uint32_t fp8q_quant_floor_min_m(uint32_t k, uint32_t sm_count, uint32_t groups_per_cta, uint32_t rows_per_cta,
                                float min_ctas_per_sm) {
    if (k < kGroup || groups_per_cta == 0 || rows_per_cta == 0 || !(min_ctas_per_sm >= 0.0f)) return 0;
    const uint64_t grid_x = ceil_div(k / kGroup, groups_per_cta);
    const uint64_t floor_ctas = floor_cta_count(sm_count, min_ctas_per_sm);
    // smallest M with grid_x * ceil(M / rows_per_cta) >= floor_ctas
    const uint64_t row_blocks = (floor_ctas + grid_x - 1) / grid_x;
    const uint64_t min_m = row_blocks == 0 ? 0 : (row_blocks - 1) * rows_per_cta + 1;
    return static_cast<uint32_t>(min_m > 0xFFFFFFFFull ? 0xFFFFFFFFull : min_m);
}

fp8q_status fp8q_quant_pick(uint32_t m, uint32_t k, uint32_t sm_count, int32_t requested,
                            fp8q_quant_pick_t* out) {
    if (!out) return FP8Q_ERR_NULL;
    if (k == 0 || k % kGroup) return FP8Q_ERR_SHAPE;
    if (sm_count == 0 || requested < FP8Q_QUANT_AUTO || requested > FP8Q_QUANT_MULTI) return FP8Q_ERR_ARG;
    const uint32_t G = k / kGroup;
    fp8q_quant_pick_t p;
    std::memset(&p, 0, sizeof p);
    // m * G < 2^24 for every m*k < 2^31 the quantizer accepts; larger
    // products are only ever asked for by the pick itself.
    const uint64_t groups = static_cast<uint64_t>(m) * G;
    const uint64_t stages = (groups + kStreamChunkGroups - 1) / kStreamChunkGroups;
    const uint64_t cap = static_cast<uint64_t>(sm_count) * kStreamCtasPerSm;
    p.multi_ctas = static_cast<uint32_t>(stages < cap ? stages : cap);
    p.floor_ctas = static_cast<uint32_t>(floor_cta_count(sm_count, kMultiMinCtasPerSm));
    int32_t v;
    if (requested == FP8Q_QUANT_AUTO) {
        // The pages' rule: the multi-group kernel only when its grid reaches
        // the CTA-count floor.
        v = p.multi_ctas >= p.floor_ctas ? FP8Q_QUANT_MULTI : FP8Q_QUANT_SINGLE;
    } else {
        v = requested;
        p.forced = 1;
    }
    p.variant = v;
    if (v == FP8Q_QUANT_MULTI) {
        p.grid_x = p.multi_ctas;
        p.block_x = kStreamThreads;
        const uint64_t per_cta = p.multi_ctas ? (stages + p.multi_ctas - 1) / p.multi_ctas : 0;
        p.groups_per_cta = static_cast<uint32_t>(per_cta * kStreamChunkGroups);
    } else {
        const uint64_t single = groups;
        p.grid_x = static_cast<uint32_t>(single > 0xFFFFFFFFull ? 0xFFFFFFFFull : single);
        p.block_x = 16;
        p.groups_per_cta = 1;
    }
    *out = p;
    return FP8Q_OK;
}

fp8q_status fp8q_quant_act_variant(const void* x, void* q, float* s_row, float* s_kmajor, uint32_t m, uint32_t k,
                                   int32_t variant, void* stream) {
    fp8q_status st = check_quant_args(x, q, s_row, s_kmajor, m, k);
    if (st != FP8Q_OK) return st;
    if (variant < FP8Q_QUANT_AUTO || variant > FP8Q_QUANT_MULTI) return FP8Q_ERR_ARG;
    if (m == 0) return FP8Q_OK;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != FP8Q_OK) return st;
    fp8q_quant_pick_t pick;
    if ((st = fp8q_quant_pick(m, k, static_cast<uint32_t>(dev.sms), variant, &pick)) != FP8Q_OK) return st;
    log_pick(pick, m, k);
    QuantLaunch L{x, q, s_row, s_kmajor, m, k, fp8q_m_pad(m), pick.variant, static_cast<uint32_t>(dev.sms)};
    return from_cuda(launch_quant_act(L, static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_quant_act(const void* x, void* q, float* s_row, float* s_kmajor, uint32_t m, uint32_t k,
                           void* stream) {
    return fp8q_quant_act_variant(x, q, s_row, s_kmajor, m, k, env_variant(), stream);
}

fp8q_status fp8q_quant_weight(const void* w, void* wq, float* w_scale, uint32_t n, uint32_t k, void* stream) {
    if (k == 0 || k % kGroup || n == 0 || n % kGroup) return FP8Q_ERR_SHAPE;
    if (!w || !wq || !w_scale) return FP8Q_ERR_NULL;
    if (static_cast<uint64_t>(n) * k >= (1ull << 31)) return FP8Q_ERR_SHAPE;
    if (!aligned16(w) || !aligned16(wq) || !aligned16(w_scale)) return FP8Q_ERR_ALIGN;
    DeviceInfo dev;
    fp8q_status st = current_device(&dev);
    if (st != FP8Q_OK) return st;
    return from_cuda(launch_quant_weight(w, wq, w_scale, n, k, static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_quant_weight_rowwise(const void* w, void* wq, float* w_scale, uint32_t n, uint32_t k,
                                      void* stream) {
    if (k == 0 || k % kGroup || n == 0) return FP8Q_ERR_SHAPE;
    if (!w || !wq || !w_scale) return FP8Q_ERR_NULL;
    if (static_cast<uint64_t>(n) * k >= (1ull << 31)) return FP8Q_ERR_SHAPE;
    if (!aligned16(w) || !aligned16(wq) || !aligned16(w_scale)) return FP8Q_ERR_ALIGN;
    DeviceInfo dev;
    fp8q_status st = current_device(&dev);
    if (st != FP8Q_OK) return st;
    return from_cuda(launch_quant_weight_rowwise(w, wq, w_scale, n, k, static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_gemm_ex(const void* q, const float* s_kmajor, const void* wq, const float* w_scale,
                         int32_t weight_format, void* y, uint32_t m, uint32_t n, uint32_t k, void* stream) {
    if (weight_format != FP8Q_WEIGHT_BLOCK128 && weight_format != FP8Q_WEIGHT_PER_ROW) return FP8Q_ERR_ARG;
    fp8q_status st = check_gemm_args(q, s_kmajor, wq, w_scale, y, m, n, k);
    if (st != FP8Q_OK) return st;
    if (m == 0) return FP8Q_OK;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != FP8Q_OK) return st;
    GemmLaunch L{q, s_kmajor, wq, w_scale, y, m, n, k, fp8q_m_pad(m), false, weight_format == FP8Q_WEIGHT_PER_ROW};
    return from_cuda(launch_gemm(L, static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_gemm_blockscaled(const void* q, const float* s_kmajor, const void* wq, const float* w_scale,
                                  void* y, uint32_t m, uint32_t n, uint32_t k, void* stream) {
    return fp8q_gemm_ex(q, s_kmajor, wq, w_scale, FP8Q_WEIGHT_BLOCK128, y, m, n, k, stream);
}

size_t fp8q_linear_scale_offset(uint32_t m, uint32_t k) {
    return round_up(static_cast<size_t>(m) * k, 256);
}

size_t fp8q_linear_workspace_bytes(uint32_t m, uint32_t k) {
    const size_t g = k / kGroup;
    return fp8q_linear_scale_offset(m, k) + round_up(g * fp8q_m_pad(m) * sizeof(float), 256);
}

fp8q_status fp8q_linear_ex(const void* x, const void* wq, const float* w_scale, int32_t weight_format, void* y,
                           void* workspace, size_t workspace_bytes, uint32_t m, uint32_t n, uint32_t k,
                           void* stream) {
    if (weight_format != FP8Q_WEIGHT_BLOCK128 && weight_format != FP8Q_WEIGHT_PER_ROW) return FP8Q_ERR_ARG;
    if (k == 0 || k % kGroup || n == 0 || n % kGroup) return FP8Q_ERR_SHAPE;
    if (m == 0) return FP8Q_OK;
    if (!x || !wq || !w_scale || !y || !workspace) return FP8Q_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FP8Q_ERR_WORKSPACE;
    if (workspace_bytes < fp8q_linear_workspace_bytes(m, k)) return FP8Q_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* s_k = reinterpret_cast<float*>(ws + fp8q_linear_scale_offset(m, k));
    fp8q_status st = check_quant_args(x, ws, nullptr, s_k, m, k);
    if (st != FP8Q_OK) return st;
    if ((st = check_gemm_args(ws, s_k, wq, w_scale, y, m, n, k)) != FP8Q_OK) return st;
    const bool per_row = weight_format == FP8Q_WEIGHT_PER_ROW;
    if ((st = fp8q_quant_act(x, ws, nullptr, s_k, m, k, stream)) != FP8Q_OK) return st;
    // The GEMM is the quantizer's programmatic dependent: its set-up (barriers,
    // TMEM, descriptor prefetch) overlaps the quantizer, and its producer waits
    // for the quantizer's grid before the first load.
    GemmLaunch L{ws, s_k, wq, w_scale, y, m, n, k, fp8q_m_pad(m), true, per_row};
    return from_cuda(launch_gemm(L, static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_linear_decode_fused(const void* x, const void* wq, const float* w_scale, int32_t weight_format,
                                     void* y, void* workspace, size_t workspace_bytes, uint32_t m, uint32_t n,
                                     uint32_t k, void* stream) {
    if (weight_format != FP8Q_WEIGHT_BLOCK128 && weight_format != FP8Q_WEIGHT_PER_ROW) return FP8Q_ERR_ARG;
    if (k == 0 || k % kGroup || n == 0 || n % kGroup || m > kFusedDecodeMaxTokens) return FP8Q_ERR_SHAPE;
    if (m == 0) return FP8Q_OK;
    if (!x || !wq || !w_scale || !y || !workspace) return FP8Q_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FP8Q_ERR_WORKSPACE;
    if (workspace_bytes < fp8q_linear_workspace_bytes(m, k)) return FP8Q_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* s_k = reinterpret_cast<float*>(ws + fp8q_linear_scale_offset(m, k));
    fp8q_status st = check_quant_args(x, ws, nullptr, s_k, m, k);
    if (st != FP8Q_OK) return st;
    if ((st = check_gemm_args(ws, s_k, wq, w_scale, y, m, n, k)) != FP8Q_OK) return st;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != FP8Q_OK) return st;
    GemmLaunch L{ws, s_k, wq, w_scale, y, m, n, k, fp8q_m_pad(m), false, weight_format == FP8Q_WEIGHT_PER_ROW, x};
    return from_cuda(launch_gemm(L, static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_diag_stalled_linear(const void* x, const void* wq, const float* w_scale, void* y, void* workspace,
                                     size_t workspace_bytes, uint32_t m, uint32_t n, uint32_t k,
                                     uint64_t wait_budget_cycles, void* stream) {
    if (wait_budget_cycles == 0 || wait_budget_cycles > static_cast<uint64_t>(kWaitBudgetCycles)) return FP8Q_ERR_ARG;
    if (k == 0 || k % kGroup || n == 0 || n % kGroup) return FP8Q_ERR_SHAPE;
    if (m == 0) return FP8Q_OK;
    if (!x || !wq || !w_scale || !y || !workspace) return FP8Q_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FP8Q_ERR_WORKSPACE;
    if (workspace_bytes < fp8q_linear_workspace_bytes(m, k)) return FP8Q_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* s_k = reinterpret_cast<float*>(ws + fp8q_linear_scale_offset(m, k));
    fp8q_status st = check_quant_args(x, ws, nullptr, s_k, m, k);
    if (st != FP8Q_OK) return st;
    if ((st = check_gemm_args(ws, s_k, wq, w_scale, y, m, n, k)) != FP8Q_OK) return st;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != FP8Q_OK) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const long long budget = static_cast<long long>(wait_budget_cycles);
    QuantLaunch Lq{x, ws, nullptr, s_k, m, k, fp8q_m_pad(m), kVariantMulti, static_cast<uint32_t>(dev.sms)};
    Lq.diag_budget = budget;
    if ((st = from_cuda(launch_quant_act(Lq, s))) != FP8Q_OK) return st;
    GemmLaunch Lg{ws, s_k, wq, w_scale, y, m, n, k, fp8q_m_pad(m), false, false};
    Lg.diag_budget = budget;
    return from_cuda(launch_gemm(Lg, s));
}

fp8q_status fp8q_linear(const void* x, const void* wq, const float* w_scale, void* y, void* workspace,
                        size_t workspace_bytes, uint32_t m, uint32_t n, uint32_t k, void* stream) {
    return fp8q_linear_ex(x, wq, w_scale, FP8Q_WEIGHT_BLOCK128, y, workspace, workspace_bytes, m, n, k, stream);
}

fp8q_status fp8q_silu_mul_quant(const void* gate, const void* up, uint32_t ld, void* q, float* s_row,
                                float* s_kmajor, uint32_t m, uint32_t i, void* stream) {
    if (i == 0 || i % kGroup || ld < i || ld % 8) return FP8Q_ERR_SHAPE;
    if (m == 0) return FP8Q_OK;
    if (!gate || !up || !q || !s_kmajor) return FP8Q_ERR_NULL;
    if (static_cast<uint64_t>(m) * ld >= (1ull << 31)) return FP8Q_ERR_SHAPE;
    if (!aligned16(gate) || !aligned16(up) || !aligned16(q) || !aligned16(s_kmajor) ||
        (s_row && !aligned16(s_row)))
        return FP8Q_ERR_ALIGN;
    DeviceInfo dev;
    fp8q_status st = current_device(&dev);
    if (st != FP8Q_OK) return st;
    SiluLaunch L{gate, up, ld, q, s_row, s_kmajor, m, i, fp8q_m_pad(m)};
    return from_cuda(launch_silu_mul_quant(L, false, static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_ffn_workspace_layout(uint32_t m, uint32_t d, uint32_t i, size_t* offsets) {
    if (!offsets) return FP8Q_ERR_NULL;
    if (d == 0 || d % kGroup || i == 0 || i % kGroup) return FP8Q_ERR_SHAPE;
    const size_t mp = fp8q_m_pad(m);
    size_t off = 0;
    offsets[0] = off;  // q_x      e4m3 [m, d]
    off += round_up(static_cast<size_t>(m) * d, 256);
    offsets[1] = off;  // s_x      fp32 [d/128, ceil16(m)]
    off += round_up((d / kGroup) * mp * sizeof(float), 256);
    offsets[2] = off;  // gate|up  bf16 [m, 2i]
    off += round_up(static_cast<size_t>(m) * 2 * i * sizeof(uint16_t), 256);
    offsets[3] = off;  // q_h      e4m3 [m, i]
    off += round_up(static_cast<size_t>(m) * i, 256);
    offsets[4] = off;  // s_h      fp32 [i/128, ceil16(m)]
    off += round_up((i / kGroup) * mp * sizeof(float), 256);
    offsets[5] = off;  // total
    return FP8Q_OK;
}

size_t fp8q_ffn_workspace_bytes(uint32_t m, uint32_t d, uint32_t i) {
    size_t off[6];
    return fp8q_ffn_workspace_layout(m, d, i, off) == FP8Q_OK ? off[5] : 0;
}

fp8q_status fp8q_ffn(const void* x, const void* w_gate_up, const float* w_gate_up_scale, const void* w_down,
                     const float* w_down_scale, void* y, void* workspace, size_t workspace_bytes, uint32_t m,
                     uint32_t d, uint32_t i, void* stream) {
    size_t off[6];
    fp8q_status st = fp8q_ffn_workspace_layout(m, d, i, off);
    if (st != FP8Q_OK) return st;
    if (m == 0) return FP8Q_OK;
    if (!x || !w_gate_up || !w_gate_up_scale || !w_down || !w_down_scale || !y || !workspace) return FP8Q_ERR_NULL;
    // gate|up is [m, 2i]: the stacked width and the element count must stay
    // below 2^31 like every other operand (2i is formed in 32 bits below)
    if (static_cast<uint64_t>(m) * 2u * i >= (1ull << 31)) return FP8Q_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < off[5]) return FP8Q_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    void* q_x = ws + off[0];
    float* s_x = reinterpret_cast<float*>(ws + off[1]);
    uint16_t* gu = reinterpret_cast<uint16_t*>(ws + off[2]);
    void* q_h = ws + off[3];
    float* s_h = reinterpret_cast<float*>(ws + off[4]);
    if ((st = check_quant_args(x, q_x, nullptr, s_x, m, d)) != FP8Q_OK) return st;
    if ((st = check_gemm_args(q_x, s_x, w_gate_up, w_gate_up_scale, gu, m, 2 * i, d)) != FP8Q_OK) return st;
    if ((st = check_gemm_args(q_h, s_h, w_down, w_down_scale, y, m, d, i)) != FP8Q_OK) return st;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != FP8Q_OK) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint32_t mp = fp8q_m_pad(m);
    // x is quantized once; gate and up come out of one GEMM over the stacked
    // [2i, d] weight. Each later launch is the programmatic dependent of the
    // one before it and waits on it before reading its output.
    if ((st = fp8q_quant_act(x, q_x, nullptr, s_x, m, d, stream)) != FP8Q_OK) return st;
    GemmLaunch gate_up{q_x, s_x, w_gate_up, w_gate_up_scale, gu, m, 2 * i, d, mp, true, false};
    if ((st = from_cuda(launch_gemm(gate_up, s))) != FP8Q_OK) return st;
    SiluLaunch act{gu, gu + i, 2 * i, q_h, nullptr, s_h, m, i, mp};
    if ((st = from_cuda(launch_silu_mul_quant(act, true, s))) != FP8Q_OK) return st;
    GemmLaunch down{q_h, s_h, w_down, w_down_scale, y, m, d, i, mp, true, false};
    return from_cuda(launch_gemm(down, s));
}

fp8q_status fp8q_check_silu_mul(unsigned long long* counts, uint32_t* max_err_bits, void* stream) {
    if (!counts || !max_err_bits) return FP8Q_ERR_NULL;
    DeviceInfo dev;
    fp8q_status st = current_device(&dev);
    if (st != FP8Q_OK) return st;
    return from_cuda(launch_check_silu_mul(counts, max_err_bits, static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- NVFP4 --

size_t fp8q_nvfp4_sf_mma_bytes(uint32_t rows, uint32_t k) { return nvfp4_sf_mma_bytes(rows, k); }

fp8q_status fp8q_nvfp4_quant(const void* x, void* q, void* sf_rowmajor, void* sf_mma, float s2, uint32_t rows,
                             uint32_t k, void* stream) {
    if (k == 0 || k % 64u) return FP8Q_ERR_SHAPE;
    if (!(s2 > 0.0f) || std::isinf(s2)) return FP8Q_ERR_ARG;
    if (rows == 0) return FP8Q_OK;
    if (!x || !q || !sf_mma) return FP8Q_ERR_NULL;
    if (static_cast<uint64_t>(rows) * k >= (1ull << 31)) return FP8Q_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(q) || !aligned16(sf_mma)) return FP8Q_ERR_ALIGN;
    DeviceInfo dev;
    fp8q_status st = current_device(&dev);
    if (st != FP8Q_OK) return st;
    return from_cuda(launch_nvfp4_quant(x, q, sf_rowmajor, sf_mma, s2, rows, k, static_cast<cudaStream_t>(stream)));
}

namespace {

fp8q_status check_nvfp4_gemm_args(const void* qa, const void* sfa, float s2a, const void* qw, const void* sfw,
                                  float s2w, const void* y, uint32_t m, uint32_t n, uint32_t k) {
    if (k == 0 || k % 256u || n == 0 || n % kGroup) return FP8Q_ERR_SHAPE;
    if (!(s2a > 0.0f) || std::isinf(s2a) || !(s2w > 0.0f) || std::isinf(s2w)) return FP8Q_ERR_ARG;
    if (m == 0) return FP8Q_OK;
    if (!qa || !sfa || !qw || !sfw || !y) return FP8Q_ERR_NULL;
    if (static_cast<uint64_t>(m) * k >= (1ull << 31) || static_cast<uint64_t>(n) * k >= (1ull << 31) ||
        static_cast<uint64_t>(m) * n >= (1ull << 31))
        return FP8Q_ERR_SHAPE;
    if (!aligned16(qa) || !aligned16(sfa) || !aligned16(qw) || !aligned16(sfw) || !aligned16(y))
        return FP8Q_ERR_ALIGN;
    return FP8Q_OK;
}

}  // namespace

fp8q_status fp8q_nvfp4_gemm(const void* qa, const void* sfa_mma, float s2a, const void* qw, const void* sfw_mma,
                            float s2w, void* y, uint32_t m, uint32_t n, uint32_t k, void* stream) {
    fp8q_status st = check_nvfp4_gemm_args(qa, sfa_mma, s2a, qw, sfw_mma, s2w, y, m, n, k);
    if (st != FP8Q_OK) return st;
    if (m == 0) return FP8Q_OK;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != FP8Q_OK) return st;
    Nvfp4GemmLaunch L{qa, sfa_mma, qw, sfw_mma, y, s2a * s2w, m, n, k, false};
    return from_cuda(launch_nvfp4_gemm(L, static_cast<cudaStream_t>(stream)));
}

size_t fp8q_nvfp4_linear_workspace_bytes(uint32_t m, uint32_t k) {
    return round_up(static_cast<size_t>(m) * (k / 2), 256) + round_up(nvfp4_sf_mma_bytes(m, k), 256);
}

fp8q_status fp8q_nvfp4_linear(const void* x, float s2a, const void* qw, const void* sfw_mma, float s2w, void* y,
                              void* workspace, size_t workspace_bytes, uint32_t m, uint32_t n, uint32_t k,
                              void* stream) {
    if (k == 0 || k % 256u || n == 0 || n % kGroup) return FP8Q_ERR_SHAPE;
    if (!(s2a > 0.0f) || std::isinf(s2a) || !(s2w > 0.0f) || std::isinf(s2w)) return FP8Q_ERR_ARG;
    if (m == 0) return FP8Q_OK;
    if (!x || !qw || !sfw_mma || !y || !workspace) return FP8Q_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FP8Q_ERR_WORKSPACE;
    if (static_cast<uint64_t>(m) * k >= (1ull << 31)) return FP8Q_ERR_SHAPE;
    if (workspace_bytes < fp8q_nvfp4_linear_workspace_bytes(m, k)) return FP8Q_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    void* qa = ws;
    void* sfa = ws + round_up(static_cast<size_t>(m) * (k / 2), 256);
    fp8q_status st = check_nvfp4_gemm_args(qa, sfa, s2a, qw, sfw_mma, s2w, y, m, n, k);
    if (st != FP8Q_OK) return st;
    if (!aligned16(x)) return FP8Q_ERR_ALIGN;
    DeviceInfo dev;
    if ((st = current_device(&dev)) != FP8Q_OK) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = from_cuda(launch_nvfp4_quant(x, qa, nullptr, sfa, s2a, m, k, s))) != FP8Q_OK) return st;
    // The GEMM is the packer's programmatic dependent: its set-up overlaps
    // the packer and its producer waits for the packer's grid before loading.
    Nvfp4GemmLaunch L{qa, sfa, qw, sfw_mma, y, s2a * s2w, m, n, k, true};
    return from_cuda(launch_nvfp4_gemm(L, s));
}

fp8q_status fp8q_dequant_fp8_bf16(const void* wq, const float* w_scale, int32_t weight_format, void* y, uint32_t n,
                                  uint32_t k, void* stream) {
    if (weight_format != FP8Q_WEIGHT_BLOCK128 && weight_format != FP8Q_WEIGHT_PER_ROW) return FP8Q_ERR_ARG;
    const bool per_row = weight_format == FP8Q_WEIGHT_PER_ROW;
    if (k == 0 || k % kGroup || n == 0 || (!per_row && n % kGroup)) return FP8Q_ERR_SHAPE;
    if (!wq || !w_scale || !y) return FP8Q_ERR_NULL;
    if (static_cast<uint64_t>(n) * k >= (1ull << 31)) return FP8Q_ERR_SHAPE;
    if (!aligned16(wq) || !aligned16(w_scale) || !aligned16(y)) return FP8Q_ERR_ALIGN;
    DeviceInfo dev;
    fp8q_status st = current_device(&dev);
    if (st != FP8Q_OK) return st;
    return from_cuda(launch_dequant_fp8_bf16(wq, w_scale, y, n, k, per_row ? 1u : kGroup, per_row ? k : kGroup,
                                             static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_convert_e2m1(const float* in, uint8_t* out, size_t count, void* stream) {
    if (!in || !out) return FP8Q_ERR_NULL;
    if (count == 0) return FP8Q_OK;
    DeviceInfo dev;
    fp8q_status st = current_device(&dev);
    if (st != FP8Q_OK) return st;
    return from_cuda(launch_convert_e2m1(in, out, count, static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_convert_e4m3(const float* in, uint8_t* out, size_t count, void* stream) {
    if (!in || !out) return FP8Q_ERR_NULL;
    if (count == 0) return FP8Q_OK;
    DeviceInfo dev;
    fp8q_status st = current_device(&dev);
    if (st != FP8Q_OK) return st;
    return from_cuda(launch_convert_e4m3(in, out, count, static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_check_division(unsigned long long* counts, void* stream) {
    if (!counts) return FP8Q_ERR_NULL;
    DeviceInfo dev;
    fp8q_status st = current_device(&dev);
    if (st != FP8Q_OK) return st;
    return from_cuda(launch_check_division(counts, static_cast<cudaStream_t>(stream)));
}

uint64_t fp8q_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

fp8q_status fp8q_device_error(void* stream, uint32_t* code) {
    if (!code) return FP8Q_ERR_NULL;
    *code = 0;
    DeviceInfo dev;
    fp8q_status st = current_device(&dev);
    if (st != FP8Q_OK) return st;
    uint32_t nvfp4_code = 0, quant_code = 0;
    if (read_clear_device_error(code, static_cast<cudaStream_t>(stream)) != cudaSuccess ||
        read_clear_nvfp4_error(&nvfp4_code, static_cast<cudaStream_t>(stream)) != cudaSuccess ||
        read_clear_quant_error(&quant_code, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return FP8Q_ERR_CUDA;
    }
    *code |= nvfp4_code | quant_code;
    return *code ? FP8Q_ERR_DEVICE_TIMEOUT : FP8Q_OK;
}

}  // extern "C"
