// fp8q_linear for callers that cannot allocate device memory.
//
// Some callers have no way to obtain a device buffer for the fused linear's
// intermediate FP8 activation and scales: a plugin inside a runtime that
// owns the whole device-memory budget and hands it only inputs and outputs,
// or a latency-critical loop where a cudaMalloc could synchronize the device.
// For them this file keeps that intermediate in a fixed, file-scope device
// array that is part of the library image, and runs the same kernels as
// fp8q_linear on it.
//
// In host code `g_linear_scratch` is only a host-side stand-in for the
// device array, not a device address. Its device address is looked up with
// cudaGetSymbolAddress, with the device current, and that address is what
// the kernels receive. The lookup is cached per device together with the
// unique ID of the CUDA context it was made in; a call that finds a
// different context current (for example after cudaDeviceReset made a new
// primary context) looks the address up again instead of reusing one that
// belonged to the old context.
#include <cuda.h>

#include <mutex>

#include "fp8q.h"
#include "internal.h"

namespace fp8q {
namespace {

// The scratch holds the FP8 activation [M, K] and the K-major scales
// [K/128, ceil16(M)] of one call (fp8q_linear_workspace_bytes(M, K)).
// 16 MiB covers, e.g., M = 1168 tokens at K = 5120 (6.2 MB) or M = 900 at
// K = 17408 (16.2 MB). Every GPU that loads the library holds this array
// until the process exits.
constexpr size_t kScratchBytes = size_t(16) << 20;

static __device__ __align__(256) uint8_t g_linear_scratch[kScratchBytes];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct DriverFns {
    CtxGetCurrentFn get_current = nullptr;
    CtxGetIdFn get_id = nullptr;
};

const DriverFns& driver_fns() {
    static DriverFns fns;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fns.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fns.get_id = reinterpret_cast<CtxGetIdFn>(p);
        cudaGetLastError();
    });
    return fns;
}

// ID of the context current on this thread, or 0 if there is none yet (the
// runtime makes the primary context current on its first call that needs one).
unsigned long long current_context_id() {
    const DriverFns& f = driver_fns();
    if (!f.get_current || !f.get_id) return 0;
    CUcontext ctx = nullptr;
    if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    unsigned long long id = 0;
    if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

struct ScratchEntry {
    unsigned long long ctx_id = 0;
    void* addr = nullptr;
};

std::mutex g_scratch_mu;
ScratchEntry g_scratch[64];

// Device address of g_linear_scratch in the current device's current context.
// The first call in a context looks it up (and so should come before any
// stream capture); later calls in the same context reuse it.
fp8q_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return FP8Q_ERR_CUDA;
    }
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return FP8Q_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return FP8Q_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchEntry& e = g_scratch[dev];
    const unsigned long long id = current_context_id();
    if (e.addr == nullptr || id == 0 || id != e.ctx_id) {
        void* p = nullptr;
        const cudaError_t err = cudaGetSymbolAddress(&p, g_linear_scratch);
        if (err != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            e = ScratchEntry{};
            return FP8Q_ERR_CUDA;
        }
        // The lookup made the device's primary context current if it was not.
        e.ctx_id = current_context_id();
        e.addr = p;
    }
    *out = e.addr;
    return FP8Q_OK;
}

}  // namespace
}  // namespace fp8q

extern "C" fp8q_status fp8q_linear_noalloc(const void* x, const void* wq, const float* w_scale, void* y,
                                           uint32_t m, uint32_t n, uint32_t k, void* stream) {
    if (k == 0 || k % 128 || n == 0 || n % 128) return FP8Q_ERR_SHAPE;
    if (m == 0) return FP8Q_OK;
    if (!x || !wq || !w_scale || !y) return FP8Q_ERR_NULL;
    if (fp8q_linear_workspace_bytes(m, k) > fp8q::kScratchBytes) return FP8Q_ERR_WORKSPACE;
    void* scratch = nullptr;
    const fp8q_status st = fp8q::scratch_address(&scratch);
    if (st != FP8Q_OK) return st;
    // The quantizer overwrites every byte the GEMM then reads (FP8 rows and
    // all K-major scales, pad rows included), so nothing left in the array
    // by an earlier call needs clearing.
    return fp8q_linear(x, wq, w_scale, y, scratch, fp8q::kScratchBytes, m, n, k, stream);
}
