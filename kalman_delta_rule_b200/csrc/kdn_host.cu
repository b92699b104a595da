// Host-side caches of the launchers: per (device, CUDA context) kernel set-up and symbol
// addresses, so that no call repeats cudaFuncSetAttribute, occupancy queries or symbol
// look-ups, and a new primary context (after cudaDeviceReset) is set up afresh.
#include <cuda.h>

#include <map>
#include <mutex>
#include <tuple>

#include "kdn_launch.h"

namespace kdn {

namespace {
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

// the driver's cuCtxGetCurrent, resolved once through the runtime (no link against libcuda)
CUcontext current_context() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    CUcontext c = nullptr;
    if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
    return c;
}

// the context current on this thread for `dev`; the runtime binds the device's primary context
// lazily, so bind it first (cudaSetDevice initialises it) when none is current yet
cudaError_t bound_context(int dev, CUcontext *ctx) {
    *ctx = current_context();
    if (*ctx) return cudaSuccess;
    cudaError_t e = cudaSetDevice(dev);
    if (e != cudaSuccess) return e;
    *ctx = current_context();
    return cudaSuccess;
}

std::mutex g_mu;
std::map<std::tuple<const void *, int, CUcontext, size_t, int, bool>, KernelSetup> g_setups;
std::map<std::tuple<const void *, int, CUcontext>, void *> g_symbols;
}  // namespace

cudaError_t kernel_setup(const void *kern, size_t smem, int threads, bool max_carveout, KernelSetup *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    CUcontext ctx = nullptr;
    e = bound_context(dev, &ctx);
    if (e != cudaSuccess) return e;
    const auto key = std::make_tuple(kern, dev, ctx, smem, threads, max_carveout);
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_setups.find(key);
    if (it != g_setups.end()) {
        *out = it->second;
        return cudaSuccess;
    }
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (max_carveout) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
    }
    KernelSetup ks{148, 1};
    e = cudaDeviceGetAttribute(&ks.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ks.blocks_per_sm, kern, threads, smem);
    if (e != cudaSuccess) return e;
    g_setups[key] = ks;
    *out = ks;
    return cudaSuccess;
}

cudaError_t symbol_address(const void *symbol, void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    CUcontext ctx = nullptr;
    e = bound_context(dev, &ctx);
    if (e != cudaSuccess) return e;
    const auto key = std::make_tuple(symbol, dev, ctx);
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_symbols.find(key);
    if (it != g_symbols.end()) {
        *out = it->second;
        return cudaSuccess;
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, symbol);
    if (e != cudaSuccess) return e;
    g_symbols[key] = p;
    *out = p;
    return cudaSuccess;
}

}  // namespace kdn
