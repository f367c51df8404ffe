// Process-wide launch settings.
//
// A kernel's dynamic shared-memory ceiling (cudaFuncAttributeMaxDynamic-
// SharedMemorySize) is a property of the function on a device, shared by
// every host thread. Setting it per call to the call's own size would let a
// call on another thread lower it between this call's set and its launch,
// and that launch would then fail. So each kernel's ceiling is raised once
// per device to the device's opt-in maximum (less the kernel's static shared
// memory); a launch still asks for exactly the shared memory it uses (the
// ceiling is only an upper bound).
#include <atomic>
#include <mutex>
#include <set>
#include <utility>

#include "kernels.h"

namespace csa {

cudaError_t smem_ceiling(const void* kern) {
    static std::mutex mu;
    static std::set<std::pair<const void*, int>> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({kern, dev})) return cudaSuccess;
    int optin = 0;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    // the kernel's static shared memory counts against the same per-block limit
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)fa.sharedSizeBytes);
    if (e != cudaSuccess) return e;
    done.insert({kern, dev});
    return cudaSuccess;
}

// Failure-path test hooks (csa_debug_set): a shorter bound for the device
// waits of the tensor-core indexer, and flags that withhold one of its copies
// so that a wait runs out. Both default to off.
static std::atomic<uint32_t> g_wait_limit{0};
static std::atomic<uint32_t> g_debug_flags{0};

uint32_t debug_wait_limit() { return g_wait_limit.load(std::memory_order_relaxed); }
uint32_t debug_flags() { return g_debug_flags.load(std::memory_order_relaxed); }

}  // namespace csa

extern "C" int csa_debug_set(uint32_t wait_limit, uint32_t flags) {
    if (flags & ~(uint32_t)(CSA_DEBUG_SKIP_FIRST_TILE | CSA_DEBUG_SCORE_BLOCK | CSA_DEBUG_TOPK_FILTER))
        return csa::set_last_error(CSA_ERR_INVALID_ARG, "csa_debug_set: unknown flags 0x%x", flags);
    csa::g_wait_limit.store(wait_limit, std::memory_order_relaxed);
    csa::g_debug_flags.store(flags, std::memory_order_relaxed);
    return CSA_OK;
}
