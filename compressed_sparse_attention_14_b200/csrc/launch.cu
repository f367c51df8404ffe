// Process-wide launch settings.
//
// A kernel's dynamic shared-memory ceiling (cudaFuncAttributeMaxDynamic-
// SharedMemorySize) is a property of the function on a device, shared by
// every host thread. Setting it per call to the call's own size would let a
// call on another thread lower it between this call's set and its launch,
// and that launch would then fail. So each kernel's ceiling is raised once
// per device to the device's opt-in maximum; a launch still asks for exactly
// the shared memory it uses (the ceiling is only an upper bound).
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
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e != cudaSuccess) return e;
    done.insert({kern, dev});
    return cudaSuccess;
}

}  // namespace csa
