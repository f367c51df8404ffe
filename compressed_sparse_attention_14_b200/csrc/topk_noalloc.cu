// Top-k selection for callers that cannot allocate device memory.
//
// Who needs this: code that must select entries at a point where it cannot
// call cudaMalloc or take memory from an allocator, e.g. a plug-in whose
// host framework owns every device allocation and hands out no workspace,
// or a serving loop that forbids allocation after start-up so that its
// memory footprint stays fixed. csa_topk_from_scores_noalloc returns exactly
// what csa_topk_from_scores returns, but takes no workspace: the candidate
// buffers of the multi-level selection live in g_topk_scratch below, a fixed
// array in the library's own device memory.
//
// Costs and rules of the fixed array:
//  * kNoAllocScratchBytes (8 MiB) of device memory on every GPU that loads
//    this code, held until the process exits;
//  * a call whose selection needs more scratch than that is rejected with
//    CSA_ERR_UNSUPPORTED before anything is launched;
//  * every call shares the one array, so calls whose kernels may run at the
//    same time on the GPU (other streams, other host threads) race on it and
//    must be serialized by the caller; a call leaves its candidates in the
//    array, and nothing in it needs to start at zero (each level writes every
//    slot it later reads);
//  * the first call on a device, with that device current, looks up the
//    array's device address (cudaGetSymbolAddress) and remembers it; make
//    that first call before any stream capture begins.
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "kernels.h"

namespace csa {

constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;

static __device__ __align__(256) unsigned char g_topk_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_topk_scratch on the current device (looked up once).
int scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_last_error(CSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return set_last_error(CSA_ERR_UNSUPPORTED, "device ordinal %d beyond %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lk(g_setup_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_topk_scratch);
        if (e != cudaSuccess || !p)
            return set_last_error(CSA_ERR_CUDA, "cudaGetSymbolAddress(g_topk_scratch): %s", cudaGetErrorString(e));
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return CSA_OK;
}
}  // namespace

}  // namespace csa

using namespace csa;

extern "C" int csa_topk_from_scores_noalloc(const float* scores, int64_t ld, const int32_t* valid, int valid_div,
                                            int nq, int64_t ncols, int k, int32_t* idx, float* top_scores,
                                            void* stream) {
    if (k < 1 || k > CSA_MAX_TOPK)
        return set_last_error(CSA_ERR_UNSUPPORTED, "k=%d outside [1, %d]", k, CSA_MAX_TOPK);
    if (nq < 0 || ncols < 0 || ld < ncols || valid_div < 1)
        return set_last_error(CSA_ERR_INVALID_ARG, "csa_topk_from_scores_noalloc: bad nq/ncols/ld/valid_div");
    if (ncols > INT32_MAX) return set_last_error(CSA_ERR_UNSUPPORTED, "ncols beyond int32 indices");
    if (nq == 0) return CSA_OK;
    const void* ptrs[3] = {scores, valid, idx};
    const char* names[3] = {"scores", "valid", "idx"};
    const bool required[3] = {ncols > 0, false, true};
    for (int i = 0; i < 3; ++i) {
        if (!ptrs[i]) {
            if (required[i]) return set_last_error(CSA_ERR_INVALID_ARG, "%s is NULL", names[i]);
            continue;
        }
        if (((uintptr_t)ptrs[i]) & 15u)
            return set_last_error(CSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
    }
    if (top_scores && (((uintptr_t)top_scores) & 15u))
        return set_last_error(CSA_ERR_INVALID_ARG, "top_scores is not 16-byte aligned");
    const size_t need = topk_workspace_bytes(nq, ncols, k);
    if (need > kNoAllocScratchBytes)
        return set_last_error(CSA_ERR_UNSUPPORTED,
                              "csa_topk_from_scores_noalloc: this selection needs %zu bytes of scratch, the fixed "
                              "array holds %zu; use csa_topk_from_scores with a workspace",
                              need, kNoAllocScratchBytes);
    void* scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc != CSA_OK) return rc;
    cudaError_t e = topk_select(scores, ld, valid, valid_div, nq, ncols, k, idx, top_scores, scratch,
                                (cudaStream_t)stream);
    if (e != cudaSuccess)
        return set_last_error(CSA_ERR_CUDA, "csa_topk_from_scores_noalloc: %s", cudaGetErrorString(e));
    return CSA_OK;
}
