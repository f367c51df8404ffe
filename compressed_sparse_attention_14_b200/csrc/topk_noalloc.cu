// Top-k selection for callers that cannot allocate device memory.
//
// Who needs this: code that must select entries at a point where it cannot
// call cudaMalloc or take memory from an allocator, e.g. a plug-in whose
// host framework owns every device allocation and hands out no workspace,
// or a serving loop that forbids allocation after start-up so that its
// memory footprint stays fixed. csa_topk_from_scores_noalloc returns exactly
// what csa_topk_from_scores returns and takes no workspace. The selection
// kernel keeps all of its scratch (sample, candidates, sort buffers) in
// shared memory, so nothing is allocated, no device memory is held between
// calls, and calls on different streams do not share state.
#include <stdarg.h>
#include <stdio.h>

#include "kernels.h"

using namespace csa;

extern "C" int csa_topk_from_scores_noalloc(const float* scores, int64_t ld, const int32_t* valid, int valid_div,
                                            int nq, int64_t ncols, int k, int32_t* idx, float* top_scores,
                                            void* stream) {
    if (k < 1 || k > CSA_MAX_TOPK)
        return set_last_error(CSA_ERR_UNSUPPORTED, "k=%d outside [1, %d]", k, CSA_MAX_TOPK);
    if (nq < 0 || ncols < 0 || ld < ncols || valid_div < 1)
        return set_last_error(CSA_ERR_INVALID_ARG, "csa_topk_from_scores_noalloc: bad nq/ncols/ld/valid_div");
    if (ncols > INT32_MAX) return set_last_error(CSA_ERR_UNSUPPORTED, "ncols beyond int32 indices");
    if (nq > 65535) return set_last_error(CSA_ERR_UNSUPPORTED, "csa_topk_from_scores_noalloc: nq=%d above 65535", nq);
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
    cudaError_t e = topk_select(scores, ld, valid, valid_div, nq, ncols, k, idx, top_scores, nullptr,
                                (cudaStream_t)stream);
    if (e != cudaSuccess)
        return set_last_error(CSA_ERR_CUDA, "csa_topk_from_scores_noalloc: %s", cudaGetErrorString(e));
    return CSA_OK;
}
