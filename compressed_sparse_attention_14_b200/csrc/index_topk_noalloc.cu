// Indexer + top-k for callers that cannot allocate device memory.
//
// csa_index_topk passes an fp32 score block of nq x Nmax floats from the
// indexer kernel to the top-k kernel, and takes it from a workspace the
// caller allocates. Some callers cannot provide one: a plug-in whose host
// framework owns every device allocation and hands it no scratch, a serving
// loop that fixes its memory footprint at start-up and must not allocate
// afterwards, or a latency-critical path that cannot afford cudaMalloc,
// which may synchronise the whole device. csa_index_topk_noalloc gives them
// the same computation with the score block in a fixed array of device
// memory owned by this library (g_noalloc_scores, CSA_NOALLOC_MAX_SCORES
// floats = 16 MiB). Every GPU that loads the library holds that array until
// the process exits. The call itself allocates nothing: no cudaMalloc,
// cudaFree or allocating library routine.
//
// Set-up: host code cannot pass the array's name to a kernel (on the host
// the name is only a stand-in for the device object), so the first call on
// each device, with that device current, looks up the array's device address
// with cudaGetSymbolAddress and keeps it; later calls reuse it. Make that
// first call before any stream capture.
//
// Sharing: every call on a device uses the same array, which keeps the last
// call's scores. Nothing in it has to start at zero: each call writes every
// score it later reads (the indexer writes all visible columns of each
// query, and the selection reads only those). Two calls that overlap on the
// GPU (on different streams, or from different host threads without
// ordering) race on the array; serialise them.
#include <mutex>

#include "kernels.h"

using namespace csa;

namespace {

__device__ __align__(256) float g_noalloc_scores[CSA_NOALLOC_MAX_SCORES];

// Device address of g_noalloc_scores on the current device (nullptr and a
// message on failure). Looked up once per device.
float* noalloc_scores_address(int* rc) {
    static std::mutex mu;
    static float* addr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        *rc = set_last_error(CSA_ERR_CUDA, "csa_index_topk_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
        return nullptr;
    }
    if (dev < 0 || dev >= 64) {
        *rc = set_last_error(CSA_ERR_UNSUPPORTED, "csa_index_topk_noalloc: device %d beyond 64", dev);
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        float* p = nullptr;
        e = cudaGetSymbolAddress((void**)&p, g_noalloc_scores);
        if (e != cudaSuccess || !p) {
            *rc = set_last_error(CSA_ERR_CUDA, "csa_index_topk_noalloc: cudaGetSymbolAddress: %s",
                                 cudaGetErrorString(e));
            return nullptr;
        }
        addr[dev] = p;
    }
    return addr[dev];
}

int check_ptr16(const void* p, const char* name, bool required) {
    if (!p) return required ? set_last_error(CSA_ERR_INVALID_ARG, "%s is NULL", name) : CSA_OK;
    if (((uintptr_t)p) & 15u) return set_last_error(CSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return CSA_OK;
}

}  // namespace

extern "C" int csa_index_topk_noalloc(const void* qI, const float* w, const void* K, const int32_t* pos,
                                      const int32_t* seq_of_q, int nq, int n_seq, int HI, int cI, int64_t Nmax,
                                      int m, int k, int32_t* idx, float* top_scores, int dtype, void* stream) {
    ElemType t = ElemType::BF16;
    if (dtype == CSA_FP32) t = ElemType::F32;
    else if (dtype != CSA_BF16)
        return set_last_error(CSA_ERR_INVALID_ARG, "dtype %d is neither CSA_BF16 nor CSA_FP32", dtype);
    if (HI < 1 || HI > CSA_MAX_INDEX_HEADS)
        return set_last_error(CSA_ERR_UNSUPPORTED, "HI=%d outside [1, %d]", HI, CSA_MAX_INDEX_HEADS);
    if (cI < 8 || cI > CSA_MAX_INDEX_DIM || cI % 8)
        return set_last_error(CSA_ERR_UNSUPPORTED, "index dim cI=%d must be a multiple of 8 in [8, %d]", cI,
                              CSA_MAX_INDEX_DIM);
    if (t == ElemType::BF16 && !index_tc_supported(HI, cI, 1))
        return set_last_error(CSA_ERR_UNSUPPORTED, "bf16 indexer needs cI a multiple of 64 (<= 256) (cI=%d)", cI);
    if (k < 1 || k > CSA_MAX_TOPK) return set_last_error(CSA_ERR_UNSUPPORTED, "k=%d outside [1, %d]", k, CSA_MAX_TOPK);
    if (nq < 0 || Nmax < 0 || m < 1 || n_seq < 1)
        return set_last_error(CSA_ERR_INVALID_ARG, "csa_index_topk_noalloc: bad nq/n_seq/Nmax/m");
    if (nq > 65535)
        return set_last_error(CSA_ERR_UNSUPPORTED, "csa_index_topk_noalloc: at most 65535 queries per call (got %d)",
                              nq);
    if (!seq_of_q && n_seq < nq)
        return set_last_error(CSA_ERR_INVALID_ARG,
                              "seq_of_q is NULL (query t reads sequence t) but n_seq < nq");
    if ((int64_t)n_seq * Nmax > INT32_MAX)
        return set_last_error(CSA_ERR_UNSUPPORTED, "cache rows n_seq*Nmax beyond int32");
    if ((int64_t)nq * Nmax > (int64_t)CSA_NOALLOC_MAX_SCORES)
        return set_last_error(CSA_ERR_UNSUPPORTED,
                              "csa_index_topk_noalloc: nq*Nmax = %lld scores exceed the fixed %d-score array "
                              "(use csa_index_topk with a workspace)",
                              (long long)nq * Nmax, CSA_NOALLOC_MAX_SCORES);
    if (nq == 0) return CSA_OK;
    int rc = CSA_OK;
    if ((rc = check_ptr16(qI, "qI", true)) || (rc = check_ptr16(w, "w", true)) ||
        (rc = check_ptr16(K, "K", Nmax > 0)) || (rc = check_ptr16(pos, "pos", true)) ||
        (rc = check_ptr16(seq_of_q, "seq_of_q", false)) || (rc = check_ptr16(idx, "idx", true)) ||
        (rc = check_ptr16(top_scores, "top_scores", false)))
        return rc;
    float* sc = noalloc_scores_address(&rc);
    if (!sc) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    QuerySpec qs{seq_of_q, pos, 0, 0};
    cudaError_t e = cudaSuccess;
    if (Nmax > 0) {
        e = t == ElemType::BF16
                ? index_scores_tc(qI, w, K, qs, nq, n_seq, HI, cI, Nmax, m, sc, Nmax, 1, false, device_status(), st)
                : index_scores(qI, w, K, qs, nq, n_seq, HI, cI, Nmax, m, sc, Nmax, t, st);
        if (e != cudaSuccess)
            return set_last_error(CSA_ERR_CUDA, "csa_index_topk_noalloc: scores: %s", cudaGetErrorString(e));
    }
    e = topk_select(sc, Nmax, pos, m, nq, Nmax, k, idx, top_scores, nullptr, st, seq_of_q, n_seq);
    if (e != cudaSuccess)
        return set_last_error(CSA_ERR_CUDA, "csa_index_topk_noalloc: top-k: %s", cudaGetErrorString(e));
    return CSA_OK;
}
