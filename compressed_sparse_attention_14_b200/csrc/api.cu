// C ABI of libcsa: argument checks, workspace planning and launch order for
// every entry point declared in include/csa.h. All checks run on the host
// before the first launch; nothing here allocates device memory.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <string>

#include "common.cuh"
#include "kernels.h"

namespace csa {

__device__ int g_status_word = 0;

int* device_status() {
    static int* addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
        addr[dev] = (int*)p;
    }
    return addr[dev];
}


static thread_local std::string g_err;

static int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int set_last_error(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

static int cuda_status(cudaError_t e, const char* where) {
    if (e == cudaSuccess) return CSA_OK;
    return fail(CSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define CSA_TRY(expr)                          \
    do {                                       \
        int _rc = (expr);                      \
        if (_rc != CSA_OK) return _rc;         \
    } while (0)

#define CSA_CUDA(expr, where)                                  \
    do {                                                       \
        cudaError_t _e = (expr);                               \
        if (_e != cudaSuccess) return cuda_status(_e, where);  \
    } while (0)

static int check_ptr(const void* p, const char* name, bool required = true) {
    if (!p) return required ? fail(CSA_ERR_INVALID_ARG, "%s is NULL", name) : CSA_OK;
    if (((uintptr_t)p) & 15u) return fail(CSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return CSA_OK;
}

static int check_dtype(int dtype, ElemType* t) {
    if (dtype == CSA_BF16) { *t = ElemType::BF16; return CSA_OK; }
    if (dtype == CSA_FP32) { *t = ElemType::F32; return CSA_OK; }
    return fail(CSA_ERR_INVALID_ARG, "dtype %d is neither CSA_BF16 nor CSA_FP32", dtype);
}

static int check_ws(void* ws, size_t have, size_t need) {
    if (need == 0) return CSA_OK;
    if (!ws) return fail(CSA_ERR_WORKSPACE, "workspace is NULL but %zu bytes are needed", need);
    if (((uintptr_t)ws) & 255u) return fail(CSA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
    if (have < need) return fail(CSA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", have, need);
    return CSA_OK;
}

static float default_scale(float scale, int c) { return scale == 0.f ? 1.f / sqrtf((float)c) : scale; }

// Carves consecutive 256-byte aligned regions out of a workspace.
struct Carve {
    char* base;
    size_t off = 0;
    explicit Carve(void* b) : base((char*)b) {}
    void* take(size_t bytes) {
        void* p = base ? base + off : nullptr;
        off += align256(bytes);
        return p;
    }
};

static int check_attn_shape(int H, int c) {
    if (H < 1 || H > CSA_MAX_HEADS) return fail(CSA_ERR_UNSUPPORTED, "H=%d outside [1, %d]", H, CSA_MAX_HEADS);
    if (c < 32 || c > CSA_MAX_HEAD_DIM || c % 32)
        return fail(CSA_ERR_UNSUPPORTED, "head dim c=%d must be a multiple of 32 in [32, %d]", c, CSA_MAX_HEAD_DIM);
    return CSA_OK;
}

static int check_attn_mode(int H, int c, ElemType t) {
    if (t == ElemType::BF16 && !mqa_tc_supported(H, c))
        return fail(CSA_ERR_UNSUPPORTED, "bf16 MQA needs c a multiple of 128 (c=%d)", c);
    return CSA_OK;
}

static int check_cache_rows(int64_t n_seq, int64_t Nmax) {
    if (n_seq * Nmax > INT32_MAX) return fail(CSA_ERR_UNSUPPORTED, "cache rows n_seq*Nmax beyond int32");
    return CSA_OK;
}

static int check_index_shape(int HI, int cI) {
    if (HI < 1 || HI > CSA_MAX_INDEX_HEADS)
        return fail(CSA_ERR_UNSUPPORTED, "HI=%d outside [1, %d]", HI, CSA_MAX_INDEX_HEADS);
    if (cI < 8 || cI > CSA_MAX_INDEX_DIM || cI % 8)
        return fail(CSA_ERR_UNSUPPORTED, "index dim cI=%d must be a multiple of 8 in [8, %d]", cI, CSA_MAX_INDEX_DIM);
    return CSA_OK;
}

static int check_k(int k) {
    if (k < 1 || k > CSA_MAX_TOPK) return fail(CSA_ERR_UNSUPPORTED, "k=%d outside [1, %d]", k, CSA_MAX_TOPK);
    return CSA_OK;
}

// Indexer of the mode: tcgen05 kernel for bf16, FFMA kernel for fp32.
static cudaError_t run_indexer(const void* qI, const float* w, const void* K, QuerySpec qs, int nq, int n_seq,
                               int HI, int cI, int64_t Nmax, int m, float* scores, int64_t ld, int group,
                               bool fill_invisible, ElemType t, cudaStream_t st, RowBlocks kb = RowBlocks{0, 0}) {
    if (t == ElemType::BF16)
        return index_scores_tc(qI, w, K, qs, nq, n_seq, HI, cI, Nmax, m, scores, ld, group, fill_invisible,
                               device_status(), st, nullptr, false, kb);
    return index_scores(qI, w, K, qs, nq, n_seq, HI, cI, Nmax, m, scores, ld, t, st);
}

static int check_index_mode(int HI, int cI, ElemType t) {
    if (t == ElemType::BF16 && !index_tc_supported(HI, cI, 1))
        return fail(CSA_ERR_UNSUPPORTED, "bf16 indexer needs cI a multiple of 64 (<= 256) and HI <= 256 (cI=%d HI=%d)",
                    cI, HI);
    return CSA_OK;
}

static int check_rows(int nq, const char* who) {
    if (nq > 65535) return fail(CSA_ERR_UNSUPPORTED, "%s: at most 65535 queries per call (got %d)", who, nq);
    return CSA_OK;
}

// ---- plans shared by the size queries and the calls ------------------------

static size_t index_topk_bytes(int nq, int64_t Nmax, int k) {
    return align256((size_t)nq * (size_t)Nmax * sizeof(float)) + topk_workspace_bytes(nq, Nmax, k);
}

// The selection stage of csa_decode / csa_prefill: the indexer's top-k filter
// (candidate lists [nq][Nmax] of 64-bit keys + their lengths) where it
// applies, else the fp32 score block; the workspace holds either.
static size_t select_bytes(int nq, int64_t Nmax, int k) {
    const size_t cand = align256((size_t)nq * (size_t)Nmax * sizeof(uint64_t)) + align256((size_t)nq * sizeof(uint32_t));
    const size_t block = index_topk_bytes(nq, Nmax, k);
    return cand > block ? cand : block;
}

// The filter is opt-in (CSA_DEBUG_TOPK_FILTER): measured on B200 it makes the
// selection cheaper (long prefill: 7.1 -> 2.5 ms of top-k, 3.9 K candidates
// per 50 K-score row) but the indexer slower (59 -> 74-82 ms), because the
// prefill indexer is paced by its epilogue and every per-tile instruction
// there adds to the tile time; decode rows are split over several CTAs,
// whose bounds stay weak.
static bool use_topk_filter(ElemType t, int HI, int cI, int group, int k) {
    const uint32_t f = debug_flags();
    return t == ElemType::BF16 && (f & CSA_DEBUG_TOPK_FILTER) && !(f & CSA_DEBUG_SCORE_BLOCK) &&
           index_cand_supported(HI, cI, group, k);
}

// indexer -> top-k for nq queries into sel, through the filter (blk holds
// select_bytes) or the score block
static cudaError_t index_then_select(const void* qI, const float* w, const void* K, QuerySpec qs, int nq, int n_seq,
                                     int HI, int cI, int64_t Nmax, int m, int group, int k, int32_t* sel, void* blk,
                                     ElemType t, cudaStream_t st, RowBlocks kb, const char*& step) {
    if (kb.rpb == 0 && use_topk_filter(t, HI, cI, group, k)) {
        uint64_t* cand = (uint64_t*)blk;
        uint32_t* cnt = (uint32_t*)((char*)blk + align256((size_t)nq * (size_t)Nmax * sizeof(uint64_t)));
        step = "indexer with top-k filter";
        cudaError_t e = index_scores_tc(qI, w, K, qs, nq, n_seq, HI, cI, Nmax, m, nullptr, Nmax, group, false,
                                        device_status(), st, nullptr, false, RowBlocks{0, 0},
                                        CandOut{cand, cnt, Nmax, k});
        if (e != cudaSuccess) return e;
        step = "top-k of the candidates";
        return topk_from_candidates(cand, cnt, Nmax, nq, k, sel, nullptr, st);
    }
    float* sc = (float*)blk;
    step = "indexer";
    cudaError_t e = run_indexer(qI, w, K, qs, nq, n_seq, HI, cI, Nmax, m, sc, Nmax, group, false, t, st, kb);
    if (e != cudaSuccess) return e;
    step = "top-k";
    if (qs.pos) return topk_select(sc, Nmax, qs.pos, m, nq, Nmax, k, sel, nullptr, nullptr, st);
    return topk_select_positions(sc, Nmax, qs.pos_base, m, nq, Nmax, k, sel, nullptr, st);
}

static int64_t prefill_query_chunk(int64_t n, int64_t Nmax, int m) {
    // bound the fp32 score block of one query chunk to 1 GiB; whole
    // compressed blocks (multiples of m tokens) and at most 65535 queries
    int64_t qc = ((int64_t)1 << 28) / (Nmax > 0 ? Nmax : 1);
    if (qc > 65535) qc = 65535;
    qc -= qc % m;
    if (qc < m) qc = m;
    if (qc > n) qc = n;
    return qc;
}

}  // namespace csa

using namespace csa;

extern "C" {

const char* csa_last_error(void) { return g_err.c_str(); }
int csa_abi_version(void) { return CSA_ABI_VERSION; }
uint64_t csa_launch_count(void) { return launch_count(); }

void csa_trace_enable(int on) { trace_enable(on); }

int csa_trace_read(int max_kernels, char* names, double* total_ms, int* counts, int* n_kernels) {
    if (max_kernels < 0 || (max_kernels > 0 && (!names || !total_ms || !counts)) || !n_kernels)
        return fail(CSA_ERR_INVALID_ARG, "csa_trace_read: bad buffers");
    int e = trace_read(max_kernels, names, total_ms, counts, n_kernels);
    if (e) return cuda_status((cudaError_t)e, "csa_trace_read");
    return CSA_OK;
}

int csa_poll_status(void* stream, int reset) {
    cudaStream_t st = (cudaStream_t)stream;
    int v = 0;
    CSA_CUDA(cudaStreamSynchronize(st), "csa_poll_status sync");
    CSA_CUDA(cudaMemcpyFromSymbol(&v, g_status_word, sizeof(int)), "csa_poll_status read");
    if (reset) {
        int z = 0;
        CSA_CUDA(cudaMemcpyToSymbol(g_status_word, &z, sizeof(int)), "csa_poll_status reset");
    }
    if (v != 0) return fail(v, "a kernel reported device error %d", v);
    return CSA_OK;
}

// ---------------------------------------------------------------- a1
int csa_project(const void* x, const void* W, int64_t n, int d, int M, float* out, int dtype,
                void* stream) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    if (n < 0 || d < 8 || d % 8 || M < 8 || M % 8)
        return fail(CSA_ERR_INVALID_ARG, "csa_project: need n>=0, d and M multiples of 8 (n=%lld d=%d M=%d)",
                    (long long)n, d, M);
    if (n == 0) return CSA_OK;
    CSA_TRY(check_ptr(x, "x"));
    CSA_TRY(check_ptr(W, "W"));
    CSA_TRY(check_ptr(out, "out"));
    CSA_CUDA(project(x, W, n, d, M, out, t, (cudaStream_t)stream), "csa_project");
    return CSA_OK;
}

// ---------------------------------------------------------------- a2 / a3
static int check_compress(int64_t n, int c, int m, int mmax, const char* who) {
    if (m < 1 || m > mmax) return fail(CSA_ERR_INVALID_ARG, "%s: compression rate %d outside [1, %d]", who, m, mmax);
    if (n < 0 || n % m) return fail(CSA_ERR_INVALID_ARG, "%s: n=%lld is not a multiple of %d", who, (long long)n, m);
    if (c < 8 || c % 8) return fail(CSA_ERR_INVALID_ARG, "%s: c=%d must be a positive multiple of 8", who, c);
    return CSA_OK;
}

int csa_compress(const void* proj, const void* left, const float* bias, int64_t n, int c, int m,
                 void* out, int dtype, void* stream) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_compress(n, c, m, 64, "csa_compress"));
    if (n == 0) return CSA_OK;
    CSA_TRY(check_ptr(proj, "proj"));
    CSA_TRY(check_ptr(left, "left", false));
    CSA_TRY(check_ptr(bias, "bias"));
    CSA_TRY(check_ptr(out, "out"));
    CSA_CUDA(compress_csa(proj, left, bias, n, c, m, out, t, t, (cudaStream_t)stream), "csa_compress");
    return CSA_OK;
}

int hca_compress(const void* proj, const float* bias, int64_t n, int c, int mp, void* out,
                 int dtype, void* stream) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_compress(n, c, mp, 1024, "hca_compress"));
    if (n == 0) return CSA_OK;
    CSA_TRY(check_ptr(proj, "proj"));
    CSA_TRY(check_ptr(bias, "bias"));
    CSA_TRY(check_ptr(out, "out"));
    CSA_CUDA(compress_hca(proj, bias, n, c, mp, out, t, t, (cudaStream_t)stream), "hca_compress");
    return CSA_OK;
}

static int compress_step_common(const float* proj_new, float* state, const float* bias, const int32_t* pos, int B,
                                int c, int m, int mmax, int64_t Nmax, void* cache, int dtype, bool overlap,
                                void* stream, const char* who, RowBlocks cb = RowBlocks{0, 0}) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_compress(0, c, m, mmax, who));
    if (B < 0 || Nmax < 0) return fail(CSA_ERR_INVALID_ARG, "%s: bad B/Nmax", who);
    if (B == 0) return CSA_OK;
    CSA_TRY(check_ptr(proj_new, "proj_new"));
    CSA_TRY(check_ptr(state, "state"));
    CSA_TRY(check_ptr(bias, "bias"));
    CSA_TRY(check_ptr(pos, "pos"));
    CSA_TRY(check_ptr(cache, "cache", Nmax > 0));
    CSA_CUDA(compress_step(proj_new, state, bias, pos, B, c, m, overlap, Nmax, cache, t, (cudaStream_t)stream, 1, cb),
             who);
    return CSA_OK;
}

int csa_compress_step(const float* proj_new, float* state, const float* bias, const int32_t* pos, int B, int c, int m,
                      int64_t Nmax, void* cache, int dtype, void* stream) {
    return compress_step_common(proj_new, state, bias, pos, B, c, m, 64, Nmax, cache, dtype, true, stream,
                                "csa_compress_step");
}

int hca_compress_step(const float* proj_new, float* state, const float* bias, const int32_t* pos, int B, int c,
                      int mp, int64_t Nmax, void* cache, int dtype, void* stream) {
    return compress_step_common(proj_new, state, bias, pos, B, c, mp, 1024, Nmax, cache, dtype, false, stream,
                                "hca_compress_step");
}

// ---------------------------------------------------------------- cache blocks
static int64_t gcd64(int64_t a, int64_t b) { return b ? gcd64(b, a % b) : a; }

int csa_cache_block_layout(int m, int mp, int c, int cI, int dtype, int* csa_rows, int* hca_rows,
                           int64_t* block_bytes, int64_t* kv_offset, int64_t* idx_offset, int64_t* hca_offset) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    if (m < 1 || mp < 1 || c < 8 || cI < 8 || c % 8 || cI % 8)
        return fail(CSA_ERR_INVALID_ARG, "csa_cache_block_layout: m=%d mp=%d c=%d cI=%d", m, mp, c, cI);
    CSA_TRY(check_ptr(csa_rows, "csa_rows"));
    CSA_TRY(check_ptr(hca_rows, "hca_rows"));
    CSA_TRY(check_ptr(block_bytes, "block_bytes"));
    const int64_t L = (int64_t)m / gcd64(m, mp) * mp;   // lcm(m, m')
    if (L > (1 << 20)) return fail(CSA_ERR_UNSUPPORTED, "csa_cache_block_layout: lcm(m, m') = %lld", (long long)L);
    const int64_t es = t == ElemType::BF16 ? 2 : 4;
    const int64_t r1 = L / m, r2 = L / mp;
    *csa_rows = (int)r1;
    *hca_rows = (int)r2;
    const int64_t kv = 0, idx = kv + r1 * c * es, hca = idx + r1 * cI * es;
    *block_bytes = hca + r2 * c * es;   // a multiple of 16: c and cI are multiples of 8
    if (kv_offset) *kv_offset = kv;
    if (idx_offset) *idx_offset = idx;
    if (hca_offset) *hca_offset = hca;
    return CSA_OK;
}

// the blocked calls: bf16 caches, rows in blocks of rpb (dividing Nmax),
// blocks 16-byte aligned and at least rpb rows of `width` long
static int check_blocks(int rpb, int64_t block_bytes, int64_t Nmax, int width, const void* base, int dtype,
                        const char* who) {
    if (dtype != CSA_BF16) return fail(CSA_ERR_UNSUPPORTED, "%s: bf16 caches only", who);
    if (rpb < 1 || block_bytes % 16 || block_bytes < (int64_t)rpb * width * 2)
        return fail(CSA_ERR_INVALID_ARG, "%s: rows_per_block=%d block_bytes=%lld (a multiple of 16 holding %d rows of "
                    "%d bf16)", who, rpb, (long long)block_bytes, rpb, width);
    if (Nmax % rpb) return fail(CSA_ERR_INVALID_ARG, "%s: Nmax=%lld is not a multiple of rows_per_block=%d", who,
                                (long long)Nmax, rpb);
    if (base && ((uintptr_t)base & 15)) return fail(CSA_ERR_INVALID_ARG, "%s: cache pointer not 16-byte aligned", who);
    return CSA_OK;
}

int hca_compress_step_blocked(const float* proj_new, float* state, const float* bias, const int32_t* pos, int B,
                              int c, int mp, int64_t Nmax, void* cache, int rows_per_block, int64_t block_bytes,
                              int dtype, void* stream) {
    CSA_TRY(check_blocks(rows_per_block, block_bytes, Nmax, c, cache, dtype, "hca_compress_step_blocked"));
    return compress_step_common(proj_new, state, bias, pos, B, c, mp, 1024, Nmax, cache, dtype, false, stream,
                                "hca_compress_step_blocked", RowBlocks{rows_per_block, block_bytes});
}

static int compress_chunk_common(const float* proj, float* state, const float* bias, int64_t start, int64_t n, int c,
                                 int m, int mmax, void* cache, int64_t Nmax, int dtype, bool overlap, void* stream,
                                 const char* who) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_compress(0, c, m, mmax, who));
    if (start < 0 || n < 0 || Nmax < 0) return fail(CSA_ERR_INVALID_ARG, "%s: bad start/n/Nmax", who);
    if ((start + n) / m > Nmax)
        return fail(CSA_ERR_INVALID_ARG, "%s: the cache holds %lld entries, %lld needed", who, (long long)Nmax,
                    (long long)((start + n) / m));
    if (n == 0) return CSA_OK;
    CSA_TRY(check_ptr(proj, "proj"));
    CSA_TRY(check_ptr(state, "state"));
    CSA_TRY(check_ptr(bias, "bias"));
    CSA_TRY(check_ptr(cache, "cache", (start + n) / m > start / m));
    CSA_CUDA(compress_chunk_state(proj, state, bias, start, n, c, m, overlap, cache, t, (cudaStream_t)stream), who);
    return CSA_OK;
}

int csa_compress_chunk(const float* proj, float* state, const float* bias, int64_t start, int64_t n, int c, int m,
                       void* cache, int64_t Nmax, int dtype, void* stream) {
    return compress_chunk_common(proj, state, bias, start, n, c, m, 64, cache, Nmax, dtype, true, stream,
                                 "csa_compress_chunk");
}

int hca_compress_chunk(const float* proj, float* state, const float* bias, int64_t start, int64_t n, int c, int mp,
                       void* cache, int64_t Nmax, int dtype, void* stream) {
    return compress_chunk_common(proj, state, bias, start, n, c, mp, 1024, cache, Nmax, dtype, false, stream,
                                 "hca_compress_chunk");
}

size_t csa_decode_compress_workspace_size(int B, int c, int cI) {
    if (B < 0 || c < 0 || cI < 0) return 0;
    // decode-time projections run split over K (a few rows, a 21 MB weight
    // stream at d = 4096) and the workspace holds every slice's partial sums;
    // the split count depends on d, which this query does not take: size for
    // the largest split project_ksplit2 can choose (64 slices)
    return align256((size_t)64 * B * 4 * c * sizeof(float)) + align256((size_t)64 * B * 4 * cI * sizeof(float));
}

static int decode_compress_impl(const void* x_new, const void* W_kv, const float* B_kv, const void* W_idx,
                                const float* B_idx, const int32_t* pos, int B, int d, int m, int c, int cI,
                                float* state_kv, float* state_idx, void* kv_cache, void* idx_cache, int64_t Nmax,
                                void* ws, size_t ws_bytes, int dtype, void* stream, RowBlocks cb) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_compress(0, c, m, 64, "csa_decode_compress"));
    CSA_TRY(check_compress(0, cI, m, 64, "csa_decode_compress"));
    if (d < 8 || d % 8) return fail(CSA_ERR_INVALID_ARG, "d=%d must be a positive multiple of 8", d);
    if (B < 0 || Nmax < 0) return fail(CSA_ERR_INVALID_ARG, "csa_decode_compress: bad B/Nmax");
    if (B == 0) return CSA_OK;
    CSA_TRY(check_ptr(x_new, "x_new"));
    CSA_TRY(check_ptr(W_kv, "W_kv"));
    CSA_TRY(check_ptr(B_kv, "B_kv"));
    CSA_TRY(check_ptr(W_idx, "W_idx"));
    CSA_TRY(check_ptr(B_idx, "B_idx"));
    CSA_TRY(check_ptr(pos, "pos"));
    CSA_TRY(check_ptr(state_kv, "state_kv"));
    CSA_TRY(check_ptr(state_idx, "state_idx"));
    CSA_TRY(check_ptr(kv_cache, "kv_cache", Nmax > 0));
    CSA_TRY(check_ptr(idx_cache, "idx_cache", Nmax > 0));
    CSA_TRY(check_ws(ws, ws_bytes, csa_decode_compress_workspace_size(B, c, cI)));
    cudaStream_t st = (cudaStream_t)stream;
    Carve cv(ws);
    float* pk = (float*)cv.take((size_t)64 * B * 4 * c * sizeof(float));
    float* pi = (float*)cv.take((size_t)64 * B * 4 * cI * sizeof(float));
    // bf16: both split-K tensor-core projections in one launch (every SM
    // streams a slice of the weights); then one launch of the step kernel
    // adds the slices' partial sums in order and compresses both streams
    int ks_kv = 1, ks_idx = 1;
    if (t == ElemType::BF16) {
        project_ksplit2(B, d, 4 * c, 4 * cI, &ks_kv, &ks_idx);
        CSA_CUDA(project_tc2(x_new, B, d, W_kv, 4 * c, pk, ks_kv, W_idx, 4 * cI, pi, ks_idx, device_status(), st),
                 "csa_decode_compress: projections");
    } else {
        CSA_CUDA(project(x_new, W_kv, B, d, 4 * c, pk, t, st), "csa_decode_compress: KV projection");
        CSA_CUDA(project(x_new, W_idx, B, d, 4 * cI, pi, t, st), "csa_decode_compress: index-key projection");
    }
    const StepStream skv{pk, state_kv, B_kv, kv_cache, c, ks_kv, (int64_t)B * 4 * c, cb};
    const StepStream sidx{pi, state_idx, B_idx, idx_cache, cI, ks_idx, (int64_t)B * 4 * cI, cb};
    CSA_CUDA(compress_step_csa2(skv, sidx, pos, B, m, Nmax, t, st), "csa_decode_compress: compressors");
    return CSA_OK;
}

int csa_decode_compress(const void* x_new, const void* W_kv, const float* B_kv, const void* W_idx, const float* B_idx,
                        const int32_t* pos, int B, int d, int m, int c, int cI, float* state_kv, float* state_idx,
                        void* kv_cache, void* idx_cache, int64_t Nmax, void* ws, size_t ws_bytes, int dtype,
                        void* stream) {
    return decode_compress_impl(x_new, W_kv, B_kv, W_idx, B_idx, pos, B, d, m, c, cI, state_kv, state_idx, kv_cache,
                                idx_cache, Nmax, ws, ws_bytes, dtype, stream, RowBlocks{0, 0});
}

int csa_decode_compress_blocked(const void* x_new, const void* W_kv, const float* B_kv, const void* W_idx,
                                const float* B_idx, const int32_t* pos, int B, int d, int m, int c, int cI,
                                float* state_kv, float* state_idx, void* kv_cache, void* idx_cache, int64_t Nmax,
                                int rows_per_block, int64_t block_bytes, void* ws, size_t ws_bytes, int dtype,
                                void* stream) {
    CSA_TRY(check_blocks(rows_per_block, block_bytes, Nmax, c, kv_cache, dtype, "csa_decode_compress_blocked"));
    CSA_TRY(check_blocks(rows_per_block, block_bytes, Nmax, cI, idx_cache, dtype, "csa_decode_compress_blocked"));
    return decode_compress_impl(x_new, W_kv, B_kv, W_idx, B_idx, pos, B, d, m, c, cI, state_kv, state_idx, kv_cache,
                                idx_cache, Nmax, ws, ws_bytes, dtype, stream, RowBlocks{rows_per_block, block_bytes});
}

size_t csa_compress_from_hidden_workspace_size(int64_t n, int d, int c, int m, int dtype) {
    (void)d; (void)dtype;
    if (n < 0 || c < 0 || m < 1) return 0;
    return align256((size_t)n * 4 * c * sizeof(float)) + align256((size_t)m * 4 * c * sizeof(float));
}

int csa_compress_from_hidden(const void* x, const void* x_left, const void* W, const float* bias,
                             int64_t n, int d, int c, int m, void* out, void* ws, size_t ws_bytes,
                             int dtype, void* stream) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_compress(n, c, m, 64, "csa_compress_from_hidden"));
    if (d < 8 || d % 8) return fail(CSA_ERR_INVALID_ARG, "d=%d must be a positive multiple of 8", d);
    if (n == 0) return CSA_OK;
    CSA_TRY(check_ptr(x, "x"));
    CSA_TRY(check_ptr(x_left, "x_left", false));
    CSA_TRY(check_ptr(W, "W"));
    CSA_TRY(check_ptr(bias, "bias"));
    CSA_TRY(check_ptr(out, "out"));
    CSA_TRY(check_ws(ws, ws_bytes, csa_compress_from_hidden_workspace_size(n, d, c, m, dtype)));
    cudaStream_t st = (cudaStream_t)stream;
    Carve cv(ws);
    float* proj = (float*)cv.take((size_t)n * 4 * c * sizeof(float));
    float* lproj = (float*)cv.take((size_t)m * 4 * c * sizeof(float));
    CSA_CUDA(project(x, W, n, d, 4 * c, proj, t, st), "csa_compress_from_hidden: projection");
    if (x_left) CSA_CUDA(project(x_left, W, m, d, 4 * c, lproj, t, st), "csa_compress_from_hidden: left projection");
    CSA_CUDA(compress_csa(proj, x_left ? lproj : nullptr, bias, n, c, m, out, ElemType::F32, t, st),
             "csa_compress_from_hidden: compress");
    return CSA_OK;
}

size_t hca_compress_from_hidden_workspace_size(int64_t n, int d, int c, int mp, int dtype) {
    (void)d; (void)mp; (void)dtype;
    if (n < 0 || c < 0) return 0;
    return align256((size_t)n * 2 * c * sizeof(float));
}

int hca_compress_from_hidden(const void* x, const void* W, const float* bias, int64_t n, int d,
                             int c, int mp, void* out, void* ws, size_t ws_bytes, int dtype,
                             void* stream) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_compress(n, c, mp, 1024, "hca_compress_from_hidden"));
    if (d < 8 || d % 8) return fail(CSA_ERR_INVALID_ARG, "d=%d must be a positive multiple of 8", d);
    if (n == 0) return CSA_OK;
    CSA_TRY(check_ptr(x, "x"));
    CSA_TRY(check_ptr(W, "W"));
    CSA_TRY(check_ptr(bias, "bias"));
    CSA_TRY(check_ptr(out, "out"));
    CSA_TRY(check_ws(ws, ws_bytes, hca_compress_from_hidden_workspace_size(n, d, c, mp, dtype)));
    cudaStream_t st = (cudaStream_t)stream;
    float* proj = (float*)ws;
    CSA_CUDA(project(x, W, n, d, 2 * c, proj, t, st), "hca_compress_from_hidden: projection");
    CSA_CUDA(compress_hca(proj, bias, n, c, mp, out, ElemType::F32, t, st), "hca_compress_from_hidden: compress");
    return CSA_OK;
}

// ---------------------------------------------------------------- a4 / a5
int csa_index_scores(const void* qI, const float* w, const void* K, const int32_t* pos,
                     const int32_t* seq_of_q, int nq, int n_seq, int HI, int cI, int64_t Nmax, int m,
                     float* scores, int dtype, void* stream) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_index_shape(HI, cI));
    CSA_TRY(check_index_mode(HI, cI, t));
    CSA_TRY(check_rows(nq, "csa_index_scores"));
    if (nq < 0 || Nmax < 0 || m < 1 || n_seq < 1) return fail(CSA_ERR_INVALID_ARG, "bad nq/n_seq/Nmax/m");
    if (!seq_of_q && n_seq < nq) return fail(CSA_ERR_INVALID_ARG, "seq_of_q is NULL (query t reads sequence t) but n_seq < nq");
    if (Nmax > INT32_MAX) return fail(CSA_ERR_UNSUPPORTED, "Nmax beyond int32 entry indices");
    CSA_TRY(check_cache_rows(n_seq, Nmax));
    if (nq == 0 || Nmax == 0) return CSA_OK;
    CSA_TRY(check_ptr(qI, "qI"));
    CSA_TRY(check_ptr(w, "w"));
    CSA_TRY(check_ptr(K, "K"));
    CSA_TRY(check_ptr(pos, "pos"));
    CSA_TRY(check_ptr(seq_of_q, "seq_of_q", false));
    CSA_TRY(check_ptr(scores, "scores"));
    QuerySpec qs{seq_of_q, pos, 0, 0};
    CSA_CUDA(run_indexer(qI, w, K, qs, nq, n_seq, HI, cI, Nmax, m, scores, Nmax, 1, true, t, (cudaStream_t)stream),
             "csa_index_scores");
    return CSA_OK;
}

size_t csa_topk_workspace_size(int nq, int64_t ncols, int k) {
    if (nq < 0 || ncols < 0 || k < 1) return 0;
    return topk_workspace_bytes(nq, ncols, k);
}

int csa_topk_from_scores(const float* scores, int64_t ld, const int32_t* valid, int valid_div,
                         int nq, int64_t ncols, int k, int32_t* idx, float* top_scores, void* ws,
                         size_t ws_bytes, void* stream) {
    CSA_TRY(check_k(k));
    if (nq < 0 || ncols < 0 || ld < ncols || valid_div < 1)
        return fail(CSA_ERR_INVALID_ARG, "csa_topk_from_scores: bad nq/ncols/ld/valid_div");
    if (ncols > INT32_MAX) return fail(CSA_ERR_UNSUPPORTED, "ncols beyond int32 indices");
    CSA_TRY(check_rows(nq, "csa_topk_from_scores"));
    if (nq == 0) return CSA_OK;
    if (ncols > 0) CSA_TRY(check_ptr(scores, "scores"));
    CSA_TRY(check_ptr(valid, "valid", false));
    CSA_TRY(check_ptr(idx, "idx"));
    CSA_TRY(check_ptr(top_scores, "top_scores", false));
    CSA_TRY(check_ws(ws, ws_bytes, topk_workspace_bytes(nq, ncols, k)));
    CSA_CUDA(topk_select(scores, ld, valid, valid_div, nq, ncols, k, idx, top_scores, ws,
                         (cudaStream_t)stream), "csa_topk_from_scores");
    return CSA_OK;
}

int csa_topk_from_scores_bf16(const void* scores, int64_t ld, const int32_t* valid, int valid_div, int nq,
                              int64_t ncols, int k, int32_t* idx, float* top_scores, void* stream) {
    CSA_TRY(check_k(k));
    if (nq < 0 || ncols < 0 || ld < ncols || valid_div < 1)
        return fail(CSA_ERR_INVALID_ARG, "csa_topk_from_scores_bf16: bad nq/ncols/ld/valid_div");
    if (ncols > INT32_MAX) return fail(CSA_ERR_UNSUPPORTED, "ncols beyond int32 indices");
    CSA_TRY(check_rows(nq, "csa_topk_from_scores_bf16"));
    if (nq == 0) return CSA_OK;
    if (ncols > 0) CSA_TRY(check_ptr(scores, "scores"));
    CSA_TRY(check_ptr(valid, "valid", false));
    CSA_TRY(check_ptr(idx, "idx"));
    CSA_TRY(check_ptr(top_scores, "top_scores", false));
    CSA_CUDA(topk_select_bf16(scores, ld, valid, valid_div, nq, ncols, k, idx, top_scores, (cudaStream_t)stream),
             "csa_topk_from_scores_bf16");
    return CSA_OK;
}

size_t csa_index_topk_workspace_size(int nq, int64_t Nmax, int k, int dtype) {
    (void)dtype;
    if (nq < 0 || Nmax < 0 || k < 1) return 0;
    return index_topk_bytes(nq, Nmax, k);
}

int csa_index_topk(const void* qI, const float* w, const void* K, const int32_t* pos,
                   const int32_t* seq_of_q, int nq, int n_seq, int HI, int cI, int64_t Nmax, int m, int k,
                   int32_t* idx, float* top_scores, void* ws, size_t ws_bytes, int dtype,
                   void* stream) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_index_shape(HI, cI));
    CSA_TRY(check_index_mode(HI, cI, t));
    CSA_TRY(check_k(k));
    CSA_TRY(check_rows(nq, "csa_index_topk"));
    if (nq < 0 || Nmax < 0 || m < 1 || n_seq < 1) return fail(CSA_ERR_INVALID_ARG, "bad nq/n_seq/Nmax/m");
    if (!seq_of_q && n_seq < nq) return fail(CSA_ERR_INVALID_ARG, "seq_of_q is NULL (query t reads sequence t) but n_seq < nq");
    if (Nmax > INT32_MAX) return fail(CSA_ERR_UNSUPPORTED, "Nmax beyond int32 entry indices");
    if (nq == 0) return CSA_OK;
    CSA_TRY(check_ptr(qI, "qI"));
    CSA_TRY(check_ptr(w, "w"));
    CSA_TRY(check_ptr(K, "K", Nmax > 0));
    CSA_TRY(check_ptr(pos, "pos"));
    CSA_TRY(check_ptr(seq_of_q, "seq_of_q", false));
    CSA_TRY(check_ptr(idx, "idx"));
    CSA_TRY(check_ptr(top_scores, "top_scores", false));
    CSA_TRY(check_ws(ws, ws_bytes, index_topk_bytes(nq, Nmax, k)));
    cudaStream_t st = (cudaStream_t)stream;
    Carve cv(ws);
    float* sc = (float*)cv.take((size_t)nq * Nmax * sizeof(float));
    void* tws = cv.take(topk_workspace_bytes(nq, Nmax, k));
    QuerySpec qs{seq_of_q, pos, 0, 0};
    CSA_CUDA(run_indexer(qI, w, K, qs, nq, n_seq, HI, cI, Nmax, m, sc, Nmax, 1, false, t, st), "csa_index_topk: scores");
    CSA_CUDA(topk_select(sc, Nmax, pos, m, nq, Nmax, k, idx, top_scores, tws, st, seq_of_q, n_seq),
             "csa_index_topk: top-k");
    return CSA_OK;
}

// ---------------------------------------------------------------- FP8 indexer
int csa_quantize_e4m3(const void* x, int64_t rows, int cols, void* out, float* scale, const float* w, float* w_out,
                      int dtype, void* stream) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    if (rows < 0 || cols < 8 || cols % 8) return fail(CSA_ERR_INVALID_ARG, "rows=%lld cols=%d: cols must be a "
                                                      "positive multiple of 8", (long long)rows, cols);
    if ((rows + 7) / 8 > INT32_MAX) return fail(CSA_ERR_UNSUPPORTED, "rows beyond one launch");
    if ((w == nullptr) != (w_out == nullptr)) return fail(CSA_ERR_INVALID_ARG, "w and w_out go together");
    if (rows == 0) return CSA_OK;
    CSA_TRY(check_ptr(x, "x"));
    CSA_TRY(check_ptr(out, "out"));
    CSA_TRY(check_ptr(scale, "scale"));
    CSA_TRY(check_ptr(w, "w", false));
    CSA_TRY(check_ptr(w_out, "w_out", false));
    CSA_CUDA(quantize_e4m3(x, rows, cols, out, scale, w, w_out, t, (cudaStream_t)stream), "csa_quantize_e4m3");
    return CSA_OK;
}

// ---------------------------------------------------------------- FP8 KV
static int check_kv_fp8(int c, int rope_dims, const char* who) {
    if (rope_dims < 0 || rope_dims % 16 || c % 16 || c - rope_dims < 16 || c > CSA_MAX_HEAD_DIM)
        return fail(CSA_ERR_INVALID_ARG, "%s: c=%d rope_dims=%d (c and rope_dims multiples of 16, at least 16 "
                    "quantised dims, c <= %d)", who, c, rope_dims, CSA_MAX_HEAD_DIM);
    return CSA_OK;
}

int csa_quantize_kv_fp8(const void* kv, int64_t rows, int c, int rope_dims, uint8_t* codes, float* scales,
                        void* rope, void* stream) {
    CSA_TRY(check_kv_fp8(c, rope_dims, "csa_quantize_kv_fp8"));
    if (rows < 0) return fail(CSA_ERR_INVALID_ARG, "csa_quantize_kv_fp8: rows=%lld", (long long)rows);
    if ((rows + 7) / 8 > INT32_MAX) return fail(CSA_ERR_UNSUPPORTED, "rows beyond one launch");
    if (rows == 0) return CSA_OK;
    CSA_TRY(check_ptr(kv, "kv"));
    CSA_TRY(check_ptr(codes, "codes"));
    CSA_TRY(check_ptr(scales, "scales"));
    CSA_TRY(check_ptr(rope, "rope", rope_dims > 0));
    CSA_CUDA(quantize_e4m3(kv, rows, c - rope_dims, codes, scales, nullptr, nullptr, ElemType::BF16,
                           (cudaStream_t)stream, c, rope_dims ? rope : nullptr, rope_dims),
             "csa_quantize_kv_fp8");
    return CSA_OK;
}

static int check_index_fp8(int HI, int cI) {
    CSA_TRY(check_index_shape(HI, cI));
    if (!index_tc_supported(HI, cI, 1, true))
        return fail(CSA_ERR_UNSUPPORTED, "FP8 indexer needs cI a multiple of 128 (<= 256) (cI=%d)", cI);
    return CSA_OK;
}

int csa_index_scores_fp8(const void* qI8, const float* wq, const void* K8, const float* k_scale, const int32_t* pos,
                         const int32_t* seq_of_q, int nq, int n_seq, int HI, int cI, int64_t Nmax, int m,
                         float* scores, void* stream) {
    CSA_TRY(check_index_fp8(HI, cI));
    CSA_TRY(check_rows(nq, "csa_index_scores_fp8"));
    if (nq < 0 || Nmax < 0 || m < 1 || n_seq < 1) return fail(CSA_ERR_INVALID_ARG, "bad nq/n_seq/Nmax/m");
    if (!seq_of_q && n_seq < nq) return fail(CSA_ERR_INVALID_ARG, "seq_of_q is NULL (query t reads sequence t) but n_seq < nq");
    if (Nmax > INT32_MAX) return fail(CSA_ERR_UNSUPPORTED, "Nmax beyond int32 entry indices");
    CSA_TRY(check_cache_rows(n_seq, Nmax));
    if (nq == 0 || Nmax == 0) return CSA_OK;
    CSA_TRY(check_ptr(qI8, "qI8"));
    CSA_TRY(check_ptr(wq, "wq"));
    CSA_TRY(check_ptr(K8, "K8"));
    CSA_TRY(check_ptr(k_scale, "k_scale"));
    CSA_TRY(check_ptr(pos, "pos"));
    CSA_TRY(check_ptr(seq_of_q, "seq_of_q", false));
    CSA_TRY(check_ptr(scores, "scores"));
    QuerySpec qs{seq_of_q, pos, 0, 0};
    CSA_CUDA(index_scores_tc(qI8, wq, K8, qs, nq, n_seq, HI, cI, Nmax, m, scores, Nmax, 1, true, device_status(),
                             (cudaStream_t)stream, k_scale), "csa_index_scores_fp8");
    return CSA_OK;
}

size_t csa_decode_fp8_workspace_size(int B, int64_t Nmax, int H, int c, int HI, int cI, int k) {
    if (B < 0 || Nmax < 0 || k < 1 || H < 1 || c < 1 || HI < 1 || cI < 1) return 0;
    return align256((size_t)B * HI * cI) + 2 * align256((size_t)B * HI * sizeof(float)) +
           index_topk_bytes(B, Nmax, k) + align256((size_t)B * k * sizeof(int32_t)) +
           mqa_workspace_bytes(B, H, c, k, ElemType::BF16);
}

int csa_decode_fp8(const void* qI, const float* w, const void* idx_cache8, const float* idx_scale, const void* q,
                   const void* kv_cache, const int32_t* ctx_len, int B, int64_t Nmax, int m, int H, int c, int HI,
                   int cI, int k, float scale, const float* sink, int flags, void* out, float* lse, int32_t* topk_idx,
                   void* ws, size_t ws_bytes, void* stream) {
    CSA_TRY(check_index_fp8(HI, cI));
    if (flags & ~CSA_SCORES_BF16) return fail(CSA_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
    const bool sbf = (flags & CSA_SCORES_BF16) != 0;
    CSA_TRY(check_attn_shape(H, c));
    CSA_TRY(check_attn_mode(H, c, ElemType::BF16));
    CSA_TRY(check_cache_rows(B, Nmax));
    CSA_TRY(check_k(k));
    CSA_TRY(check_rows(B, "csa_decode_fp8"));
    if (B < 0 || Nmax < 0 || m < 1) return fail(CSA_ERR_INVALID_ARG, "bad B/Nmax/m");
    if (Nmax > INT32_MAX) return fail(CSA_ERR_UNSUPPORTED, "Nmax beyond int32 entry indices");
    if (B == 0) return CSA_OK;
    CSA_TRY(check_ptr(qI, "qI"));
    CSA_TRY(check_ptr(w, "w"));
    CSA_TRY(check_ptr(idx_cache8, "idx_cache8", Nmax > 0));
    CSA_TRY(check_ptr(idx_scale, "idx_scale", Nmax > 0));
    CSA_TRY(check_ptr(q, "q"));
    CSA_TRY(check_ptr(kv_cache, "kv_cache", Nmax > 0));
    CSA_TRY(check_ptr(ctx_len, "ctx_len"));
    CSA_TRY(check_ptr(sink, "sink", false));
    CSA_TRY(check_ptr(out, "out"));
    CSA_TRY(check_ptr(lse, "lse", false));
    CSA_TRY(check_ptr(topk_idx, "topk_idx", false));
    CSA_TRY(check_ws(ws, ws_bytes, csa_decode_fp8_workspace_size(B, Nmax, H, c, HI, cI, k)));
    cudaStream_t st = (cudaStream_t)stream;
    Carve cv(ws);
    void* q8 = cv.take((size_t)B * HI * cI);
    float* qs8 = (float*)cv.take((size_t)B * HI * sizeof(float));
    float* wq = (float*)cv.take((size_t)B * HI * sizeof(float));
    float* sc = (float*)cv.take((size_t)B * Nmax * sizeof(float));
    void* tws = cv.take(topk_workspace_bytes(B, Nmax, k));
    int32_t* sel = (int32_t*)cv.take((size_t)B * k * sizeof(int32_t));
    void* mws = cv.take(mqa_workspace_bytes(B, H, c, k, ElemType::BF16));
    if (topk_idx) sel = topk_idx;
    QuerySpec qs{nullptr, ctx_len, 0, 0};
    CSA_CUDA(quantize_e4m3(qI, (int64_t)B * HI, cI, q8, qs8, w, wq, ElemType::BF16, st), "csa_decode_fp8: quantize q");
    CSA_CUDA(index_scores_tc(q8, wq, idx_cache8, qs, B, B, HI, cI, Nmax, m, sc, Nmax, 1, false, device_status(), st,
                             idx_scale, sbf), "csa_decode_fp8: indexer");
    if (sbf)
        CSA_CUDA(topk_select_bf16(sc, Nmax, ctx_len, m, B, Nmax, k, sel, nullptr, st), "csa_decode_fp8: top-k");
    else
        CSA_CUDA(topk_select(sc, Nmax, ctx_len, m, B, Nmax, k, sel, nullptr, tws, st), "csa_decode_fp8: top-k");
    CSA_CUDA(mqa(q, kv_cache, sel, k, qs, 1, B, B, H, c, Nmax, default_scale(scale, c), sink, out, lse, mws,
                 ElemType::BF16, st), "csa_decode_fp8: mqa");
    return CSA_OK;
}

// ---------------------------------------------------------------- a6 / a7
size_t csa_sparse_mqa_workspace_size(int nq, int H, int c, int k, int dtype) {
    ElemType t = dtype == CSA_FP32 ? ElemType::F32 : ElemType::BF16;
    if (nq < 0 || H < 1 || c < 1 || k < 1) return 0;
    return mqa_workspace_bytes(nq, H, c, k, t);
}

int csa_sparse_mqa(const void* q, const void* KV, const int32_t* idx, const int32_t* seq_of_q,
                   int nq, int n_seq, int H, int c, int64_t Nmax, int k, float scale, const float* sink,
                   void* out, float* lse, void* ws, size_t ws_bytes, int dtype, void* stream) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_attn_shape(H, c));
    CSA_TRY(check_attn_mode(H, c, t));
    CSA_TRY(check_cache_rows(n_seq, Nmax));
    CSA_TRY(check_k(k));
    CSA_TRY(check_rows(nq, "csa_sparse_mqa"));
    if (nq < 0 || Nmax < 0 || n_seq < 1) return fail(CSA_ERR_INVALID_ARG, "bad nq/n_seq/Nmax");
    if (!seq_of_q && n_seq < nq) return fail(CSA_ERR_INVALID_ARG, "seq_of_q is NULL (query t reads sequence t) but n_seq < nq");
    if (nq == 0) return CSA_OK;
    CSA_TRY(check_ptr(q, "q"));
    CSA_TRY(check_ptr(KV, "KV", Nmax > 0));
    CSA_TRY(check_ptr(idx, "idx"));
    CSA_TRY(check_ptr(seq_of_q, "seq_of_q", false));
    CSA_TRY(check_ptr(sink, "sink", false));
    CSA_TRY(check_ptr(out, "out"));
    CSA_TRY(check_ptr(lse, "lse", false));
    CSA_TRY(check_ws(ws, ws_bytes, mqa_workspace_bytes(nq, H, c, k, t)));
    QuerySpec qs{seq_of_q, nullptr, 0, 0};
    CSA_CUDA(mqa(q, KV, idx, k, qs, 1, nq, n_seq, H, c, Nmax, default_scale(scale, c), sink, out, lse, ws, t,
                 (cudaStream_t)stream), "csa_sparse_mqa");
    return CSA_OK;
}

size_t hca_dense_mqa_workspace_size(int nq, int H, int c, int64_t Nmax, int dtype) {
    ElemType t = dtype == CSA_FP32 ? ElemType::F32 : ElemType::BF16;
    if (nq < 0 || H < 1 || c < 1 || Nmax < 0) return 0;
    return mqa_workspace_bytes(nq, H, c, Nmax, t);
}

static int hca_dense_mqa_impl(const void* q, const void* KV, const int32_t* pos, const int32_t* seq_of_q,
                              int nq, int n_seq, int H, int c, int64_t Nmax, int mp, float scale, const float* sink,
                              void* out, float* lse, void* ws, size_t ws_bytes, int dtype, void* stream,
                              RowBlocks kvb) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_attn_shape(H, c));
    CSA_TRY(check_attn_mode(H, c, t));
    CSA_TRY(check_cache_rows(n_seq, Nmax));
    CSA_TRY(check_rows(nq, "hca_dense_mqa"));
    if (nq < 0 || Nmax < 0 || mp < 1 || n_seq < 1) return fail(CSA_ERR_INVALID_ARG, "bad nq/n_seq/Nmax/mp");
    if (!seq_of_q && n_seq < nq) return fail(CSA_ERR_INVALID_ARG, "seq_of_q is NULL (query t reads sequence t) but n_seq < nq");
    if (Nmax > INT32_MAX) return fail(CSA_ERR_UNSUPPORTED, "Nmax beyond int32 entry indices");
    if (nq == 0) return CSA_OK;
    CSA_TRY(check_ptr(q, "q"));
    CSA_TRY(check_ptr(KV, "KV", Nmax > 0));
    CSA_TRY(check_ptr(pos, "pos"));
    CSA_TRY(check_ptr(seq_of_q, "seq_of_q", false));
    CSA_TRY(check_ptr(sink, "sink", false));
    CSA_TRY(check_ptr(out, "out"));
    CSA_TRY(check_ptr(lse, "lse", false));
    CSA_TRY(check_ws(ws, ws_bytes, mqa_workspace_bytes(nq, H, c, Nmax, t)));
    QuerySpec qs{seq_of_q, pos, 0, 0};
    CSA_CUDA(mqa(q, KV, nullptr, 0, qs, mp, nq, n_seq, H, c, Nmax, default_scale(scale, c), sink, out, lse, ws,
                 t, (cudaStream_t)stream, kvb), "hca_dense_mqa");
    return CSA_OK;
}

int hca_dense_mqa(const void* q, const void* KV, const int32_t* pos, const int32_t* seq_of_q,
                  int nq, int n_seq, int H, int c, int64_t Nmax, int mp, float scale, const float* sink,
                  void* out, float* lse, void* ws, size_t ws_bytes, int dtype, void* stream) {
    return hca_dense_mqa_impl(q, KV, pos, seq_of_q, nq, n_seq, H, c, Nmax, mp, scale, sink, out, lse, ws, ws_bytes,
                              dtype, stream, RowBlocks{0, 0});
}

// ---------------------------------------------------------------- fused
size_t csa_decode_workspace_size(int B, int64_t Nmax, int H, int c, int HI, int cI, int k, int dtype) {
    (void)HI; (void)cI;
    ElemType t = dtype == CSA_FP32 ? ElemType::F32 : ElemType::BF16;
    if (B < 0 || Nmax < 0 || k < 1 || H < 1 || c < 1) return 0;
    return select_bytes(B, Nmax, k) + align256((size_t)B * k * sizeof(int32_t)) + mqa_workspace_bytes(B, H, c, k, t);
}

static int csa_decode_impl(const void* qI, const float* w, const void* idx_cache, const void* q,
                           const void* kv_cache, const int32_t* ctx_len, int B, int64_t Nmax, int m, int H,
                           int c, int HI, int cI, int k, float scale, const float* sink, void* out, float* lse,
                           int32_t* topk_idx, void* ws, size_t ws_bytes, int dtype, void* stream, RowBlocks cb) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_index_shape(HI, cI));
    CSA_TRY(check_index_mode(HI, cI, t));
    CSA_TRY(check_attn_shape(H, c));
    CSA_TRY(check_attn_mode(H, c, t));
    CSA_TRY(check_cache_rows(B, Nmax));
    CSA_TRY(check_k(k));
    CSA_TRY(check_rows(B, "csa_decode"));
    if (B < 0 || Nmax < 0 || m < 1) return fail(CSA_ERR_INVALID_ARG, "bad B/Nmax/m");
    if (Nmax > INT32_MAX) return fail(CSA_ERR_UNSUPPORTED, "Nmax beyond int32 entry indices");
    if (B == 0) return CSA_OK;
    CSA_TRY(check_ptr(qI, "qI"));
    CSA_TRY(check_ptr(w, "w"));
    CSA_TRY(check_ptr(idx_cache, "idx_cache", Nmax > 0));
    CSA_TRY(check_ptr(q, "q"));
    CSA_TRY(check_ptr(kv_cache, "kv_cache", Nmax > 0));
    CSA_TRY(check_ptr(ctx_len, "ctx_len"));
    CSA_TRY(check_ptr(sink, "sink", false));
    CSA_TRY(check_ptr(out, "out"));
    CSA_TRY(check_ptr(lse, "lse", false));
    CSA_TRY(check_ptr(topk_idx, "topk_idx", false));
    CSA_TRY(check_ws(ws, ws_bytes, csa_decode_workspace_size(B, Nmax, H, c, HI, cI, k, dtype)));
    cudaStream_t st = (cudaStream_t)stream;
    Carve cv(ws);
    void* blk = cv.take(select_bytes(B, Nmax, k));
    int32_t* sel = (int32_t*)cv.take((size_t)B * k * sizeof(int32_t));
    void* mws = cv.take(mqa_workspace_bytes(B, H, c, k, t));
    if (topk_idx) sel = topk_idx;
    QuerySpec qs{nullptr, ctx_len, 0, 0};
    const char* step = "indexer";
    const cudaError_t se = index_then_select(qI, w, idx_cache, qs, B, B, HI, cI, Nmax, m, 1, k, sel, blk, t, st, cb,
                                             step);
    if (se != cudaSuccess) return fail(CSA_ERR_CUDA, "csa_decode: %s: %s", step, cudaGetErrorString(se));
    CSA_CUDA(mqa(q, kv_cache, sel, k, qs, 1, B, B, H, c, Nmax, default_scale(scale, c), sink, out, lse, mws, t, st,
                 cb),
             "csa_decode: mqa");
    return CSA_OK;
}

int csa_decode(const void* qI, const float* w, const void* idx_cache, const void* q,
               const void* kv_cache, const int32_t* ctx_len, int B, int64_t Nmax, int m, int H,
               int c, int HI, int cI, int k, float scale, const float* sink, void* out, float* lse,
               int32_t* topk_idx, void* ws, size_t ws_bytes, int dtype, void* stream) {
    return csa_decode_impl(qI, w, idx_cache, q, kv_cache, ctx_len, B, Nmax, m, H, c, HI, cI, k, scale, sink, out, lse,
                           topk_idx, ws, ws_bytes, dtype, stream, RowBlocks{0, 0});
}

int csa_decode_blocked(const void* qI, const float* w, const void* idx_cache, const void* q, const void* kv_cache,
                       const int32_t* ctx_len, int B, int64_t Nmax, int m, int H, int c, int HI, int cI, int k,
                       float scale, const float* sink, void* out, float* lse, int32_t* topk_idx, int rows_per_block,
                       int64_t block_bytes, void* ws, size_t ws_bytes, int dtype, void* stream) {
    CSA_TRY(check_blocks(rows_per_block, block_bytes, Nmax, c, kv_cache, dtype, "csa_decode_blocked"));
    CSA_TRY(check_blocks(rows_per_block, block_bytes, Nmax, cI, idx_cache, dtype, "csa_decode_blocked"));
    if (128 % rows_per_block)
        return fail(CSA_ERR_UNSUPPORTED, "csa_decode_blocked: rows_per_block=%d must divide the indexer's 128-key tile",
                    rows_per_block);
    return csa_decode_impl(qI, w, idx_cache, q, kv_cache, ctx_len, B, Nmax, m, H, c, HI, cI, k, scale, sink, out, lse,
                           topk_idx, ws, ws_bytes, dtype, stream, RowBlocks{rows_per_block, block_bytes});
}

size_t hca_decode_workspace_size(int B, int64_t Nmax, int H, int c, int dtype) {
    return hca_dense_mqa_workspace_size(B, H, c, Nmax, dtype);
}

size_t csa_decode_fp8kv_workspace_size(int B, int64_t Nmax, int H, int c, int HI, int cI, int k) {
    (void)HI; (void)cI;
    if (B < 0 || Nmax < 0 || k < 1 || H < 1 || c < 1) return 0;
    return select_bytes(B, Nmax, k) + align256((size_t)B * k * sizeof(int32_t)) +
           align256((size_t)B * k * c * sizeof(uint16_t)) + align256((size_t)B * k * sizeof(int32_t)) +
           mqa_workspace_bytes(B, H, c, k, ElemType::BF16);
}

int csa_decode_fp8kv(const void* qI, const float* w, const void* idx_cache, const void* q, const uint8_t* kv_codes,
                     const float* kv_scales, const void* kv_rope, const int32_t* ctx_len, int B, int64_t Nmax, int m,
                     int H, int c, int rope_dims, int HI, int cI, int k, float scale, const float* sink, void* out,
                     float* lse, int32_t* topk_idx, void* ws, size_t ws_bytes, void* stream) {
    CSA_TRY(check_kv_fp8(c, rope_dims, "csa_decode_fp8kv"));
    CSA_TRY(check_index_shape(HI, cI));
    CSA_TRY(check_index_mode(HI, cI, ElemType::BF16));
    CSA_TRY(check_attn_shape(H, c));
    CSA_TRY(check_attn_mode(H, c, ElemType::BF16));
    CSA_TRY(check_cache_rows(B, Nmax));
    CSA_TRY(check_k(k));
    CSA_TRY(check_rows(B, "csa_decode_fp8kv"));
    if (B < 0 || Nmax < 0 || m < 1) return fail(CSA_ERR_INVALID_ARG, "bad B/Nmax/m");
    if (Nmax > INT32_MAX) return fail(CSA_ERR_UNSUPPORTED, "Nmax beyond int32 entry indices");
    if (B == 0) return CSA_OK;
    CSA_TRY(check_ptr(qI, "qI"));
    CSA_TRY(check_ptr(w, "w"));
    CSA_TRY(check_ptr(idx_cache, "idx_cache", Nmax > 0));
    CSA_TRY(check_ptr(q, "q"));
    CSA_TRY(check_ptr(kv_codes, "kv_codes", Nmax > 0));
    CSA_TRY(check_ptr(kv_scales, "kv_scales", Nmax > 0));
    CSA_TRY(check_ptr(kv_rope, "kv_rope", Nmax > 0 && rope_dims > 0));
    CSA_TRY(check_ptr(ctx_len, "ctx_len"));
    CSA_TRY(check_ptr(sink, "sink", false));
    CSA_TRY(check_ptr(out, "out"));
    CSA_TRY(check_ptr(lse, "lse", false));
    CSA_TRY(check_ptr(topk_idx, "topk_idx", false));
    CSA_TRY(check_ws(ws, ws_bytes, csa_decode_fp8kv_workspace_size(B, Nmax, H, c, HI, cI, k)));
    cudaStream_t st = (cudaStream_t)stream;
    const ElemType t = ElemType::BF16;
    Carve cv(ws);
    void* blk = cv.take(select_bytes(B, Nmax, k));
    int32_t* sel = (int32_t*)cv.take((size_t)B * k * sizeof(int32_t));
    void* rows = cv.take((size_t)B * k * c * sizeof(uint16_t));
    int32_t* slots = (int32_t*)cv.take((size_t)B * k * sizeof(int32_t));
    void* mws = cv.take(mqa_workspace_bytes(B, H, c, k, t));
    if (topk_idx) sel = topk_idx;
    QuerySpec qs{nullptr, ctx_len, 0, 0};
    const char* step = "indexer";
    const cudaError_t se = index_then_select(qI, w, idx_cache, qs, B, B, HI, cI, Nmax, m, 1, k, sel, blk, t, st,
                                             RowBlocks{0, 0}, step);
    if (se != cudaSuccess) return fail(CSA_ERR_CUDA, "csa_decode_fp8kv: %s: %s", step, cudaGetErrorString(se));
    // the selected entries, dequantised into one row list per query; the
    // attention then runs on those rows (query t over "sequence" t of k rows)
    CSA_CUDA(gather_kv_fp8(kv_codes, kv_scales, kv_rope, sel, B, k, Nmax, c, rope_dims, rows, slots, st),
             "csa_decode_fp8kv: dequantise the selection");
    QuerySpec qs_rows{nullptr, ctx_len, 0, 0};
    CSA_CUDA(mqa(q, rows, slots, k, qs_rows, 1, B, B, H, c, k, default_scale(scale, c), sink, out, lse, mws, t, st),
             "csa_decode_fp8kv: mqa");
    return CSA_OK;
}

int hca_decode(const void* q, const void* kv_cache, const int32_t* ctx_len, int B, int64_t Nmax,
               int mp, int H, int c, float scale, const float* sink, void* out, float* lse,
               void* ws, size_t ws_bytes, int dtype, void* stream) {
    return hca_dense_mqa(q, kv_cache, ctx_len, nullptr, B, B, H, c, Nmax, mp, scale, sink, out, lse, ws,
                         ws_bytes, dtype, stream);
}

int hca_decode_blocked(const void* q, const void* kv_cache, const int32_t* ctx_len, int B, int64_t Nmax, int mp,
                       int H, int c, float scale, const float* sink, void* out, float* lse, int rows_per_block,
                       int64_t block_bytes, void* ws, size_t ws_bytes, int dtype, void* stream) {
    CSA_TRY(check_blocks(rows_per_block, block_bytes, Nmax, c, kv_cache, dtype, "hca_decode_blocked"));
    if (rows_per_block != 1)
        return fail(CSA_ERR_UNSUPPORTED, "hca_decode_blocked: one HCA entry per block (rows_per_block=%d)",
                    rows_per_block);
    return hca_dense_mqa_impl(q, kv_cache, ctx_len, nullptr, B, B, H, c, Nmax, mp, scale, sink, out, lse, ws, ws_bytes,
                              dtype, stream, RowBlocks{rows_per_block, block_bytes});
}

size_t csa_prefill_workspace_size(int64_t n, int64_t Nmax, int d, int m, int c, int cI, int H,
                                  int HI, int k, int dtype) {
    (void)d; (void)HI;
    ElemType t = dtype == CSA_FP32 ? ElemType::F32 : ElemType::BF16;
    if (n < 0 || Nmax < 0 || m < 1 || c < 1 || cI < 1 || k < 1) return 0;
    const int cw = c > cI ? c : cI;
    int64_t qc = prefill_query_chunk(n, Nmax, m);
    size_t b = align256((size_t)n * 4 * cw * sizeof(float)) + align256((size_t)m * 4 * cw * sizeof(float));
    b += select_bytes((int)qc, Nmax, k) + align256((size_t)qc * k * sizeof(int32_t));
    b += mqa_workspace_bytes((int)qc, H, c, k, t);
    return b;
}

int csa_prefill(const void* x, const void* x_left, const void* W_kv, const float* B_kv,
                const void* W_idx, const float* B_idx, int64_t start, int64_t n, int d, int m,
                int c, int cI, void* kv_cache, void* idx_cache, int64_t Nmax, float* state_kv,
                float* state_idx, const void* qI, const float* w, const void* q, int H, int HI, int k,
                float scale, const float* sink, void* out, float* lse, int32_t* topk_idx, void* ws,
                size_t ws_bytes, int dtype, void* stream) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_index_shape(HI, cI));
    CSA_TRY(check_index_mode(HI, cI, t));
    CSA_TRY(check_attn_shape(H, c));
    CSA_TRY(check_attn_mode(H, c, t));
    CSA_TRY(check_k(k));
    const bool stateful = state_kv || state_idx;
    if (stateful && !(state_kv && state_idx))
        return fail(CSA_ERR_INVALID_ARG, "state_kv and state_idx go together (both or neither)");
    // no weights: the chunk's entries are already in the caches (compressed
    // elsewhere, e.g. gathered from the ranks that own them); attend only
    const bool attend_only = !W_kv && !W_idx;
    if (attend_only && stateful)
        return fail(CSA_ERR_INVALID_ARG, "state rings given without compressor weights");
    CSA_TRY(check_compress(stateful ? 0 : n, c, m, 64, "csa_prefill"));
    if (n < 0) return fail(CSA_ERR_INVALID_ARG, "n=%lld is negative", (long long)n);
    if (d < 8 || d % 8) return fail(CSA_ERR_INVALID_ARG, "d=%d must be a positive multiple of 8", d);
    if (start < 0) return fail(CSA_ERR_INVALID_ARG, "start=%lld is negative", (long long)start);
    if (!stateful && !attend_only && start % m)
        return fail(CSA_ERR_INVALID_ARG, "start=%lld is not a multiple of m (pass the state rings to start "
                    "mid-block)", (long long)start);
    if (!stateful && !attend_only && start > 0 && !x_left)
        return fail(CSA_ERR_INVALID_ARG, "x_left is required when start > 0 (or pass the state rings)");
    if ((start + n) / m > Nmax) return fail(CSA_ERR_INVALID_ARG, "caches hold %lld entries, %lld needed",
                                            (long long)Nmax, (long long)((start + n) / m));
    if (Nmax > INT32_MAX || start + n > INT32_MAX) return fail(CSA_ERR_UNSUPPORTED, "positions beyond int32");
    if (n == 0) return CSA_OK;
    CSA_TRY(check_ptr(x, "x", !attend_only));
    CSA_TRY(check_ptr(x_left, "x_left", false));
    CSA_TRY(check_ptr(W_kv, "W_kv", !attend_only));
    CSA_TRY(check_ptr(B_kv, "B_kv", !attend_only));
    CSA_TRY(check_ptr(W_idx, "W_idx", !attend_only));
    CSA_TRY(check_ptr(B_idx, "B_idx", !attend_only));
    if (attend_only != (!W_kv || !W_idx))
        return fail(CSA_ERR_INVALID_ARG, "W_kv and W_idx go together (both, or neither to attend only)");
    CSA_TRY(check_ptr(kv_cache, "kv_cache"));
    CSA_TRY(check_ptr(idx_cache, "idx_cache"));
    CSA_TRY(check_ptr(state_kv, "state_kv", false));
    CSA_TRY(check_ptr(state_idx, "state_idx", false));
    CSA_TRY(check_ptr(qI, "qI"));
    CSA_TRY(check_ptr(w, "w"));
    CSA_TRY(check_ptr(q, "q"));
    CSA_TRY(check_ptr(sink, "sink", false));
    CSA_TRY(check_ptr(out, "out"));
    CSA_TRY(check_ptr(lse, "lse", false));
    CSA_TRY(check_ptr(topk_idx, "topk_idx", false));
    CSA_TRY(check_ws(ws, ws_bytes, csa_prefill_workspace_size(n, Nmax, d, m, c, cI, H, HI, k, dtype)));
    cudaStream_t st = (cudaStream_t)stream;
    const size_t es = elem_size(t);
    const int cw = c > cI ? c : cI;
    const int64_t qc = prefill_query_chunk(n, Nmax, m);
    Carve cv(ws);
    float* proj = (float*)cv.take((size_t)n * 4 * cw * sizeof(float));
    float* lproj = (float*)cv.take((size_t)m * 4 * cw * sizeof(float));
    void* blk = cv.take(select_bytes((int)qc, Nmax, k));
    int32_t* sel_ws = (int32_t*)cv.take((size_t)qc * k * sizeof(int32_t));
    void* mws = cv.take(mqa_workspace_bytes((int)qc, H, c, k, t));

    // 1-2. compress the chunk into both caches: aligned chunks from their own
    // rows and the m rows before (entries start/m ..); with the state rings,
    // any chunk: every block that ends inside it, earlier window tokens from
    // the ring, which then keeps the chunk's last 2m projected rows
    const int64_t e0 = start / m;
    struct { const void* W; const float* B; int cc; void* cache; float* state; } streams[2] = {
        {W_kv, B_kv, c, kv_cache, state_kv}, {W_idx, B_idx, cI, idx_cache, state_idx}};
    for (auto& s : streams) {
        if (attend_only) break;
        CSA_CUDA(project(x, s.W, n, d, 4 * s.cc, proj, t, st), "csa_prefill: projection");
        if (stateful) {
            CSA_CUDA(compress_chunk_state(proj, s.state, s.B, start, n, s.cc, m, true, s.cache, t, st),
                     "csa_prefill: compress");
            continue;
        }
        if (start > 0) CSA_CUDA(project(x_left, s.W, m, d, 4 * s.cc, lproj, t, st), "csa_prefill: left projection");
        CSA_CUDA(compress_csa(proj, start > 0 ? lproj : nullptr, s.B, n, s.cc, m,
                              (char*)s.cache + (size_t)e0 * s.cc * es, ElemType::F32, t, st),
                 "csa_prefill: compress");
    }
    // 3. indexer -> top-k -> sparse MQA per query chunk; a chunk that starts
    // mid-block first takes the queries up to the next block boundary alone
    const float sc_scale = default_scale(scale, c);
    const int64_t head = (m - start % m) % m;
    for (int64_t q0 = 0; q0 < n;) {
        const int64_t span = (q0 == 0 && head > 0) ? head : qc;
        const int nqc = (int)((n - q0) < span ? (n - q0) : span);
        QuerySpec qs{nullptr, nullptr, start + q0, 1};
        int32_t* sel = topk_idx ? topk_idx + q0 * k : sel_ws;
        // the m tokens of one compressed block see the same entries: score them
        // together against each key tile when the group fits one MMA (the
        // group starts on a block boundary)
        const int group = (m <= 4 && (start + q0) % m == 0 && index_tc_supported(HI, cI, m)) ? m : 1;
        // the visible count of query t is floor((start + q0 + t) / m)
        const char* step = "indexer";
        const cudaError_t se = index_then_select((const char*)qI + (size_t)q0 * HI * cI * es, w + q0 * HI, idx_cache,
                                                 qs, nqc, 1, HI, cI, Nmax, m, group, k, sel, blk, t, st,
                                                 RowBlocks{0, 0}, step);
        if (se != cudaSuccess) return fail(CSA_ERR_CUDA, "csa_prefill: %s: %s", step, cudaGetErrorString(se));
        CSA_CUDA(mqa((const char*)q + (size_t)q0 * H * c * es, kv_cache, sel, k, qs, 1, nqc, 1, H, c, Nmax,
                     sc_scale, sink, (char*)out + (size_t)q0 * H * c * es, lse ? lse + q0 * H : nullptr, mws,
                     t, st), "csa_prefill: mqa");
        q0 += nqc;
    }
    return CSA_OK;
}

// ---------------------------------------------------------------- attention output completion
static int check_norm_rope(int c, int rope_dims, float rope_base, float eps) {
    if (!norm_rope_supported(c, rope_dims))
        return fail(CSA_ERR_UNSUPPORTED, "norm/rotary needs c a multiple of 8 in [8, %d] and rope_dims a multiple "
                    "of 8 in [0, c] (c=%d rope_dims=%d)", CSA_MAX_HEAD_DIM, c, rope_dims);
    if (rope_dims > 0 && !(rope_base > 0.f)) return fail(CSA_ERR_INVALID_ARG, "rope_base must be positive");
    if (!(eps >= 0.f)) return fail(CSA_ERR_INVALID_ARG, "eps must be non-negative");
    return CSA_OK;
}

static int check_window(int n_win, int64_t ring_off, int64_t ring_len) {
    if (n_win < 0) return fail(CSA_ERR_INVALID_ARG, "n_win=%d is negative", n_win);
    if (n_win > 0 && ring_len < n_win)
        return fail(CSA_ERR_INVALID_ARG, "the window ring (%lld rows) is shorter than the window (%d)",
                    (long long)ring_len, n_win);
    if (ring_off < 0 || ring_off + ring_len > INT32_MAX)
        return fail(CSA_ERR_UNSUPPORTED, "window ring rows beyond int32 entry indices");
    return CSA_OK;
}

int csa_norm_rope(const void* x, void* y, int64_t rows, int group, int c, const float* gamma, float eps,
                  int rope_dims, float rope_base, const int32_t* pos, int64_t pos0, int64_t pos_step, int inverse,
                  int dtype, void* stream) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_norm_rope(c, rope_dims, rope_base, eps));
    if (rows < 0 || group < 1 || rows % group)
        return fail(CSA_ERR_INVALID_ARG, "rows=%lld must be a non-negative multiple of group=%d", (long long)rows, group);
    if ((rows + 15) / 16 > INT32_MAX) return fail(CSA_ERR_UNSUPPORTED, "rows=%lld beyond one launch", (long long)rows);
    if (rows == 0) return CSA_OK;
    CSA_TRY(check_ptr(x, "x"));
    CSA_TRY(check_ptr(y, "y"));
    CSA_TRY(check_ptr(gamma, "gamma", false));
    CSA_TRY(check_ptr(pos, "pos", false));
    if (x != y && (const char*)x < (const char*)y + rows * c * elem_size(t) &&
        (const char*)y < (const char*)x + rows * c * elem_size(t))
        return fail(CSA_ERR_INVALID_ARG, "x and y overlap without being the same array");
    CSA_CUDA(norm_rope(x, y, rows, group, c, gamma, eps, rope_dims, (double)rope_base, pos, pos0, pos_step,
                       inverse ? 1 : 0, t, (cudaStream_t)stream), "csa_norm_rope");
    return CSA_OK;
}

int csa_window_entries(const int32_t* sel, int k, const int32_t* pos, int64_t pos0, int nq, int n_win,
                       int64_t ring_off, int64_t ring_len, int32_t* ent, void* stream) {
    CSA_TRY(check_window(n_win, ring_off, ring_len));
    if (nq < 0 || k < 0) return fail(CSA_ERR_INVALID_ARG, "bad nq/k");
    if ((int64_t)k + n_win > INT32_MAX / 2) return fail(CSA_ERR_UNSUPPORTED, "entry list too wide");
    if (((int64_t)nq * ((int64_t)k + n_win) + 255) / 256 > INT32_MAX)
        return fail(CSA_ERR_UNSUPPORTED, "entry lists beyond one launch");
    if (nq == 0 || k + n_win == 0) return CSA_OK;
    CSA_TRY(check_ptr(sel, "sel", k > 0));
    CSA_TRY(check_ptr(pos, "pos", false));
    CSA_TRY(check_ptr(ent, "ent"));
    if (sel && sel == ent) return fail(CSA_ERR_INVALID_ARG, "ent must not be the selection array");
    CSA_CUDA(window_entries(sel, k, pos, pos0, nq, n_win, ring_off, ring_len, ent, (cudaStream_t)stream),
             "csa_window_entries");
    return CSA_OK;
}

size_t csa_attend_decode_workspace_size(int B, int64_t Nmax, int64_t ring_len, int n_win, int H, int c, int HI,
                                        int cI, int k, int dtype) {
    (void)HI; (void)cI; (void)ring_len;
    ElemType t = dtype == CSA_FP32 ? ElemType::F32 : ElemType::BF16;
    if (B < 0 || Nmax < 0 || k < 1 || n_win < 0 || H < 1 || c < 1) return 0;
    const int ke = k + n_win;
    return select_bytes(B, Nmax, k) + align256((size_t)B * k * sizeof(int32_t)) +
           align256((size_t)B * ke * sizeof(int32_t)) + align256((size_t)B * H * c * elem_size(t)) +
           mqa_workspace_bytes(B, H, c, ke, t);
}

int csa_attend_decode(const void* qI, const float* w, const void* idx_cache, const void* q, const void* kv_cache,
                      const int32_t* ctx_len, int B, int64_t Nmax, int64_t ring_len, int n_win, int m, int H, int c,
                      int HI, int cI, int k, float scale, const float* q_gamma, float eps, int rope_dims,
                      float rope_base, const float* sink, void* out, float* lse, int32_t* topk_idx, void* ws,
                      size_t ws_bytes, int dtype, void* stream) {
    ElemType t = ElemType::BF16;   // set by check_dtype
    CSA_TRY(check_dtype(dtype, &t));
    CSA_TRY(check_index_shape(HI, cI));
    CSA_TRY(check_index_mode(HI, cI, t));
    CSA_TRY(check_attn_shape(H, c));
    CSA_TRY(check_attn_mode(H, c, t));
    CSA_TRY(check_norm_rope(c, rope_dims, rope_base, eps));
    CSA_TRY(check_k(k));
    CSA_TRY(check_rows(B, "csa_attend_decode"));
    if (B < 0 || Nmax < 0 || m < 1 || ring_len < 0) return fail(CSA_ERR_INVALID_ARG, "bad B/Nmax/m/ring_len");
    CSA_TRY(check_window(n_win, Nmax, ring_len));
    if (k + n_win > CSA_MAX_TOPK)
        return fail(CSA_ERR_UNSUPPORTED, "k + n_win = %d beyond %d entries per query", k + n_win, CSA_MAX_TOPK);
    const int64_t rows = Nmax + ring_len;   // cache rows per sequence
    CSA_TRY(check_cache_rows(B, rows));
    if (B == 0) return CSA_OK;
    CSA_TRY(check_ptr(qI, "qI"));
    CSA_TRY(check_ptr(w, "w"));
    CSA_TRY(check_ptr(idx_cache, "idx_cache", Nmax > 0));
    CSA_TRY(check_ptr(q, "q"));
    CSA_TRY(check_ptr(kv_cache, "kv_cache", rows > 0));
    CSA_TRY(check_ptr(ctx_len, "ctx_len"));
    CSA_TRY(check_ptr(q_gamma, "q_gamma", false));
    CSA_TRY(check_ptr(sink, "sink", false));
    CSA_TRY(check_ptr(out, "out"));
    CSA_TRY(check_ptr(lse, "lse", false));
    CSA_TRY(check_ptr(topk_idx, "topk_idx", false));
    CSA_TRY(check_ws(ws, ws_bytes,
                     csa_attend_decode_workspace_size(B, Nmax, ring_len, n_win, H, c, HI, cI, k, dtype)));
    cudaStream_t st = (cudaStream_t)stream;
    const int ke = k + n_win;
    Carve cv(ws);
    void* blk = cv.take(select_bytes(B, Nmax, k));
    int32_t* sel = (int32_t*)cv.take((size_t)B * k * sizeof(int32_t));
    int32_t* ent = (int32_t*)cv.take((size_t)B * ke * sizeof(int32_t));
    void* qn = cv.take((size_t)B * H * c * elem_size(t));
    void* mws = cv.take(mqa_workspace_bytes(B, H, c, ke, t));
    if (topk_idx) sel = topk_idx;
    const bool prep_q = q_gamma || rope_dims > 0;
    QuerySpec qs{nullptr, ctx_len, 0, 0};
    if (prep_q)
        CSA_CUDA(norm_rope(q, qn, (int64_t)B * H, H, c, q_gamma, eps, rope_dims, (double)rope_base, ctx_len, 0, 0, 0,
                           t, st), "csa_attend_decode: query norm/rotary");
    const char* step = "indexer";
    const cudaError_t se = index_then_select(qI, w, idx_cache, qs, B, B, HI, cI, Nmax, m, 1, k, sel, blk, t, st,
                                             RowBlocks{0, 0}, step);
    if (se != cudaSuccess) return fail(CSA_ERR_CUDA, "csa_attend_decode: %s: %s", step, cudaGetErrorString(se));
    CSA_CUDA(window_entries(sel, k, ctx_len, 0, B, n_win, Nmax, ring_len > 0 ? ring_len : 1, ent, st),
             "csa_attend_decode: window entries");
    CSA_CUDA(mqa(prep_q ? qn : q, kv_cache, ent, ke, qs, 1, B, B, H, c, rows, default_scale(scale, c), sink, out,
                 lse, mws, t, st), "csa_attend_decode: mqa");
    if (rope_dims > 0)
        CSA_CUDA(norm_rope(out, out, (int64_t)B * H, H, c, nullptr, 0.f, rope_dims, (double)rope_base, ctx_len, 0, 0,
                           1, t, st), "csa_attend_decode: output back-rotation");
    return CSA_OK;
}

}  // extern "C"
