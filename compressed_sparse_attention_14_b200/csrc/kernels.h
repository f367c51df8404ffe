// Internal launchers of libcsa (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "csa.h"

namespace csa {

enum class ElemType { BF16 = 0, F32 = 1 };

// trace.cu: launch accounting and optional per-kernel event timing. Every
// kernel launch goes through CSA_LAUNCH(stream, "name", kernel<<<...>>>(...)).
int trace_begin(cudaStream_t st);
void trace_end(int token, cudaStream_t st, const char* name);
uint64_t launch_count();
void trace_enable(int on);
int trace_read(int max_kernels, char* names, double* total_ms, int* counts, int* n_out);

#define CSA_LAUNCH(st, name, ...)                  \
    do {                                           \
        int _csa_tok = ::csa::trace_begin(st);     \
        __VA_ARGS__;                               \
        ::csa::trace_end(_csa_tok, st, name);      \
    } while (0)

// Launch `kern` with programmatic dependent launch allowed (the kernel must
// call pdl_wait() before touching global memory) and, when cluster_x > 0,
// as clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       unsigned cluster_x, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_x > 0) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// launch.cu: raise `kern`'s dynamic shared-memory ceiling to the device's
// opt-in maximum, once per (kernel, device); thread-safe. Every launcher calls
// this instead of setting the attribute to its own size per call, which would
// race with calls on other host threads.
cudaError_t smem_ceiling(const void* kern);
template <typename... KArgs>
cudaError_t smem_ceiling(void (*kern)(KArgs...)) {
    return smem_ceiling(reinterpret_cast<const void*>(kern));
}

// launch.cu: the failure-path test hooks set by csa_debug_set (0 = off).
uint32_t debug_wait_limit();
uint32_t debug_flags();

inline size_t elem_size(ElemType t) { return t == ElemType::BF16 ? 2 : 4; }
inline size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

// Query -> (sequence, position) description passed to attention launchers.
struct QuerySpec {
    const int32_t* seq;   // nullable
    const int32_t* pos;   // nullable: then pos = pos_base + t
    int64_t pos_base;
    int single_seq;
};

// Where row R of a cache lives (R = sequence * Nmax + entry). rpb == 0: a
// contiguous [rows, width] matrix. rpb > 0: rows come in blocks of rpb, block
// j at j * block_bytes from the cache pointer (the other parts of a block,
// such as the other cache types of the same raw tokens, lie between them).
struct RowBlocks {
    int rpb;
    int64_t block_bytes;
};
__host__ __device__ __forceinline__ int64_t row_byte_offset(int64_t R, int64_t row_bytes, RowBlocks L) {
    return L.rpb ? (R / L.rpb) * L.block_bytes + (R % L.rpb) * row_bytes : R * row_bytes;
}

// api.cu: record the thread's last error message (csa_last_error) and
// return `code`.
int set_last_error(int code, const char* fmt, ...);

// compress.cu
cudaError_t compress_csa(const void* proj, const void* left, const float* bias, int64_t n, int c,
                         int m, void* out, ElemType in_t, ElemType out_t, cudaStream_t st);
cudaError_t compress_hca(const void* proj, const float* bias, int64_t n, int c, int mp, void* out,
                         ElemType in_t, ElemType out_t, cudaStream_t st);

// compress.cu, decode time: store the newest token's projected row of each
// sequence in its state ring (2m rows of [C^a|C^b|Z^a|Z^b] when overlap, m
// rows of [C|Z] otherwise) and write the entry of a block the token closes.
// proj_new may hold nsplit partial sums (slice s at proj_new + s * B * row
// width), added in slice order.
cudaError_t compress_step(const float* proj_new, float* state, const float* bias, const int32_t* pos, int B, int c,
                          int m, bool overlap, int64_t Nmax, void* cache, ElemType out_t, cudaStream_t st,
                          int nsplit = 1, RowBlocks cb = RowBlocks{0, 0});
// One CSA compressor stream of a decode step: proj holds nsplit partial sums
// [B, 4c] fp32, slice s at proj + s * pstride; state [B, 2m, 4c]; bias [2m, c];
// cache [B, Nmax, c] of the output type.
struct StepStream {
    const float* proj;
    float* state;
    const float* bias;
    void* cache;
    int c, nsplit;
    int64_t pstride;
    RowBlocks cb;   // where the cache's entry rows live
};
// both CSA streams of a decode step (same m, positions and output type) in
// one launch; s1.c == 0 leaves the second out
cudaError_t compress_step_csa2(const StepStream& s0, const StepStream& s1, const int32_t* pos, int B, int m,
                               int64_t Nmax, ElemType out_t, cudaStream_t st);

// compress.cu, chunks at any start and length: the entries of every block
// that ends inside the chunk [start, start+n) (proj rows fp32, one sequence),
// earlier window tokens read from the state ring (2m rows for CSA, m' for
// HCA, slot tau mod ring rows), which is then refreshed with the chunk's last
// tokens. cache is the sequence's [Nmax, c] cache; entry i at row i.
cudaError_t compress_chunk_state(const float* proj, float* state, const float* bias, int64_t start, int64_t n, int c,
                                 int m, bool overlap, void* cache, ElemType out_t, cudaStream_t st);

// gemm.cu: out[n, M] (fp32) = x[n, d] . W[M, d]^T (bf16 -> gemm_tc.cu)
cudaError_t project(const void* x, const void* W, int64_t n, int d, int M, float* out, ElemType t,
                    cudaStream_t st);
// ksplit > 1: the contraction is cut into ksplit slices whose fp32 partial
// sums go to out + s * n * M (out holds ksplit * n * M floats).
cudaError_t project_tc(const void* x, const void* W, int64_t n, int d, int M, float* out, int* status,
                       cudaStream_t st, int ksplit = 1);
// Two projections of the same rows in one launch: x [n, d] times W0 [M0, d]
// into out0 (ks0 K slices) and times W1 [M1, d] into out1 (ks1 slices), each
// laid out as project_tc lays out its output.
cudaError_t project_tc2(const void* x, int64_t n, int d, const void* W0, int M0, float* out0, int ks0, const void* W1,
                        int M1, float* out1, int ks1, int* status, cudaStream_t st);
// K slices for two projections of n rows sharing one launch: the slices of
// the one with the longer weight stream per work item double while the work
// items fit on the SMs and a slice keeps at least 4 blocks of 64
void project_ksplit2(int64_t n, int d, int M0, int M1, int* ks0, int* ks1);

// indexer.cu (FFMA, fp32 mode): scores[t, 0..Nmax) with ld = ld_scores;
// -inf past the visible range (the whole row for a query whose sequence is
// outside [0, n_seq))
cudaError_t index_scores(const void* qI, const float* w, const void* K, QuerySpec qs, int nq, int n_seq,
                         int HI, int cI, int64_t Nmax, int m, float* scores, int64_t ld_scores,
                         ElemType t, cudaStream_t st);
// indexer_tc.cu (tcgen05, bf16): groups of `group` consecutive queries share
// one visible range; fill_invisible writes -inf past each visible range.
// With kscale (fp32 [n_seq * Nmax]) qI and K are e4m3 bytes, w holds the
// head weights times the query-head scales, and each key's sum is scaled.
// score_bf16: scores are stored as bf16 (nearest, ties to even), row stride
// ld bf16 values (no fill_invisible).
bool index_tc_supported(int HI, int cI, int group, bool fp8 = false);
// Top-k filter on the indexer epilogue: instead of the score block, each
// query's scores that can still be among its k largest are appended to
// cand[t * ld ...] as 64-bit composite keys (order key << 32 | ~column),
// cnt[t] counting them (at most the row's visible columns; ld >= Nmax). The
// kernel zeroes cnt first. bf16 operands, contiguous keys.
struct CandOut {
    uint64_t* cand = nullptr;
    uint32_t* cnt = nullptr;
    int64_t ld = 0;
    int k = 0;
};
bool index_cand_supported(int HI, int cI, int group, int k);
// K in blocks (kb.rpb > 0; bf16 keys only): rpb must divide the 128-key tile
// and Nmax.
cudaError_t index_scores_tc(const void* qI, const float* w, const void* K, QuerySpec qs, int nq, int n_seq, int HI,
                            int cI, int64_t Nmax, int m, float* scores, int64_t ld, int group, bool fill_invisible,
                            int* status, cudaStream_t st, const float* kscale = nullptr,
                            bool score_bf16 = false, RowBlocks kb = RowBlocks{0, 0}, CandOut co = CandOut{});

// quant.cu: row-wise e4m3 codes out [rows, cols] and fp32 scales
// s = max|row| / 448 (1 for a zero row), decided in fp64; w_out = w * s when
// w is given (one head weight per row).
cudaError_t quantize_e4m3(const void* x, int64_t rows, int cols, void* out, float* scale, const float* w, float* w_out,
                          ElemType t, cudaStream_t st, int64_t ld = 0, void* rope = nullptr, int rope_dims = 0);
// FP8 KV entries of a selection dequantised into bf16 rows out [nq, k, c]
// (codes [n_seq*Nmax, c-R] e4m3, scales [n_seq*Nmax], rope [n_seq*Nmax, R]
// bf16; query t reads sequence t); idx_out [nq, k]: i for a selected slot,
// -1 for an empty one.
cudaError_t gather_kv_fp8(const uint8_t* codes, const float* scales, const void* rope, const int32_t* idx, int nq,
                          int k, int64_t Nmax, int c, int rope_dims, void* out, int32_t* idx_out, cudaStream_t st);

// api.cu: device address of the status word on the current device
int* device_status();

// topk.cu. With seq given, a row whose sequence seq[t] is outside
// [0, n_seq) has no candidate (its indexer row was never written).
size_t topk_workspace_bytes(int nq, int64_t ncols, int k);
cudaError_t topk_select(const float* scores, int64_t ld, const int32_t* valid, int valid_div,
                        int nq, int64_t ncols, int k, int32_t* idx, float* top_scores, void* ws,
                        cudaStream_t st, const int32_t* seq = nullptr, int n_seq = 0);
// as topk_select on bf16 scores (row stride ld bf16 values)
cudaError_t topk_select_bf16(const void* scores, int64_t ld, const int32_t* valid, int valid_div, int nq,
                             int64_t ncols, int k, int32_t* idx, float* top_scores, cudaStream_t st,
                             const int32_t* seq = nullptr, int n_seq = 0);
// as topk_select with the candidate count of row t = (pos_base + t) / m
cudaError_t topk_select_positions(const float* scores, int64_t ld, int64_t pos_base, int m, int nq,
                                  int64_t ncols, int k, int32_t* idx, void* ws, cudaStream_t st);
// exact top-k of the candidate lists the indexer's filter wrote (row t:
// cand[t * ld ...], cnt[t] entries); the same order and padding as topk_select
cudaError_t topk_from_candidates(const uint64_t* cand, const uint32_t* cnt, int64_t ld, int nq, int k, int32_t* idx,
                                 float* top_scores, cudaStream_t st);

// mqa_tc.cu: tensor-core shared-KV MQA (bf16); ws holds split partials when nsplit > 1
bool mqa_tc_supported(int H, int c);
int mqa_tc_nsplit(int nq, int H, int64_t max_entries, int num_sms);
// two splits run as a cluster of two and merge on chip (no workspace, no combine launch)
bool mqa_tc_pair(int nsplit);
// KV in blocks (kvb.rpb > 0): any rpb dividing Nmax for the sparse path, rpb
// == 1 for the dense one (its rows are read by TMA with the block as the row
// pitch).
cudaError_t mqa_tc(const void* q, const void* KV, const int32_t* idx, int k, QuerySpec qs, int mp, int nq, int n_seq,
                   int H, int c, int64_t Nmax, float scale, const float* sink, void* out, float* lse, void* ws,
                   int nsplit, int* status, cudaStream_t st, RowBlocks kvb = RowBlocks{0, 0});

// mqa.cu: sparse (idx != nullptr) or dense (entries s < pos/mp) shared-KV MQA
size_t mqa_workspace_bytes(int nq, int H, int c, int64_t max_entries, ElemType t);
cudaError_t mqa(const void* q, const void* KV, const int32_t* idx, int k, QuerySpec qs, int mp,
                int nq, int n_seq, int H, int c, int64_t Nmax, float scale, const float* sink, void* out,
                float* lse, void* ws, ElemType t, cudaStream_t st, RowBlocks kvb = RowBlocks{0, 0});

// norm_rope.cu: RMSNorm (gamma != nullptr) then rotary encoding of the last R
// channels of every row of c channels; row r takes the position of group
// r / group: pos[g], or pos0 + g * pos_step when pos is null. y may equal x.
bool norm_rope_supported(int c, int R);
cudaError_t norm_rope(const void* x, void* y, int64_t rows, int group, int c, const float* gamma, float eps, int R,
                      double base, const int32_t* pos, int64_t pos0, int64_t pos_step, int inverse, ElemType t,
                      cudaStream_t st);
// ent[t] = sel[t][0..k) then the window rows of tokens p_t - n_win + 1 .. p_t
// (ring_off + tau mod ring_len; -1 before the sequence start), p_t = pos[t]
// or pos0 + t when pos is null.
cudaError_t window_entries(const int32_t* sel, int k, const int32_t* pos, int64_t pos0, int nq, int n_win,
                           int64_t ring_off, int64_t ring_len, int32_t* ent, cudaStream_t st);

}  // namespace csa
