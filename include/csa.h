/*
 * csa.h — C ABI of libcsa: the DeepSeek-V4 compressed attention hot path
 * (CSA: overlapping token compressor, lightning indexer, top-k selection and
 * shared-KV MQA over the selected entries; HCA: non-overlapping heavy
 * compression and dense shared-KV MQA) for NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page title and section:
 *   [Notes] "DeepSeek-V4: 迈向高效百万级上下文智能" — study notes on the
 *           DeepSeek-V4 report (notes.kuangjux.top): §1.1 CSA (compressor and
 *           indexer equations), §1.2 HCA (comparison table), §1.3 (partial
 *           RoPE, sliding window, sink equation, mixed-precision storage),
 *           §2.6 Fig. 6 (state cache), model configuration table.
 *   [Walk]  mlpod.com walk-through of "DeepSeek-V4: Towards Highly Efficient
 *           Million-Token Context Intelligence": §2.3.1 CSA, §2.3.2 HCA and
 *           MQA, §2.3.3 attention details (query/KV RMSNorm, partial RoPE,
 *           sliding window, sink; causality), §5 item 2 (state cache).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every pointer argument is a DEVICE pointer owned by the caller, unless
 *    stated otherwise, 16-byte aligned. The library never allocates device
 *    memory; calls that need scratch take a caller-provided workspace `ws`
 *    of at least the size returned by the matching *_workspace_size query.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and does not synchronize.
 *  - Arrays are dense and row-major with the shapes given in brackets.
 *  - dtype selects the storage type of activations, weights, caches and
 *    outputs: CSA_BF16 (bfloat16; fp32 accumulation) or CSA_FP32 (fp32 in
 *    and out, fp32 arithmetic). Biases, indexer head weights `w`, sink
 *    logits, scores and lse are always fp32; indices are int32.
 *  - Return value: CSA_OK, or an error code with a message readable through
 *    csa_last_error() on the calling thread. Argument errors are found on the
 *    host before anything is launched, so nothing is written on error.
 *  - Positions are 0-based token positions. A query at position p sees
 *    compressed entry s iff s < floor(p / m) (m' for HCA): it sees only
 *    blocks that end at or before it [Walk §2.3.3 item 3; Walk §2.3.1].
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CSA_ABI_VERSION 2

enum csa_status {
    CSA_OK = 0,
    CSA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or shape   */
    CSA_ERR_UNSUPPORTED = 2,  /* shape outside what the kernels implement     */
    CSA_ERR_WORKSPACE = 3,    /* ws missing or smaller than the query's size  */
    CSA_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed         */
    CSA_ERR_TIMEOUT = 5       /* a device-side wait hit its bound             */
};

enum csa_dtype { CSA_BF16 = 0, CSA_FP32 = 1 };

/* Limits of this build (checked; larger values give CSA_ERR_UNSUPPORTED). */
#define CSA_MAX_TOPK 2048
#define CSA_MAX_HEADS 128
#define CSA_MAX_HEAD_DIM 512
#define CSA_MAX_INDEX_HEADS 64
#define CSA_MAX_INDEX_DIM 256

/* Message of the last failing call on this thread ("" if none). The string
 * is owned by the library and valid until the next call on this thread. */
const char* csa_last_error(void);
int csa_abi_version(void);

/* Number of kernels this library has launched in this process (all devices,
 * all threads). Lets a caller count the launches inside a timed region. */
uint64_t csa_launch_count(void);

/* Per-kernel device timing (tracing). While enabled, every kernel launch is
 * bracketed by CUDA events recorded on the launching stream. Enabling (or
 * disabling) discards the records gathered so far. */
void csa_trace_enable(int on);
/* Waits for the recorded events and aggregates them per kernel name:
 * names [max_kernels][64] (NUL-terminated), total_ms [max_kernels] (sum of
 * device times), counts [max_kernels] (launches); *n_kernels receives the
 * number of distinct kernels written. Host pointers. */
int csa_trace_read(int max_kernels, char* names, double* total_ms, int* counts, int* n_kernels);

/* Device-side status word: the first CSA_ERR_TIMEOUT (or other device error)
 * raised by a kernel since the last reset. Synchronizes `stream`. Returns
 * CSA_OK when no kernel reported an error; resets the word when `reset`. */
int csa_poll_status(void* stream, int reset);

/* Failure-path test hooks (for the tests of the timeout path; leave off in
 * production). csa_debug_set(wait_limit, flags): wait_limit > 0 bounds every
 * device wait of the tensor-core indexer to that many polls (0 restores the
 * built-in bound); flags CSA_DEBUG_SKIP_FIRST_TILE makes the indexer never
 * load its first key tile, so the wait for it runs out: the kernel records
 * CSA_ERR_TIMEOUT in the status word (csa_poll_status), stops every role,
 * drains its copies, frees its tensor memory and returns. Process-wide;
 * affects launches made after the call. */
#define CSA_DEBUG_SKIP_FIRST_TILE 1u
/* Selection paths of csa_decode, csa_prefill, csa_decode_fp8kv and
 * csa_attend_decode (bf16, contiguous caches). By default the indexer stores
 * every score (the fp32 score block) and a top-k kernel selects on it.
 * CSA_DEBUG_TOPK_FILTER switches to the top-k filter on the indexer's
 * epilogue: it writes only the scores that can still be among each query's
 * k best (a running lower bound of the k-th score) and an exact selection
 * runs over those (for k up to 1024 in the grouped prefill of 64 index
 * heads, up to 2048 otherwise). Both give the same selection. The filter
 * cuts the selection's reads but slows the indexer, whose epilogue paces it,
 * so it is not the default. CSA_DEBUG_SCORE_BLOCK forces the score block
 * (it wins when both are set). */
#define CSA_DEBUG_SCORE_BLOCK 2u
#define CSA_DEBUG_TOPK_FILTER 4u
int csa_debug_set(uint32_t wait_limit, uint32_t flags);

/* ------------------------------------------------------------------------
 * a1. Projection [Walk §2.3.1 "KV compression": the KV streams and their
 * compression weights are learnable linear maps of the hidden state H].
 *   out[t][o] = sum_k x[t][k] * W[o][k]
 * x [n, d], W [M, d] (one row per output feature, i.e. nn.Linear layout),
 * out [n, M] always fp32. n >= 0, d % 8 == 0, M % 8 == 0.
 * ------------------------------------------------------------------------ */
int csa_project(const void* x, const void* W, int64_t n, int d, int M, float* out, int dtype,
                void* stream);

/* ------------------------------------------------------------------------
 * a2. CSA overlapping compressor [Notes §1.1, equation C^Comp_i and the
 * sentence after it]. Per block i and channel j, ONE softmax over the 2m
 * logits Z^a[mi+r][j] + B[r][j] and Z^b[m(i-1)+r][j] + B[m+r][j] (r < m),
 * then out[i][j] = sum S^a C^a[mi+r][j] + sum S^b C^b[m(i-1)+r][j].
 *   proj [n, 4c]: each row C^a | C^b | Z^a | Z^b (dtype)
 *   left [m, 4c]: the m projected rows just before this chunk, or NULL at
 *                 the start of a sequence (block 0 then has no b-window)
 *   bias [2m, c] fp32: rows 0..m-1 pair with the a-window, m..2m-1 with b
 *   out  [n/m, c] (dtype), written in full.
 * n % m == 0, c % 8 == 0, 1 <= m <= 64.
 * ------------------------------------------------------------------------ */
int csa_compress(const void* proj, const void* left, const float* bias, int64_t n, int c, int m,
                 void* out, int dtype, void* stream);

/* a3. HCA compressor [Notes §1.2 and its comparison table; Walk §2.3.2]:
 * per block i of mp tokens, one softmax per channel over Z[i*mp+r][j] +
 * B'[r][j], out[i][j] = sum_r S_r C[i*mp+r][j]; no overlap.
 *   proj [n, 2c]: rows C | Z (dtype); bias [mp, c] fp32; out [n/mp, c].
 * n % mp == 0, c % 8 == 0, 1 <= mp <= 1024. */
int hca_compress(const void* proj, const float* bias, int64_t n, int c, int mp, void* out,
                 int dtype, void* stream);

/* a1+a2 fused: projection of the hidden states then CSA compression.
 *   x [n, d], x_left [m, d] or NULL (sequence start), W [4c, d] packing the
 *   a-KV, b-KV, a-weight and b-weight maps (rows 0..c-1, c..2c-1, ...),
 *   bias [2m, c], out [n/m, c]. */
size_t csa_compress_from_hidden_workspace_size(int64_t n, int d, int c, int m, int dtype);
int csa_compress_from_hidden(const void* x, const void* x_left, const void* W, const float* bias,
                             int64_t n, int d, int c, int m, void* out, void* ws, size_t ws_bytes,
                             int dtype, void* stream);

/* a1+a3 fused: x [n, d], W [2c, d] (C map rows then Z map rows), bias
 * [mp, c], out [n/mp, c]. */
size_t hca_compress_from_hidden_workspace_size(int64_t n, int d, int c, int mp, int dtype);
int hca_compress_from_hidden(const void* x, const void* W, const float* bias, int64_t n, int d,
                             int c, int mp, void* out, void* ws, size_t ws_bytes, int dtype,
                             void* stream);

/* ------------------------------------------------------------------------
 * Decode-time compression through the per-sequence state cache [Walk §5
 * item 2: CSA keeps the "tail" tokens that have not yet formed a block, in a
 * fixed-size per-request state; Notes §2.6 Fig. 6, state cache]. One new
 * token per sequence per step; the entry of a block is written by the step
 * whose token closes it, and equals what csa_compress gives for the same
 * rows (the same operations in the same order).
 *
 * csa_compress_step:
 *   proj_new [B, 4c] fp32: the newest token's projections (C^a|C^b|Z^a|Z^b,
 *            as csa_project writes them) of sequence b;
 *   state    [B, 2m, 4c] fp32, caller-owned and kept across steps: the ring
 *            of the last 2m tokens' projections (token tau in slot
 *            tau mod 2m); only slots of the last 2m tokens are ever read;
 *   bias     [2m, c] fp32 (as csa_compress);
 *   pos      [B] int32 (device): the newest token's position (= tokens
 *            before it); a negative position skips the sequence;
 *   cache    [B, Nmax, c] (dtype): when (pos+1) % m == 0, entry
 *            i = (pos+1)/m - 1 (if i < Nmax) is written from the ring:
 *            a-window tokens mi..mi+m-1, b-window m(i-1)..mi-1 (none for
 *            i = 0); nothing else is written.
 * c % 8 == 0, 1 <= m <= 64. */
int csa_compress_step(const float* proj_new, float* state, const float* bias, const int32_t* pos, int B, int c, int m,
                      int64_t Nmax, void* cache, int dtype, void* stream);

/* hca_compress_step: the same for HCA: proj_new [B, 2c] (C|Z), state
 * [B, mp, 2c] (token tau in slot tau mod mp), bias [mp, c]; entry
 * (pos+1)/mp - 1 is written when (pos+1) % mp == 0. 1 <= mp <= 1024. */
int hca_compress_step(const float* proj_new, float* state, const float* bias, const int32_t* pos, int B, int c,
                      int mp, int64_t Nmax, void* cache, int dtype, void* stream);

/* csa_compress_chunk: a chunk of ONE sequence at ANY start and length
 * through the same state ring, so prefill chunks and decode steps can split
 * a sequence anywhere (a chunk that ends mid-block leaves its tail in the
 * ring; the next chunk or step closes the block):
 *   proj  [n, 4c] fp32: the projections of tokens start .. start+n-1;
 *   state [2m, 4c] fp32: this sequence's ring (as csa_compress_step); on
 *         entry it holds the tokens before start that are among the last
 *         2m, on return the last 2m tokens up to start+n;
 *   cache [Nmax, c] (dtype): the sequence's entries; every block that ends
 *         inside the chunk, i = floor(start/m) .. floor((start+n)/m) - 1, is
 *         written at row i, its window tokens before start read from the
 *         ring. Nmax >= floor((start+n)/m). Entries equal csa_compress's for
 *         the same rows (the same operations in the same order).
 * c % 8 == 0, 1 <= m <= 64; n may be 0 (nothing happens). */
int csa_compress_chunk(const float* proj, float* state, const float* bias, int64_t start, int64_t n, int c, int m,
                       void* cache, int64_t Nmax, int dtype, void* stream);

/* hca_compress_chunk: the same for HCA: proj [n, 2c] (C|Z), state [mp, 2c]
 * (token tau in slot tau mod mp), bias [mp, c]; blocks of mp tokens. */
int hca_compress_chunk(const float* proj, float* state, const float* bias, int64_t start, int64_t n, int c, int mp,
                       void* cache, int64_t Nmax, int dtype, void* stream);

/* csa_decode_compress: a1 + csa_compress_step for both CSA streams of one
 * decode step: x_new [B, d] (dtype) projected by W_kv [4c, d] and W_idx
 * [4cI, d], then stepped through state_kv [B, 2m, 4c] and state_idx
 * [B, 2m, 4cI] (fp32) into kv_cache [B, Nmax, c] and idx_cache [B, Nmax, cI]
 * with B_kv [2m, c], B_idx [2m, cI]; pos as csa_compress_step. */
size_t csa_decode_compress_workspace_size(int B, int c, int cI);
int csa_decode_compress(const void* x_new, const void* W_kv, const float* B_kv, const void* W_idx, const float* B_idx,
                        const int32_t* pos, int B, int d, int m, int c, int cI, float* state_kv, float* state_idx,
                        void* kv_cache, void* idx_cache, int64_t Nmax, void* ws, size_t ws_bytes, int dtype,
                        void* stream);

/* ------------------------------------------------------------------------
 * a4. Lightning indexer [Notes §1.1, equation I_{t,s}; Walk §2.3.1]:
 *   scores[t][s] = sum_h w[t][h] * ReLU(qI[t][h] . K[seq_t][s]),
 *   for s < floor(pos[t] / m); columns s >= that are set to -inf.
 *   qI [nq, HI, cI] (dtype), w [nq, HI] fp32, K [B, Nmax, cI] (dtype),
 *   pos [nq] int32, seq_of_q [nq] int32 or NULL (query t reads sequence t),
 *   n_seq = B (sequences in K; a query whose sequence is outside [0, n_seq)
 *   sees no entry), scores [nq, Nmax] fp32.
 * cI % 8 == 0, cI <= CSA_MAX_INDEX_DIM, HI <= CSA_MAX_INDEX_HEADS; in bf16
 * mode (tensor cores) cI % 64 == 0. nq <= 65535.
 * ------------------------------------------------------------------------ */
int csa_index_scores(const void* qI, const float* w, const void* K, const int32_t* pos,
                     const int32_t* seq_of_q, int nq, int n_seq, int HI, int cI, int64_t Nmax, int m,
                     float* scores, int dtype, void* stream);

/* a5. Top-k selection [Walk §2.3.1: the k highest-scoring compressed blocks
 * are kept; Notes model table: k = 512 / 1024]. Row t's candidates are
 * columns 0 .. min(valid[t] / valid_div, ncols) - 1 of scores (row stride
 * ld floats). Output idx [nq, k]: the min(k, candidates) best, ordered by
 * (score descending, column ascending), padded with -1; top_scores [nq, k]
 * (NULL allowed) gets their scores, -inf in padded slots. Deterministic and
 * bit-exact: equal scores are resolved by the lower column. -0.0 == +0.0.
 * 1 <= k <= CSA_MAX_TOPK, nq <= 65535. csa_topk_workspace_size returns 0:
 * the selection needs no workspace (ws may be NULL). */
size_t csa_topk_workspace_size(int nq, int64_t ncols, int k);
int csa_topk_from_scores(const float* scores, int64_t ld, const int32_t* valid, int valid_div,
                         int nq, int64_t ncols, int k, int32_t* idx, float* top_scores, void* ws,
                         size_t ws_bytes, void* stream);

/* a5 on bf16 scores [Notes §2.4]: as csa_topk_from_scores with scores
 * [nq, ld] bf16 (row stride ld bf16 values); a bf16 score widens exactly to
 * fp32, so the result is csa_topk_from_scores's on those values. No
 * workspace. */
int csa_topk_from_scores_bf16(const void* scores, int64_t ld, const int32_t* valid, int valid_div, int nq,
                              int64_t ncols, int k, int32_t* idx, float* top_scores, void* stream);

/* a4+a5: indexer then top-k over the visible entries of each query. */
size_t csa_index_topk_workspace_size(int nq, int64_t Nmax, int k, int dtype);
int csa_index_topk(const void* qI, const float* w, const void* K, const int32_t* pos,
                   const int32_t* seq_of_q, int nq, int n_seq, int HI, int cI, int64_t Nmax, int m, int k,
                   int32_t* idx, float* top_scores, void* ws, size_t ws_bytes, int dtype,
                   void* stream);

/* a4+a5 without a workspace, for callers that cannot allocate device memory
 * at the point of the call: a plug-in whose host framework owns every device
 * allocation and gives it no scratch, a serving loop whose memory footprint
 * is fixed after start-up, a latency-critical path that cannot afford
 * cudaMalloc (which may synchronise the device). The pages have no
 * counterpart: this is a library convenience. Same arguments and exactly the
 * same result as csa_index_topk, minus ws/ws_bytes.
 *
 * The score block between the indexer and the selection lives in a fixed
 * array of device memory inside the library, CSA_NOALLOC_MAX_SCORES fp32
 * scores (16 MiB), held by every GPU that loads the library until the
 * process exits. nq * Nmax above CSA_NOALLOC_MAX_SCORES returns
 * CSA_ERR_UNSUPPORTED (use csa_index_topk). The call makes no cudaMalloc,
 * cudaFree or other allocating call.
 *  - The first call on a device (with that device current) looks up the
 *    array's device address; make it before any stream capture.
 *  - All calls on a device share the array, which keeps the last call's
 *    scores; nothing in it must start at zero (each call writes every score
 *    it reads). Calls that overlap on the GPU (other streams, other host
 *    threads) race on it: serialise them. */
#define CSA_NOALLOC_MAX_SCORES (4 * 1024 * 1024)
int csa_index_topk_noalloc(const void* qI, const float* w, const void* K, const int32_t* pos,
                           const int32_t* seq_of_q, int nq, int n_seq, int HI, int cI, int64_t Nmax, int m, int k,
                           int32_t* idx, float* top_scores, int dtype, void* stream);

/* ------------------------------------------------------------------------
 * FP8 indexer [Notes §2.4: the indexer's query-key products run in low
 * precision; Notes §1.3: FP8 storage; Walk §2.3.4]. q^I and the indexer keys
 * are stored as e4m3 (OCP FP8: 4 exponent bits, 3 mantissa bits, largest
 * magnitude 448, no infinity) with one fp32 scale per row.
 *
 * csa_quantize_e4m3: x [rows, cols] (dtype) -> out [rows, cols] e4m3 bytes
 *   and scale [rows] fp32, s = max|row| / 448 (1 for an all-zero row);
 *   out = the e4m3 value nearest x / s (ties to even, saturating at 448),
 *   with s and x / s taken in fp64. With w [rows] fp32 given, w_out [rows]
 *   = w * s: for q^I rows (one per query head) this folds the query scale into
 *   the head weight, since ReLU(s x) = s ReLU(x) for s > 0.
 *   cols % 8 == 0.
 * csa_index_scores_fp8: as csa_index_scores on e4m3 operands, on tensor cores
 *   (kind::f8f6f4, fp32 accumulation):
 *     scores[t][s] = k_scale[seq_t][s] * sum_h wq[t][h] * ReLU(qI8[t][h] . K8[seq_t][s])
 *   qI8 [nq, HI, cI] e4m3, wq [nq, HI] fp32 (w times the query-head scale, as
 *   csa_quantize_e4m3 writes it), K8 [B, Nmax, cI] e4m3, k_scale [B, Nmax]
 *   fp32; invisible columns -inf. cI % 128 == 0, cI <= 256.
 * csa_decode_fp8: csa_decode with the FP8 indexer: qI [B, HI, cI] bf16 is
 *   quantized per head row inside the call, the indexer reads idx_cache8
 *   [B, Nmax, cI] e4m3 with idx_scale [B, Nmax] fp32 (the keys quantized once
 *   when their entries were written, csa_quantize_e4m3), top-k over the
 *   scores, sparse MQA over kv_cache [B, Nmax, c] bf16. flags: 0, or
 *   CSA_SCORES_BF16 to store the index scores as bf16 (nearest, ties to even)
 *   and select on those [Notes §2.4: BF16 index scores halve the selector's
 *   reads]; ties among rounded scores go to the lower entry index.
 * ------------------------------------------------------------------------ */
#define CSA_SCORES_BF16 1
int csa_quantize_e4m3(const void* x, int64_t rows, int cols, void* out, float* scale, const float* w, float* w_out,
                      int dtype, void* stream);
int csa_index_scores_fp8(const void* qI8, const float* wq, const void* K8, const float* k_scale, const int32_t* pos,
                         const int32_t* seq_of_q, int nq, int n_seq, int HI, int cI, int64_t Nmax, int m,
                         float* scores, void* stream);
size_t csa_decode_fp8_workspace_size(int B, int64_t Nmax, int H, int c, int HI, int cI, int k);
int csa_decode_fp8(const void* qI, const float* w, const void* idx_cache8, const float* idx_scale, const void* q,
                   const void* kv_cache, const int32_t* ctx_len, int B, int64_t Nmax, int m, int H, int c, int HI,
                   int cI, int k, float scale, const float* sink, int flags, void* out, float* lse, int32_t* topk_idx,
                   void* ws, size_t ws_bytes, void* stream);

/* FP8 KV storage with bf16 rotary dims [Notes §1.3 and §2.4: compressed
 * entries stored in FP8 except the rotary dims, which stay BF16]. An entry
 * row x of c values (bf16) becomes: codes [c - R] e4m3 with one fp32 scale
 * s = max|x[0 .. c-R)| / 448 (1 for an all-zero part), decided in fp64 as
 * csa_quantize_e4m3 does, and its last R = rope_dims values unchanged (bf16).
 * In attention the entry is bf16(code * s) for the first c - R dims (the
 * product in fp32) and the stored rotary values after them.
 *
 * csa_quantize_kv_fp8: kv [rows, c] bf16 -> codes [rows, c-R] u8, scales
 * [rows] fp32, rope [rows, R] bf16 (may be NULL when R == 0). c and R
 * multiples of 16, c - R >= 16. */
int csa_quantize_kv_fp8(const void* kv, int64_t rows, int c, int rope_dims, uint8_t* codes, float* scales,
                        void* rope, void* stream);

/* csa_decode_fp8kv: csa_decode (bf16 index keys, bf16 out) with the KV
 * entries in FP8 storage: kv_codes [B, Nmax, c-R], kv_scales [B, Nmax],
 * kv_rope [B, Nmax, R] as csa_quantize_kv_fp8 writes them. The selected
 * entries are dequantised into the workspace (k rows per query) and the
 * sparse MQA runs on those rows; the selection equals csa_decode's. */
size_t csa_decode_fp8kv_workspace_size(int B, int64_t Nmax, int H, int c, int HI, int cI, int k);
int csa_decode_fp8kv(const void* qI, const float* w, const void* idx_cache, const void* q, const uint8_t* kv_codes,
                     const float* kv_scales, const void* kv_rope, const int32_t* ctx_len, int B, int64_t Nmax, int m,
                     int H, int c, int rope_dims, int HI, int cI, int k, float scale, const float* sink, void* out,
                     float* lse, int32_t* topk_idx, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * a6. Sparse shared-KV MQA [Notes §1.1 last paragraph: every compressed
 * entry is both key and value, all query heads share it; Walk §2.3.2; sink
 * from Notes §1.3 equation s_{h,i,j}]:
 *   z_s = scale * q[t][h] . KV[seq_t][s] for s in idx[t][0..k) (-1 = none),
 *   out[t][h] = sum_s exp(z_s) KV[s] / (sum_s exp(z_s) + exp(sink[h])),
 *   lse[t][h] = log of that denominator (-inf for an empty set, no sink).
 *   q [nq, H, c] (dtype), KV [B, Nmax, c] (dtype), idx [nq, k] int32,
 *   seq_of_q [nq] or NULL (identity), n_seq = B (sequences in KV), sink [H]
 *   fp32 or NULL (no sink term),
 *   out [nq, H, c] (dtype), lse [nq, H] fp32 or NULL.
 *   scale == 0 selects 1/sqrt(c).
 * c % 32 == 0, c <= CSA_MAX_HEAD_DIM, H <= CSA_MAX_HEADS, k <= CSA_MAX_TOPK,
 * nq <= 65535.
 * ------------------------------------------------------------------------ */
size_t csa_sparse_mqa_workspace_size(int nq, int H, int c, int k, int dtype);
int csa_sparse_mqa(const void* q, const void* KV, const int32_t* idx, const int32_t* seq_of_q,
                   int nq, int n_seq, int H, int c, int64_t Nmax, int k, float scale, const float* sink,
                   void* out, float* lse, void* ws, size_t ws_bytes, int dtype, void* stream);

/* a7. Dense shared-KV MQA over every visible HCA entry [Walk §2.3.2: after
 * heavy compression full attention is affordable; Notes §1.2 table]: as a6
 * with the entry set s < floor(pos[t] / mp). */
size_t hca_dense_mqa_workspace_size(int nq, int H, int c, int64_t Nmax, int dtype);
int hca_dense_mqa(const void* q, const void* KV, const int32_t* pos, const int32_t* seq_of_q,
                  int nq, int n_seq, int H, int c, int64_t Nmax, int mp, float scale, const float* sink,
                  void* out, float* lse, void* ws, size_t ws_bytes, int dtype, void* stream);

/* ------------------------------------------------------------------------
 * Fused steps.
 *
 * csa_decode: one decode query per sequence b against its cached entries:
 * indexer (a4) over idx_cache[b][0 .. floor(ctx_len[b]/m)), top-k (a5),
 * sparse MQA (a6) over kv_cache[b]. The query position is ctx_len[b].
 *   qI [B, HI, cI], w [B, HI], idx_cache [B, Nmax, cI], q [B, H, c],
 *   kv_cache [B, Nmax, c], ctx_len [B] int32 (device), out [B, H, c],
 *   lse [B, H] or NULL, topk_idx [B, k] or NULL (selected entries).
 * ------------------------------------------------------------------------ */
size_t csa_decode_workspace_size(int B, int64_t Nmax, int H, int c, int HI, int cI, int k,
                                 int dtype);
int csa_decode(const void* qI, const float* w, const void* idx_cache, const void* q,
               const void* kv_cache, const int32_t* ctx_len, int B, int64_t Nmax, int m, int H,
               int c, int HI, int cI, int k, float scale, const float* sink, void* out, float* lse,
               int32_t* topk_idx, void* ws, size_t ws_bytes, int dtype, void* stream);

/* hca_decode: dense MQA (a7) of query b over kv_cache[b][0 .. floor(ctx_len[b]/mp)). */
size_t hca_decode_workspace_size(int B, int64_t Nmax, int H, int c, int dtype);
int hca_decode(const void* q, const void* kv_cache, const int32_t* ctx_len, int B, int64_t Nmax,
               int mp, int H, int c, float scale, const float* sink, void* out, float* lse,
               void* ws, size_t ws_bytes, int dtype, void* stream);

/* csa_prefill: one chunk of n new tokens of ONE sequence at positions
 * start .. start+n-1. Without state rings (state_kv = state_idx = NULL)
 * start % m == 0 and n % m == 0, and x_left supplies the b-window of the
 * first block. With both state rings ([2m, 4c] and [2m, 4cI] fp32, as
 * csa_compress_chunk) start and n are free: the blocks that end inside the
 * chunk are written (earlier window tokens from the rings), the rings then
 * hold the chunk's last 2m projected rows, and x_left is not read. With
 * W_kv = W_idx = NULL the chunk's entries are already in the caches
 * (compressed elsewhere, e.g. gathered from other ranks): steps 1-2 are
 * skipped and x, x_left, B_kv, B_idx are not read. Steps:
 *   1. compress the chunk's KV entries (a1+a2 with W_kv [4c, d], B_kv
 *      [2m, c]) into kv_cache rows start/m .. (start+n)/m - 1;
 *   2. the same for the indexer keys (W_idx [4cI, d], B_idx [2m, cI]) into
 *      idx_cache;
 *   3. for each new token t: indexer over the visible entries, top-k, and
 *      sparse MQA over kv_cache.
 *   x [n, d], x_left [m, d] (the m hidden rows before the chunk; NULL when
 *   start == 0), kv_cache [Nmax, c] and idx_cache [Nmax, cI] with
 *   Nmax >= (start+n)/m (rows before start/m already filled by earlier
 *   chunks), qI [n, HI, cI], w [n, HI], q [n, H, c], out [n, H, c],
 *   lse [n, H] or NULL, topk_idx [n, k] or NULL.
 * ------------------------------------------------------------------------ */
size_t csa_prefill_workspace_size(int64_t n, int64_t Nmax, int d, int m, int c, int cI, int H,
                                  int HI, int k, int dtype);
int csa_prefill(const void* x, const void* x_left, const void* W_kv, const float* B_kv,
                const void* W_idx, const float* B_idx, int64_t start, int64_t n, int d, int m,
                int c, int cI, void* kv_cache, void* idx_cache, int64_t Nmax, float* state_kv,
                float* state_idx, const void* qI, const float* w, const void* q, int H, int HI, int k,
                float scale, const float* sink, void* out, float* lse, int32_t* topk_idx, void* ws,
                size_t ws_bytes, int dtype, void* stream);

/* ------------------------------------------------------------------------
 * Completion of the attention output around a6 [Walk §2.3.3 items 1-3;
 * Notes §1.3 "Partial RoPE" and "sliding window branch"; the window's state
 * cache: Walk §5 item 2, Notes §2.6 Fig. 6].
 *
 * csa_norm_rope: RMSNorm then partial rotary encoding, row by row. For each
 * row of c channels:
 *   y_j = x_j / sqrt(mean_j(x_j^2) + eps) * gamma_j       (gamma NULL: y = x)
 * then the last R = rope_dims channels, as adjacent pairs (c-R+2i,
 * c-R+2i+1), are turned by the angle p * rope_base^(-2i/R):
 *   (a, b) -> (a cos - b sin, a sin + b cos)               (inverse: angle -p)
 * Row r has the position of group r / group: pos[r / group] (device int32
 * [rows / group]) or, with pos NULL, pos0 + (r / group) * pos_step. Queries
 * [nq, H, c] use group = H and their positions; compressed KV entries use
 * group = 1; the attention output is turned back with inverse = 1 and no
 * gamma. x, y [rows, c] (dtype); y == x (in place) is allowed, other overlap
 * is not. gamma [c] fp32 or NULL. c % 8 == 0, 8 <= c <= CSA_MAX_HEAD_DIM,
 * rope_dims % 8 == 0, 0 <= rope_dims <= c, rows % group == 0. Angles are
 * formed in fp64 (positions up to 2^31 keep their accuracy).
 * ------------------------------------------------------------------------ */
int csa_norm_rope(const void* x, void* y, int64_t rows, int group, int c, const float* gamma, float eps,
                  int rope_dims, float rope_base, const int32_t* pos, int64_t pos0, int64_t pos_step, int inverse,
                  int dtype, void* stream);

/* csa_window_entries: entry lists that join the sliding window to the
 * selected compressed entries, for one softmax over both (a6 with
 * k' = k + n_win). Row t of ent [nq, k + n_win] int32 is sel[t][0..k)
 * followed by the window rows of the n_win most recent tokens, the query's
 * own included: slot k + j holds token tau = p_t - n_win + 1 + j at row
 * ring_off + (tau mod ring_len) of the query's sequence, or -1 when tau < 0.
 * p_t = pos[t] (device int32 [nq]) or, with pos NULL, pos0 + t. sel [nq, k]
 * (NULL only when k == 0) and ent must not be the same array.
 * n_win <= ring_len, ring_off + ring_len <= INT32_MAX. */
int csa_window_entries(const int32_t* sel, int k, const int32_t* pos, int64_t pos0, int nq, int n_win,
                       int64_t ring_off, int64_t ring_len, int32_t* ent, void* stream);

/* csa_attend_decode: csa_decode with the complete attention output. Per
 * sequence b (query position p = ctx_len[b]):
 *   1. q' = csa_norm_rope(q[b]) with q_gamma, eps, rope_dims, rope_base at p
 *      (skipped when q_gamma is NULL and rope_dims is 0);
 *   2. indexer (a4) over idx_cache[b][0 .. floor(p/m)) and top-k (a5);
 *   3. the entry list: the selection, then the window rows of tokens
 *      p-n_win+1 .. p;
 *   4. sparse MQA (a6) of q' over those entries of kv_cache[b], ONE softmax
 *      (and the sink, if given) over selection and window together;
 *   5. out turned back by p on the last rope_dims channels.
 *   kv_cache [B, Nmax + ring_len, c]: rows 0..Nmax-1 hold the compressed
 *   entries (already normalised and rotated at their positions), rows
 *   Nmax + (tau mod ring_len) the window ring (token tau's uncompressed KV;
 *   the caller has written the current token's row). idx_cache [B, Nmax, cI].
 *   Other arguments as csa_decode. k + n_win <= CSA_MAX_TOPK,
 *   n_win <= ring_len (ring_len may be 0 when n_win is 0). */
size_t csa_attend_decode_workspace_size(int B, int64_t Nmax, int64_t ring_len, int n_win, int H, int c, int HI,
                                        int cI, int k, int dtype);
int csa_attend_decode(const void* qI, const float* w, const void* idx_cache, const void* q, const void* kv_cache,
                      const int32_t* ctx_len, int B, int64_t Nmax, int64_t ring_len, int n_win, int m, int H, int c,
                      int HI, int cI, int k, float scale, const float* q_gamma, float eps, int rope_dims,
                      float rope_base, const float* sink, void* out, float* lse, int32_t* topk_idx, void* ws,
                      size_t ws_bytes, int dtype, void* stream);

/* ------------------------------------------------------------------------
 * The lcm(m, m')-token cache block [Notes §2.6, the compressed KV cache: one
 * block covers lcm(m, m') raw tokens and holds their lcm/m CSA entries and
 * lcm/m' HCA entries; Walk §5 item 2]. The entries of one sequence live in
 * consecutive blocks; block j (raw tokens j*L .. j*L+L-1, L = lcm(m, m'))
 * holds, in this order:
 *   CSA KV entries   [L/m][c]   (entries j*L/m ..),
 *   CSA index keys   [L/m][cI],
 *   HCA entries      [L/m'][c]  (entries j*L/m' ..),
 * each row in the cache dtype. The compressor state rings of the tail tokens
 * (csa_compress_step, hca_compress_step) stay per sequence, outside the
 * blocks. Sequence b's blocks start Nmax/(L/m) blocks after sequence b-1's,
 * Nmax being the CSA entry capacity per sequence (a multiple of L/m); the HCA
 * capacity is then Nmax*m/m'.
 *
 * csa_cache_block_layout: the block for (m, m', c, cI, dtype): rows of each
 * part per block, bytes per block (a multiple of 16: c and cI multiples of
 * 8) and the byte offset of each part in a block (offset pointers may be
 * NULL). The *_blocked calls below take a cache as (pointer to the part in
 * block 0 = block base + its offset, rows_per_block, block_bytes); they
 * compute exactly what the contiguous calls compute (same kernels, same
 * arithmetic), bf16 caches only. CSA_ERR_INVALID_ARG for an inconsistent
 * layout (rows_per_block < 1, block_bytes not a multiple of 16 or too short
 * for its rows, Nmax not a multiple of rows_per_block, a cache pointer not
 * 16-byte aligned); CSA_ERR_UNSUPPORTED for fp32 caches, a CSA rows_per_block
 * that does not divide 128 (the indexer's key tile), or more than one HCA row
 * per block. Nothing is allocated.
 * ------------------------------------------------------------------------ */
int csa_cache_block_layout(int m, int mp, int c, int cI, int dtype, int* csa_rows, int* hca_rows,
                           int64_t* block_bytes, int64_t* kv_offset, int64_t* idx_offset, int64_t* hca_offset);

/* csa_decode over block caches: kv_cache -> block 0's CSA KV part,
 * idx_cache -> block 0's index-key part, rows_per_block = L/m. Workspace as
 * csa_decode_workspace_size. */
int csa_decode_blocked(const void* qI, const float* w, const void* idx_cache, const void* q, const void* kv_cache,
                       const int32_t* ctx_len, int B, int64_t Nmax, int m, int H, int c, int HI, int cI, int k,
                       float scale, const float* sink, void* out, float* lse, int32_t* topk_idx, int rows_per_block,
                       int64_t block_bytes, void* ws, size_t ws_bytes, int dtype, void* stream);

/* hca_decode over block caches: kv_cache -> block 0's HCA part,
 * rows_per_block = L/m' = 1, Nmax = the HCA capacity per sequence. Workspace
 * as hca_decode_workspace_size. */
int hca_decode_blocked(const void* q, const void* kv_cache, const int32_t* ctx_len, int B, int64_t Nmax, int mp,
                       int H, int c, float scale, const float* sink, void* out, float* lse, int rows_per_block,
                       int64_t block_bytes, void* ws, size_t ws_bytes, int dtype, void* stream);

/* csa_decode_compress writing the closed blocks' entries into block caches
 * (kv_cache, idx_cache as for csa_decode_blocked). Workspace as
 * csa_decode_compress_workspace_size. */
int csa_decode_compress_blocked(const void* x_new, const void* W_kv, const float* B_kv, const void* W_idx,
                                const float* B_idx, const int32_t* pos, int B, int d, int m, int c, int cI,
                                float* state_kv, float* state_idx, void* kv_cache, void* idx_cache, int64_t Nmax,
                                int rows_per_block, int64_t block_bytes, void* ws, size_t ws_bytes, int dtype,
                                void* stream);

/* hca_compress_step writing into block caches (cache -> block 0's HCA part,
 * rows_per_block = 1, Nmax = the HCA capacity per sequence). */
int hca_compress_step_blocked(const float* proj_new, float* state, const float* bias, const int32_t* pos, int B,
                              int c, int mp, int64_t Nmax, void* cache, int rows_per_block, int64_t block_bytes,
                              int dtype, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
