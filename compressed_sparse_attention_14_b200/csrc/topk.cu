// Top-k entry selection [Walk §2.3.1: keep the k highest-scoring compressed
// blocks; Notes model table: k = 512 for Flash, 1024 for Pro].
// ([Walk] = mlpod.com walk-through of the DeepSeek-V4 report; [Notes] = the
// "DeepSeek-V4: 迈向高效百万级上下文智能" study notes.)
//
// Order: score descending, then column ascending. Each candidate becomes the
// 64-bit composite key
//     (orderable(score) << 32) | (0xFFFFFFFF - column)
// where orderable() maps fp32 to uint32 monotonically (-0.0 folded into
// +0.0). Composite keys are distinct and their descending order is exactly
// the selection order, so the k largest composites ARE the answer.
//
// Exact selection (one CTA): an MSB-first radix select on the composites
// (8-bit digits, warp-aggregated shared-memory histograms, a warp scan picks
// the digit) finds the k-th largest composite T; the winners are all
// composites >= T; a bitonic network sorts them.
//
// Rows longer than one CTA's shared memory take two steps:
//   1. threshold (one CTA per row): from a strided sample of 1024 scores take
//      an estimate low enough that, for any row that is not adversarial,
//      well over k scores reach it (the sample value of rank ~1.25x the
//      expected count plus 16); filter (several CTAs per row): each appends
//      the composites of its slice that reach it to the row's candidate
//      buffer;
//   2. final (one CTA per row): when at least min(k, n) and at most the
//      buffer's capacity of candidates arrived, the exact selection runs on
//      them; otherwise it runs on the whole row, streamed from global memory.
// Either way the result is exact: the k best are among the candidates
// whenever at least k scores reach the threshold.
#include "common.cuh"
#include "kernels.h"

namespace csa {

__device__ __forceinline__ uint32_t orderable(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;  // -0.0 == +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_orderable(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}
__device__ __forceinline__ uint64_t composite(float s, int64_t col) {
    return ((uint64_t)orderable(s) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)col);
}

// Small CTAs: these steps are dominated by barrier latency, not arithmetic.
constexpr int kThreads = 256;
constexpr int kSegMax = 16384;     // composites one CTA holds (128 KB)
constexpr int kSample = 1024;      // sample for the threshold estimate
constexpr int kSlice = 4096;       // scores per filter CTA

// The candidate columns of each row: 0 .. count(row) - 1.
struct RowSpec {
    const float* scores;
    int64_t ld;
    const int32_t* valid;     // nullable
    int valid_div;
    int64_t pos_base;         // used when use_pos
    int use_pos;
    int64_t ncols;
    __device__ __forceinline__ int64_t count(int row) const {
        if (!valid && !use_pos) return ncols;
        int64_t v = (valid ? (int64_t)valid[row] : pos_base + row) / valid_div;
        return v < 0 ? 0 : (v < ncols ? v : ncols);
    }
};

struct SelShared {
    uint32_t hist[256];
    uint64_t prefix;
    uint32_t remaining;
    int done;
    uint32_t cnt, tie;
};

struct SmemSrc {
    const uint64_t* e;
    __device__ __forceinline__ uint64_t operator()(int64_t i) const { return e[i]; }
};
struct RowSrc {
    const float* row;
    __device__ __forceinline__ uint64_t operator()(int64_t i) const { return composite(row[i], i); }
};

// Largest T such that exactly min(k, n) elements are >= T (distinct keys).
// Called by every thread of the CTA.
template <class Src>
__device__ uint64_t radix_threshold(const Src& src, int64_t n, int k, SelShared& sh) {
    const int tid = threadIdx.x, lane = tid & 31;
    if (n <= k) return 0ull;
    if (tid == 0) { sh.prefix = 0; sh.remaining = (uint32_t)k; sh.done = 0; }
    __syncthreads();
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int b = tid; b < 256; b += kThreads) sh.hist[b] = 0;
        __syncthreads();
        const uint64_t prefix = sh.prefix;
        const uint64_t hi_mask = (shift == 56) ? 0ull : (~0ull << (shift + 8));
        // warp-aggregated histogram: the leading digits of similar scores
        // coincide, so plain atomics would serialize on a few bins
        for (int64_t i0 = tid - lane; i0 < n; i0 += kThreads) {
            const int64_t i = i0 + lane;
            uint32_t d = 256u;
            if (i < n) {
                const uint64_t x = src(i);
                if ((x & hi_mask) == prefix) d = (uint32_t)((x >> shift) & 255u);
            }
            const unsigned peers = __match_any_sync(0xffffffffu, d);
            if (d < 256u && lane == __ffs(peers) - 1) atomicAdd(&sh.hist[d], (uint32_t)__popc(peers));
        }
        __syncthreads();
        if (tid < 32) {
            // lane l owns digits 255-8l .. 248-8l (high to low)
            uint32_t h[8];
            uint32_t sum = 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) { h[u] = sh.hist[255 - 8 * tid - u]; sum += h[u]; }
            uint32_t incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (tid >= o) incl += y;
            }
            const uint32_t excl = incl - sum;
            const uint32_t rem = sh.remaining;
            if (excl < rem && incl >= rem) {
                uint32_t cum = excl;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (cum + h[u] >= rem) {
                        const uint32_t r2 = rem - cum;
                        sh.prefix = prefix | ((uint64_t)(255u - 8u * tid - u) << shift);
                        sh.remaining = r2;
                        sh.done = (h[u] == r2);
                        break;
                    }
                    cum += h[u];
                }
            }
        }
        __syncthreads();
        if (sh.done) break;
    }
    return sh.prefix;  // bits below the last digit are zero: select x >= prefix
}

// Winners (x >= thr, exactly kk of them) into sel[0..kk), order arbitrary:
// everything above the threshold, then copies of it up to kk.
template <class Src>
__device__ void collect(const Src& src, int64_t n, uint64_t thr, int kk, uint64_t* sel, SelShared& sh) {
    const int tid = threadIdx.x;
    if (tid == 0) { sh.cnt = 0; sh.tie = 0; }
    __syncthreads();
    for (int64_t i = tid; i < n; i += kThreads) {
        const uint64_t x = src(i);
        if (x > thr) {
            const uint32_t slot = atomicAdd(&sh.cnt, 1u);
            if (slot < (uint32_t)CSA_MAX_TOPK) sel[slot] = x;
        }
    }
    __syncthreads();
    const uint32_t n_gt = sh.cnt;
    for (int64_t i = tid; i < n; i += kThreads) {
        const uint64_t x = src(i);
        if (x == thr) {
            const uint32_t t = atomicAdd(&sh.tie, 1u);
            if (n_gt + t < (uint32_t)kk) sel[n_gt + t] = x;
        }
    }
    __syncthreads();
}

// Bitonic sort of up to 2048 64-bit keys, descending, by all threads of the
// CTA. Element e = j * kThreads + t lives in register v[j] of thread t. A
// compare-exchange partner at distance `stride` is in the same warp
// (stride < 32: shuffle), in another warp (stride < kThreads: double-buffered
// shared memory, one barrier), or in the same thread (register swap).
constexpr int kSortMax = CSA_MAX_TOPK;
constexpr int kPerThread = kSortMax / kThreads;

template <int SJ>
__device__ __forceinline__ void swap_in_thread(uint64_t (&v)[kPerThread], int E, int size, int t) {
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) {
        if ((j & SJ) == 0 && j < E) {
            const int e = j * kThreads + t;
            const bool desc = (e & size) == 0;
            const uint64_t a = v[j], b = v[j ^ SJ];
            const bool sw = (a < b) == desc;
            v[j] = sw ? b : a;
            v[j ^ SJ] = sw ? a : b;
        }
    }
}

__device__ void bitonic_desc(uint64_t (&v)[kPerThread], int P, uint64_t* xbuf /* [2][kSortMax] */) {
    const int t = threadIdx.x;
    const int E = P / kThreads;          // P >= kThreads here
    int pb = 0;
    for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            if (stride >= kThreads) {
                const int sj = stride / kThreads;
                if (sj == 1) swap_in_thread<1>(v, E, size, t);
                else if (sj == 2) swap_in_thread<2>(v, E, size, t);
                else swap_in_thread<4>(v, E, size, t);
            } else if (stride >= 32) {
#pragma unroll
                for (int j = 0; j < kPerThread; ++j)
                    if (j < E) xbuf[pb * kSortMax + j * kThreads + t] = v[j];
                __syncthreads();
#pragma unroll
                for (int j = 0; j < kPerThread; ++j) {
                    if (j < E) {
                        const int e = j * kThreads + t;
                        const uint64_t y = xbuf[pb * kSortMax + j * kThreads + (t ^ stride)];
                        const bool keep_max = ((e & stride) == 0) == ((e & size) == 0);
                        v[j] = keep_max ? (v[j] > y ? v[j] : y) : (v[j] < y ? v[j] : y);
                    }
                }
                pb ^= 1;
            } else {
#pragma unroll
                for (int j = 0; j < kPerThread; ++j) {
                    if (j < E) {
                        const int e = j * kThreads + t;
                        const uint64_t y = __shfl_xor_sync(0xffffffffu, v[j], stride);
                        const bool keep_max = ((e & stride) == 0) == ((e & size) == 0);
                        v[j] = keep_max ? (v[j] > y ? v[j] : y) : (v[j] < y ? v[j] : y);
                    }
                }
            }
        }
    }
}

// Sort sel[0..kk) (the winners, arbitrary order) descending and write the
// row's idx / scores; slots past kk get -1 / -inf.
__device__ void sort_and_write(uint64_t* sel, int kk, int k, int32_t* idx_row, float* score_row,
                               uint64_t* xbuf) {
    const int tid = threadIdx.x;
    int P = kThreads;
    while (P < kk) P <<= 1;
    uint64_t v[kPerThread];
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) {
        const int e = j * kThreads + tid;
        v[j] = (e < kk) ? sel[e] : 0ull;
    }
    __syncthreads();   // sel may alias xbuf
    bitonic_desc(v, P, xbuf);
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) {
        const int e = j * kThreads + tid;
        if (e < k) {
            const uint64_t x = (e < kk) ? v[j] : 0ull;
            if (x == 0ull) {
                idx_row[e] = -1;
                if (score_row) score_row[e] = -INFINITY;
            } else {
                idx_row[e] = (int32_t)(0xFFFFFFFFu - (uint32_t)(x & 0xFFFFFFFFull));
                if (score_row) score_row[e] = from_orderable((uint32_t)(x >> 32));
            }
        }
    }
}

// ---------------------------------------------------------------- kernels

// Rows of at most kSegMax candidates: one CTA per row, the row in smem.
__global__ void __launch_bounds__(kThreads) topk_rows_kernel(RowSpec R, int k, int32_t* idx, float* top) {
    extern __shared__ uint64_t s_elems[];
    __shared__ uint64_t s_x[2 * kSortMax];
    uint64_t* s_sel = s_x;
    __shared__ SelShared sh;
    const int row = blockIdx.x;
    const int64_t n = R.count(row);
    const float* srow = R.scores + (int64_t)row * R.ld;
    for (int64_t i = threadIdx.x; i < n; i += kThreads) s_elems[i] = composite(srow[i], i);
    __syncthreads();
    const int kk = (int)(n < k ? n : k);
    SmemSrc src{s_elems};
    const uint64_t thr = radix_threshold(src, n, k, sh);
    collect(src, n, thr, kk, s_sel, sh);
    sort_and_write(s_sel, kk, k, idx + (int64_t)row * k, top ? top + (int64_t)row * k : nullptr, s_x);
}

// Step 1a of long rows: one CTA per row takes a strided sample of 1024
// scores, sorts it (one element per thread; shuffles inside a warp, shared
// memory across warps) and keeps the sample value of rank r as the row's
// threshold estimate (an orderable key).
constexpr int kThrThreads = kSample;
__global__ void __launch_bounds__(kThrThreads) topk_threshold_kernel(RowSpec R, int k, uint32_t* thr_out) {
    __shared__ uint32_t s_key[2][kSample];
    const int row = blockIdx.x;
    const int t = threadIdx.x;
    const int64_t n = R.count(row);
    if (n <= kSegMax) return;   // the final step reads such rows whole
    const float* srow = R.scores + (int64_t)row * R.ld;
    uint32_t x = orderable(srow[(int64_t)t * n / kSample]);
    int pb = 0;
    for (int size = 2; size <= kSample; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            uint32_t y;
            if (stride >= 32) {
                s_key[pb][t] = x;
                __syncthreads();
                y = s_key[pb][t ^ stride];
                pb ^= 1;
            } else {
                y = __shfl_xor_sync(0xffffffffu, x, stride);
            }
            const bool keep_max = ((t & stride) == 0) == ((t & size) == 0);
            x = keep_max ? max(x, y) : min(x, y);
        }
    }
    // expected sample entries at or above the k-th score: k * S / n
    int64_t r = (int64_t)((1.25 * (double)k * kSample) / (double)n) + 16;
    if (r > kSample - 1) r = kSample - 1;
    if (t == (int)r) thr_out[row] = x;
}

// Step 1b: each CTA collects the composites of its slice that reach the
// row's threshold in shared memory, reserves room in the row's candidate
// buffer with one atomic, and copies them there.
__global__ void __launch_bounds__(kThreads) topk_filter_kernel(RowSpec R, const uint32_t* thr_in, uint64_t* cand,
                                                               int cap, uint32_t* cnt) {
    __shared__ uint64_t s_out[kSlice];
    __shared__ uint32_t s_n, s_base;
    const int row = blockIdx.y;
    const int tid = threadIdx.x;
    const int64_t n = R.count(row);
    if (n <= kSegMax) return;
    const int64_t beg = (int64_t)blockIdx.x * kSlice;
    if (beg >= n) return;
    const float* srow = R.scores + (int64_t)row * R.ld;
    const uint32_t thr = thr_in[row];
    int64_t end = beg + kSlice;
    if (end > n) end = n;
    if (tid == 0) s_n = 0;
    __syncthreads();
    const int lane = tid & 31;
    for (int64_t i0 = beg + tid - lane; i0 < end; i0 += kThreads) {
        const int64_t i = i0 + lane;
        const float s = (i < end) ? srow[i] : 0.f;
        const bool take = (i < end) && orderable(s) >= thr;
        const unsigned m = __ballot_sync(0xffffffffu, take);
        if (!m) continue;
        const int leader = __ffs(m) - 1;
        uint32_t base = 0;
        if (lane == leader) base = atomicAdd(&s_n, (uint32_t)__popc(m));
        base = __shfl_sync(0xffffffffu, base, leader);
        if (take) s_out[base + __popc(m & ((1u << lane) - 1u))] = composite(s, i);
    }
    __syncthreads();
    const uint32_t c = s_n;
    if (tid == 0) s_base = c ? atomicAdd(&cnt[row], c) : 0u;
    __syncthreads();
    const uint32_t base = s_base;
    uint64_t* crow = cand + (int64_t)row * cap;
    for (uint32_t j = tid; j < c; j += kThreads)
        if (base + j < (uint32_t)cap) crow[base + j] = s_out[j];
}

// Step 2 of long rows (short rows are read whole): exact selection.
__global__ void __launch_bounds__(kThreads) topk_final_kernel(RowSpec R, int k, const uint64_t* cand, int cap,
                                                              const uint32_t* cnt, int32_t* idx, float* top) {
    extern __shared__ uint64_t s_elems[];
    __shared__ uint64_t s_x[2 * kSortMax];
    uint64_t* s_sel = s_x;
    __shared__ SelShared sh;
    const int row = blockIdx.x;
    const int64_t n = R.count(row);
    const int kk = (int)(n < k ? n : k);
    const float* srow = R.scores + (int64_t)row * R.ld;
    if (n <= kSegMax) {
        for (int64_t i = threadIdx.x; i < n; i += kThreads) s_elems[i] = composite(srow[i], i);
        __syncthreads();
        SmemSrc src{s_elems};
        const uint64_t thr = radix_threshold(src, n, k, sh);
        collect(src, n, thr, kk, s_sel, sh);
    } else {
        const uint32_t c = cnt[row];
        if (c >= (uint32_t)kk && c <= (uint32_t)cap) {
            const uint64_t* crow = cand + (int64_t)row * cap;
            for (int64_t i = threadIdx.x; i < (int64_t)c; i += kThreads) s_elems[i] = crow[i];
            __syncthreads();
            SmemSrc src{s_elems};
            const uint64_t thr = radix_threshold(src, (int64_t)c, k, sh);
            collect(src, (int64_t)c, thr, kk, s_sel, sh);
        } else {
            // the estimate missed (ties, adversarial rows): exact on the whole row
            RowSrc src{srow};
            const uint64_t thr = radix_threshold(src, n, k, sh);
            collect(src, n, thr, kk, s_sel, sh);
        }
    }
    sort_and_write(s_sel, kk, k, idx + (int64_t)row * k, top ? top + (int64_t)row * k : nullptr, s_x);
}

// ---------------------------------------------------------------- host side

static int candidate_cap(int k) {
    int cap = 8 * k;
    if (cap > kSegMax) cap = kSegMax;
    return cap;
}

size_t topk_workspace_bytes(int nq, int64_t ncols, int k) {
    if (ncols <= kSegMax) return 0;
    return align256((size_t)nq * candidate_cap(k) * sizeof(uint64_t)) + align256((size_t)nq * 2 * sizeof(uint32_t));
}

static cudaError_t topk_run(const RowSpec& R, int nq, int k, int32_t* idx, float* top, void* ws, cudaStream_t st) {
    if (nq == 0) return cudaSuccess;
    const size_t smem = (size_t)kSegMax * sizeof(uint64_t);
    cudaError_t e;
    if (R.ncols <= kSegMax) {
        e = cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const size_t need = (size_t)(R.ncols > 0 ? R.ncols : 1) * sizeof(uint64_t);
        CSA_LAUNCH(st, "topk_select", topk_rows_kernel<<<nq, kThreads, need, st>>>(R, k, idx, top));
        return cudaGetLastError();
    }
    const int cap = candidate_cap(k);
    uint64_t* cand = (uint64_t*)ws;
    uint32_t* cnt = (uint32_t*)((char*)ws + align256((size_t)nq * cap * sizeof(uint64_t)));
    uint32_t* thr = cnt + nq;
    e = cudaMemsetAsync(cnt, 0, (size_t)nq * sizeof(uint32_t), st);
    if (e != cudaSuccess) return e;
    CSA_LAUNCH(st, "topk_threshold", topk_threshold_kernel<<<nq, kThrThreads, 0, st>>>(R, k, thr));
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int slices = (int)((R.ncols + kSlice - 1) / kSlice);
    CSA_LAUNCH(st, "topk_filter", topk_filter_kernel<<<dim3(slices, nq), kThreads, 0, st>>>(R, thr, cand, cap, cnt));
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(topk_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    CSA_LAUNCH(st, "topk_select", topk_final_kernel<<<nq, kThreads, smem, st>>>(R, k, cand, cap, cnt, idx, top));
    return cudaGetLastError();
}

cudaError_t topk_select(const float* scores, int64_t ld, const int32_t* valid, int valid_div, int nq, int64_t ncols,
                        int k, int32_t* idx, float* top_scores, void* ws, cudaStream_t st) {
    RowSpec R{scores, ld, valid, valid_div, 0, 0, ncols};
    return topk_run(R, nq, k, idx, top_scores, ws, st);
}

cudaError_t topk_select_positions(const float* scores, int64_t ld, int64_t pos_base, int m, int nq, int64_t ncols,
                                  int k, int32_t* idx, void* ws, cudaStream_t st) {
    RowSpec R{scores, ld, nullptr, m, pos_base, 1, ncols};
    return topk_run(R, nq, k, idx, nullptr, ws, st);
}

}  // namespace csa
