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
//   1. threshold (one CTA per row): sort a strided sample of 2048 scores and
//      take an estimate low enough that, for any row that is not
//      adversarial, well over k scores reach it (a rank ~1.25x the expected
//      count plus 16); filter (several CTAs per row): each appends the
//      composites of its slice that reach it to the row's candidate buffer;
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

constexpr int kThreads = 1024;
constexpr int kSegMax = 16384;     // composites one CTA holds (128 KB)
constexpr int kSample = 2048;      // sample for the threshold estimate
constexpr int kSlice = 8192;       // scores per filter CTA

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

// Bitonic sort of sel[0..P) descending (P a power of two >= kk; the slots
// above kk are filled with 0), then idx / score output for one row.
__device__ void sort_and_write(uint64_t* sel, int kk, int k, int32_t* idx_row, float* score_row) {
    const int tid = threadIdx.x;
    int P = 1;
    while (P < kk) P <<= 1;
    for (int j = kk + tid; j < P; j += kThreads) sel[j] = 0ull;
    __syncthreads();
    for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < (P >> 1); i += kThreads) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const uint64_t a = sel[lo], b = sel[hi];
                if ((a < b) == desc) { sel[lo] = b; sel[hi] = a; }
            }
            __syncthreads();
        }
    }
    for (int j = tid; j < k; j += kThreads) {
        const uint64_t x = (j < kk) ? sel[j] : 0ull;
        if (x == 0ull) {
            idx_row[j] = -1;
            if (score_row) score_row[j] = -INFINITY;
        } else {
            idx_row[j] = (int32_t)(0xFFFFFFFFu - (uint32_t)(x & 0xFFFFFFFFull));
            if (score_row) score_row[j] = from_orderable((uint32_t)(x >> 32));
        }
    }
}

// ---------------------------------------------------------------- kernels

// Rows of at most kSegMax candidates: one CTA per row, the row in smem.
__global__ void __launch_bounds__(kThreads) topk_rows_kernel(RowSpec R, int k, int32_t* idx, float* top) {
    extern __shared__ uint64_t s_elems[];
    __shared__ uint64_t s_sel[CSA_MAX_TOPK];
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
    sort_and_write(s_sel, kk, k, idx + (int64_t)row * k, top ? top + (int64_t)row * k : nullptr);
}

// Step 1a of long rows: one CTA per row sorts a strided sample of 2048
// scores and keeps a threshold estimate (an orderable key) for the filter.
__global__ void __launch_bounds__(kThreads) topk_threshold_kernel(RowSpec R, int k, uint32_t* thr_out) {
    __shared__ uint32_t s_key[kSample];
    const int row = blockIdx.x;
    const int tid = threadIdx.x;
    const int64_t n = R.count(row);
    if (n <= kSegMax) return;   // the final step reads such rows whole
    const float* srow = R.scores + (int64_t)row * R.ld;
    for (int j = tid; j < kSample; j += kThreads) s_key[j] = orderable(srow[(int64_t)j * n / kSample]);
    __syncthreads();
    for (int size = 2; size <= kSample; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < kSample / 2; i += kThreads) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const bool desc = (lo & size) == 0;
                const uint32_t a = s_key[lo], b = s_key[hi];
                if ((a < b) == desc) { s_key[lo] = b; s_key[hi] = a; }
            }
            __syncthreads();
        }
    }
    if (tid == 0) {
        // expected sample entries at or above the k-th score: k * S / n
        int64_t r = (int64_t)((1.25 * (double)k * kSample) / (double)n) + 16;
        if (r > kSample - 1) r = kSample - 1;
        thr_out[row] = s_key[r];
    }
}

// Step 1b: each CTA appends the composites of its slice that reach the
// row's threshold to the row's candidate buffer.
__global__ void __launch_bounds__(kThreads) topk_filter_kernel(RowSpec R, const uint32_t* thr_in, uint64_t* cand,
                                                               int cap, uint32_t* cnt) {
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
    uint64_t* crow = cand + (int64_t)row * cap;
    const int lane = tid & 31;
    for (int64_t i0 = beg + tid - lane; i0 < end; i0 += kThreads) {
        const int64_t i = i0 + lane;
        const float s = (i < end) ? srow[i] : 0.f;
        const bool take = (i < end) && orderable(s) >= thr;
        const unsigned m = __ballot_sync(0xffffffffu, take);
        if (!m) continue;
        const int leader = __ffs(m) - 1;
        uint32_t base = 0;
        if (lane == leader) base = atomicAdd(&cnt[row], (uint32_t)__popc(m));
        base = __shfl_sync(0xffffffffu, base, leader);
        if (take) {
            const uint32_t slot = base + __popc(m & ((1u << lane) - 1u));
            if (slot < (uint32_t)cap) crow[slot] = composite(s, i);
        }
    }
}

// Step 2 of long rows (short rows are read whole): exact selection.
__global__ void __launch_bounds__(kThreads) topk_final_kernel(RowSpec R, int k, const uint64_t* cand, int cap,
                                                              const uint32_t* cnt, int32_t* idx, float* top) {
    extern __shared__ uint64_t s_elems[];
    __shared__ uint64_t s_sel[CSA_MAX_TOPK];
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
    sort_and_write(s_sel, kk, k, idx + (int64_t)row * k, top ? top + (int64_t)row * k : nullptr);
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
    CSA_LAUNCH(st, "topk_threshold", topk_threshold_kernel<<<nq, kThreads, 0, st>>>(R, k, thr));
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
