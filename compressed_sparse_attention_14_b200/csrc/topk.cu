// Top-k entry selection [Walk §2.3.1: keep the k highest-scoring compressed
// blocks; Notes model table: k = 512 for Flash, 1024 for Pro].
// ([Walk] = mlpod.com walk-through of the DeepSeek-V4 report; [Notes] = the
// "DeepSeek-V4: 迈向高效百万级上下文智能" study notes.)
//
// Order: score descending, then column ascending. Each candidate becomes the
// 64-bit composite key
//     (orderable(score) << 32) | (0xFFFFFFFF - column)
// where orderable() maps fp32 to uint32 monotonically (-0.0 folded into
// +0.0). Composite keys are unique and their descending order is exactly the
// selection order, so the k largest composites ARE the answer: no tie pass.
//
// One CTA selects the k largest of one segment held in shared memory with an
// MSB-first radix select (8-bit digits, shared-memory histograms, a warp scan
// to pick the digit), stopping as soon as the digit's bucket fills the
// remaining quota exactly. Segments larger than shared memory are reduced
// in levels: each segment emits its k best, the next level selects among
// those. The last level sorts its k winners with a bitonic network.
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

constexpr int kTopkThreads = 1024;

// Input of one level: either a raw score row (column = position) or a row of
// composite candidates from the previous level (0 = empty slot).
struct TopkLevel {
    const float* scores;      // level 0
    int64_t ld;
    const int32_t* valid;     // nullable: then pos_base rule or every column
    int valid_div;
    int64_t pos_base;         // use_pos: candidates = (pos_base + row) / valid_div
    int use_pos;
    int64_t ncols;
    const uint64_t* cand;     // level >= 1
    int64_t cand_ld;
    int seg_len;
    int k;
    uint64_t* cand_out;       // non-final
    int64_t cand_out_ld;
    int32_t* idx_out;         // final
    float* score_out;         // final, nullable
};

template <bool kRaw, bool kFinal>
__global__ void __launch_bounds__(kTopkThreads) topk_select_kernel(TopkLevel L) {
    extern __shared__ uint64_t s_elems[];
    __shared__ uint64_t s_sel[CSA_MAX_TOPK];
    __shared__ uint32_t s_hist[256];
    __shared__ uint32_t s_cnt;
    __shared__ uint64_t s_prefix;
    __shared__ uint32_t s_remaining;
    __shared__ int s_done;
    __shared__ uint32_t s_n, s_tie;

    const int row = blockIdx.y;
    const int seg = blockIdx.x;
    const int tid = threadIdx.x;
    const int k = L.k;

    int64_t n_row;
    if (kRaw) {
        n_row = L.ncols;
        if (L.valid || L.use_pos) {
            int64_t v = (L.valid ? (int64_t)L.valid[row] : L.pos_base + row) / L.valid_div;
            n_row = v < 0 ? 0 : (v < L.ncols ? v : L.ncols);
        }
    } else {
        n_row = L.cand_ld;
    }
    const int64_t beg = (int64_t)seg * L.seg_len;
    int64_t n64 = n_row - beg;
    const int n_in = n64 <= 0 ? 0 : (n64 > L.seg_len ? L.seg_len : (int)n64);

    if (tid == 0) { s_prefix = 0; s_remaining = (uint32_t)k; s_done = 0; s_cnt = 0; s_n = 0; s_tie = 0; }
    __syncthreads();
    if (kRaw) {
        for (int i = tid; i < n_in; i += kTopkThreads) {
            float s = L.scores[(int64_t)row * L.ld + beg + i];
            s_elems[i] = ((uint64_t)orderable(s) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)(beg + i));
        }
    } else {
        // candidate rows carry empty slots (0); keep only real candidates, so
        // every composite in shared memory is distinct
        for (int i = tid; i < n_in; i += kTopkThreads) {
            uint64_t x = L.cand[(int64_t)row * L.cand_ld + beg + i];
            if (x != 0ull) s_elems[atomicAdd(&s_n, 1u)] = x;
        }
    }
    __syncthreads();
    const int n = kRaw ? n_in : (int)s_n;

    // ---- radix select: threshold T such that exactly min(k, n) elements are >= T
    uint64_t thr = 0;
    if (n > k) {
        for (int shift = 56; shift >= 0; shift -= 8) {
            for (int b = tid; b < 256; b += kTopkThreads) s_hist[b] = 0;
            __syncthreads();
            const uint64_t prefix = s_prefix;
            const uint64_t hi_mask = (shift == 56) ? 0ull : (~0ull << (shift + 8));
            // warp-aggregated histogram: one atomic per distinct digit per warp
            // (the leading digits of similar scores coincide, so plain atomics
            // would serialize on one or two bins)
            const int lane = tid & 31;
            for (int i0 = tid - lane; i0 < n; i0 += kTopkThreads) {
                const int i = i0 + lane;
                uint32_t d = 256u;
                if (i < n) {
                    uint64_t x = s_elems[i];
                    if ((x & hi_mask) == prefix) d = (uint32_t)((x >> shift) & 255u);
                }
                const unsigned peers = __match_any_sync(0xffffffffu, d);
                if (d < 256u && lane == __ffs(peers) - 1) atomicAdd(&s_hist[d], (uint32_t)__popc(peers));
            }
            __syncthreads();
            if (tid < 32) {
                // lane l owns digits 255-8l .. 248-8l (high to low)
                uint32_t h[8];
                uint32_t sum = 0;
#pragma unroll
                for (int u = 0; u < 8; ++u) { h[u] = s_hist[255 - 8 * tid - u]; sum += h[u]; }
                uint32_t incl = sum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (tid >= o) incl += y;
                }
                const uint32_t excl = incl - sum;
                const uint32_t rem = s_remaining;
                const bool mine = excl < rem && incl >= rem;
                const uint32_t ballot = __ballot_sync(0xffffffffu, mine);
                if (mine) {
                    uint32_t cum = excl;
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        if (cum + h[u] >= rem) {
                            const uint32_t digit = 255u - 8u * tid - u;
                            const uint32_t r2 = rem - cum;
                            s_prefix = prefix | ((uint64_t)digit << shift);
                            s_remaining = r2;
                            s_done = (h[u] == r2);
                            break;
                        }
                        cum += h[u];
                    }
                }
                (void)ballot;
            }
            __syncthreads();
            if (s_done) break;
        }
        thr = s_prefix;  // low bits below the last digit are zero: select x >= thr
    }
    const int kk = n < k ? n : k;

    // ---- collect the winners (order arbitrary): everything above the
    // threshold, then copies of the threshold value up to exactly kk (the
    // composites are distinct, so at most one element equals thr; the second
    // pass keeps the count exact regardless)
    for (int i = tid; i < n; i += kTopkThreads) {
        uint64_t x = s_elems[i];
        if (x > thr) {
            uint32_t slot = atomicAdd(&s_cnt, 1u);
            if (slot < (uint32_t)CSA_MAX_TOPK) s_sel[slot] = x;
        }
    }
    __syncthreads();
    const uint32_t n_gt = s_cnt;
    for (int i = tid; i < n; i += kTopkThreads) {
        uint64_t x = s_elems[i];
        if (x == thr) {
            uint32_t t = atomicAdd(&s_tie, 1u);
            if (n_gt + t < (uint32_t)kk) s_sel[n_gt + t] = x;
        }
    }
    __syncthreads();

    if (!kFinal) {
        uint64_t* dst = L.cand_out + (int64_t)row * L.cand_out_ld + (int64_t)seg * k;
        for (int j = tid; j < k; j += kTopkThreads) dst[j] = (j < kk) ? s_sel[j] : 0ull;
        return;
    }

    // ---- final level: bitonic sort of the winners, descending
    int P = 1;
    while (P < kk) P <<= 1;
    for (int j = kk + tid; j < P; j += kTopkThreads) s_sel[j] = 0ull;
    __syncthreads();
    for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < (P >> 1); i += kTopkThreads) {
                int lo = 2 * i - (i & (stride - 1));
                int hi = lo + stride;
                bool desc = (lo & size) == 0;
                uint64_t a = s_sel[lo], b = s_sel[hi];
                if ((a < b) == desc) { s_sel[lo] = b; s_sel[hi] = a; }
            }
            __syncthreads();
        }
    }
    int32_t* io = L.idx_out + (int64_t)row * k;
    float* so = L.score_out ? L.score_out + (int64_t)row * k : nullptr;
    for (int j = tid; j < k; j += kTopkThreads) {
        uint64_t x = (j < kk) ? s_sel[j] : 0ull;
        if (x == 0ull) {
            io[j] = -1;
            if (so) so[j] = -INFINITY;
        } else {
            io[j] = (int32_t)(0xFFFFFFFFu - (uint32_t)(x & 0xFFFFFFFFull));
            if (so) so[j] = from_orderable((uint32_t)(x >> 32));
        }
    }
}

// Largest segment one CTA holds: 16384 composites = 128 KB of shared memory.
constexpr int kTopkSegMax = 16384;

// Segment length of the first level: the whole row when it fits, else
// shorter segments (down to 4k, at least 4096) while few rows would leave
// SMs idle.
static int topk_seg_len(int64_t n, int k, int nq) {
    if (n <= kTopkSegMax) return (int)(n > 0 ? n : 1);
    int seg = kTopkSegMax;
    const int min_seg = 4 * k > 4096 ? 4 * k : 4096;
    while (seg / 2 >= min_seg && (int64_t)nq * ((n + seg - 1) / seg) < 2 * 148) seg /= 2;
    return seg;
}

// Candidate slots needed by the levels (the same plan topk_run follows).
size_t topk_workspace_bytes(int nq, int64_t ncols, int k) {
    int64_t n = ncols;
    size_t best = 0;
    bool first = true;
    while (n > kTopkSegMax) {
        int64_t seg = first ? topk_seg_len(n, k, nq) : kTopkSegMax;
        int64_t nseg = (n + seg - 1) / seg;
        n = nseg * k;
        size_t b = (size_t)nq * (size_t)n * sizeof(uint64_t);
        if (b > best) best = b;
        first = false;
    }
    // two ping-pong buffers, 256-byte aligned
    return best ? 2 * ((best + 255) & ~(size_t)255) : 0;
}

template <bool kRaw, bool kFinal>
static cudaError_t launch_level(const TopkLevel& L, int nq, int nseg, int seg_len, cudaStream_t st) {
    size_t smem = (size_t)seg_len * sizeof(uint64_t);
    auto kern = topk_select_kernel<kRaw, kFinal>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(kTopkSegMax * sizeof(uint64_t)));
    if (e != cudaSuccess) return e;
    CSA_LAUNCH(st, "topk_select", kern<<<dim3(nseg, nq), kTopkThreads, smem, st>>>(L));
    return cudaGetLastError();
}

static cudaError_t topk_run(TopkLevel L, int nq, int64_t ncols, int k, void* ws, cudaStream_t st) {
    if (nq == 0) return cudaSuccess;
    if (ncols <= kTopkSegMax) {
        L.seg_len = topk_seg_len(ncols, k, nq);
        return launch_level<true, true>(L, nq, 1, L.seg_len, st);
    }
    size_t half = topk_workspace_bytes(nq, ncols, k) / 2;
    uint64_t* buf[2] = {(uint64_t*)ws, (uint64_t*)((char*)ws + half)};
    int64_t n = ncols;
    int which = 0;
    bool raw = true;
    cudaError_t e = cudaSuccess;
    while (true) {
        if (n <= kTopkSegMax) {
            L.seg_len = (int)(n > 0 ? n : 1);
            L.cand_ld = n;
            return raw ? launch_level<true, true>(L, nq, 1, L.seg_len, st)
                       : launch_level<false, true>(L, nq, 1, L.seg_len, st);
        }
        const int seg = raw ? topk_seg_len(n, k, nq) : kTopkSegMax;
        int nseg = (int)((n + seg - 1) / seg);
        L.seg_len = seg;
        L.cand_ld = n;
        L.cand_out = buf[which];
        L.cand_out_ld = (int64_t)nseg * k;
        e = raw ? launch_level<true, false>(L, nq, nseg, seg, st)
                : launch_level<false, false>(L, nq, nseg, seg, st);
        if (e != cudaSuccess) return e;
        L.cand = buf[which];
        n = (int64_t)nseg * k;
        which ^= 1;
        raw = false;
    }
}

cudaError_t topk_select(const float* scores, int64_t ld, const int32_t* valid, int valid_div,
                        int nq, int64_t ncols, int k, int32_t* idx, float* top_scores, void* ws,
                        cudaStream_t st) {
    TopkLevel L{};
    L.scores = scores; L.ld = ld; L.valid = valid; L.valid_div = valid_div; L.ncols = ncols;
    L.k = k; L.idx_out = idx; L.score_out = top_scores;
    return topk_run(L, nq, ncols, k, ws, st);
}

cudaError_t topk_select_positions(const float* scores, int64_t ld, int64_t pos_base, int m, int nq,
                                  int64_t ncols, int k, int32_t* idx, void* ws, cudaStream_t st) {
    TopkLevel L{};
    L.scores = scores; L.ld = ld; L.valid = nullptr; L.valid_div = m; L.ncols = ncols;
    L.pos_base = pos_base; L.use_pos = 1;
    L.k = k; L.idx_out = idx; L.score_out = nullptr;
    return topk_run(L, nq, ncols, k, ws, st);
}

}  // namespace csa
