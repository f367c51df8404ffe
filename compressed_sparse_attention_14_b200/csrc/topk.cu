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
// Scores are read as fp32, or as bf16 [Notes §2.4: index scores quantized
// to BF16 halve the selector's reads]: a bf16 score widens exactly to fp32,
// so the order is the same as on fp32 scores holding those values.
//
// One launch, no global scratch; a row is served by one CTA, or by a cluster
// of G CTAs (G = 2, 4, 8 when there are few long rows, so that the row's
// pass over its scores has G SMs' worth of loads in flight):
//   * a row of at most kCap candidates is read whole into shared memory;
//   * a longer row is first narrowed to a candidate set: every CTA of the
//     cluster takes the same strided sample of kSample scores and finds
//     (radix select) the sample score of rank r = mu + 4 sqrt(mu) + 4,
//     mu = k * kSample / n being the expected number of samples at or above
//     the row's k-th score; CTA g keeps every score of its slice of the row
//     at or above it (16-byte loads, warp-aggregated appends to its shared
//     memory); CTA 0 then pulls the other CTAs' candidates over distributed
//     shared memory. If at least min(k, n) and at most kCap scores reach the
//     estimate, the k best are all among them; otherwise (ties, a row
//     ordered against the strided sample) CTA 0 selects exactly on the whole
//     row, streamed from global memory.
//   * exact selection on the candidates: up to kSortMax of them are simply
//     sorted (bitonic network); more go through an MSB-first radix select on
//     the composites (8-bit digits, warp-aggregated shared-memory
//     histograms, a warp scan picks the digit) that finds the k-th largest
//     composite T; the winners are the composites >= T, and those are sorted.
#include <cooperative_groups.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace csa {

// One score, widened to fp32 (L2-cached load: each is read once).
__device__ __forceinline__ float ld_score(const float* p) { return __ldcg(p); }
__device__ __forceinline__ float ld_score(const bf16* p) {
    return __uint_as_float((uint32_t)__ldcg(reinterpret_cast<const unsigned short*>(p)) << 16);
}
// Score e of a 16-byte vector of scores kept as raw words (4 fp32 or 8 bf16),
// widened to fp32 where it is used, so the vectors in flight take 4
// registers each whatever the score type.
template <typename TS>
__device__ __forceinline__ float vec_score(const uint4& q, int e) {
    const uint32_t w = (e & (16 / (int)sizeof(TS) / 2)) ? ((e & (16 / (int)sizeof(TS) / 4)) ? q.w : q.z)
                                                         : ((e & (16 / (int)sizeof(TS) / 4)) ? q.y : q.x);
    if constexpr (sizeof(TS) == 4) return __uint_as_float(w);
    else return __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
}

namespace cg = cooperative_groups;

constexpr int kThreads = 512;
constexpr int kMaxCluster = 8;
constexpr int kCap = 8192;          // candidates one CTA holds (64 KB)
constexpr int kSample = 4096;       // sample for the threshold estimate
constexpr int kSortMax = CSA_MAX_TOPK;
constexpr int kPerThread = kSortMax / kThreads;
// Dynamic shared memory: the candidates, then a scratch area that holds the
// sample, later the winners and the sort's exchange buffer (the sort reads
// the winners into registers before it reuses the area).
constexpr size_t kCandBytes = (size_t)kCap * sizeof(uint64_t);
constexpr size_t kScratchBytes = (size_t)2 * kSortMax * sizeof(uint64_t);
static_assert(kScratchBytes >= (size_t)kSample * sizeof(uint64_t), "the sample must fit the scratch area");
constexpr size_t kSmemBytes = kCandBytes + kScratchBytes;
// When the launch has no more CTAs than SMs, each asks for more shared
// memory than two CTAs can share, so that every CTA gets an SM of its own.
constexpr size_t kSmemSpread = 160 * 1024;

// The candidate columns of each row: 0 .. count(row) - 1.
struct RowSpec {
    const void* scores;       // fp32, or bf16 when bf16 != 0
    int bf16;
    int64_t ld;
    const int32_t* valid;     // nullable
    int valid_div;
    int64_t pos_base;         // used when use_pos
    int use_pos;
    int64_t ncols;
    const int32_t* seq;       // nullable: row t reads sequence seq[t]
    int n_seq;                // a row whose sequence is outside [0, n_seq) has no candidate
    __device__ __forceinline__ int64_t count(int row) const {
        if (seq && (seq[row] < 0 || seq[row] >= n_seq)) return 0;
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
template <typename TS>
struct RowSrc {
    const TS* row;
    __device__ __forceinline__ uint64_t operator()(int64_t i) const { return composite(ld_score(row + i), i); }
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
            if (slot < (uint32_t)kSortMax) sel[slot] = x;
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

// Bitonic sort of up to kSortMax 64-bit keys, descending, by all threads of
// the CTA. Element e = j * kThreads + t lives in register v[j] of thread t. A
// compare-exchange partner at distance `stride` is in the same warp
// (stride < 32: shuffle), in another warp (stride < kThreads: double-buffered
// shared memory, one barrier), or in the same thread (register swap).
static_assert(kSortMax <= 4 * kThreads, "in-thread strides above 2 * kThreads are not generated");

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
                if (stride == kThreads) swap_in_thread<1>(v, E, size, t);
                else swap_in_thread<2>(v, E, size, t);
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

// Sort src[0..cnt) (cnt <= kSortMax, arbitrary order) descending and write
// the first kk = min(cnt, k) as the row's idx / scores; slots past kk get
// -1 / -inf. src may alias xbuf.
__device__ void sort_and_write(const uint64_t* src, int cnt, int kk, int k, int32_t* idx_row, float* score_row,
                               uint64_t* xbuf) {
    const int tid = threadIdx.x;
    int P = kThreads;
    while (P < cnt) P <<= 1;
    uint64_t v[kPerThread];
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) {
        const int e = j * kThreads + tid;
        v[j] = (e < cnt) ? src[e] : 0ull;
    }
    __syncthreads();   // src may alias xbuf
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

// ---------------------------------------------------------------- key bins
// Counting by value: a key (orderable score) falls into bin
// (key - kmin) >> shift, shift chosen so that the keys span at most kBins
// bins; bin order is value order. Exact integer arithmetic, so the smallest
// key of bin B is kmin + (B << shift).
constexpr int kBins = 2 * kThreads;     // two per thread in the scans
constexpr int kBucketMax = 4096;        // candidates placed by counting in the smaller scratch area
constexpr uint32_t kMaxBinLoad = 64;    // larger bins (heavy ties): bitonic path
static_assert(kScratchBytes >= (size_t)kBucketMax * sizeof(uint64_t), "buckets must fit the scratch area");

// Entries the scratch area holds: the dynamic shared memory past the
// candidates (a CTA launched with an SM to itself gets a larger one).
__device__ __forceinline__ int scratch_entries() {
    uint32_t dyn;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
    return (int)((dyn - (uint32_t)kCandBytes) / sizeof(uint64_t));
}

struct BinShared {
    uint32_t cnt[kBins];
    uint32_t start[kBins];
    uint32_t cur[kBins];
    uint32_t red[2][kThreads / 32];
    uint32_t B;
    int overflow;
};

struct KeyBins {
    uint32_t kmin;
    int shift;
    __device__ __forceinline__ int bin(uint32_t key) const { return (int)((key - kmin) >> shift); }
};

// Min and max over the CTA of the keys each thread passes (have = false: none).
__device__ KeyBins key_bins(uint32_t lo, uint32_t hi, BinShared& bs) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (lane == 0) { bs.red[0][warp] = lo; bs.red[1][warp] = hi; }
    __syncthreads();
    uint32_t mn = 0xffffffffu, mx = 0u;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) { mn = min(mn, bs.red[0][w]); mx = max(mx, bs.red[1][w]); }
    KeyBins kb;
    kb.kmin = mn;
    const uint32_t span = mx > mn ? mx - mn : 0u;
    const int bits = 32 - __clz(span);
    kb.shift = bits > 10 ? bits - 10 : 0;    // (span >> shift) < 1024 = kBins
    static_assert(kBins == 1024, "shift rule assumes 1024 bins");
    return kb;
}

// start[b] = elements in the bins above b (descending exclusive scan of
// cnt); cur[b] = start[b]. Thread t owns bins kBins-1-2t and kBins-2-2t.
// Also flags bins holding more than kMaxBinLoad. Ends with a barrier.
__device__ void bins_scan_desc(BinShared& bs) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b0 = kBins - 1 - 2 * tid, b1 = b0 - 1;
    const uint32_t c0 = bs.cnt[b0], c1 = bs.cnt[b1];
    uint32_t incl = c0 + c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) bs.red[0][warp] = incl;
    if (c0 > kMaxBinLoad || c1 > kMaxBinLoad) bs.overflow = 1;
    __syncthreads();
    uint32_t base = 0;
    for (int w = 0; w < warp; ++w) base += bs.red[0][w];
    const uint32_t excl = base + incl - (c0 + c1);
    bs.start[b0] = excl;
    bs.start[b1] = excl + c0;
    bs.cur[b0] = excl;
    bs.cur[b1] = excl + c0;
    __syncthreads();
}

__device__ __forceinline__ void bins_clear(BinShared& bs) {
    for (int b = threadIdx.x; b < kBins; b += kThreads) bs.cnt[b] = 0;
    if (threadIdx.x == 0) bs.overflow = 0;
}

// Threshold estimate from the row's strided sample: the smallest key of the
// bin that holds the sample's r-th largest score, so that at least r sample
// scores reach it. (Ranking the samples inside that bin to return the exact
// r-th key was measured: the bins near the sample's top are narrow, the
// candidates did not shrink and the two extra barriers cost 0.3 us.)
template <typename TS>
__device__ uint32_t sample_threshold(const TS* srow, int64_t n, int r, BinShared& bs) {
    constexpr int kPer = kSample / kThreads;
    const int tid = threadIdx.x;
    uint32_t key[kPer];
    uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int t = u * kThreads + tid;
        key[u] = orderable(ld_score(srow + ((int64_t)t * n) / kSample));
        lo = min(lo, key[u]);
        hi = max(hi, key[u]);
    }
    bins_clear(bs);
    const KeyBins kb = key_bins(lo, hi, bs);   // its barrier also orders the clear
#pragma unroll
    for (int u = 0; u < kPer; ++u) atomicAdd(&bs.cnt[kb.bin(key[u])], 1u);
    __syncthreads();
    bins_scan_desc(bs);
    const uint32_t ur = (uint32_t)r;
    for (int b = tid; b < kBins; b += kThreads)
        if (bs.start[b] < ur && bs.start[b] + bs.cnt[b] >= ur) bs.B = (uint32_t)b;
    __syncthreads();
    return kb.kmin + (bs.B << kb.shift);
}

// Exact top-k of e[0..n) (n <= kBucketMax, distinct composites) by counting:
// place each key in its value bin (bins in descending order, arbitrary order
// inside a bin), then each key's output slot is its bin's start plus the
// number of keys of its bin above it. Writes the first k slots (padding
// past n). Returns false, having written nothing, when some bin holds more
// than kMaxBinLoad keys.
__device__ bool select_by_bins(const uint64_t* e, int n, int k, int32_t* idx_row, float* score_row, uint64_t* bucket,
                               BinShared& bs) {
    const int tid = threadIdx.x;
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int i = tid; i < n; i += kThreads) {
        const uint32_t key = (uint32_t)(e[i] >> 32);
        lo = min(lo, key);
        hi = max(hi, key);
    }
    bins_clear(bs);
    const KeyBins kb = key_bins(lo, hi, bs);
    for (int i = tid; i < n; i += kThreads) atomicAdd(&bs.cnt[kb.bin((uint32_t)(e[i] >> 32))], 1u);
    __syncthreads();
    bins_scan_desc(bs);
    if (bs.overflow) return false;
    for (int i = tid; i < n; i += kThreads) {
        const uint64_t x = e[i];
        bucket[atomicAdd(&bs.cur[kb.bin((uint32_t)(x >> 32))], 1u)] = x;
    }
    __syncthreads();
    for (int p = tid; p < n; p += kThreads) {
        const uint64_t x = bucket[p];
        const int b = kb.bin((uint32_t)(x >> 32));
        if ((int)bs.start[b] >= k) continue;
        const int s0 = (int)bs.start[b], s1 = (int)bs.cur[b];
        int rank = 0;
        for (int q = s0; q < s1; ++q) rank += bucket[q] > x;
        const int pos = s0 + rank;
        if (pos < k) {
            idx_row[pos] = (int32_t)(0xFFFFFFFFu - (uint32_t)(x & 0xFFFFFFFFull));
            if (score_row) score_row[pos] = from_orderable((uint32_t)(x >> 32));
        }
    }
    for (int pos = n + tid; pos < k; pos += kThreads) {
        idx_row[pos] = -1;
        if (score_row) score_row[pos] = -INFINITY;
    }
    return true;
}

// Exact selection among n distinct composites (in shared memory, or the row
// in global memory): by counting when they fit the buckets, else all of
// them sorted when they fit the network, else radix select of the k-th,
// collect the winners, sort those.
template <class Src>
__device__ void select_exact(const Src& src, int64_t n, int k, int32_t* idx_row, float* score_row,
                             uint64_t* scratch, SelShared& sh, BinShared& bs) {
    const int kk = (int)(n < k ? n : k);
    if constexpr (std::is_same<Src, SmemSrc>::value) {
        if (n <= scratch_entries() && select_by_bins(src.e, (int)n, k, idx_row, score_row, scratch, bs)) return;
        __syncthreads();   // the scratch area may hold buckets
        if (n <= kSortMax) {
            sort_and_write(src.e, (int)n, kk, k, idx_row, score_row, scratch);
            return;
        }
    }
    const uint64_t thr = radix_threshold(src, n, k, sh);
    collect(src, n, thr, kk, scratch, sh);
    sort_and_write(scratch, kk, kk, k, idx_row, score_row, scratch);
}

// Warp-aggregated append of s (column i) to buf when it reaches thr
// (orderable); *cnt counts every taker, also past cap.
__device__ __forceinline__ void append_if(float s, int64_t i, bool in, uint32_t thr, uint64_t* buf, uint32_t cap,
                                          uint32_t* cnt) {
    const int lane = threadIdx.x & 31;
    const bool take = in && orderable(s) >= thr;
    const unsigned m = __ballot_sync(0xffffffffu, take);
    if (m) {
        const int leader = __ffs(m) - 1;
        uint32_t base = 0;
        if (lane == leader) base = atomicAdd(cnt, (uint32_t)__popc(m));
        base = __shfl_sync(0xffffffffu, base, leader);
        const uint32_t slot = base + __popc(m & ((1u << lane) - 1u));
        if (take && slot < cap) buf[slot] = composite(s, i);
    }
}

// Every score of srow[lo, hi) that reaches thr, appended to buf; kU 16-byte
// loads (kV scores each) in flight per thread.
template <int kU, typename TS>
__device__ void filter_slice(const TS* srow, int64_t lo, int64_t hi, uint32_t thr, uint64_t* buf, uint32_t cap,
                             uint32_t* cnt) {
    constexpr int kV = 16 / (int)sizeof(TS);
    const int tid = threadIdx.x, lane = tid & 31;
    // scalar head up to the first 16-byte boundary, 16-byte body, scalar
    // tail; the head and tail loads are issued first and used last
    int64_t lo_v = lo + (int64_t)(((16u - ((uint32_t)(uintptr_t)(srow + lo) & 15u)) & 15u) / sizeof(TS));
    if (lo_v > hi) lo_v = hi;
    const int64_t nvec = (hi - lo_v) / kV;
    const int64_t hi_v = lo_v + kV * nvec;
    const int64_t ih = lo + tid, it = hi_v + tid;
    const bool inh = ih < lo_v, intl = it < hi;
    const float sh = inh ? ld_score(srow + ih) : 0.f;
    const float stl = intl ? ld_score(srow + it) : 0.f;
    static_assert(kV * kU <= 64, "one mask bit per value");
    for (int64_t b0 = 0; b0 < nvec; b0 += kU * kThreads) {
        uint4 raw[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t j = b0 + u * kThreads + tid;
            raw[u] = j < nvec ? __ldcg(reinterpret_cast<const uint4*>(srow + lo_v + kV * j)) : make_uint4(0, 0, 0, 0);
        }
        // this thread's takers, then one reservation per warp
        uint64_t mask = 0;
#pragma unroll
        for (int e = 0; e < kV * kU; ++e) {
            const int64_t j = b0 + (e / kV) * kThreads + tid;
            if (j < nvec && orderable(vec_score<TS>(raw[e / kV], e % kV)) >= thr) mask |= 1ull << e;
        }
        const uint32_t mine = __popcll(mask);
        uint32_t incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
        if (total == 0) continue;
        uint32_t base = 0;
        if (lane == 31) base = atomicAdd(cnt, total);
        uint32_t slot = __shfl_sync(0xffffffffu, base, 31) + incl - mine;
#pragma unroll
        for (int e = 0; e < kV * kU; ++e) {
            if (mask & (1ull << e)) {
                const int64_t i = lo_v + kV * (b0 + (e / kV) * kThreads + tid) + (e % kV);
                if (slot < cap) buf[slot] = composite(vec_score<TS>(raw[e / kV], e % kV), i);
                ++slot;
            }
        }
    }
    append_if(sh, ih, inh, thr, buf, cap, cnt);
    append_if(stl, it, intl, thr, buf, cap, cnt);
}

__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

constexpr int kFilterLoads = 4;   // 16-byte filter loads in flight per thread

// Bulk prefetch of the bytes [b, e) into L2 (the 16-byte-aligned part, in
// 32 KB pieces); a hint only.
template <typename TS>
__device__ __forceinline__ void prefetch_l2(const TS* b, const TS* e) {
    uintptr_t p = ((uintptr_t)b + 15) & ~(uintptr_t)15;
    const uintptr_t end = (uintptr_t)e & ~(uintptr_t)15;
    for (; p + 16 <= end; p += 32768) {
        const uint32_t bytes = (uint32_t)(end - p < 32768 ? end - p : 32768);
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
    }
}

template <typename TS>
__global__ void __launch_bounds__(kThreads, 2) topk_kernel(RowSpec R, int k, int32_t* idx, float* top) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint64_t* cand = reinterpret_cast<uint64_t*>(smem_raw);
    uint64_t* scratch = reinterpret_cast<uint64_t*>(smem_raw + kCandBytes);
    __shared__ SelShared sh;
    __shared__ BinShared bs;
    __shared__ uint32_t s_cnt, s_total, s_base;
    pdl_wait();
    pdl_launch_next();
    cg::cluster_group cluster = cg::this_cluster();
    const int G = (int)cluster.num_blocks();
    const int g = (int)cluster.block_rank();
    const int row = blockIdx.x / G;
    const int tid = threadIdx.x;
    const int64_t n = R.count(row);
    const TS* srow = reinterpret_cast<const TS*>(R.scores) + (int64_t)row * R.ld;
    int32_t* idx_row = idx + (int64_t)row * k;
    float* score_row = top ? top + (int64_t)row * k : nullptr;
    const int kk = (int)(n < k ? n : k);

    if (n <= kCap) {   // the same branch for every CTA of the cluster
        if (g != 0) return;
        for (int64_t i = tid; i < n; i += kThreads) cand[i] = composite(ld_score(srow + i), i);
        __syncthreads();
        select_exact(SmemSrc{cand}, n, k, idx_row, score_row, scratch, sh, bs);
        return;
    }

    // ---- this CTA's slice starts on its way to L2 while the threshold is
    // worked out (bulk prefetches: no registers or shared memory held)
    const int64_t lo = n * g / G, hi = n * (g + 1) / G;
    if (tid == 0) prefetch_l2(srow + lo, srow + hi);

    // ---- threshold from the sample (identical in every CTA of the cluster)
    if (tid == 0) { s_cnt = 0; s_total = 0; }
    // CTA 0's total must be zero before any CTA of the cluster adds to it:
    // arrive here, wait just before the first addition
    if (G > 1) cluster_arrive_release();
    const double mu = (double)k * kSample / (double)n;
    int r = (int)(mu + 4.0 * sqrt(mu) + 4.0);
    if (r > kSample) r = kSample;
    const uint32_t thr = sample_threshold(srow, n, r, bs);

    // ---- this CTA's slice: keep every score that reaches it
    if (G == 1) {
        filter_slice<kFilterLoads>(srow, lo, hi, thr, cand, kCap, &s_cnt);
        __syncthreads();
    } else {
        // CTA 0 filters into its scratch area; every CTA then reserves a
        // range of CTA 0's candidate array with one remote addition and
        // stores its candidates there over distributed shared memory
        uint64_t* buf = g == 0 ? scratch : cand;
        const uint32_t cap = g == 0 ? (uint32_t)scratch_entries() : (uint32_t)kCap;
        filter_slice<kFilterLoads>(srow, lo, hi, thr, buf, cap, &s_cnt);
        __syncthreads();
        const uint32_t mine = s_cnt;
        cluster_wait_acquire();
        if (tid == 0) {
            // a CTA that dropped candidates forces the exact fallback
            const uint32_t add = mine <= cap ? mine : (uint32_t)kCap + 1u;
            s_base = add ? atomicAdd(cluster.map_shared_rank(&s_total, 0), add) : 0u;
        }
        __syncthreads();
        const uint32_t base = s_base;
        uint64_t* dst = cluster.map_shared_rank(cand, 0);
        if (mine <= cap)
            for (uint32_t j = tid; j < mine && base + j < (uint32_t)kCap; j += kThreads) dst[base + j] = buf[j];
        cluster.sync();   // every CTA's candidates are in CTA 0
        if (g != 0) return;
    }
    const uint32_t c = G == 1 ? s_cnt : s_total;
    if (c >= (uint32_t)kk && c <= (uint32_t)kCap)
        select_exact(SmemSrc{cand}, (int64_t)c, k, idx_row, score_row, scratch, sh, bs);
    else
        select_exact(RowSrc<TS>{srow}, n, k, idx_row, score_row, scratch, sh, bs);   // the estimate missed
}

// ---------------------------------------------------------------- candidate lists
// Exact top-k of the lists the indexer's top-k filter wrote (composite keys
// of distinct columns, in arbitrary order): a list of at most kCap entries is
// read into shared memory and selected there like a short score row
// (counting, sorting or radix select); a longer one is selected in place,
// the radix passes streaming it from global memory.
struct GmemKeySrc {
    const uint64_t* e;
    __device__ __forceinline__ uint64_t operator()(int64_t i) const { return __ldcg(e + i); }
};

__global__ void __launch_bounds__(kThreads, 2) topk_cand_kernel(const uint64_t* cand, const uint32_t* cnt, int64_t ld,
                                                                int k, int32_t* idx, float* top) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint64_t* c = reinterpret_cast<uint64_t*>(smem_raw);
    uint64_t* scratch = reinterpret_cast<uint64_t*>(smem_raw + kCandBytes);
    __shared__ SelShared sh;
    __shared__ BinShared bs;
    pdl_wait();
    pdl_launch_next();
    const int row = blockIdx.x;
    const int64_t n = (int64_t)cnt[row] < ld ? (int64_t)cnt[row] : ld;
    const uint64_t* src = cand + (int64_t)row * ld;
    int32_t* idx_row = idx + (int64_t)row * k;
    float* score_row = top ? top + (int64_t)row * k : nullptr;
    if (n <= kCap) {
#pragma unroll 4
        for (int64_t i = threadIdx.x; i < n; i += kThreads) c[i] = __ldcg(src + i);
        __syncthreads();
        select_exact(SmemSrc{c}, n, k, idx_row, score_row, scratch, sh, bs);
    } else {
        select_exact(GmemKeySrc{src}, n, k, idx_row, score_row, scratch, sh, bs);
    }
}

// ---------------------------------------------------------------- host side

size_t topk_workspace_bytes(int nq, int64_t ncols, int k) {
    (void)nq;
    (void)ncols;
    (void)k;
    return 0;
}

static int sm_count() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    }
    return n;
}

static cudaError_t topk_run(const RowSpec& R, int nq, int k, int32_t* idx, float* top, cudaStream_t st) {
    if (nq == 0) return cudaSuccess;
    // CTAs per row: enough to give long rows most of the SMs when rows are few
    int G = 1;
    if (R.ncols > kCap)
        while (G < kMaxCluster && (int64_t)nq * G * 2 <= sm_count()) G <<= 1;
    const bool spread = (int64_t)nq * G <= sm_count();
    auto kern = R.bf16 ? topk_kernel<bf16> : topk_kernel<float>;
    const size_t smem = spread ? kSmemSpread : kSmemBytes;
    cudaError_t e = smem_ceiling(kern);
    if (e != cudaSuccess) return e;
    cudaError_t le = cudaSuccess;
    CSA_LAUNCH(st, "topk_select",
               le = launch_pdl(kern, dim3((unsigned)nq * G), dim3(kThreads), smem, st, (unsigned)G, R, k, idx, top));
    if (le != cudaSuccess) return le;
    return cudaGetLastError();
}

cudaError_t topk_from_candidates(const uint64_t* cand, const uint32_t* cnt, int64_t ld, int nq, int k, int32_t* idx,
                                 float* top_scores, cudaStream_t st) {
    if (nq == 0) return cudaSuccess;
    cudaError_t e = smem_ceiling(topk_cand_kernel);
    if (e != cudaSuccess) return e;
    const size_t smem = nq <= sm_count() ? kSmemSpread : kSmemBytes;
    cudaError_t le = cudaSuccess;
    CSA_LAUNCH(st, "topk_candidates",
               le = launch_pdl(topk_cand_kernel, dim3((unsigned)nq), dim3(kThreads), smem, st, 0, cand, cnt, ld, k,
                               idx, top_scores));
    if (le != cudaSuccess) return le;
    return cudaGetLastError();
}

cudaError_t topk_select(const float* scores, int64_t ld, const int32_t* valid, int valid_div, int nq, int64_t ncols,
                        int k, int32_t* idx, float* top_scores, void* ws, cudaStream_t st, const int32_t* seq,
                        int n_seq) {
    (void)ws;
    RowSpec R{scores, 0, ld, valid, valid_div, 0, 0, ncols, seq, n_seq};
    return topk_run(R, nq, k, idx, top_scores, st);
}

cudaError_t topk_select_positions(const float* scores, int64_t ld, int64_t pos_base, int m, int nq, int64_t ncols,
                                  int k, int32_t* idx, void* ws, cudaStream_t st) {
    (void)ws;
    RowSpec R{scores, 0, ld, nullptr, m, pos_base, 1, ncols, nullptr, 0};
    return topk_run(R, nq, k, idx, nullptr, st);
}

cudaError_t topk_select_bf16(const void* scores, int64_t ld, const int32_t* valid, int valid_div, int nq,
                             int64_t ncols, int k, int32_t* idx, float* top_scores, cudaStream_t st,
                             const int32_t* seq, int n_seq) {
    RowSpec R{scores, 1, ld, valid, valid_div, 0, 0, ncols, seq, n_seq};
    return topk_run(R, nq, k, idx, top_scores, st);
}

}  // namespace csa
