// Shared-KV multi-query attention on the 5th-generation tensor cores
// [Notes §1.1 last paragraph: each compressed entry is both key and value,
// shared by all query heads; Walk §2.3.2; sink from Notes §1.3, equation
// s_{h,i,j}] ([Notes] = "DeepSeek-V4: 迈向高效百万级上下文智能" study notes;
// [Walk] = the mlpod.com walk-through of the DeepSeek-V4 report).
//
// One CTA serves (query t, a group of up to 64 heads, one split of t's entry
// list) and walks the split in tiles of 128 entries. Because key and value
// are the same row, ONE shared-memory copy of a tile (128 entries x c dims,
// 128-byte swizzle, 64-dim blocks) feeds both products:
//   S^T  = KV_tile . q^T       M = 128 entries, N = heads, K = c  (KV K-major)
//   O^T += KV_tile^T . P^T     M = 128 dims,    N = heads, K = 128 (KV MN-major)
// with S^T (double-buffered) and O^T in tensor memory. A TMEM lane of S^T
// holds one entry's logits for every head, so the softmax threads work per
// entry; the per-head running max is a reference value that only moves (and
// then O^T and the partial sums are rescaled in place) when a logit exceeds
// it by more than 2^8 — exact, since the final normalisation uses the same
// reference, and cheap, since it rarely moves after the first tile.
//
// Entry sources. CSA (sparse): one tile buffer; the selected rows are
// gathered with 16-byte cp.async (the producer warp moves four rows'
// 128-byte block per instruction), and the tile's 64-dim blocks are released
// one by one as the second product finishes with them, so the next tile's
// gather overlaps it. HCA (dense): consecutive rows stream through two rings
// of 32 KB slots (a pair of 64-dim blocks per slot, one TMA box per block):
// every tile passes through twice, once through the S ring for the first
// product and again (mostly from L2) through the O ring for the second, each
// ring with its own loading thread and its own MMA-issuing thread, so the
// HBM read of the next tiles runs while tile j waits for its softmax.
//
// Warp roles: warp 0 loads (sparse: all lanes issue gathers; dense: the S
// ring), warp 1 allocates TMEM, one lane each of warps 1 and 6 issues MMAs,
// warps 2-5 run the softmax and the epilogue, warp 7 loads the dense O ring.
// A single split writes the normalised output directly. Up to
// kMaxClusterSplits splits of one query run as one thread-block cluster and
// merge on chip: each CTA stages its unnormalised O (fp32) in the shared
// memory its KV tile used, and after a cluster barrier CTA g combines the
// g-th slice of the head dimension from every split's O over distributed
// shared memory (fixed order: deterministic). Otherwise the splits write
// partials (O, max, sum) to the workspace for mqa_combine. Waits are bounded
// (CSA_ERR_TIMEOUT).
#include <cooperative_groups.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tmap.h"

namespace csa {

namespace cg = cooperative_groups;

namespace {

// warp 0 loads (dense: the S-pass ring), warps 1 and 6 issue MMAs (warp 1
// also owns TMEM), warps 2-5 run the softmax and the epilogue, warp 7 loads
// the O-pass ring of the dense path
constexpr int kThreads = 256;
constexpr int kE = 128;                 // entries per tile
constexpr int kMaxDBlocks = 8;          // c <= 512
constexpr uint32_t kWaitLimit = 1u << 24;
constexpr float kRescaleLog2 = 8.0f;    // move the reference max past 2^8
// Splits merged in one cluster: at most 8 (the portable cluster size); the
// host takes a cluster only when all of the launch's clusters can be resident
// at once.
constexpr int kMaxClusterSplits = 8;

struct MqaArgs {
    QueryMap qm;
    int n_seq, mp;
    const void* KV;           // [n_seq * Nmax][c] bf16
    const int32_t* idx;       // sparse entry lists, or nullptr (dense)
    int k;
    int nq, H, c;
    int hg;                   // heads per CTA (MMA N) = 64
    int64_t Nmax;
    float scale_log2;
    const float* sink;
    int nsplit;
    int cluster;              // the splits of a query form one cluster
    int64_t split_len;
    bf16* out;
    float* lse;
    float* part_o;
    float* part_ml;
    int* status;
    int dblocks, mtiles;
    int ring;                 // dense: 32 KB slots (a pair of 64-dim blocks) in the KV ring; 0 for sparse
    uint32_t tmem_cols, q_bytes;
};

// 16-byte asynchronous global -> shared copy (L1 bypassed) and its groups.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most n (0..7) of this thread's most recent groups are pending.
__device__ __forceinline__ void cp_async_wait_pending(int n) {
    switch (n) {
        case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
        case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
        case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
        case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
        case 4: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
        case 5: asm volatile("cp.async.wait_group 5;" ::: "memory"); break;
        case 6: asm volatile("cp.async.wait_group 6;" ::: "memory"); break;
        default: asm volatile("cp.async.wait_group 7;" ::: "memory"); break;
    }
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              int* status) {
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && *abort_flag) return false;
    }
    report_device_error(status, CSA_ERR_TIMEOUT);
    *abort_flag = 1;
    return false;
}

__device__ __forceinline__ bool bar_or_128(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, 1, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void bar_sync_128() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

}  // namespace

// The splits of query t (one cluster, rank = split) merge on chip: after a
// cluster barrier, CTA `split` combines its slice of the head dimension for
// every head from all splits' staged O (fp32, [head][dim] where the KV tile
// was), their reference maxima and sums (log2 domain) and the sink. kG is the
// largest cluster the instance handles (G <= kG splits take part).
// (The launch parameters come in by value: read through a pointer to the
// kernel's parameter block inside this out-of-line function, every access
// would be a slow generic load.)
template <int kG>
__device__ __noinline__ void cluster_merge(int G, int c, int H, const float* sink, float* lse_out, bf16* out, int t,
                                           int h0, int split, float* obuf, float* mref_s, float* lsum_s,
                                           float (*coef_s)[64]) {
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();   // every split's obuf, reference max and sum are final
    const int tid = threadIdx.x;
    if (tid < 64) {
        const int h = h0 + tid;
        // every split's max and sum loaded at once (fully unrolled, so the
        // arrays stay in registers)
        const float sk = (sink && h < H) ? sink[h] * 1.4426950408889634f : -INFINITY;
        float mq[kG], lq[kG];
#pragma unroll
        for (int q = 0; q < kG; ++q) {
            mq[q] = q < G ? cl.map_shared_rank(mref_s, q)[tid] : -INFINITY;
            lq[q] = q < G ? cl.map_shared_rank(lsum_s, q)[tid] : 0.f;
        }
        float M = sk;
#pragma unroll
        for (int q = 0; q < kG; ++q) M = fmaxf(M, mq[q]);
        float L = (sk == -INFINITY) ? 0.f : exp2f(sk - M);
#pragma unroll
        for (int q = 0; q < kG; ++q)
            if (mq[q] != -INFINITY) L += lq[q] * exp2f(mq[q] - M);
        const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
        for (int q = 0; q < kG; ++q)
            if (q < G) coef_s[q][tid] = (mq[q] == -INFINITY) ? 0.f : exp2f(mq[q] - M) * inv;
        if (split == 0 && lse_out && h < H)
            lse_out[(int64_t)t * H + h] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
    }
    __syncthreads();
    // this CTA's slice of the head dimension, every head, in units of 4
    // dims (16-byte aligned, whatever G): sum over the splits in rank order.
    // The (head, 4-dim chunk) items of the slice are spread over all threads,
    // consecutive threads on consecutive chunks of one head; kR items per
    // thread per round, every load of the round issued before any is used
    // (the rounds are bound by the latency of the distributed-shared-memory
    // reads)
    const int n4 = c / 4;
    const int lo4 = split * n4 / G, dn4 = (split + 1) * n4 / G - lo4;
    const int nh = H - h0 < 64 ? H - h0 : 64;
    const int total = nh * dn4;
    constexpr int kR = 16 / kG;
    const float* src[kG];
#pragma unroll
    for (int q = 0; q < kG; ++q)   // this CTA's own split straight from its shared memory
        src[q] = q < G ? (q == split ? obuf : cl.map_shared_rank(obuf, q)) : obuf;
    for (int base = tid; base < total; base += kR * kThreads) {
        float4 v[kR][kG];
        float w[kR][kG];
        int hi[kR], ji[kR];
#pragma unroll
        for (int u = 0; u < kR; ++u) {
            const int item = base + u * kThreads;
            const bool ok = item < total;
            hi[u] = ok ? item / dn4 : 0;
            ji[u] = ok ? item - hi[u] * dn4 : 0;
#pragma unroll
            for (int q = 0; q < kG; ++q) {
                w[u][q] = (ok && q < G) ? coef_s[q][hi[u]] : 0.f;
                v[u][q] = w[u][q] != 0.f   // an empty split staged no O
                              ? *reinterpret_cast<const float4*>(src[q] + hi[u] * c + 4 * (lo4 + ji[u]))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int u = 0; u < kR; ++u) {
            if (base + u * kThreads >= total) continue;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int q = 0; q < kG; ++q) {
                if (w[u][q] == 0.f) continue;
                acc.x = fmaf(w[u][q], v[u][q].x, acc.x);
                acc.y = fmaf(w[u][q], v[u][q].y, acc.y);
                acc.z = fmaf(w[u][q], v[u][q].z, acc.z);
                acc.w = fmaf(w[u][q], v[u][q].w, acc.w);
            }
            __nv_bfloat162 lo2 = __floats2bfloat162_rn(acc.x, acc.y), hi2 = __floats2bfloat162_rn(acc.z, acc.w);
            uint2 pk;
            pk.x = *reinterpret_cast<uint32_t*>(&lo2);
            pk.y = *reinterpret_cast<uint32_t*>(&hi2);
            *reinterpret_cast<uint2*>(out + ((int64_t)t * H + h0 + hi[u]) * c + 4 * (lo4 + ji[u])) = pk;
        }
    }
    cl.sync();   // the other CTAs' shared memory stays alive until read
}

// Dense path: one ring of 32 KB slots (a pair of 64-dim blocks each),
// slots [r_lo, r_lo + r_n), filled with every tile of the split pair by pair,
// in order; one producer and one consumer per ring.
__device__ __noinline__ void dense_ring_load(const MqaArgs& a, uint8_t* kv_s, const CUtensorMap* tm, uint64_t* kv_full,
                                             uint64_t* kv_empty, int r_lo, int r_n, int ntiles, int64_t row_base,
                                             volatile int* abort_flag) {
    uint32_t cnt = 0;
    bool ok = true;
    for (int jt = 0; ok && jt < ntiles; ++jt) {
        const int row = (int)(row_base + (int64_t)jt * kE);
        for (int mt = 0; mt < a.mtiles; ++mt, ++cnt) {
            const int slot = r_lo + (int)(cnt % (uint32_t)r_n);
            if (cnt >= (uint32_t)r_n &&
                !(ok = wait_or_abort(&kv_empty[slot], ((cnt / r_n) - 1) & 1, abort_flag, a.status)))
                break;
            uint8_t* dst = kv_s + (size_t)slot * 2 * kE * 128;
            tc::mbar_expect_tx(&kv_full[slot], 2 * kE * 128);
            tc::tma_load_2d(dst, tm, &kv_full[slot], 2 * mt * 64, row);
            tc::tma_load_2d(dst + kE * 128, tm, &kv_full[slot], (2 * mt + 1) * 64, row);
        }
    }
    // drain: the copies still in flight must land
    for (uint32_t i = cnt > (uint32_t)r_n ? cnt - r_n : 0; i < cnt; ++i)
        tc::mbar_wait(&kv_full[r_lo + i % r_n], (i / r_n) & 1, kWaitLimit);
}

__global__ void __launch_bounds__(kThreads, 1) mqa_tc_kernel(const __grid_constant__ MqaArgs a,
                                                             const __grid_constant__ CUtensorMap tmQ,
                                                             const __grid_constant__ CUtensorMap tmTile) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* kv_s = base;                                        // dblocks x 16 KB
    // KV area: sparse, one tile (dblocks x 16 KB); dense, a ring of `ring`
    // 32 KB slots
    const size_t kv_bytes = a.ring ? (size_t)a.ring * 2 * kE * 128 : (size_t)a.dblocks * kE * 128;
    uint8_t* q_s = kv_s + kv_bytes;                              // dblocks x hg*128
    uint8_t* p_s = q_s + a.q_bytes;                              // 128 x 128 B
    float* mref_s = (float*)(p_s + kE * 128);                    // [64]
    float* alpha_s = mref_s + 64;                                // [64]
    float* red_s = alpha_s + 64;                                 // [4][64]
    float* lsum_s = red_s + 256;                                 // [64]
    uint64_t* bars = (uint64_t*)(lsum_s + 64);
    uint64_t* kv_full = bars;                                    // [8]
    uint64_t* kv_empty = bars + kMaxDBlocks;                     // [8]
    uint64_t* s_full = bars + 2 * kMaxDBlocks;                   // [2]
    uint64_t* s_empty = s_full + 2;                              // [2]
    uint64_t* q_full = s_empty + 2;
    uint64_t* p_full = q_full + 1;
    uint64_t* o_done = p_full + 1;
    uint64_t* fin = o_done + 1;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ float merge_coef[kMaxClusterSplits][64];   // cluster merge: each split's weight per head

    pdl_wait();
    pdl_launch_next();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.z;
    const int h0 = blockIdx.y * a.hg;
    const int split = blockIdx.x;
    const int seq = a.qm.seq_of(t);
    const bool seq_ok = seq >= 0 && seq < a.n_seq;
    int64_t n_ent = 0;
    if (seq_ok) n_ent = a.idx ? (int64_t)a.k : visible_entries(a.qm.pos_of(t), a.mp, a.Nmax);
    const int64_t e_beg = (int64_t)split * a.split_len;
    int64_t e_end = e_beg + a.split_len;
    if (e_end > n_ent) e_end = n_ent;
    const int ntiles = e_end > e_beg ? (int)((e_end - e_beg + kE - 1) / kE) : 0;
    const int64_t row0 = (int64_t)(seq_ok ? seq : 0) * a.Nmax;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kMaxDBlocks; ++i) { tc::mbar_init(&kv_full[i], 1); tc::mbar_init(&kv_empty[i], 1); }
        // sparse: both issuers commit their half of S and of O; dense: the
        // first issuer makes S, the second O
        const uint32_t nis = a.idx ? 2u : 1u;
        for (int i = 0; i < 2; ++i) { tc::mbar_init(&s_full[i], nis); tc::mbar_init(&s_empty[i], 4); }
        tc::mbar_init(q_full, 1);
        tc::mbar_init(p_full, 4);
        tc::mbar_init(o_done, nis);
        tc::mbar_init(fin, 2);
        tc::fence_mbar_init();
        s_abort = 0;
    }
    if (warp == 1) {
        tc::tmem_alloc(&s_tmem, a.tmem_cols);
        tc::tmem_relinquish();
        tc::tc_fence_before();
    }
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = s_tmem;
    // S^T (double-buffered); sparse: the second issuer's half of S^T beside
    // it; then O^T (mtiles x hg columns)
    const uint32_t tmem_S = tmem;                                      // 2 x hg columns
    const uint32_t tmem_SB = tmem + 2 * (uint32_t)a.hg;                // 2 x hg columns (sparse)
    const uint32_t tmem_O = tmem + (a.idx ? 4u : 2u) * (uint32_t)a.hg; // mtiles x hg columns
    volatile int* abort_flag = &s_abort;

    if (warp == 0) {
        // ---------------------------------------------------------------- loads
        if (ntiles > 0) {
            if (lane == 0) {
                tc::mbar_expect_tx(q_full, a.q_bytes);
                for (int b = 0; b < a.dblocks; ++b)
                    tc::tma_load_2d(q_s + (size_t)b * a.hg * 128, &tmQ, q_full, b * 64, t * a.H + h0);
            }
            int j = 0;
            if (a.idx) {
                // Sparse rows: 16-byte cp.async by the whole warp. One warp
                // instruction moves one 64-dim block (128 B) of four rows, so
                // every access is a full, aligned 128-byte line; the chunk
                // lands at its 128-byte-swizzle position. (A TMA gather4 moves
                // the same 512 B per instruction but its issue rate, not DRAM,
                // bounded the tile load.) Block b is handed to the MMA once
                // this warp's copies of it have completed.
                const int chunk = lane & 7, rsub = lane >> 3;
                const char* kv_g = (const char*)a.KV;
                const int64_t row_bytes = (int64_t)a.c * 2;
                for (; j < ntiles; ++j) {
                    const int64_t e0 = e_beg + (int64_t)j * kE;
                    int rows[kE / 4];
#pragma unroll
                    for (int i = 0; i < kE / 4; ++i) {
                        const int64_t e = e0 + 4 * i + rsub;
                        int s = -1;
                        if (e < e_end) s = a.idx[(int64_t)t * a.k + e];
                        if (s < 0 || s >= a.Nmax) s = 0;   // masked in the softmax
                        rows[i] = (int)(row0 + s);
                    }
                    bool ok = true;
                    for (int b = 0; b < a.dblocks; ++b) {
                        if (j > 0 && lane == 0) ok = wait_or_abort(&kv_empty[b], (j - 1) & 1, abort_flag, a.status);
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (!ok) break;
                        uint8_t* dst = kv_s + (size_t)b * kE * 128;
#pragma unroll
                        for (int i = 0; i < kE / 4; ++i) {
                            const int r = 4 * i + rsub;
                            cp_async16(dst + r * 128 + ((chunk ^ (r & 7)) << 4),
                                       kv_g + (int64_t)rows[i] * row_bytes + b * 128 + chunk * 16);
                        }
                        cp_async_commit();
                    }
                    // hand the blocks over in order as they complete
                    const int issued = ok ? a.dblocks : 0;
                    for (int b = 0; b < issued; ++b) {
                        cp_async_wait_pending(issued - 1 - b);
                        tc::fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) tc::mbar_arrive(&kv_full[b]);
                    }
                    if (!ok) {
                        cp_async_wait_pending(0);
                        break;
                    }
                }
            } else if (lane == 0) {
                // Dense rows stream through the ring twice per tile, pair by
                // pair of 64-dim blocks: for the first product (S) through
                // this thread's ring, and again (mostly from L2) for the
                // second (O) through warp 7's ring
                dense_ring_load(a, kv_s, &tmTile, kv_full, kv_empty, 0, a.ring / 2, ntiles, row0 + e_beg, abort_flag);
                j = 0;
            }
            // drain (sparse): the last issued tile and q must have landed
            if (a.idx && lane == 0 && j > 0)
                for (int b = 0; b < a.dblocks; ++b) tc::mbar_wait(&kv_full[b], (j - 1) & 1, kWaitLimit);
            if (lane == 0) tc::mbar_wait(q_full, 0, kWaitLimit);
        }
    } else if (warp == 7) {
        // ---------------------------------------------------------------- dense: O-pass ring
        if (!a.idx && lane == 0 && ntiles > 0)
            dense_ring_load(a, kv_s, &tmTile, kv_full, kv_empty, a.ring / 2, a.ring - a.ring / 2, ntiles,
                            row0 + e_beg, abort_flag);
    } else if (warp == 1 || warp == 6) {
        // ---------------------------------------------------------------- MMA
        // Two issuing threads (each tcgen05.mma costs its issuer tens of
        // ns, and a tile takes 32 for S and 32 for O). Sparse: issuer mi
        // accumulates S^T over its half of the 64-dim blocks into its own
        // accumulator (the softmax adds the two) and O^T for the dim tiles
        // mt with mt % 2 == mi; both wait for the same phases of every
        // barrier they share, in the same order. Dense: issuer 0 makes S from
        // the S-pass ring, issuer 1 makes O from the O-pass ring; each ring
        // has one producer and one consumer, which take its slots' phases in
        // order (a parity wait can only tell consecutive phases apart).
        const int mi = warp == 6 ? 1 : 0;
        if (lane == 0 && ntiles > 0) {
            const uint32_t idesc1 = tc::idesc_bf16_f32(128, a.hg, 0, 0);
            const uint32_t idesc2 = tc::idesc_bf16_f32(128, a.hg, 1, 1);
            const uint32_t kv_addr = tc::smem_u32(kv_s);
            const uint32_t q_addr = tc::smem_u32(q_s);
            const uint32_t p_addr = tc::smem_u32(p_s);
            bool ok = wait_or_abort(q_full, 0, abort_flag, a.status);
            int j = 0;
            if (!a.idx) {
                // dense: this issuer's ring, in the order its producer fills it
                const int r_lo = mi ? a.ring / 2 : 0, r_n = mi ? a.ring - a.ring / 2 : a.ring / 2;
                uint32_t cnt = 0;
                for (int jt = 0; ok && jt < ntiles; ++jt) {
                    const int sb = jt & 1;
                    if (mi == 0) {
                        if (jt >= 2 && !(ok = wait_or_abort(&s_empty[sb], ((jt >> 1) - 1) & 1, abort_flag, a.status)))
                            break;
                    } else {
                        if (!(ok = wait_or_abort(p_full, jt & 1, abort_flag, a.status))) break;
                        tc::tc_fence_after();
                    }
                    for (int mt = 0; mt < a.mtiles; ++mt, ++cnt) {
                        const int slot = r_lo + (int)(cnt % (uint32_t)r_n);
                        if (!(ok = wait_or_abort(&kv_full[slot], (cnt / r_n) & 1, abort_flag, a.status))) break;
                        tc::tc_fence_after();
                        const uint32_t sa = kv_addr + (uint32_t)slot * 2 * kE * 128;
                        if (mi == 0) {
                            // S^T += KV[:, blocks 2mt, 2mt+1] . q[:, same]^T
                            for (int bb = 0; bb < 2; ++bb)
                                for (int kk = 0; kk < 4; ++kk) {
                                    uint64_t ad = tc::sdesc_sw128(sa + bb * (kE * 128) + kk * 32, 16, 1024);
                                    uint64_t bd = tc::sdesc_sw128(q_addr + (2 * mt + bb) * (a.hg * 128) + kk * 32,
                                                                  16, 1024);
                                    tc::umma_bf16(tmem_S + sb * a.hg, ad, bd, idesc1, (mt | bb | kk) ? 1u : 0u);
                                }
                        } else {
                            // O^T[dims of mt] += KV^T . P^T
                            for (int ke = 0; ke < kE / 16; ++ke) {
                                uint64_t ad = tc::sdesc_sw128(sa + ke * 2048, kE * 128, 1024);
                                uint64_t bd = tc::sdesc_sw128(p_addr + ke * 2048, kE * 128, 1024);
                                tc::umma_bf16(tmem_O + mt * a.hg, ad, bd, idesc2, (jt > 0 || ke > 0) ? 1u : 0u);
                            }
                        }
                        tc::umma_commit(&kv_empty[slot]);
                    }
                    if (!ok) break;
                    tc::umma_commit(mi == 0 ? &s_full[sb] : o_done);
                }
                j = ntiles;   // skip the sparse loop below
            }
            const int b_lo = mi * (a.dblocks / 2), b_hi = b_lo + a.dblocks / 2;
            const uint32_t my_S = mi ? tmem_SB : tmem_S;
            for (; ok && j < ntiles; ++j) {
                const int sb = j & 1;
                if (j >= 2 && !(ok = wait_or_abort(&s_empty[sb], ((j >> 1) - 1) & 1, abort_flag, a.status))) break;
                // this issuer's part of S^T = KV . q^T (its 64-dim blocks)
                for (int b = b_lo; b < b_hi && ok; ++b) {
                    if (!(ok = wait_or_abort(&kv_full[b], j & 1, abort_flag, a.status))) break;
                    tc::tc_fence_after();
                    for (int kk = 0; kk < 4; ++kk) {
                        uint64_t ad = tc::sdesc_sw128(kv_addr + b * (kE * 128) + kk * 32, 16, 1024);
                        uint64_t bd = tc::sdesc_sw128(q_addr + b * (a.hg * 128) + kk * 32, 16, 1024);
                        tc::umma_bf16(my_S + sb * a.hg, ad, bd, idesc1, (b > b_lo || kk) ? 1u : 0u);
                    }
                }
                if (!ok) break;
                tc::umma_commit(&s_full[sb]);
                // O^T += KV^T . P^T once the softmax has written P
                if (!(ok = wait_or_abort(p_full, j & 1, abort_flag, a.status))) break;
                tc::tc_fence_after();
                for (int mt = mi; mt < a.mtiles; mt += 2) {
                    for (int ke = 0; ke < kE / 16; ++ke) {
                        uint64_t ad = tc::sdesc_sw128(kv_addr + (2 * mt) * (kE * 128) + ke * 2048, kE * 128, 1024);
                        uint64_t bd = tc::sdesc_sw128(p_addr + ke * 2048, kE * 128, 1024);
                        tc::umma_bf16(tmem_O + mt * a.hg, ad, bd, idesc2, (j > 0 || ke > 0) ? 1u : 0u);
                    }
                    tc::umma_commit(&kv_empty[2 * mt]);
                    tc::umma_commit(&kv_empty[2 * mt + 1]);
                }
                tc::umma_commit(o_done);
            }
            // a last commit covers every MMA this thread issued (also on abort)
            tc::umma_commit(fin);
            tc::mbar_wait(fin, 0, kWaitLimit);
        }
    } else if (warp < 6) {
        // ---------------------------------------------------------------- softmax + epilogue
        const int quad = warp & 3;
        const int row = quad * 32 + lane;            // entry within the tile / dim within an M tile
        const int eth = threadIdx.x - 64;            // 0..127
        const int hg = a.hg;
        if (eth < 64) { mref_s[eth] = -INFINITY; lsum_s[eth] = 0.f; }
        float lpart[64];
#pragma unroll
        for (int h = 0; h < 64; ++h) lpart[h] = 0.f;
        bar_sync_128();
        bool ok = true;
        int j = 0;
        for (; j < ntiles; ++j) {
            const int sb = j & 1;
            // this row's entry (its index is read before the wait, so the
            // load's latency hides behind it)
            const int64_t e = e_beg + (int64_t)j * kE + row;
            bool valid = e < e_end;
            if (valid && a.idx) {
                int s = a.idx[(int64_t)t * a.k + e];
                valid = s >= 0 && s < a.Nmax;
            }
            if (!(ok = wait_or_abort(&s_full[sb], (j >> 1) & 1, abort_flag, a.status))) break;
            tc::tc_fence_after();
            float z[64];
            const uint32_t taddr = tmem_S + ((uint32_t)(quad * 32) << 16) + sb * hg;
            const uint32_t taddr_b = tmem_SB + ((uint32_t)(quad * 32) << 16) + sb * hg;
#pragma unroll
            for (int cc = 0; cc < 64; cc += 16) {
                if (cc < hg) {
                    float v[16];
                    tc::tmem_ld16(taddr + cc, v);
                    if (a.idx) {
                        // sparse: S^T is the sum of the two issuers' halves
                        float v2[16];
                        tc::tmem_ld16(taddr_b + cc, v2);
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] += v2[i];
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) z[cc + i] = v[i];
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) z[cc + i] = -INFINITY;
                }
            }
            tc::tmem_ld_wait();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&s_empty[sb]);
            bool need = false;
#pragma unroll
            for (int h = 0; h < 64; ++h) {
                z[h] = valid ? z[h] * a.scale_log2 : -INFINITY;
                need |= z[h] > mref_s[h] + kRescaleLog2;
            }
            if (bar_or_128(need)) {
                // new reference: per-head max over the tile's 128 entries. A
                // butterfly reduce-scatter over the warp leaves lane l with the
                // maxima of heads 2l and 2l+1 (62 shuffles instead of 320).
                {
                    float v[64];
#pragma unroll
                    for (int h = 0; h < 64; ++h) v[h] = z[h];
#pragma unroll
                    for (int r = 0; r < 5; ++r) {
                        const int o = 16 >> r, nh = 32 >> r;
                        const bool upper = (lane & o) != 0;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            if (i < nh) {
                                const float send = upper ? v[i] : v[i + nh];
                                const float keep = upper ? v[i + nh] : v[i];
                                v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, o));
                            }
                        }
                    }
                    red_s[quad * 64 + 2 * lane] = v[0];
                    red_s[quad * 64 + 2 * lane + 1] = v[1];
                }
                bar_sync_128();
                if (eth < 64) {
                    float old = mref_s[eth];
                    float nm = fmaxf(fmaxf(fmaxf(red_s[eth], red_s[64 + eth]), fmaxf(red_s[128 + eth], red_s[192 + eth])),
                                     old);
                    alpha_s[eth] = (old == -INFINITY) ? 0.f : exp2f(old - nm);
                    mref_s[eth] = nm;
                }
                bar_sync_128();
#pragma unroll
                for (int h = 0; h < 64; ++h) lpart[h] *= alpha_s[h];
                if (j > 0) {
                    // rescale O^T (all previous products must have landed)
                    if (!(ok = wait_or_abort(o_done, (j - 1) & 1, abort_flag, a.status))) break;
                    tc::tc_fence_after();
                    for (int mt = 0; mt < a.mtiles; ++mt) {
                        for (int cc = 0; cc < hg; cc += 16) {
                            float v[16];
                            const uint32_t oaddr = tmem_O + ((uint32_t)(quad * 32) << 16) + mt * hg + cc;
                            tc::tmem_ld16(oaddr, v);
                            tc::tmem_ld_wait();
#pragma unroll
                            for (int i = 0; i < 16; ++i) v[i] *= alpha_s[cc + i];
                            tc::tmem_st16(oaddr, v);
                        }
                    }
                    tc::tmem_st_wait();
                    tc::tc_fence_before();
                }
            }
            // P = 2^(z - m), rows of 64 bf16 (128 bytes), 128-byte swizzle
            uint32_t pk[32];
#pragma unroll
            for (int h = 0; h < 64; h += 2) {
                float p0 = (z[h] == -INFINITY) ? 0.f : exp2f(z[h] - mref_s[h]);
                float p1 = (z[h + 1] == -INFINITY) ? 0.f : exp2f(z[h + 1] - mref_s[h + 1]);
                lpart[h] += p0;
                lpart[h + 1] += p1;
                __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                pk[h >> 1] = *reinterpret_cast<uint32_t*>(&b2);
            }
            // the previous tile's second product must be done reading P
            if (j > 0 && !(ok = wait_or_abort(o_done, (j - 1) & 1, abort_flag, a.status))) break;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint4 v = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
                *reinterpret_cast<uint4*>(p_s + row * 128 + ((ch ^ (row & 7)) * 16)) = v;
            }
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(p_full);
        }
        // ------------------------------------------------------------ epilogue
        if (ok && ntiles > 0) ok = wait_or_abort(o_done, (ntiles - 1) & 1, abort_flag, a.status);
        tc::tc_fence_after();
        // per-head sums of the 128 per-entry partials (fixed order): a
        // butterfly reduce-scatter within each warp leaves lane l with the
        // warp's sums of heads 2l and 2l+1 (62 shuffles), then the four warps'
        // sums are added through shared memory
        {
#pragma unroll
            for (int r = 0; r < 5; ++r) {
                const int o = 16 >> r, nh = 32 >> r;
                const bool upper = (lane & o) != 0;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if (i < nh) {
                        const float send = upper ? lpart[i] : lpart[i + nh];
                        const float keep = upper ? lpart[i + nh] : lpart[i];
                        lpart[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                    }
                }
            }
            bar_sync_128();   // red_s may still be read by the last max update
            red_s[quad * 64 + 2 * lane] = lpart[0];
            red_s[quad * 64 + 2 * lane + 1] = lpart[1];
            bar_sync_128();
            if (eth < 64)
                lsum_s[eth] = (red_s[eth] + red_s[64 + eth]) + (red_s[128 + eth] + red_s[192 + eth]);
            bar_sync_128();
        }
        const bool have_o = ok && ntiles > 0;
        if (a.cluster) {
            // stage this split's O^T as obuf[head][dim] (fp32) where the KV
            // tile was; the combine after the role branches reads it
            float* obuf = (float*)kv_s;
            if (eth < 64 && !have_o) { mref_s[eth] = -INFINITY; lsum_s[eth] = 0.f; }
            if (have_o) {
                for (int mt = 0; mt < a.mtiles; ++mt) {
                    const int dim = mt * 128 + row;
                    float v[64];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        tc::tmem_ld16(tmem_O + ((uint32_t)(quad * 32) << 16) + mt * hg + 16 * u,
                                      *reinterpret_cast<float(*)[16]>(v + 16 * u));
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 64; ++i) obuf[i * a.c + dim] = v[i];
                }
            }
        } else if (a.nsplit == 1) {
            // normalise: denominator = sum + sink term (same reference max)
            if (eth < 64) {
                const int h = h0 + eth;
                float m = mref_s[eth];
                float L = lsum_s[eth];
                float sk = (a.sink && h < a.H) ? a.sink[h] * 1.4426950408889634f : -INFINITY;
                float lse;
                if (m == -INFINITY) {              // no visible entry
                    alpha_s[eth] = 0.f;
                    lse = (sk == -INFINITY) ? -INFINITY : sk * 0.6931471805599453f;
                } else {
                    float Lt = L + ((sk == -INFINITY) ? 0.f : exp2f(sk - m));
                    alpha_s[eth] = 1.f / Lt;
                    lse = (m + log2f(Lt)) * 0.6931471805599453f;
                }
                if (a.lse && h < a.H) a.lse[(int64_t)t * a.H + h] = lse;
            }
            bar_sync_128();
            // the normalised O goes through shared memory (the KV area,
            // [head][dim] bf16) so that the output rows leave in 16-byte
            // stores: a thread holds one dim of every head, and 2-byte
            // stores at a head stride are slow
            bf16* stage = reinterpret_cast<bf16*>(kv_s);
            for (int mt = 0; mt < a.mtiles; ++mt) {
                const int dim = mt * 128 + row;
                float v[64];
                if (have_o) {
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        tc::tmem_ld16(tmem_O + ((uint32_t)(quad * 32) << 16) + mt * hg + 16 * u,
                                      *reinterpret_cast<float(*)[16]>(v + 16 * u));
                    tc::tmem_ld_wait();
                }
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    const float o = (have_o && mref_s[i] != -INFINITY) ? v[i] * alpha_s[i] : 0.f;
                    stage[i * a.c + dim] = __float2bfloat16_rn(o);
                }
            }
            bar_sync_128();
            const int nh = a.H - h0 < 64 ? a.H - h0 : 64;
            const int cpr = a.c / 8;   // 16-byte chunks per head row
            for (int e = eth; e < nh * cpr; e += 128) {
                const int i = e / cpr, ch = e - i * cpr;
                *reinterpret_cast<uint4*>(a.out + ((int64_t)t * a.H + h0 + i) * a.c + ch * 8) =
                    *reinterpret_cast<const uint4*>(stage + i * a.c + ch * 8);
            }
        } else {
            if (eth < 64 && h0 + eth < a.H) {
                float* pm = a.part_ml + (((int64_t)t * a.nsplit + split) * a.H + h0 + eth) * 2;
                pm[0] = (have_o && mref_s[eth] != -INFINITY) ? mref_s[eth] * 0.6931471805599453f : -INFINITY;
                pm[1] = have_o ? lsum_s[eth] : 0.f;
            }
            if (have_o) {
                for (int mt = 0; mt < a.mtiles; ++mt) {
                    const int dim = mt * 128 + row;
                    float v[64];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        tc::tmem_ld16(tmem_O + ((uint32_t)(quad * 32) << 16) + mt * hg + 16 * u,
                                      *reinterpret_cast<float(*)[16]>(v + 16 * u));
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 64; ++i) {
                        const int h = h0 + i;
                        if (h < a.H) a.part_o[(((int64_t)t * a.nsplit + split) * a.H + h) * a.c + dim] = v[i];
                    }
                }
            }
        }
        tc::tc_fence_before();
    }

    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, a.tmem_cols);
    }
    if (a.cluster) {
        if (a.nsplit <= 2)
            cluster_merge<2>(a.nsplit, a.c, a.H, a.sink, a.lse, a.out, t, h0, split, (float*)kv_s, mref_s, lsum_s,
                             merge_coef);
        else if (a.nsplit <= 4)
            cluster_merge<4>(a.nsplit, a.c, a.H, a.sink, a.lse, a.out, t, h0, split, (float*)kv_s, mref_s, lsum_s,
                             merge_coef);
        else
            cluster_merge<8>(a.nsplit, a.c, a.H, a.sink, a.lse, a.out, t, h0, split, (float*)kv_s, mref_s, lsum_s,
                             merge_coef);
    }
}

bool mqa_tc_supported(int H, int c) { return c % 128 == 0 && c <= 512 && H >= 1; }

int mqa_tc_nsplit(int nq, int H, int64_t max_entries, int num_sms) {
    const int hgroups = (H + 63) / 64;
    const int64_t ctas = (int64_t)nq * hgroups;
    int64_t ns = ctas > 0 ? num_sms / ctas : 1;
    const int64_t tiles = (max_entries + kE - 1) / kE;
    if (ns > tiles) ns = tiles;
    if (ns < 1) ns = 1;
    if (ns > 64) ns = 64;
    // splits are whole tiles: as many as the tiles per split need (9 splits
    // of 64 tiles take 8 tiles each, so 8 splits do the same work)
    if (tiles > 0) ns = (tiles + (tiles + ns - 1) / ns - 1) / ((tiles + ns - 1) / ns);
    return (int)ns;
}

// Whether the nsplit splits of every (query, head group) run as one cluster
// and merge on chip: clusters of up to 4 one-CTA-per-SM blocks always; of 5
// to 8 only when every cluster of the launch can be resident at once (the
// device's count of such clusters, asked once per cluster size).
bool mqa_tc_cluster(int nsplit, int nq, int H) {
    if (nsplit < 2 || nsplit > kMaxClusterSplits) return false;
    if (nsplit <= 4) return true;
    static std::mutex mu;
    static int dev_seen[kMaxClusterSplits + 1][64];   // per (cluster size, device): 0 unknown, else count + 1
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lock(mu);
    int& cached = dev_seen[nsplit][dev];
    if (cached == 0) {
        int n = 0;
        if (smem_ceiling(mqa_tc_kernel) == cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = (unsigned)nsplit;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.gridDim = dim3((unsigned)nsplit, 1, 1);
            cfg.blockDim = dim3(kThreads);
            cfg.dynamicSmemBytes = 200 * 1024;   // one CTA per SM, as every launch of this kernel
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n, mqa_tc_kernel, &cfg) != cudaSuccess) {
                (void)cudaGetLastError();
                n = 0;
            }
        }
        cached = n + 1;
    }
    const int64_t clusters = (int64_t)nq * ((H + 63) / 64);
    return clusters <= (int64_t)(cached - 1);
}

cudaError_t mqa_tc(const void* q, const void* KV, const int32_t* idx, int k, QuerySpec qs, int mp, int nq, int n_seq,
                   int H, int c, int64_t Nmax, float scale, const float* sink, void* out, float* lse, void* ws,
                   int nsplit, int* status, cudaStream_t st) {
    if (nq == 0) return cudaSuccess;
    MqaArgs a{};
    a.qm = QueryMap{qs.seq, qs.pos, qs.pos_base, qs.single_seq};
    a.n_seq = n_seq;
    a.mp = mp;
    a.KV = KV;
    a.idx = idx;
    a.k = k;
    a.nq = nq;
    a.H = H;
    a.c = c;
    a.hg = 64;   // heads per CTA; smaller H pads with rows that are never written out
    a.Nmax = Nmax;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.sink = sink;
    a.nsplit = nsplit;
    a.cluster = mqa_tc_cluster(nsplit, nq, H) ? 1 : 0;
    const int64_t max_entries = idx ? k : Nmax;
    int64_t per = (max_entries + nsplit - 1) / nsplit;
    a.split_len = ((per + kE - 1) / kE) * kE;
    if (a.split_len == 0) a.split_len = kE;
    a.out = (bf16*)out;
    a.lse = lse;
    a.part_o = (float*)ws;
    a.part_ml = (float*)((char*)ws + align256((size_t)nq * nsplit * H * c * sizeof(float)));
    a.status = status;
    a.dblocks = c / 64;
    a.mtiles = c / 128;
    a.q_bytes = (uint32_t)(a.hg * c * 2);
    uint32_t need = (idx ? 4 : 2) * a.hg + a.mtiles * a.hg, cols = 32;
    while (cols < need) cols <<= 1;
    a.tmem_cols = cols;

    CUtensorMap tmQ, tmTile;
    if (!make_tmap_bf16_2d(&tmQ, q, (uint64_t)nq * H, c, c, a.hg, 64)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_2d(&tmTile, KV, (uint64_t)n_seq * Nmax, c, c, kE, 64)) return cudaErrorInvalidValue;

    const size_t fixed = 1024 + a.q_bytes + kE * 128 + (64 * 4 + 256) * sizeof(float) + 32 * sizeof(uint64_t);
    size_t kv_bytes = (size_t)a.dblocks * kE * 128;
    if (!idx) {
        // dense ring: as many 32 KB slots as fit (at most 8, at least the
        // KV tile's size so the staging areas that reuse it still fit, and
        // at least 2: half the slots carry the S pass, half the O pass)
        // (4 KB left for the kernel's static shared memory)
        int ring = (int)((223 * 1024 - fixed) / (2 * kE * 128));
        if (ring > kMaxDBlocks) ring = kMaxDBlocks;
        if (ring < a.mtiles) ring = a.mtiles;
        if (ring < 2) ring = 2;
        a.ring = ring;
        kv_bytes = (size_t)ring * 2 * kE * 128;
    }
    const size_t smem = fixed + kv_bytes;
    cudaError_t e = smem_ceiling(mqa_tc_kernel);
    if (e != cudaSuccess) return e;
    cudaError_t le = cudaSuccess;
    CSA_LAUNCH(st, "mqa_tc",
               le = launch_pdl(mqa_tc_kernel, dim3(nsplit, (H + a.hg - 1) / a.hg, nq), dim3(kThreads), smem, st,
                               a.cluster ? (unsigned)nsplit : 0u, a, tmQ, tmTile));
    if (le != cudaSuccess) return le;
    return cudaGetLastError();
}

}  // namespace csa
