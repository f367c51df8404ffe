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
// gathered with 16-byte cp.async (two producer warps, half the rows each; a
// warp moves four rows' 128-byte block per instruction), and the tile's
// 64-dim blocks are released
// one by one as the second product finishes with them, so the next tile's
// gather overlaps it. HCA (dense): consecutive rows stream through two rings
// of 32 KB slots (a pair of 64-dim blocks per slot, one TMA box per block):
// every tile passes through twice, once through the S ring for the first
// product and again (mostly from L2) through the O ring for the second, each
// ring with its own loading thread and its own MMA-issuing thread, so the
// HBM read of the next tiles runs while tile j waits for its softmax.
//
// Warp roles: warps 0 and 7 load (sparse: all their lanes gather, half a
// tile each; dense: one lane each fills the S ring and the O ring), warp 1
// allocates TMEM, one lane each of warps 1 and 6 issues MMAs, warps 2-5 run
// the softmax and the epilogue.
// A single split writes the normalised output directly. More splits stage
// their unnormalised O^T (fp32, [head][dim]) in the shared memory the KV
// tile used, and one thread writes it to the workspace with bulk copies,
// beside the split's reference maxima and sums; mqa_combine then merges the
// splits in split order (deterministic). Waits are bounded (CSA_ERR_TIMEOUT).
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tmap.h"

namespace csa {

namespace {

// warps 0 and 7 load, warps 1 and 6 issue MMAs (warp 1 also owns TMEM),
// warps 2-5 run the softmax and the epilogue
constexpr int kThreads = 256;
constexpr int kE = 128;                 // entries per tile
constexpr int kMaxDBlocks = 8;          // c <= 512
constexpr uint32_t kWaitLimit = 1u << 24;
constexpr float kRescaleLog2 = 8.0f;    // move the reference max past 2^8

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
    int pair;                 // nsplit == 2: the query's two splits form a cluster and merge on chip
    RowBlocks kvb;            // where the cache rows live (sparse gather)
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

// Sparse rows: 16-byte cp.async by whole warps, kGatherWarps of them, warp
// `part` taking rows [part, part + 1) * kE / kGatherWarps of every tile. One
// warp instruction moves one 64-dim block (128 B) of four rows, so every
// access is a full, aligned 128-byte line; the chunk lands at its
// 128-byte-swizzle position. (A TMA gather4 moves the same 512 B per
// instruction but its issue rate, not DRAM, bounded the tile load.) Each
// warp arrives on block b's barrier once its copies of it have completed.
// Returns the tiles handed over.
constexpr int kGatherWarps = 2;
template <bool kBlk>
__device__ __forceinline__ int sparse_gather(const MqaArgs& a, uint8_t* kv_s, uint64_t* kv_full, uint64_t* kv_empty,
                                             int part, int lane, int t, int ntiles, int64_t e_beg, int64_t e_end,
                                             int64_t row0, volatile int* abort_flag) {
    constexpr int kRows = kE / kGatherWarps;   // rows per warp per tile
    const int chunk = lane & 7, rsub = lane >> 3;
    const char* kv_g = (const char*)a.KV;
    const int64_t row_bytes = (int64_t)a.c * 2;
    int j = 0;
    for (; j < ntiles; ++j) {
        const int64_t e0 = e_beg + (int64_t)j * kE + part * kRows;
        // rows: the row indices (contiguous cache), or their byte offsets
        // (rows in blocks)
        std::conditional_t<kBlk, int64_t, int> rows[kRows / 4];
#pragma unroll
        for (int i = 0; i < kRows / 4; ++i) {
            const int64_t e = e0 + 4 * i + rsub;
            int s = -1;
            if (e < e_end) s = a.idx[(int64_t)t * a.k + e];
            if (s < 0 || s >= a.Nmax) s = 0;   // masked in the softmax
            if constexpr (kBlk) rows[i] = row_byte_offset(row0 + s, row_bytes, a.kvb);
            else rows[i] = (int)(row0 + s);
        }
        bool ok = true;
        for (int b = 0; b < a.dblocks; ++b) {
            if (j > 0 && lane == 0) ok = wait_or_abort(&kv_empty[b], (j - 1) & 1, abort_flag, a.status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            uint8_t* dst = kv_s + (size_t)b * kE * 128;
#pragma unroll
            for (int i = 0; i < kRows / 4; ++i) {
                const int r = part * kRows + 4 * i + rsub;
                const int64_t off = kBlk ? (int64_t)rows[i] : (int64_t)rows[i] * row_bytes;
                cp_async16(dst + r * 128 + ((chunk ^ (r & 7)) << 4), kv_g + off + b * 128 + chunk * 16);
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
    return j;
}

// Dense path: one ring of 32 KB slots (a pair of 64-dim blocks each),
// slots [r_lo, r_lo + r_n), filled with every tile of the split pair by pair,
// in order; one producer and one consumer per ring.
__device__ __noinline__ void dense_ring_load(const MqaArgs& a, uint8_t* kv_s, const CUtensorMap* tm, uint64_t* kv_full,
                                             uint64_t* kv_empty, int r_lo, int r_n, int ntiles, int64_t row_base,
                                             volatile int* abort_flag) {
    uint32_t cnt = 0;
    bool ok = true;
    // ring position without a division per slot: index, use parity, wrapped
    int pos = 0;
    uint32_t phase = 0;
    bool wrapped = false;
    for (int jt = 0; ok && jt < ntiles; ++jt) {
        const int row = (int)(row_base + (int64_t)jt * kE);
        for (int mt = 0; mt < a.mtiles; ++mt, ++cnt) {
            const int slot = r_lo + pos;
            if (wrapped && !(ok = wait_or_abort(&kv_empty[slot], phase ^ 1u, abort_flag, a.status))) break;
            if (++pos == r_n) {
                pos = 0;
                phase ^= 1u;
                wrapped = true;
            }
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

// The two splits of query t (a cluster of two, rank = split) merge on chip.
// Each has staged its unnormalised O^T as [half][head][dim in half] fp32; after
// a cluster barrier (both staged, maxima and sums final, receive areas free)
// one thread of each sends the other split's half to it with one bulk copy
// over distributed shared memory (into the peer's q area), counted on the
// peer's mbarrier. Both work out the two weights per head from both splits'
// reference maxima and sums and the sink (the same arithmetic on each side),
// then split g writes half g of every head: w0 O_0 + w1 O_1, in split order,
// 4 dims per 8-byte store. A last cluster barrier keeps each CTA's shared
// memory alive until the peer's copy of it has landed.
__device__ __noinline__ void pair_merge(int c, int H, const float* sink, float* lse_out, bf16* out, int t, int h0,
                                        uint32_t split, bool have_o, const float* obuf, float* recv, float* mref_s,
                                        float* lsum_s, uint64_t* xbar, float (*coef_s)[64], volatile int* abort_flag,
                                        int* status) {
    const int tid = threadIdx.x;
    const uint32_t peer = split ^ 1u;
    const int half = c / 2;
    const uint32_t bytes = 64u * (uint32_t)half * 4u;
    if (tid == 0) tc::mbar_expect_tx(xbar, bytes);
    if (tid < 64 && !have_o) { mref_s[tid] = -INFINITY; lsum_s[tid] = 0.f; }
    tc::cluster_sync();
    if (tid == 0)
        tc::bulk_copy_to_peer(tc::mapa(tc::smem_u32(recv), peer), obuf + (size_t)peer * 64 * half, bytes,
                              tc::mapa(tc::smem_u32(xbar), peer));
    if (tid < 64) {
        const int h = h0 + tid;
        const float sk = (sink && h < H) ? sink[h] * 1.4426950408889634f : -INFINITY;
        const float m_own = mref_s[tid], l_own = lsum_s[tid];
        const float m_peer = tc::ld_cluster_f32(tc::mapa(tc::smem_u32(mref_s + tid), peer));
        const float l_peer = tc::ld_cluster_f32(tc::mapa(tc::smem_u32(lsum_s + tid), peer));
        const float mq[2] = {split == 0 ? m_own : m_peer, split == 0 ? m_peer : m_own};
        const float lq[2] = {split == 0 ? l_own : l_peer, split == 0 ? l_peer : l_own};
        const float M = fmaxf(sk, fmaxf(mq[0], mq[1]));
        float L = (sk == -INFINITY) ? 0.f : exp2f(sk - M);
#pragma unroll
        for (int q = 0; q < 2; ++q)
            if (mq[q] != -INFINITY) L += lq[q] * exp2f(mq[q] - M);
        const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
        for (int q = 0; q < 2; ++q) coef_s[q][tid] = (mq[q] == -INFINITY) ? 0.f : exp2f(mq[q] - M) * inv;
        if (split == 0 && lse_out && h < H)
            lse_out[(int64_t)t * H + h] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
    }
    // every thread waits for the peer's half (a bounded wait: on a timeout the
    // status word says so and the half read below is stale)
    wait_or_abort(xbar, 0, abort_flag, status);
    __syncthreads();   // coef_s
    const float* mine = obuf + (size_t)split * 64 * half;
    const int nh = H - h0 < 64 ? H - h0 : 64;
    const int h4 = half / 4;
    for (int e = tid; e < nh * h4; e += kThreads) {
        const int i = e / h4, j = e - i * h4;
        const float4 va = *reinterpret_cast<const float4*>(mine + i * half + 4 * j);
        const float4 vb = *reinterpret_cast<const float4*>(recv + i * half + 4 * j);
        const float4 o0 = split == 0 ? va : vb, o1 = split == 0 ? vb : va;
        const float w0 = coef_s[0][i], w1 = coef_s[1][i];
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (w0 != 0.f) { acc.x = w0 * o0.x; acc.y = w0 * o0.y; acc.z = w0 * o0.z; acc.w = w0 * o0.w; }
        if (w1 != 0.f) {
            acc.x = fmaf(w1, o1.x, acc.x); acc.y = fmaf(w1, o1.y, acc.y);
            acc.z = fmaf(w1, o1.z, acc.z); acc.w = fmaf(w1, o1.w, acc.w);
        }
        store4(out + ((int64_t)t * H + h0 + i) * c + (int)split * half + 4 * j, acc.x, acc.y, acc.z, acc.w);
    }
    tc::cluster_sync();
}

// kBlk: the cache rows come in blocks (a separate instantiation, so that the
// contiguous path's gather stays as it was)
template <bool kBlk>
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
    uint64_t* xbar = fin + 1;   // pair merge: the peer's slice has arrived
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    __shared__ float pair_coef[2][64];   // pair merge: each split's weight per head

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
        // sparse: every gathering warp arrives on a block's full barrier
        for (int i = 0; i < kMaxDBlocks; ++i) {
            tc::mbar_init(&kv_full[i], a.idx ? (uint32_t)kGatherWarps : 1u);
            tc::mbar_init(&kv_empty[i], 1);
        }
        // sparse: both issuers commit their half of S and of O; dense: the
        // first issuer makes S, the second O
        const uint32_t nis = a.idx ? 2u : 1u;
        for (int i = 0; i < 2; ++i) { tc::mbar_init(&s_full[i], nis); tc::mbar_init(&s_empty[i], 4); }
        tc::mbar_init(q_full, 1);
        tc::mbar_init(p_full, 4);
        tc::mbar_init(o_done, nis);
        tc::mbar_init(fin, 2);
        tc::mbar_init(xbar, 1);
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
                j = sparse_gather<kBlk>(a, kv_s, kv_full, kv_empty, 0, lane, t, ntiles, e_beg, e_end, row0, abort_flag);
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
        // ---------------------------------------------------------------- loads: sparse second half, dense O ring
        if (a.idx) {
            if (ntiles > 0)
                sparse_gather<kBlk>(a, kv_s, kv_full, kv_empty, 1, lane, t, ntiles, e_beg, e_end, row0, abort_flag);
        } else if (lane == 0 && ntiles > 0) {
            dense_ring_load(a, kv_s, &tmTile, kv_full, kv_empty, a.ring / 2, a.ring - a.ring / 2, ntiles,
                            row0 + e_beg, abort_flag);
        }
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
                int pos = 0;          // ring position (no division per slot)
                uint32_t phase = 0;
                for (int jt = 0; ok && jt < ntiles; ++jt) {
                    const int sb = jt & 1;
                    if (mi == 0) {
                        if (jt >= 2 && !(ok = wait_or_abort(&s_empty[sb], ((jt >> 1) - 1) & 1, abort_flag, a.status)))
                            break;
                    } else {
                        if (!(ok = wait_or_abort(p_full, jt & 1, abort_flag, a.status))) break;
                        tc::tc_fence_after();
                    }
                    for (int mt = 0; mt < a.mtiles; ++mt) {
                        const int slot = r_lo + pos;
                        if (!(ok = wait_or_abort(&kv_full[slot], phase, abort_flag, a.status))) break;
                        if (++pos == r_n) {
                            pos = 0;
                            phase ^= 1u;
                        }
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
        if (a.nsplit == 1) {
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
            // stores (a thread holds one dim of every head). The heads'
            // factors are read into registers once (0 for a head without
            // entries): with them read from shared memory inside the staging
            // loop, every load waited behind the staging stores before it
            // and the loop took 15 us per query; storing each head's row
            // straight from registers (64 contiguous bytes per warp store)
            // measured 8.7 us, this 7.4 us.
            float al[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) al[i] = (have_o && mref_s[i] != -INFINITY) ? alpha_s[i] : 0.f;
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
                for (int i = 0; i < 64; ++i)
                    stage[i * a.c + dim] = __float2bfloat16_rn(al[i] != 0.f ? v[i] * al[i] : 0.f);
            }
            bar_sync_128();
            const int nh = a.H - h0 < 64 ? a.H - h0 : 64;
            const int cpr = a.c / 8;   // 16-byte chunks per head row
            for (int e = eth; e < nh * cpr; e += 128) {
                const int i = e / cpr, ch = e - i * cpr;
                *reinterpret_cast<uint4*>(a.out + ((int64_t)t * a.H + h0 + i) * a.c + ch * 8) =
                    *reinterpret_cast<const uint4*>(stage + i * a.c + ch * 8);
            }
        } else if (a.pair) {
            // stage O^T as [slice][head][dim in slice] fp32 where the KV tile
            // was (slice g = the half of the head dimension split g writes
            // out); the merge after the role branches sends the peer's half
            if (ntiles > 0) {
                float* obuf = (float*)kv_s;
                const int half = a.c / 2;
                // (a short loop body of 16 columns: code run once per block
                // is fetched cold, so a compact loop beats a long unrolled one)
#pragma unroll 1
                for (int k = 0; k < a.mtiles * 4; ++k) {
                    const int mt = k >> 2, u = k & 3;
                    const int dim = mt * 128 + row;
                    float* dst = obuf + (size_t)(dim / half) * 64 * half + dim % half + (size_t)(16 * u) * half;
                    float v[16];
                    tc::tmem_ld16(tmem_O + ((uint32_t)(quad * 32) << 16) + mt * hg + 16 * u, v);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) dst[i * half] = v[i];
                }
                tc::fence_proxy_async_smem();
            }
        } else {
            if (eth < 64 && h0 + eth < a.H) {
                float* pm = a.part_ml + (((int64_t)t * a.nsplit + split) * a.H + h0 + eth) * 2;
                pm[0] = (have_o && mref_s[eth] != -INFINITY) ? mref_s[eth] * 0.6931471805599453f : -INFINITY;
                pm[1] = have_o ? lsum_s[eth] : 0.f;
            }
            if (ntiles > 0) {   // (a block-uniform test: the barrier below takes all four warps)
                // O^T staged as [head][dim] fp32 where the KV tile was: this
                // split's heads h0.. are one contiguous block of part_o,
                // which one thread then writes with bulk copies
                float* obuf = (float*)kv_s;
#pragma unroll 1
                for (int k = 0; k < a.mtiles * 4; ++k) {
                    const int mt = k >> 2, u = k & 3;
                    float* dst = obuf + (size_t)(16 * u) * a.c + mt * 128 + row;
                    float v[16];
                    tc::tmem_ld16(tmem_O + ((uint32_t)(quad * 32) << 16) + mt * hg + 16 * u, v);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) dst[i * a.c] = v[i];
                }
                tc::fence_proxy_async_smem();
                bar_sync_128();
                if (eth == 0 && have_o) {
                    const int nh = a.H - h0 < 64 ? a.H - h0 : 64;
                    const uint32_t bytes = (uint32_t)nh * a.c * 4, chunk = 32768;
                    char* dst = (char*)(a.part_o + (((int64_t)t * a.nsplit + split) * a.H + h0) * a.c);
                    for (uint32_t off = 0; off < bytes; off += chunk)
                        tc::bulk_store(dst + off, (const char*)obuf + off, bytes - off < chunk ? bytes - off : chunk);
                    tc::bulk_commit();
                    tc::bulk_wait_all();
                }
            }
        }
        tc::tc_fence_before();
    }

    __syncthreads();
    if (a.pair)
        pair_merge(a.c, a.H, a.sink, a.lse, a.out, t, h0, (uint32_t)split, ntiles > 0 && !s_abort, (const float*)kv_s,
                   (float*)q_s, mref_s, lsum_s, xbar, pair_coef, abort_flag, a.status);
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, a.tmem_cols);
    }
}

bool mqa_tc_supported(int H, int c) { return c % 128 == 0 && c <= 512 && H >= 1; }

bool mqa_tc_pair(int nsplit) { return nsplit == 2; }

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

cudaError_t mqa_tc(const void* q, const void* KV, const int32_t* idx, int k, QuerySpec qs, int mp, int nq, int n_seq,
                   int H, int c, int64_t Nmax, float scale, const float* sink, void* out, float* lse, void* ws,
                   int nsplit, int* status, cudaStream_t st, RowBlocks kvb) {
    if (nq == 0) return cudaSuccess;
    if (kvb.rpb > 0 && (Nmax % kvb.rpb || (!idx && kvb.rpb != 1) || kvb.block_bytes % 16))
        return cudaErrorInvalidValue;
    MqaArgs a{};
    a.kvb = kvb;
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
    a.pair = mqa_tc_pair(nsplit) ? 1 : 0;
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
    // dense rows in blocks (one per block): the block is the row pitch
    const uint64_t kv_pitch = kvb.rpb ? (uint64_t)kvb.block_bytes / 2 : (uint64_t)c;
    if (!make_tmap_bf16_2d(&tmTile, KV, (uint64_t)n_seq * Nmax, c, kv_pitch, kE, 64)) return cudaErrorInvalidValue;

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
    auto kern = kvb.rpb ? mqa_tc_kernel<true> : mqa_tc_kernel<false>;
    cudaError_t e = smem_ceiling(kern);
    if (e != cudaSuccess) return e;
    cudaError_t le = cudaSuccess;
    CSA_LAUNCH(st, "mqa_tc",
               le = launch_pdl(kern, dim3(nsplit, (H + a.hg - 1) / a.hg, nq), dim3(kThreads), smem, st,
                               a.pair ? 2u : 0u, a, tmQ, tmTile));
    if (le != cudaSuccess) return le;
    return cudaGetLastError();
}

}  // namespace csa
