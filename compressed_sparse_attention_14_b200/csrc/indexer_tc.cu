// Lightning indexer on the 5th-generation tensor cores [Notes §1.1, equation
// I_{t,s}; Walk §2.3.1] ([Notes] = "DeepSeek-V4: 迈向高效百万级上下文智能" study
// notes; [Walk] = the mlpod.com walk-through of the DeepSeek-V4 report):
//   I[t][s] = sum_h w[t][h] * ReLU(qI[t][h] . K[s]),  s < floor(p_t / m).
//
// The head contraction is a dense GEMM: for a tile of 128 keys and a group
// of g queries that see the same entries (decode: g = 1; prefill: the m
// tokens of one compressed block share floor(p/m), so g = m),
//   S^T[key][(query, head)] = K_tile (128 x cI) . Q_group^T (cI x g*HI)
// runs as tcgen05.mma with M = 128 keys, N = g*HI (padded to a multiple of
// 16), K = cI, operands in shared memory with 128-byte swizzle, fp32
// accumulator in tensor memory. Each TMEM lane then holds one key's g*HI
// dot products, so the epilogue thread owning that lane reduces
// sum_h w_h * max(x_h, 0) with no cross-thread traffic.
//
// Persistent CTAs, one per SM. The (group, key tile) work list is cut into
// equal contiguous ranges, one per CTA (the visible length of each group is
// read on the device). Warp roles:
//   warp 0     TMA producer: the group's Q rows once per group, then the key
//              tiles through a ring of `stages` shared-memory buffers;
//   warps 1,10 one lane of each issues the MMAs of alternate tiles into one
//              of 2-4 accumulator buffers and commits their completion
//              (warp 1 also allocates TMEM). A single issuing thread was the
//              bottleneck: each tcgen05.mma costs its thread ~70 ns to issue,
//              so one thread issuing 8 per 32 KB key tile capped the stream
//              near 4 TB/s; two threads issuing alternate tiles bring it to
//              the memory rate;
//   warps 2-9  epilogue, two sets of four warps taking alternate tiles:
//              tcgen05.ld of the accumulator, ReLU/weight/head reduction,
//              coalesced fp32 score stores.
// Every wait is bounded; a timeout records CSA_ERR_TIMEOUT in the status
// word, stops all roles, drains the copies in flight and frees TMEM.
//
// FP8 variant [Notes §2.4 (low-precision indexer arithmetic) and §1.3
// (FP8 storage)]: q^I and K stored as e4m3 with one fp32 scale per query-head
// row and per key row; tcgen05.mma kind::f8f6f4 (K = 32 per instruction, so a
// 128-byte shared-memory row holds 128 channels). The scales are positive, so
// they leave the ReLU: sum_h w_h ReLU(sq_h sk x_h) = sk sum_h (w_h sq_h)
// ReLU(x_h). The caller passes w_h sq_h as the head weights and the key
// scales; the epilogue multiplies each key's sum by its scale.
//
// Top-k filter on the epilogue [Notes §1.1: the indexer's scores choose each
// query's k entries] (bf16, contiguous keys): instead of storing every
// score, the epilogue appends to the query's candidate list only the scores
// that can still be among its k largest, as 64-bit composite keys (order
// key << 32 | ~column); a small selection over the lists finishes the top-k.
// Per query it scores, each epilogue warp queues the scores that reach the
// current bound in shared memory (a ballot and one 8-byte store per taker:
// no global atomics in the per-tile path). Every 32 queued entries make a
// batch, one entry per lane: each lane inserts its entry's order key into a
// list of the kCandR largest keys it has been handed, the batch is reserved
// in the row's global list with one addition (whose result is first needed
// at the next batch, so its latency hides) and stored as 256 contiguous
// bytes. The warp then finds p_w, a lower bound of the kk-th largest key in
// its lanes' lists (kk = ceil(k / warps scoring the query)), and publishes
// it in shared memory: the listed keys belong to distinct columns, so at
// least k scores of the row reach min_w p_w over the warps scoring the
// query, which is therefore at most the row's k-th largest score. A score
// below the bound can never be selected; every other one is kept. The bound
// only rises, it is local to the CTA (a row split over two CTAs gets two
// valid bounds), and a row's list never holds more entries than it has
// visible columns. The bound is only tight when a CTA scores long stretches
// of a row (many rows per launch).
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tmap.h"

namespace csa {

namespace {

// warp 0 producer, warp 1 MMA issuer 0 (and TMEM owner), then the epilogue
// sets of 4 warps, then MMA issuer 1. The grouped prefill (N = 256: four
// queries of 64 heads) has four sets, each reducing one query's 64 columns
// of every tile, and the FP8 decode (256-key tiles: twice the epilogue work
// per byte) four sets taking every fourth tile, so that four epilogue warps
// share each SM sub-partition to hide the TMEM-read and arithmetic latency
// the tile time waits on; every other shape has two sets taking alternate
// tiles.
constexpr int kIssuers = 2;
__host__ __device__ constexpr int epi_warps(int kN, int kH = 1) { return (kN == 256 || (kN == 64 && kH == 2)) ? 16 : 8; }
__host__ __device__ constexpr int kernel_threads(int kN, int kH = 1) { return (epi_warps(kN, kH) + 3) * 32; }
constexpr int kKeys = 128;      // keys per MMA (M) and per TMA box
constexpr uint32_t kWaitLimit = 1u << 24;

struct IdxArgs {
    QueryMap qm;
    int nq, n_seq;
    int group;          // queries sharing one key stream
    int HI, cI;
    int npad;           // MMA N
    int kblocks;        // cI / 64
    int stages;
    int64_t Nmax;
    int m;
    const float* w;     // [nq][HI] (FP8: w times the query-head scale)
    const float* kscale;    // FP8: [n_seq * Nmax] key scales; nullptr for bf16
    int blk_elems;      // elements per 128-byte row of a tile (64 bf16, 128 e4m3)
    int key_rpb;        // keys in blocks of key_rpb rows (a 3D key map); 0: contiguous rows
    float* scores;      // [nq][ld] fp32, or bf16 values when score_bf16
    int score_bf16;
    int64_t ld;
    int* status;
    uint32_t stage_bytes, q_bytes, tmem_cols;
    uint32_t wait_limit;    // polls before a wait gives up (CSA_ERR_TIMEOUT)
    int skip_first_tile;    // failure-path test hook: the first key tile is never loaded
    int nbuf;           // TMEM accumulator buffers (2..4)
    int kpt;            // keys per tile: kKeys, or 2 * kKeys (FP8 decode: a
                        // 32 KB stage, so per-tile costs spread over 256 keys)
    uint64_t* cand;     // candidate lists [nq][cand_ld] (top-k filter), else nullptr
    uint32_t* cand_cnt; // [nq] entries appended to each list (zeroed before the launch)
    int64_t cand_ld;
    uint32_t cand_kk;   // keys each publishing warp vouches for: ceil(k / warps per query)
};

struct Smem {
    uint8_t* stage0;    // stages x stage_bytes
    uint8_t* q;         // q_bytes
    float* w;           // [8][256], one copy per epilogue warp
    uint64_t* full;     // [stages]
    uint64_t* empty;    // [stages]
    uint64_t* tfull;    // [4]
    uint64_t* tempty;   // [4]
    uint64_t* qfull;
    uint64_t* qempty;
    uint64_t* fin;
    uint8_t* cq;        // top-k filter: [8 warps][1-2 query slots] queue and lists (kCandSlotBytes each)
};

__device__ __forceinline__ Smem carve(uint8_t* base, const IdxArgs& a) {
    Smem s;
    s.stage0 = base;
    s.q = base + (size_t)a.stages * a.stage_bytes;
    s.w = (float*)(s.q + a.q_bytes);
    uint64_t* bars = (uint64_t*)(s.w + 8 * 256);
    s.full = bars;
    s.empty = bars + a.stages;
    s.tfull = bars + 2 * a.stages;
    s.tempty = s.tfull + 4;
    s.qfull = s.tempty + 4;
    s.qempty = s.qfull + 1;
    s.fin = s.qempty + 1;
    s.cq = (uint8_t*)(bars + 64);
    return s;
}

__device__ __forceinline__ int group_seq(const IdxArgs& a, int g) {
    int s = a.qm.seq_of(g * a.group);
    return (s >= 0 && s < a.n_seq) ? s : -1;
}
__device__ __forceinline__ int64_t group_visible(const IdxArgs& a, int g) {
    if (group_seq(a, g) < 0) return 0;
    return visible_entries(a.qm.pos_of(g * a.group), a.m, a.Nmax);
}
__device__ __forceinline__ int64_t group_tiles(const IdxArgs& a, int g) {
    return (group_visible(a, g) + a.kpt - 1) / a.kpt;
}

// Warp-cooperative: total tiles, and the (group, tile) at flat index `target`.
__device__ int64_t total_tiles(const IdxArgs& a, int ngroups, int lane) {
    int64_t sum = 0;
    for (int g0 = 0; g0 < ngroups; g0 += 32) {
        int g = g0 + lane;
        sum += (g < ngroups) ? group_tiles(a, g) : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    return sum;
}
__device__ void locate(const IdxArgs& a, int ngroups, int64_t target, int lane, int& g_out, int64_t& t_out) {
    int64_t base = 0;
    for (int g0 = 0; g0 < ngroups; g0 += 32) {
        int g = g0 + lane;
        int64_t c = (g < ngroups) ? group_tiles(a, g) : 0;
        int64_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int64_t tot = __shfl_sync(0xffffffffu, incl, 31);
        if (base + tot > target) {
            unsigned mask = __ballot_sync(0xffffffffu, base + incl > target);
            int L = __ffs(mask) - 1;
            int64_t excl = __shfl_sync(0xffffffffu, incl - c, L);
            g_out = g0 + L;
            t_out = target - (base + excl);
            return;
        }
        base += tot;
    }
    g_out = ngroups;
    t_out = 0;
}

// Iterator over this CTA's (group, tile) range.
struct Walk {
    int g;
    int64_t t, tiles_g;
    __device__ void start(const IdxArgs& a, int g0, int64_t t0) {
        g = g0;
        t = t0;
        tiles_g = (g < (a.nq + a.group - 1) / a.group) ? group_tiles(a, g) : 0;
    }
    __device__ void next(const IdxArgs& a, int ngroups) {
        if (++t < tiles_g) return;
        t = 0;
        do {
            ++g;
            tiles_g = (g < ngroups) ? group_tiles(a, g) : 1;
        } while (tiles_g == 0);
    }
    __device__ bool last_of_group() const { return t + 1 == tiles_g; }
};

// Position in a ring of n slots as the tile counter advances: slot, the
// parity of the slot's current use, and whether the ring has wrapped (the
// counter's quotient and remainder without a 64-bit division per tile).
struct RingPos {
    int n, slot = 0;
    uint32_t phase = 0;
    bool wrapped = false;
    __device__ explicit RingPos(int n_) : n(n_) {}
    __device__ void advance() {
        if (++slot == n) {
            slot = 0;
            phase ^= 1u;
            wrapped = true;
        }
    }
};

// Paired fp32: two values in one 64-bit register; d = a * b + c lane by
// lane, round to nearest (sm_100 packed FMA).
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// The head reduction of one key's accumulator row: sc[q] += sum over the
// heads h of query q of w[q][h] * max(x[q][h], 0), kRound columns per round
// (kRound / 16 TMEM loads in flight, one wait), four independent partial sums
// per 16 columns in paired fp32 FMAs (each lane rounds as a separate fmaf
// would).
// kN > 0: the row has kN columns and each query kHI heads, known at compile
// time (the loop unrolls and each 16-column block's query is a constant);
// kN == 0: npad and HI at run time.
template <int kN, int kHI, int kRound = 64>
__device__ __forceinline__ void head_reduce(uint32_t taddr, const float* wv, int npad, int HI, int group,
                                            float (&sc)[4]) {
    const int n = kN > 0 ? kN : npad;
#pragma unroll(kN > 0 ? 4 : 1)
    for (int c0 = 0; c0 < n; c0 += kRound) {
        float v[kRound];
#pragma unroll
        for (int u = 0; u < kRound / 16; ++u) {
            if (kN > 0 || c0 + 16 * u < n) {
                float* vv = v + 16 * u;
                tc::tmem_ld16(taddr + c0 + 16 * u, *reinterpret_cast<float(*)[16]>(vv));
            }
        }
        tc::tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < kRound / 16; ++u) {
            const int cc = c0 + 16 * u;
            if (kN > 0 || cc < n) {
                uint64_t p01 = 0, p23 = 0;
#pragma unroll
                for (int i = 0; i < 16; i += 4) {
                    const float4 w4 = *reinterpret_cast<const float4*>(wv + cc + i);
                    p01 = fma2(pack2(w4.x, w4.y),
                               pack2(fmaxf(v[16 * u + i], 0.f), fmaxf(v[16 * u + i + 1], 0.f)), p01);
                    p23 = fma2(pack2(w4.z, w4.w),
                               pack2(fmaxf(v[16 * u + i + 2], 0.f), fmaxf(v[16 * u + i + 3], 0.f)), p23);
                }
                float p4[4];
                unpack2(p01, p4[0], p4[1]);
                unpack2(p23, p4[2], p4[3]);
                const float part = (p4[0] + p4[1]) + (p4[2] + p4[3]);
                if constexpr (kN > 0) {
                    sc[cc / kHI] += part;
                } else {
                    const int gq = (group > 1) ? cc / HI : 0;
                    if (gq == 0) sc[0] += part;
                    else if (gq == 1) sc[1] += part;
                    else if (gq == 2) sc[2] += part;
                    else sc[3] += part;
                }
            }
        }
    }
}

// ---- top-k filter helpers
constexpr int kCandR = 8;                  // order keys each thread keeps per query
constexpr uint32_t kTagNone = 0xFFFFFFFFu; // no bound published yet

// Insert order key u into the descending list t (u = 0 leaves it as it is).
__device__ __forceinline__ void cand_insert(uint32_t (&t)[kCandR], uint32_t u) {
#pragma unroll
    for (int i = 0; i < kCandR; ++i) {
        const uint32_t hi = max(t[i], u);
        u = min(t[i], u);
        t[i] = hi;
    }
}
// A lane's list lives in shared memory ([i][lane]: conflict-free), loaded
// into registers only while a batch is handled.
__device__ __forceinline__ void list_load(const uint32_t* l, int lane, uint32_t (&t)[kCandR]) {
#pragma unroll
    for (int i = 0; i < kCandR; ++i) t[i] = l[i * 32 + lane];
}
__device__ __forceinline__ void list_store(uint32_t* l, int lane, const uint32_t (&t)[kCandR]) {
#pragma unroll
    for (int i = 0; i < kCandR; ++i) l[i * 32 + lane] = t[i];
}

// The largest multiple of 2^16 that at least kk keys of the warp's lists
// reach (0 when fewer are listed): a lower bound of the warp's kk-th largest
// listed key, digit by digit from the top bit (16 rounds, one warp sum each).
__device__ __forceinline__ uint32_t warp_kth_bound(const uint32_t (&t)[kCandR], uint32_t kk) {
    uint32_t p = 0;
#pragma unroll 1
    for (int b = 31; b >= 16; --b) {
        const uint32_t c = p | (1u << b);
        uint32_t n = 0;
#pragma unroll
        for (int i = 0; i < kCandR; ++i) n += t[i] >= c ? 1u : 0u;
        if (__reduce_add_sync(0xffffffffu, n) >= kk) p = c;
    }
    return p;
}

constexpr int kCandQueue = 64;              // queued entries per (warp, query): a batch + one tile
// per (epilogue warp, query slot): the queue, then the lanes' lists
constexpr uint32_t kCandSlotBytes = kCandQueue * sizeof(uint64_t) + kCandR * 32 * sizeof(uint32_t);

// One warp's filter state for one query (qn, nb, pend_n and pend_row are
// the same in every lane; pend_base lives in lane 0).
struct CandState {
    uint32_t tau;           // the bound in force
    int qn;                 // entries in the queue
    int nb;                 // batches handled for the current row
    int pend_n;             // entries of the last batch still to store
    uint32_t pend_base;     // their reservation (lane 0)
    uint64_t pend_x;        // this lane's entry of that batch
    uint64_t* pend_row;
};

__device__ __forceinline__ void cand_reset(CandState& st, uint32_t* list, int lane) {
#pragma unroll
    for (int i = 0; i < kCandR; ++i) list[i * 32 + lane] = 0u;
    st.tau = 0u;
    st.qn = 0;
    st.nb = 0;
}

// The stores of the last batch (its reservation was issued a batch earlier).
__device__ __forceinline__ void cand_complete(CandState& st, int64_t cap, int lane) {
    if (st.pend_n == 0) return;
    const uint32_t b = __shfl_sync(0xffffffffu, st.pend_base, 0);
    if (lane < st.pend_n && (int64_t)b + lane < cap) st.pend_row[b + lane] = st.pend_x;
    st.pend_n = 0;
}

// The first n (<= 32) queued entries as a batch: into the lanes' lists
// (left in t), the previous batch stored, this one reserved in the row's
// list, the rest of the queue moved to its front.
__device__ __forceinline__ void cand_batch(CandState& st, uint64_t* qb, uint32_t* list, int n, uint64_t* row,
                                           uint32_t* cnt, int64_t cap, int lane, uint32_t (&t)[kCandR]) {
    __syncwarp();
    const uint64_t x = lane < n ? qb[lane] : 0ull;
    list_load(list, lane, t);
    cand_insert(t, (uint32_t)(x >> 32));
    list_store(list, lane, t);
    ++st.nb;
    cand_complete(st, cap, lane);
    if (lane == 0) st.pend_base = atomicAdd(cnt, (uint32_t)n);
    st.pend_x = x;
    st.pend_n = n;
    st.pend_row = row;
    const int rest = st.qn - n;
    const uint64_t y = lane < rest ? qb[n + lane] : 0ull;
    __syncwarp();
    if (lane < rest) qb[lane] = y;
    st.qn = rest;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              int* status, uint32_t limit) {
    for (uint32_t i = 0; i < limit; ++i) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 255u && *abort_flag) return false;
    }
    report_device_error(status, CSA_ERR_TIMEOUT);
    *abort_flag = 1;
    return false;
}

}  // namespace

// kBlk: the keys come in blocks (a 3D key map); a separate instantiation, so
// that the contiguous path's producer loop stays as it was. kCand: the top-k
// filter replaces the score stores (bf16, one 128-key half per tile).
template <bool kFp8, int kN, int kHI, int kH, bool kBlk = false, bool kCand = false>
__global__ void __launch_bounds__(kernel_threads(kN, kH), 1) index_scores_tc_kernel(const __grid_constant__ IdxArgs a,
                                                                      const __grid_constant__ CUtensorMap tmK,
                                                                      const __grid_constant__ CUtensorMap tmQ) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    Smem sm = carve(base, a);
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    // top-k filter: [query of the group][epilogue warp] = (group << 32) | bound
    constexpr int kEpi = epi_warps(kN, kH);
    constexpr int kIssuer1 = kEpi + 2;   // warp of MMA issuer 1
    __shared__ uint64_t s_pub[4 * kEpi];
    static_assert(!kCand || (!kFp8 && kH == 1), "the top-k filter runs on bf16 tiles of 128 keys");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ngroups = (a.nq + a.group - 1) / a.group;

    if (threadIdx.x == 0) {
        for (int i = 0; i < a.stages; ++i) { tc::mbar_init(&sm.full[i], 1); tc::mbar_init(&sm.empty[i], 1); }
        // prefill (kN == 256): every epilogue set reduces every tile, so all its warps release it
        for (int i = 0; i < 4; ++i) { tc::mbar_init(&sm.tfull[i], 1); tc::mbar_init(&sm.tempty[i], kN == 256 ? kEpi : 4); }
        tc::mbar_init(sm.qfull, 1);
        tc::mbar_init(sm.qempty, kIssuers);   // every issuer releases each group's q
        tc::mbar_init(sm.fin, kIssuers);
        tc::fence_mbar_init();
        s_abort = 0;
        for (int i = 0; i < 4 * kEpi; ++i) s_pub[i] = (uint64_t)kTagNone << 32;
    }
    if (warp == 1) {
        tc::tmem_alloc(&s_tmem, a.tmem_cols);
        tc::tmem_relinquish();
        tc::tc_fence_before();
    }
    if (warp == 0 && lane == 0) {
        tc::tma_prefetch_desc(&tmK);
        tc::tma_prefetch_desc(&tmQ);
    }
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = s_tmem;
    pdl_wait();
    pdl_launch_next();

    // this CTA's share of the work list
    const int64_t T = total_tiles(a, ngroups, lane);
    const int64_t begin = T * blockIdx.x / gridDim.x;
    const int64_t end = T * (blockIdx.x + 1) / gridDim.x;
    const int64_t my = end - begin;
    int g0 = ngroups;
    int64_t t0 = 0;
    if (my > 0) locate(a, ngroups, begin, lane, g0, t0);
    volatile int* abort_flag = &s_abort;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && my > 0) {
            Walk wk;
            wk.start(a, g0, t0);
            int cur = -1;
            uint32_t switches = 0;
            int64_t it = 0;
            RingPos st(a.stages);
            for (; it < my; ++it, st.advance()) {
                if (wk.g != cur) {
                    if (switches > 0 && !wait_or_abort(sm.qempty, (switches - 1) & 1, abort_flag, a.status, a.wait_limit)) break;
                    tc::mbar_expect_tx(sm.qfull, a.q_bytes);
                    for (int kb = 0; kb < a.kblocks; ++kb)
                        tc::tma_load_2d(sm.q + (size_t)kb * a.npad * 128, &tmQ, sm.qfull, kb * a.blk_elems,
                                        wk.g * a.group * a.HI);
                    cur = wk.g;
                    ++switches;
                }
                const int s = st.slot;
                if (st.wrapped && !wait_or_abort(&sm.empty[s], st.phase ^ 1u, abort_flag, a.status, a.wait_limit))
                    break;
                if (!(a.skip_first_tile && it == 0)) {
                    tc::mbar_expect_tx(&sm.full[s], a.stage_bytes);
                    const int row = (int)((int64_t)group_seq(a, wk.g) * a.Nmax + wk.t * a.kpt);
                    uint8_t* dst = sm.stage0 + (size_t)s * a.stage_bytes;
                    // the stage holds kH halves of 128 keys, each kblocks
                    // 128-byte column blocks of 128 rows
#pragma unroll
                    for (int hh = 0; hh < kH; ++hh)
                        for (int kb = 0; kb < a.kblocks; ++kb)
                            if constexpr (kBlk)   // kKeys / key_rpb blocks of key_rpb rows
                                tc::tma_load_3d(dst + (size_t)(hh * a.kblocks + kb) * kKeys * 128, &tmK, &sm.full[s],
                                                kb * a.blk_elems, 0, (row + hh * kKeys) / a.key_rpb);
                            else
                                tc::tma_load_2d(dst + (size_t)(hh * a.kblocks + kb) * kKeys * 128, &tmK, &sm.full[s],
                                                kb * a.blk_elems, row + hh * kKeys);
                }
                wk.next(a, ngroups);
            }
            // drain: the copies of the last `stages` tiles (and the last Q) must land
            for (int64_t j = (it > a.stages ? it - a.stages : 0); j < it; ++j)
                if (!(a.skip_first_tile && j == 0)) tc::mbar_wait(&sm.full[j % a.stages], (j / a.stages) & 1, kWaitLimit);
            if (switches > 0) tc::mbar_wait(sm.qfull, (switches - 1) & 1, kWaitLimit);
        }
    } else if (warp == 1 || warp == kIssuer1) {
        // ------------------------------------------------------------ MMA issuers
        // issuer mi takes the tiles with it % kIssuers == mi; both walk the
        // whole list, wait for each group's q and release it at the group's end
        const int mi = warp == kIssuer1 ? 1 : 0;
        if (lane == 0 && my > 0) {
            Walk wk;
            wk.start(a, g0, t0);
            int cur = -1;
            uint32_t switches = 0;
            const uint32_t idesc = kFp8 ? tc::idesc_e4m3_f32(128, a.npad, 0, 0) : tc::idesc_bf16_f32(128, a.npad, 0, 0);
            // descriptors built once; a K step or a stage only moves the start
            // address field (bits 0-13, in 16-byte units), so it is added in place
            const uint64_t a_desc0 = tc::sdesc_sw128(tc::smem_u32(sm.stage0), 16, 1024);
            const uint64_t b_desc0 = tc::sdesc_sw128(tc::smem_u32(sm.q), 16, 1024);
            const uint32_t stage_step = a.stage_bytes >> 4;
            const uint32_t a_kb_step = (kKeys * 128) >> 4;
            const uint32_t b_kb_step = (uint32_t)(a.npad * 128) >> 4;
            int64_t it = 0;
            RingPos st(a.stages), bf(a.nbuf);
            for (; it < my; ++it, st.advance(), bf.advance()) {
                if (wk.g != cur) {
                    if (!wait_or_abort(sm.qfull, switches & 1, abort_flag, a.status, a.wait_limit)) break;
                    cur = wk.g;
                    ++switches;
                }
                if ((int)(it % kIssuers) != mi) {
                    if (wk.last_of_group() || it + 1 == my) tc::umma_commit(sm.qempty);
                    wk.next(a, ngroups);
                    continue;
                }
                const int s = st.slot;
                const int buf = bf.slot;
                if (!wait_or_abort(&sm.full[s], st.phase, abort_flag, a.status, a.wait_limit)) break;
                if (bf.wrapped && !wait_or_abort(&sm.tempty[buf], bf.phase ^ 1u, abort_flag, a.status, a.wait_limit))
                    break;
                tc::tc_fence_after();
                const uint64_t a_s = a_desc0 + (uint64_t)(s * stage_step);
#pragma unroll
                for (int hh = 0; hh < kH; ++hh) {
                    // half hh: keys hh*128 .. +127 into accumulator columns hh*npad
                    const uint32_t d = tmem + (uint32_t)((buf * kH + hh) * a.npad);
                    for (int kb = 0; kb < a.kblocks; ++kb) {
                        const uint64_t ad = a_s + (uint64_t)((hh * a.kblocks + kb) * a_kb_step);
                        const uint64_t bd = b_desc0 + (uint64_t)(kb * b_kb_step);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {   // 32 bytes = 2 units per K step
                            if constexpr (kFp8) tc::umma_f8(d, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) ? 1u : 0u);
                            else tc::umma_bf16(d, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) ? 1u : 0u);
                        }
                    }
                }
                tc::umma_commit(&sm.empty[s]);
                tc::umma_commit(&sm.tfull[buf]);
                if (wk.last_of_group() || it + 1 == my) tc::umma_commit(sm.qempty);
                wk.next(a, ngroups);
            }
            // a last commit covers every MMA this thread issued (also on abort)
            tc::umma_commit(sm.fin);
            tc::mbar_wait(sm.fin, 0, kWaitLimit);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // two sets of four warps take alternate tiles (prefill, kN == 256:
        // every set takes every tile, set s reducing the kSetCols columns of
        // its kQS queries, which shortens the per-tile latency of the
        // epilogue that paces the two accumulator buffers); within a set,
        // warp w reads TMEM lane quadrant w % 4
        const int set = (warp - 2) >> 2;
        const int quad = warp & 3;
        const int row = quad * 32 + lane;          // key within the tile
        constexpr int kQS = kN == 256 ? 4 / (kEpi / 4) : 4;   // queries a set reduces per tile (at most)
        constexpr int kSetCols = kN == 256 ? kN / (kEpi / 4) : 256;
        constexpr int kSets = kEpi / 4;                        // sets taking turns (kN != 256)
        // each epilogue warp keeps its own copy of its set's head weights, so
        // that no barrier ties the warps of a set together (a warp that stops
        // on a timeout can never leave the others waiting)
        float* wv = sm.w + (warp - 2) * (kN == 256 ? kSetCols : (kEpi > 8 ? 64 : 256));
        Walk wk;
        wk.start(a, g0, t0);
        int cur = -1;
        int64_t vis = 0;
        RingPos bf(a.nbuf);
        // top-k filter: this warp's queries (the grouped prefill: its set's;
        // otherwise one) and their queues
        constexpr int kQ = kN == 256 ? kQS : 1;
        CandState cst[kQ];
        uint8_t* cslot = sm.cq + (size_t)(warp - 2) * kQ * kCandSlotBytes;
        auto cq_of = [&](int q) { return reinterpret_cast<uint64_t*>(cslot + q * kCandSlotBytes); };
        auto cl_of = [&](int q) {
            return reinterpret_cast<uint32_t*>(cslot + q * kCandSlotBytes + kCandQueue * sizeof(uint64_t));
        };
        uint32_t ctop[kCandR];
        if constexpr (kCand) {
#pragma unroll
            for (int q = 0; q < kQ; ++q) {
                cand_reset(cst[q], cl_of(q), lane);
                cst[q].pend_n = 0;
                cst[q].pend_base = 0;
                cst[q].pend_x = 0;
                cst[q].pend_row = nullptr;
            }
        }
        // the row of this warp's query slot gs in group g (nullptr: none)
        auto cand_row = [&](int g, int gs, uint32_t*& cnt) -> uint64_t* {
            const int gq = kN == 256 ? kQS * set + gs : gs;
            const int tq = g * a.group + gq;
            if (g < 0 || gq >= a.group || tq >= a.nq) return nullptr;
            cnt = a.cand_cnt + tq;
            return a.cand + (int64_t)tq * a.cand_ld;
        };
        for (int64_t it = 0; it < my; ++it, wk.next(a, ngroups), bf.advance()) {
            if (kN != 256 && (int)(it & (kSets - 1)) != set) continue;
            if (wk.g != cur) {
                __syncwarp();
                const int c0w = kN == 256 ? set * kSetCols : 0;   // first column of this warp's copy
                for (int c = lane; c < (kN == 256 ? kSetCols : a.npad); c += 32) {
                    const int gq = (c0w + c) / a.HI, h = (c0w + c) % a.HI;
                    const int tq = wk.g * a.group + gq;
                    wv[c] = (gq < a.group && tq < a.nq) ? a.w[(int64_t)tq * a.HI + h] : 0.f;
                }
                __syncwarp();
                if constexpr (kCand) {
                    // the previous group's queued entries go out before its state is reset
#pragma unroll
                    for (int q = 0; q < kQ; ++q) {
                        uint32_t* cnt = nullptr;
                        uint64_t* rowp = cand_row(cur, q, cnt);
                        if (rowp && cst[q].qn > 0)
                            cand_batch(cst[q], cq_of(q), cl_of(q), cst[q].qn, rowp, cnt, a.cand_ld, lane, ctop);
                        cand_reset(cst[q], cl_of(q), lane);
                    }
                }
                cur = wk.g;
                vis = group_visible(a, wk.g);
            }
            const int buf = bf.slot;
            // this thread's keys: row of each 128-key half of the tile
            int64_t key[kH];
            float kscale[kH];
#pragma unroll
            for (int hh = 0; hh < kH; ++hh) {
                key[hh] = wk.t * a.kpt + hh * kKeys + row;
                // FP8: the key's scale, loaded before the wait so its latency hides
                kscale[hh] = 1.f;
                if constexpr (kFp8)
                    if (key[hh] < vis) kscale[hh] = __ldg(a.kscale + (int64_t)group_seq(a, wk.g) * a.Nmax + key[hh]);
            }
            if (!wait_or_abort(&sm.tfull[buf], bf.phase, abort_flag, a.status, a.wait_limit)) break;
            tc::tc_fence_after();
            // sc[hh][q]: the scores of query q of the group; with kN == 256
            // this set's queries (kQS set + q) sit in sc[hh][0..kQS) (the set
            // is a run-time value: indexing by it would put the array in
            // local memory)
            float sc[kH][4];
#pragma unroll
            for (int hh = 0; hh < kH; ++hh) {
                sc[hh][0] = sc[hh][1] = sc[hh][2] = sc[hh][3] = 0.f;
                const uint32_t taddr =
                    tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)((buf * kH + hh) * a.npad);
                if constexpr (kN == 256)
                    // (the wide layout's warps get fewer registers: 32-column rounds)
                    head_reduce<kSetCols, kHI, (kEpi > 8 ? 32 : 64)>(taddr + set * kSetCols, wv, a.npad, a.HI,
                                                                     a.group, sc[hh]);
                else
                    head_reduce<kN, kHI, (kEpi > 8 ? 32 : 64)>(taddr, wv, a.npad, a.HI, a.group, sc[hh]);
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&sm.tempty[buf]);
            if constexpr (kCand) {
                const bool in = key[0] < vis;
                const int c0 = kN == 256 ? 4 * set : 0;          // warps scoring this warp's queries
                constexpr int nc = kN == 256 ? 4 : kEpi;
#pragma unroll
                for (int gs = 0; gs < kQ; ++gs) {
                    uint32_t* cnt = nullptr;
                    uint64_t* rowp = cand_row(wk.g, gs, cnt);
                    if (!rowp) continue;                            // the same for the whole warp
                    CandState& st = cst[gs];
                    uint64_t* qb = cq_of(gs);
                    const uint32_t u = in ? orderable(sc[0][gs]) : 0u;
                    const bool take = in && u >= st.tau;
                    const unsigned mk = __ballot_sync(0xffffffffu, take);
                    if (!mk) continue;
                    if (take) qb[st.qn + __popc(mk & ((1u << lane) - 1u))] = composite_key(u, key[0]);
                    st.qn += __popc(mk);
                    if (st.qn < 32) continue;
                    cand_batch(st, qb, cl_of(gs), 32, rowp, cnt, a.cand_ld, lane, ctop);
                    // publish this warp's bound (after batches 1, 2, 4, then
                    // every fourth: it rises fastest early in the row) and take
                    // the minimum over the warps scoring the query once all of
                    // them have published for it
                    if ((st.nb & (st.nb - 1)) != 0 && (st.nb & 3) != 0) continue;
                    const int gq = kN == 256 ? kQS * set + gs : gs;
                    const uint32_t p = warp_kth_bound(ctop, a.cand_kk);
                    volatile uint64_t* slots = s_pub + gq * kEpi;
                    if (lane == 0) slots[warp - 2] = ((uint64_t)(uint32_t)wk.g << 32) | p;
                    __syncwarp();
                    uint32_t lo = 0xFFFFFFFFu;
                    bool all = true;
#pragma unroll
                    for (int j = 0; j < nc; ++j) {
                        const uint64_t v = slots[c0 + j];
                        all = all && (uint32_t)(v >> 32) == (uint32_t)wk.g;
                        lo = min(lo, (uint32_t)v);
                    }
                    if (all) st.tau = max(st.tau, lo);
                }
                continue;
            }
#pragma unroll
            for (int hh = 0; hh < kH; ++hh) {
                if (key[hh] >= vis) continue;
#pragma unroll
                for (int gs = 0; gs < kQS; ++gs) {
                    const int gq = kN == 256 ? kQS * set + gs : gs;   // query within the group
                    const int tq = wk.g * a.group + gq;
                    if (gq < a.group && tq < a.nq) {
                        const float v = kFp8 ? sc[hh][gs] * kscale[hh] : sc[hh][gs];
                        if (a.score_bf16)
                            reinterpret_cast<bf16*>(a.scores)[(int64_t)tq * a.ld + key[hh]] = __float2bfloat16_rn(v);
                        else
                            a.scores[(int64_t)tq * a.ld + key[hh]] = v;
                    }
                }
            }
        }
        if constexpr (kCand) {
            // the last group's queued entries, then every pending store
#pragma unroll
            for (int q = 0; q < kQ; ++q) {
                uint32_t* cnt = nullptr;
                uint64_t* rowp = cand_row(cur, q, cnt);
                if (rowp && cst[q].qn > 0)
                    cand_batch(cst[q], cq_of(q), cl_of(q), cst[q].qn, rowp, cnt, a.cand_ld, lane, ctop);
                cand_complete(cst[q], a.cand_ld, lane);
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, a.tmem_cols);
    }
}

// -inf for the columns a query cannot see (s >= floor(p/m)), so the score
// matrix is complete; the fused paths skip it (top-k reads only visible ones).
__global__ void fill_invisible_kernel(float* scores, int64_t ld, QueryMap qm, int nq, int n_seq, int64_t Nmax,
                                      int m) {
    pdl_wait();
    pdl_launch_next();
    const int t = blockIdx.x;
    int s = qm.seq_of(t);
    int64_t vis = (s >= 0 && s < n_seq) ? visible_entries(qm.pos_of(t), m, Nmax) : 0;
    for (int64_t c = vis + (int64_t)blockIdx.y * blockDim.x + threadIdx.x; c < Nmax; c += (int64_t)gridDim.y * blockDim.x)
        scores[(int64_t)t * ld + c] = -INFINITY;
}

static int num_sms() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

// warps whose lanes score one query: the 4 of its set in the grouped
// prefill instantiation, all 8 elsewhere (the sets alternate tiles)
static int cand_warps(int HI, int group) { return (HI == 64 && group == 4) ? 4 : 8; }

bool index_cand_supported(int HI, int cI, int group, int k) {
    // one query per epilogue warp, or the grouped prefill's two
    if (!index_tc_supported(HI, cI, group, false) || k < 1 || !(group == 1 || (HI == 64 && group == 4)))
        return false;
    const int w = cand_warps(HI, group);
    return (k + w - 1) / w <= 32 * kCandR;
}

bool index_tc_supported(int HI, int cI, int group, bool fp8) {
    if (cI % (fp8 ? 128 : 64) != 0 || cI > 256) return false;
    if (group < 1 || group > 4) return false;
    if (group > 1 && HI % 16 != 0) return false;
    int n = group * HI;
    return n <= 256;
}

cudaError_t index_scores_tc(const void* qI, const float* w, const void* K, QuerySpec qs, int nq, int n_seq, int HI,
                            int cI, int64_t Nmax, int m, float* scores, int64_t ld, int group, bool fill_invisible,
                            int* status, cudaStream_t st, const float* kscale, bool score_bf16, RowBlocks kb,
                            CandOut co) {
    if (score_bf16 && fill_invisible) return cudaErrorInvalidValue;
    const bool fp8 = kscale != nullptr;
    const bool cand = co.cand != nullptr;
    if (cand && (fp8 || score_bf16 || fill_invisible || kb.rpb > 0 || !co.cnt || co.ld < Nmax ||
                 !index_cand_supported(HI, cI, group, co.k)))
        return cudaErrorInvalidValue;
    // keys in blocks: bf16 only, whole blocks per 128-key tile and per sequence
    if (kb.rpb > 0 && (fp8 || kKeys % kb.rpb || Nmax % kb.rpb || kb.block_bytes % 16)) return cudaErrorInvalidValue;
    const int es = fp8 ? 1 : 2;
    if (cand && nq > 0) {
        const cudaError_t ze = cudaMemsetAsync(co.cnt, 0, (size_t)nq * sizeof(uint32_t), st);
        if (ze != cudaSuccess) return ze;
    }
    if (nq == 0 || Nmax == 0) return cudaSuccess;
    IdxArgs a{};
    a.qm = QueryMap{qs.seq, qs.pos, qs.pos_base, qs.single_seq};
    a.nq = nq;
    a.n_seq = n_seq;
    a.group = group;
    a.HI = HI;
    a.cI = cI;
    int n = group * HI;
    a.npad = n < 16 ? 16 : ((n + 15) / 16) * 16;
    a.kblocks = cI * es / 128;
    a.blk_elems = 128 / es;
    a.kscale = kscale;
    a.Nmax = Nmax;
    a.m = m;
    a.w = w;
    a.scores = scores;
    a.score_bf16 = score_bf16 ? 1 : 0;
    a.wait_limit = debug_wait_limit() ? debug_wait_limit() : kWaitLimit;
    a.skip_first_tile = (debug_flags() & CSA_DEBUG_SKIP_FIRST_TILE) ? 1 : 0;
    a.ld = ld;
    a.status = status;
    if (cand) {
        a.cand = co.cand;
        a.cand_cnt = co.cnt;
        a.cand_ld = co.ld;
        const int cw = cand_warps(HI, group);
        a.cand_kk = (uint32_t)((co.k + cw - 1) / cw);
    }
    // FP8 decode (one query of at most 128 heads per MMA): tiles of 256 keys
    const int kh = (fp8 && group == 1 && n <= 128) ? 2 : 1;
    a.kpt = kh * kKeys;
    a.stage_bytes = (uint32_t)(a.kpt * cI * es);
    a.q_bytes = (uint32_t)(a.npad * cI * es);
    // as many accumulator buffers (2..4) as fit 512 TMEM columns
    a.nbuf = 512 / (kh * a.npad);
    if (a.nbuf > 4) a.nbuf = 4;
    if (a.nbuf < 2) a.nbuf = 2;
    uint32_t cols = 32;
    while (cols < (uint32_t)(a.nbuf * kh * a.npad)) cols <<= 1;
    a.tmem_cols = cols;
    const size_t fixed = 1024 + a.q_bytes + 8 * 256 * sizeof(float) + 64 * sizeof(uint64_t) +
                         (cand ? (size_t)(group == 4 ? epi_warps(256) * (4 / (epi_warps(256) / 4))
                                                     : epi_warps(0)) * kCandSlotBytes : 0);
    const size_t budget = 226 * 1024;
    int stages = (int)((budget - fixed) / a.stage_bytes);
    if (stages > (fp8 ? 12 : 8)) stages = fp8 ? 12 : 8;
    if (stages < 2) return cudaErrorInvalidConfiguration;
    a.stages = stages;
    const size_t smem = fixed + (size_t)stages * a.stage_bytes;

    CUtensorMap tmK, tmQ;
    if (fp8) {
        if (!make_tmap_u8_2d(&tmK, K, (uint64_t)n_seq * Nmax, cI, cI, kKeys, 128)) return cudaErrorInvalidValue;
        if (!make_tmap_u8_2d(&tmQ, qI, (uint64_t)nq * HI, cI, cI, a.npad, 128)) return cudaErrorInvalidValue;
    } else {
        if (kb.rpb > 0) {
            a.key_rpb = kb.rpb;
            if (!make_tmap_bf16_blocks(&tmK, K, (uint64_t)n_seq * Nmax / kb.rpb, (uint32_t)kb.rpb, cI,
                                       (uint64_t)kb.block_bytes, (uint32_t)(kKeys / kb.rpb), 64))
                return cudaErrorInvalidValue;
        } else if (!make_tmap_bf16_2d(&tmK, K, (uint64_t)n_seq * Nmax, cI, cI, kKeys, 64)) {
            return cudaErrorInvalidValue;
        }
        if (!make_tmap_bf16_2d(&tmQ, qI, (uint64_t)nq * HI, cI, cI, a.npad, 64)) return cudaErrorInvalidValue;
    }

    cudaError_t e;
    if (fill_invisible) {
        QueryMap qm = a.qm;
        CSA_LAUNCH(st, "index_fill_invisible",
                   e = launch_pdl(fill_invisible_kernel, dim3(nq, 8), dim3(256), 0, st, 0, scores, ld, qm, nq, n_seq,
                                  Nmax, m));
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // the two shapes of the workloads get a fully unrolled epilogue: decode
    // (one query of 64 heads per MMA) and grouped prefill (4 queries of 64)
    auto kern = fp8 ? (kh == 2 ? index_scores_tc_kernel<true, 0, 0, 2> : index_scores_tc_kernel<true, 0, 0, 1>)
                    : index_scores_tc_kernel<false, 0, 0, 1>;
    if (a.npad == 64 && HI == 64 && group == 1)
        kern = fp8 ? index_scores_tc_kernel<true, 64, 64, 2> : index_scores_tc_kernel<false, 64, 64, 1>;
    else if (a.npad == 256 && HI == 64 && group == 4)
        kern = fp8 ? index_scores_tc_kernel<true, 256, 64, 1> : index_scores_tc_kernel<false, 256, 64, 1>;
    if (a.key_rpb)   // bf16 keys in blocks (decode shape, or any other)
        kern = (a.npad == 64 && HI == 64 && group == 1) ? index_scores_tc_kernel<false, 64, 64, 1, true>
                                                          : index_scores_tc_kernel<false, 0, 0, 1, true>;
    if (cand) {
        if (a.npad == 64 && HI == 64 && group == 1) kern = index_scores_tc_kernel<false, 64, 64, 1, false, true>;
        else if (a.npad == 256 && HI == 64 && group == 4) kern = index_scores_tc_kernel<false, 256, 64, 1, false, true>;
        else kern = index_scores_tc_kernel<false, 0, 0, 1, false, true>;
    }
    // the block size of the instantiation chosen above
    int threads = kernel_threads(0);
    if (!a.key_rpb && a.npad == 256 && HI == 64 && group == 4) threads = kernel_threads(256);
    else if (fp8 && a.npad == 64 && HI == 64 && group == 1) threads = kernel_threads(64, kh);
    e = smem_ceiling(kern);
    if (e != cudaSuccess) return e;
    CSA_LAUNCH(st, fp8 ? "index_scores_tc_fp8" : (cand ? "index_topk_filter_tc" : "index_scores_tc"),
               e = launch_pdl(kern, dim3(num_sms()), dim3(threads), smem, st, 0, a, tmK, tmQ));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace csa
