// Projection of hidden states onto the compressor streams on the tensor cores
// [Walk §2.3.1 "KV compression": the KV streams and their weight logits are
// learnable linear maps of the hidden state] ([Walk] = mlpod.com
// walk-through of the DeepSeek-V4 report):
//   out[t][o] = sum_k x[t][k] * W[o][k]       (bf16 in, fp32 accumulate and out)
//
// Persistent CTAs, one per SM, walk the 128 x 256 output tiles round-robin
// with the 256-column index fastest, so the CTAs that share an X row block
// run together and read it from L2 after the first. Per tile:
//   warp 0     TMA producer: X tile [128 x 64] and W tile [256 x 64] per
//              64-deep K block into a 4-stage shared-memory ring (128-byte
//              swizzle; out-of-range rows and K read as zeros);
//   warp 1     allocates TMEM; one lane issues tcgen05.mma M=128, N=256,
//              K=16 (four per K block) into one of two TMEM accumulators;
//   warps 2-5  epilogue: tcgen05.ld of the finished accumulator (one row per
//              thread), 16-byte fp32 stores, masked at the matrix edges.
// The two accumulators let the epilogue of one tile overlap the main loop of
// the next. Waits are bounded (CSA_ERR_TIMEOUT in the status word).
//
// Split K (project_tc_splitk): for a few rows (one decode step's new tokens)
// the 128 x 256 tiles are too few to stream the weights from every SM, so
// the contraction is also cut into ksplit slices: a work item is (row tile,
// column tile, K slice), and slice s writes its fp32 partial sums to
// out + s * n * M. The consumer adds the ksplit partials in slice order
// (deterministic).
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"
#include "tmap.h"

namespace csa {

namespace {

constexpr int kThreads = 192;
constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr uint32_t kStageBytes = (kBM + kBN) * kBK * 2;   // 48 KB
constexpr uint32_t kWaitLimit = 1u << 24;

struct GemmArgs {
    int64_t n;      // rows of x / out
    int d;          // contraction
    int M;          // rows of W / columns of out
    float* out;
    int* status;
    int tiles_m, tiles_n;
    int ksplit;     // K slices (1: no split); slice s covers 64-deep blocks [s*kbs, (s+1)*kbs)
    int kbs;        // 64-deep K blocks per slice
    int items0;     // work items of this problem; items past it belong to the second problem
    // second problem (same x): W2 [M2, d] into out2
    int M2;
    float* out2;
    int tiles_n2, ksplit2, kbs2, items2;
};

// A work item: problem, K slice, row tile, column tile and its K blocks.
struct Item {
    int prob, ks, tm, tn, kb0, kb1;
};

__device__ __forceinline__ Item item_of(const GemmArgs& a, int tile, int kblocks_all) {
    Item it;
    it.prob = tile >= a.items0;
    if (it.prob) tile -= a.items0;
    const int ksplit = it.prob ? a.ksplit2 : a.ksplit, tiles_n = it.prob ? a.tiles_n2 : a.tiles_n;
    const int kbs = it.prob ? a.kbs2 : a.kbs;
    it.ks = tile % ksplit;
    const int mn = tile / ksplit;
    it.tm = mn / tiles_n;
    it.tn = mn % tiles_n;
    it.kb0 = it.ks * kbs;
    it.kb1 = min(kblocks_all, it.kb0 + kbs);
    return it;
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

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) project_tc_kernel(const __grid_constant__ GemmArgs a,
                                                                 const __grid_constant__ CUtensorMap tmX,
                                                                 const __grid_constant__ CUtensorMap tmW,
                                                                 const __grid_constant__ CUtensorMap tmW2) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* full = (uint64_t*)(base + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* tfull = empty + kStages;   // [2]
    uint64_t* tempty = tfull + 2;        // [2]
    uint64_t* fin = tempty + 2;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = a.items0 + a.items2;
    const int kblocks_all = (a.d + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) { tc::mbar_init(&full[i], 1); tc::mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) { tc::mbar_init(&tfull[i], 1); tc::mbar_init(&tempty[i], 4); }
        tc::mbar_init(fin, 1);
        tc::fence_mbar_init();
        s_abort = 0;
    }
    if (warp == 1) {
        tc::tmem_alloc(&s_tmem, 512);
        tc::tmem_relinquish();
        tc::tc_fence_before();
    }
    if (warp == 0 && lane == 0) {
        tc::tma_prefetch_desc(&tmX);
        tc::tma_prefetch_desc(&tmW);
        if (a.items2) tc::tma_prefetch_desc(&tmW2);
    }
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = s_tmem;
    volatile int* abort_flag = &s_abort;
    pdl_wait();
    pdl_launch_next();

    if (warp == 0) {
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
                const Item w = item_of(a, tile, kblocks_all);
                const CUtensorMap* tw = w.prob ? &tmW2 : &tmW;
                for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
                    const int s = (int)(it % kStages);
                    if (it >= kStages && !(ok = wait_or_abort(&empty[s], ((it / kStages) - 1) & 1, abort_flag,
                                                              a.status)))
                        break;
                    uint8_t* st = base + (size_t)s * kStageBytes;
                    tc::mbar_expect_tx(&full[s], kStageBytes);
                    tc::tma_load_2d(st, &tmX, &full[s], kb * kBK, w.tm * kBM);
                    tc::tma_load_2d(st + kBM * 128, tw, &full[s], kb * kBK, w.tn * kBN);
                }
            }
            // drain the copies of the last stages
            for (uint32_t j = (it > kStages ? it - kStages : 0); j < it; ++j)
                tc::mbar_wait(&full[j % kStages], (j / kStages) & 1, kWaitLimit);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16_f32(kBM, kBN, 0, 0);
            const uint64_t a0 = tc::sdesc_sw128(tc::smem_u32(base), 16, 1024);
            const uint64_t b0 = tc::sdesc_sw128(tc::smem_u32(base + kBM * 128), 16, 1024);
            const uint32_t stage_step = kStageBytes >> 4;
            uint32_t it = 0, tcount = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++tcount) {
                const int buf = (int)(tcount & 1);
                if (tcount >= 2 && !(ok = wait_or_abort(&tempty[buf], ((tcount >> 1) - 1) & 1, abort_flag, a.status)))
                    break;
                tc::tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * kBN);
                const Item w = item_of(a, tile, kblocks_all);
                const int kb0 = w.kb0;
                for (int kb = kb0; kb < w.kb1; ++kb, ++it) {
                    const int s = (int)(it % kStages);
                    if (!(ok = wait_or_abort(&full[s], (it / kStages) & 1, abort_flag, a.status))) break;
                    tc::tc_fence_after();
                    const uint64_t ad = a0 + (uint64_t)(s * stage_step);
                    const uint64_t bd = b0 + (uint64_t)(s * stage_step);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::umma_bf16(d, ad + 2 * kk, bd + 2 * kk, idesc, (kb > kb0 || kk) ? 1u : 0u);
                    tc::umma_commit(&empty[s]);
                }
                if (ok) tc::umma_commit(&tfull[buf]);
            }
            tc::umma_commit(fin);
            tc::mbar_wait(fin, 0, kWaitLimit);
        }
    } else {
        const int quad = warp & 3;
        const int row_in_tile = quad * 32 + lane;
        uint32_t tcount = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tcount) {
            const int buf = (int)(tcount & 1);
            if (!wait_or_abort(&tfull[buf], (tcount >> 1) & 1, abort_flag, a.status)) break;
            tc::tc_fence_after();
            const Item w = item_of(a, tile, kblocks_all);
            const int M = w.prob ? a.M2 : a.M;
            const int64_t row = (int64_t)w.tm * kBM + row_in_tile;
            const int col0 = w.tn * kBN;
            const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * kBN);
            float* orow = (w.prob ? a.out2 : a.out) + (int64_t)w.ks * a.n * M + row * M;
            for (int c0 = 0; c0 < kBN; c0 += 64) {
                float v[64];
#pragma unroll
                for (int u = 0; u < 4; ++u) tc::tmem_ld16(taddr + c0 + 16 * u, *reinterpret_cast<float(*)[16]>(v + 16 * u));
                tc::tmem_ld_wait();
                if (row < a.n) {
#pragma unroll
                    for (int j = 0; j < 64; j += 4) {
                        const int col = col0 + c0 + j;
                        if (col + 3 < M) {
                            *reinterpret_cast<float4*>(orow + col) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
                        } else {
                            for (int u = 0; u < 4; ++u)
                                if (col + u < M) orow[col + u] = v[j + u];
                        }
                    }
                }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&tempty[buf]);
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
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

static int clamp_ksplit(int ks, int kblocks_all) { return ks < 1 ? 1 : ks > kblocks_all ? kblocks_all : ks; }

cudaError_t project_tc2(const void* x, int64_t n, int d, const void* W0, int M0, float* out0, int ks0, const void* W1,
                        int M1, float* out1, int ks1, int* status, cudaStream_t st) {
    if (n == 0 || (M0 == 0 && M1 == 0)) return cudaSuccess;
    const int kblocks_all = (d + kBK - 1) / kBK;
    GemmArgs a{};
    a.n = n;
    a.d = d;
    a.status = status;
    a.tiles_m = (int)((n + kBM - 1) / kBM);
    a.M = M0;
    a.out = out0;
    a.ksplit = clamp_ksplit(ks0, kblocks_all);
    a.kbs = (kblocks_all + a.ksplit - 1) / a.ksplit;
    a.tiles_n = (M0 + kBN - 1) / kBN;
    a.items0 = a.tiles_m * a.tiles_n * a.ksplit;
    a.M2 = W1 ? M1 : 0;
    a.out2 = out1;
    a.ksplit2 = clamp_ksplit(ks1, kblocks_all);
    a.kbs2 = (kblocks_all + a.ksplit2 - 1) / a.ksplit2;
    a.tiles_n2 = (a.M2 + kBN - 1) / kBN;
    a.items2 = a.tiles_m * a.tiles_n2 * a.ksplit2;
    CUtensorMap tmX, tmW, tmW2;
    if (!make_tmap_bf16_2d(&tmX, x, (uint64_t)n, d, d, kBM, kBK)) return cudaErrorInvalidValue;
    if (M0 > 0 && !make_tmap_bf16_2d(&tmW, W0, (uint64_t)M0, d, d, kBN, kBK)) return cudaErrorInvalidValue;
    if (a.items2 > 0 && !make_tmap_bf16_2d(&tmW2, W1, (uint64_t)a.M2, d, d, kBN, kBK)) return cudaErrorInvalidValue;
    if (M0 == 0) tmW = tmW2;
    if (a.items2 == 0) tmW2 = tmW;
    const size_t smem = 1024 + (size_t)kStages * kStageBytes + 16 * sizeof(uint64_t);
    cudaError_t e = smem_ceiling(project_tc_kernel);
    if (e != cudaSuccess) return e;
    const int ntiles = a.items0 + a.items2;
    const int grid = ntiles < sm_count() ? ntiles : sm_count();
    CSA_LAUNCH(st, "project_tc",
               e = launch_pdl(project_tc_kernel, dim3(grid), dim3(kThreads), smem, st, 0, a, tmX, tmW, tmW2));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t project_tc(const void* x, const void* W, int64_t n, int d, int M, float* out, int* status,
                       cudaStream_t st, int ksplit) {
    if (M == 0) return cudaSuccess;
    return project_tc2(x, n, d, W, M, out, ksplit, nullptr, 0, nullptr, 1, status, st);
}

void project_ksplit2(int64_t n, int d, int M0, int M1, int* ks0, int* ks1) {
    const int64_t rows = (n + kBM - 1) / kBM;
    const int64_t t0 = rows * ((M0 + kBN - 1) / kBN), t1 = rows * ((M1 + kBN - 1) / kBN);
    const int kblocks = (d + kBK - 1) / kBK;
    int k0 = 1, k1 = 1;
    for (;;) {
        // the problem whose items stream the most weight blocks splits next
        const int64_t w0 = t0 ? (kblocks + k0 - 1) / k0 : 0, w1 = t1 ? (kblocks + k1 - 1) / k1 : 0;
        const bool first = w0 >= w1;
        const int kn = 2 * (first ? k0 : k1);
        const int64_t items = first ? t0 * kn + t1 * k1 : t0 * k0 + t1 * kn;
        if (kn > 64 || kblocks / kn < 4 || items > sm_count()) break;
        (first ? k0 : k1) = kn;
    }
    *ks0 = k0;
    *ks1 = k1;
}

}  // namespace csa
