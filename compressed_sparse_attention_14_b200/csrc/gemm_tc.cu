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
};

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
                                                                 const __grid_constant__ CUtensorMap tmW) {
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
    const int ntiles = a.tiles_m * a.tiles_n;
    const int kblocks = (a.d + kBK - 1) / kBK;

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
                const int tm = tile / a.tiles_n, tn = tile % a.tiles_n;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = (int)(it % kStages);
                    if (it >= kStages && !(ok = wait_or_abort(&empty[s], ((it / kStages) - 1) & 1, abort_flag,
                                                              a.status)))
                        break;
                    uint8_t* st = base + (size_t)s * kStageBytes;
                    tc::mbar_expect_tx(&full[s], kStageBytes);
                    tc::tma_load_2d(st, &tmX, &full[s], kb * kBK, tm * kBM);
                    tc::tma_load_2d(st + kBM * 128, &tmW, &full[s], kb * kBK, tn * kBN);
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
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = (int)(it % kStages);
                    if (!(ok = wait_or_abort(&full[s], (it / kStages) & 1, abort_flag, a.status))) break;
                    tc::tc_fence_after();
                    const uint64_t ad = a0 + (uint64_t)(s * stage_step);
                    const uint64_t bd = b0 + (uint64_t)(s * stage_step);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc::umma_bf16(d, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) ? 1u : 0u);
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
            const int tm = tile / a.tiles_n, tn = tile % a.tiles_n;
            const int64_t row = (int64_t)tm * kBM + row_in_tile;
            const int col0 = tn * kBN;
            const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * kBN);
            float* orow = a.out + row * a.M;
            for (int c0 = 0; c0 < kBN; c0 += 64) {
                float v[64];
#pragma unroll
                for (int u = 0; u < 4; ++u) tc::tmem_ld16(taddr + c0 + 16 * u, *reinterpret_cast<float(*)[16]>(v + 16 * u));
                tc::tmem_ld_wait();
                if (row < a.n) {
#pragma unroll
                    for (int j = 0; j < 64; j += 4) {
                        const int col = col0 + c0 + j;
                        if (col + 3 < a.M) {
                            *reinterpret_cast<float4*>(orow + col) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
                        } else {
                            for (int u = 0; u < 4; ++u)
                                if (col + u < a.M) orow[col + u] = v[j + u];
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

cudaError_t project_tc(const void* x, const void* W, int64_t n, int d, int M, float* out, int* status,
                       cudaStream_t st) {
    if (n == 0 || M == 0) return cudaSuccess;
    GemmArgs a{};
    a.n = n;
    a.d = d;
    a.M = M;
    a.out = out;
    a.status = status;
    a.tiles_m = (int)((n + kBM - 1) / kBM);
    a.tiles_n = (M + kBN - 1) / kBN;
    CUtensorMap tmX, tmW;
    if (!make_tmap_bf16_2d(&tmX, x, (uint64_t)n, d, d, kBM, kBK)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_2d(&tmW, W, (uint64_t)M, d, d, kBN, kBK)) return cudaErrorInvalidValue;
    const size_t smem = 1024 + (size_t)kStages * kStageBytes + 16 * sizeof(uint64_t);
    cudaError_t e = smem_ceiling(project_tc_kernel);
    if (e != cudaSuccess) return e;
    const int ntiles = a.tiles_m * a.tiles_n;
    const int grid = ntiles < sm_count() ? ntiles : sm_count();
    CSA_LAUNCH(st, "project_tc", e = launch_pdl(project_tc_kernel, dim3(grid), dim3(kThreads), smem, st, 0, a, tmX, tmW));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace csa
