// Projection of hidden states onto the compressor streams [Walk §2.3.1 "KV
// compression": the KV streams and their weight logits are learnable linear
// maps of the hidden state] ([Walk] = mlpod.com walk-through of the
// DeepSeek-V4 report):  out[t][o] = sum_k x[t][k] * W[o][k], fp32 result.
//
// bf16 inputs run on the tensor cores (gemm_tc.cu); this FFMA kernel serves
// the fp32 mode: 64x64 output tile per CTA, k-steps of 16 staged in
// shared memory as fp32 (transposed so a warp reads consecutive rows), each
// thread accumulates a 4x4 register block.
#include "common.cuh"
#include "kernels.h"

namespace csa {

constexpr int kBM = 64, kBN = 64, kBK = 16;

template <typename T>
__global__ void __launch_bounds__(256) project_ffma_kernel(const T* __restrict__ X,
                                                           const T* __restrict__ W, int64_t n,
                                                           int d, int M, float* __restrict__ out) {
    __shared__ float As[kBK][kBM + 4];
    __shared__ float Bs[kBK][kBN + 4];
    const int64_t row0 = (int64_t)blockIdx.y * kBM;
    const int col0 = blockIdx.x * kBN;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < d; k0 += kBK) {
        // 64 rows x 16 k of X and of W: 1024 elements each, 4 per thread
        for (int i = threadIdx.x; i < kBM * kBK; i += 256) {
            int r = i / kBK, kk = i % kBK;
            int64_t gr = row0 + r;
            int gk = k0 + kk;
            As[kk][r] = (gr < n && gk < d) ? to_f32(X[gr * d + gk]) : 0.f;
            int gc = col0 + r;
            Bs[kk][r] = (gc < M && gk < d) ? to_f32(W[(int64_t)gc * d + gk]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kBK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int64_t r = row0 + ty * 4 + i;
        if (r >= n) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int cc = col0 + tx * 4 + j;
            if (cc < M) out[r * M + cc] = acc[i][j];
        }
    }
}

cudaError_t project(const void* x, const void* W, int64_t n, int d, int M, float* out, ElemType t,
                    cudaStream_t st) {
    if (n == 0 || M == 0) return cudaSuccess;
    if (t == ElemType::BF16) return project_tc(x, W, n, d, M, out, device_status(), st);
    dim3 grid((M + kBN - 1) / kBN, (unsigned)((n + kBM - 1) / kBM));
    if (t == ElemType::BF16)
        CSA_LAUNCH(st, "project_ffma", project_ffma_kernel<bf16><<<grid, 256, 0, st>>>((const bf16*)x, (const bf16*)W, n, d, M, out));
    else
        CSA_LAUNCH(st, "project_ffma", project_ffma_kernel<float><<<grid, 256, 0, st>>>((const float*)x, (const float*)W, n, d, M, out));
    return cudaGetLastError();
}

}  // namespace csa
