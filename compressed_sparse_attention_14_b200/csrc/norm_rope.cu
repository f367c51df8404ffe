// Completion of the attention output around the MQA: query / KV RMSNorm with
// partial rotary encoding (and the output's back-rotation), and the entry
// lists that join the sliding window to the selected compressed entries.
//
// [Walk §2.3.3 items 1-3; Notes §1.3 "Partial RoPE" and "sliding window
// branch"]: every query head and every compressed KV entry is RMS-normalised
// before the core attention; the last R channels of both carry a rotary
// encoding of the position, and the attention output is turned back by the
// query's position so that it holds relative position only. Besides its
// top-k entries every query attends to the uncompressed KV of the n_win most
// recent tokens, kept in a per-sequence window ring [Walk §5 item 2, the
// SWA state cache; Notes §2.6 Fig. 6].
//
// ([Walk] = mlpod.com walk-through of "DeepSeek-V4: Towards Highly Efficient
// Million-Token Context Intelligence"; [Notes] = "DeepSeek-V4: 迈向高效百万级
// 上下文智能", study notes on the DeepSeek-V4 report, notes.kuangjux.top.)
//
// Norm + rotary is HBM-bound: one read and one write of every row. A warp
// owns two rows and takes each in 8-channel pieces (lane l holds pieces l and
// l + 32), so each warp-wide load covers 512 contiguous bytes of bf16; the
// loads of both rows are issued before anything else, and the sum of squares
// is one warp reduction per row. Rotation angles p * theta_i are formed in
// fp64 (positions reach 2^20 and more, where an fp32 product would already be
// off by a sizeable part of a radian), reduced to [-pi, pi] by subtracting the
// nearest multiple of 2*pi (one fused multiply-add in fp64, the first step of
// Cody and Waite's reduction scheme), and only then handed to the fp32
// sincosf. The frequencies theta_i are computed once per CTA, one per thread,
// while the row loads are in flight.
//
// The window entry list is integer bookkeeping, one thread per output slot.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kWarps = 8;
constexpr int kRowsPerWarp = 2;
constexpr int kPieces = CSA_MAX_HEAD_DIM / (8 * 32);   // 8-channel pieces per lane
constexpr double kTwoPi = 6.283185307179586;            // 2*pi rounded to fp64
constexpr double kInvTwoPi = 0.15915494309189535;       // 1/(2*pi) rounded to fp64

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) norm_rope_kernel(const T* x, T* y, int64_t rows, int group, int c,
                                                                const float* __restrict__ gamma, float eps, int R,
                                                                double base, const int32_t* __restrict__ pos,
                                                                int64_t pos0, int64_t pos_step, int inverse) {
    __shared__ double s_theta[CSA_MAX_HEAD_DIM / 2];
    pdl_wait();
    pdl_launch_next();
    const int lane = threadIdx.x & 31;
    const int64_t r0 = ((int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5)) * kRowsPerWarp;
    const int pieces = c / 8;
    const int rope0 = c - R;   // first rotated channel; a multiple of 8

    float v[kRowsPerWarp][kPieces][8];
#pragma unroll
    for (int j = 0; j < kRowsPerWarp; ++j) {
        const int64_t r = r0 + j;
#pragma unroll
        for (int pc = 0; pc < kPieces; ++pc) {
            const int q = lane + 32 * pc;
            if (r < rows && q < pieces) load8(x + r * c + 8 * q, v[j][pc]);
        }
    }
    for (int i = threadIdx.x; i < R / 2; i += blockDim.x) s_theta[i] = pow(base, -2.0 * i / R);
    __syncthreads();

#pragma unroll
    for (int j = 0; j < kRowsPerWarp; ++j) {
        const int64_t r = r0 + j;
        if (r >= rows) break;
        float ss = 0.f;
#pragma unroll
        for (int pc = 0; pc < kPieces; ++pc) {
            const int q = lane + 32 * pc;
            if (q < pieces)
#pragma unroll
                for (int e = 0; e < 8; ++e) ss = fmaf(v[j][pc][e], v[j][pc][e], ss);
        }
        if (gamma) {
            ss = warp_sum(ss);
            const float inv = rsqrtf(ss / (float)c + eps);
#pragma unroll
            for (int pc = 0; pc < kPieces; ++pc) {
                const int q = lane + 32 * pc;
                if (q < pieces) {
                    float gm[8];
                    load8(gamma + 8 * q, gm);
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[j][pc][e] = v[j][pc][e] * inv * gm[e];
                }
            }
        }
        if (R > 0) {
            const int64_t g = r / group;
            const double p = (double)(pos ? (int64_t)pos[g] : pos0 + g * pos_step);
#pragma unroll
            for (int pc = 0; pc < kPieces; ++pc) {
                const int q = lane + 32 * pc;
                if (q < pieces && 8 * q >= rope0) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        double ang = p * s_theta[(8 * q + 2 * u - rope0) / 2];
                        if (inverse) ang = -ang;
                        const double turns = rint(ang * kInvTwoPi);
                        float sn, cs;
                        sincosf((float)fma(-turns, kTwoPi, ang), &sn, &cs);
                        const float a = v[j][pc][2 * u], b = v[j][pc][2 * u + 1];
                        v[j][pc][2 * u] = a * cs - b * sn;
                        v[j][pc][2 * u + 1] = a * sn + b * cs;
                    }
                }
            }
        }
        T* yr = y + r * c;
#pragma unroll
        for (int pc = 0; pc < kPieces; ++pc) {
            const int q = lane + 32 * pc;
            if (q < pieces) store8(yr + 8 * q, v[j][pc]);
        }
    }
}

__global__ void __launch_bounds__(256) window_entries_kernel(const int32_t* __restrict__ sel, int k,
                                                             const int32_t* __restrict__ pos, int64_t pos0, int nq,
                                                             int n_win, int64_t ring_off, int64_t ring_len,
                                                             int32_t* __restrict__ ent) {
    pdl_wait();
    pdl_launch_next();
    const int64_t width = (int64_t)k + n_win;
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)nq * width) return;
    const int64_t t = i / width;
    const int64_t j = i - t * width;
    int32_t v;
    if (j < k) {
        v = sel ? sel[t * k + j] : -1;
    } else {
        const int64_t p = pos ? (int64_t)pos[t] : pos0 + t;
        const int64_t tau = p - n_win + 1 + (j - k);
        v = tau < 0 ? -1 : (int32_t)(ring_off + tau % ring_len);
    }
    ent[i] = v;
}

template <typename T>
cudaError_t launch_norm_rope(const void* x, void* y, int64_t rows, int group, int c, const float* gamma, float eps,
                             int R, double base, const int32_t* pos, int64_t pos0, int64_t pos_step, int inverse,
                             cudaStream_t st) {
    const int64_t warps = (rows + kRowsPerWarp - 1) / kRowsPerWarp;
    const int64_t blocks = (warps + kWarps - 1) / kWarps;
    cudaError_t e = cudaSuccess;
    CSA_LAUNCH(st, "norm_rope",
               e = launch_pdl(norm_rope_kernel<T>, dim3((unsigned)blocks), dim3(kWarps * 32), 0, st, 0,
                              (const T*)x, (T*)y, rows, group, c, gamma, eps, R, base, pos, pos0, pos_step,
                              inverse));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

bool norm_rope_supported(int c, int R) {
    return c >= 8 && c <= CSA_MAX_HEAD_DIM && c % 8 == 0 && R >= 0 && R <= c && R % 8 == 0;
}

cudaError_t norm_rope(const void* x, void* y, int64_t rows, int group, int c, const float* gamma, float eps, int R,
                      double base, const int32_t* pos, int64_t pos0, int64_t pos_step, int inverse, ElemType t,
                      cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (t == ElemType::BF16)
        return launch_norm_rope<bf16>(x, y, rows, group, c, gamma, eps, R, base, pos, pos0, pos_step, inverse, st);
    return launch_norm_rope<float>(x, y, rows, group, c, gamma, eps, R, base, pos, pos0, pos_step, inverse, st);
}

cudaError_t window_entries(const int32_t* sel, int k, const int32_t* pos, int64_t pos0, int nq, int n_win,
                           int64_t ring_off, int64_t ring_len, int32_t* ent, cudaStream_t st) {
    const int64_t total = (int64_t)nq * ((int64_t)k + n_win);
    if (total == 0) return cudaSuccess;
    cudaError_t e = cudaSuccess;
    CSA_LAUNCH(st, "window_entries",
               e = launch_pdl(window_entries_kernel, dim3((unsigned)((total + 255) / 256)), dim3(256), 0, st, 0,
                              sel, k, pos, pos0, nq, n_win, ring_off, ring_len, ent));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace csa
