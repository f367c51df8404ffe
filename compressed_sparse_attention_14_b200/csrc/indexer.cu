// Lightning indexer scores [Notes §1.1, equation I_{t,s}; Walk §2.3.1]:
//   I[t][s] = sum_h w[t][h] * ReLU(qI[t][h] . K[s]),  s < floor(p_t / m).
// ([Notes] = "DeepSeek-V4: 迈向高效百万级上下文智能" study notes; [Walk] = the
// mlpod.com walk-through of the DeepSeek-V4 report.)
//
// FFMA kernel (fp32 arithmetic): one CTA scores a tile of 64 keys for one
// query. q and w of the query and the key tile are staged in shared memory
// as fp32 (key rows padded to an odd stride so the 32 lanes of a warp, each
// on its own key, hit distinct banks); each of the 4 warp groups takes every
// 4th head, and the 4 partial head sums are added in a fixed order.
#include "common.cuh"
#include "kernels.h"

namespace csa {

constexpr int kIdxTile = 64;

template <typename T>
__global__ void __launch_bounds__(256) index_scores_ffma_kernel(
    const T* __restrict__ qI, const float* __restrict__ w, const T* __restrict__ K, QueryMap qm,
    int n_seq, int HI, int cI, int64_t Nmax, int m, float* __restrict__ scores, int64_t ld) {
    extern __shared__ float smem[];
    const int kstride = cI + 1;
    float* q_s = smem;                       // [HI][cI]
    float* w_s = q_s + HI * cI;              // [HI]
    float* k_s = w_s + HI;                   // [64][cI+1]
    float* red = k_s + kIdxTile * kstride;   // [4][64]

    const int t = blockIdx.y;
    const int64_t s0 = (int64_t)blockIdx.x * kIdxTile;
    const int tid = threadIdx.x;
    if (s0 >= Nmax) return;
    // a query whose sequence is outside [0, n_seq) sees no entry
    const int seq = qm.seq_of(t);
    const int64_t vis = (seq >= 0 && seq < n_seq) ? visible_entries(qm.pos_of(t), m, Nmax) : 0;
    float* srow = scores + (int64_t)t * ld;
    if (s0 >= vis) {
        for (int i = tid; i < kIdxTile; i += 256)
            if (s0 + i < Nmax) srow[s0 + i] = -INFINITY;
        return;
    }
    const T* Kb = K + (int64_t)seq * Nmax * cI;
    for (int i = tid * 8; i < HI * cI; i += 256 * 8) {
        float v[8];
        load8(qI + (int64_t)t * HI * cI + i, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) q_s[i + u] = v[u];
    }
    for (int h = tid; h < HI; h += 256) w_s[h] = w[(int64_t)t * HI + h];
    const int nk = (int)((vis - s0) < kIdxTile ? (vis - s0) : kIdxTile);
    const int vec_per_row = cI / 8;
    for (int i = tid; i < kIdxTile * vec_per_row; i += 256) {
        int r = i / vec_per_row, e = (i % vec_per_row) * 8;
        float v[8];
        if (r < nk) load8(Kb + (s0 + r) * cI + e, v);
        else {
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) k_s[r * kstride + e + u] = v[u];
    }
    __syncthreads();

    const int key = tid & 63;
    const int hg = tid >> 6;
    float part = 0.f;
    const float* kr = k_s + key * kstride;
    for (int h = hg; h < HI; h += 4) {
        const float* qh = q_s + h * cI;
        float dot = 0.f;
        for (int e = 0; e < cI; ++e) dot = fmaf(qh[e], kr[e], dot);
        part = fmaf(w_s[h], fmaxf(dot, 0.f), part);
    }
    red[hg * kIdxTile + key] = part;
    __syncthreads();
    if (tid < kIdxTile) {
        int64_t s = s0 + tid;
        if (s < Nmax) {
            float v = ((red[tid] + red[kIdxTile + tid]) + red[2 * kIdxTile + tid]) + red[3 * kIdxTile + tid];
            srow[s] = (s < vis) ? v : -INFINITY;
        }
    }
}

cudaError_t index_scores(const void* qI, const float* w, const void* K, QuerySpec qs, int nq, int n_seq,
                         int HI, int cI, int64_t Nmax, int m, float* scores, int64_t ld_scores,
                         ElemType t, cudaStream_t st) {
    if (nq == 0 || Nmax == 0) return cudaSuccess;
    QueryMap qm{qs.seq, qs.pos, qs.pos_base, qs.single_seq};
    size_t smem = sizeof(float) * ((size_t)HI * cI + HI + (size_t)kIdxTile * (cI + 1) + 4 * kIdxTile);
    dim3 grid((unsigned)((Nmax + kIdxTile - 1) / kIdxTile), nq);
    cudaError_t e;
    if (t == ElemType::BF16) {
        auto kern = index_scores_ffma_kernel<bf16>;
        e = smem_ceiling(kern);
        if (e != cudaSuccess) return e;
        CSA_LAUNCH(st, "index_scores_ffma", kern<<<grid, 256, smem, st>>>((const bf16*)qI, w, (const bf16*)K, qm, n_seq, HI, cI, Nmax, m,
                                      scores, ld_scores));
    } else {
        auto kern = index_scores_ffma_kernel<float>;
        e = smem_ceiling(kern);
        if (e != cudaSuccess) return e;
        CSA_LAUNCH(st, "index_scores_ffma", kern<<<grid, 256, smem, st>>>((const float*)qI, w, (const float*)K, qm, n_seq, HI, cI, Nmax, m,
                                      scores, ld_scores));
    }
    return cudaGetLastError();
}

}  // namespace csa
