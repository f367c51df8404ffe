// CSA / HCA token compressors on projected inputs.
//
// CSA [Notes §1.1, equation C^Comp_i]: entry i mixes the a-stream of its own
// m tokens and the b-stream of the previous block's m tokens with ONE
// softmax per channel over the 2m logits Z + B (positional bias).
// HCA [Notes §1.2, comparison table]: one non-overlapping window of m' tokens.
//
// ([Notes] = "DeepSeek-V4: 迈向高效百万级上下文智能", study notes on the DeepSeek-V4
// report, notes.kuangjux.top.)
//
// HBM-bound elementwise work: one thread owns (entry, 8 channels), reads each
// projected row of its window with 16-byte vector loads (consecutive threads
// take consecutive channel groups, so a warp reads 512 contiguous bytes of
// bf16), runs the windowed softmax online in registers and writes 8 output
// channels with one vector store. Every projected element is read once.
#include "common.cuh"
#include "kernels.h"

namespace csa {

struct OnlineSoftmax8 {
    float mx[8], den[8], acc[8];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int u = 0; u < 8; ++u) { mx[u] = -INFINITY; den[u] = 0.f; acc[u] = 0.f; }
    }
    __device__ __forceinline__ void push(const float (&logit)[8], const float (&val)[8]) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            float nm = fmaxf(mx[u], logit[u]);
            float keep = expf(mx[u] - nm);   // 0 for the first push (mx = -inf)
            float p = expf(logit[u] - nm);
            den[u] = den[u] * keep + p;
            acc[u] = acc[u] * keep + p * val[u];
            mx[u] = nm;
        }
    }
};

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(256) csa_compress_kernel(const TIn* __restrict__ proj,
                                                           const TIn* __restrict__ left,
                                                           const float* __restrict__ bias,
                                                           int64_t nb, int c, int m,
                                                           TOut* __restrict__ out) {
    pdl_wait();
    pdl_launch_next();
    const int groups = c / 8;
    int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= nb * groups) return;
    const int64_t i = gid / groups;
    const int j = (int)(gid % groups) * 8;
    const int64_t ld = 4 * (int64_t)c;

    OnlineSoftmax8 sm;
    sm.init();
    float z[8], b[8], v[8];
    // a-window: tokens m*i .. m*i+m-1, C^a and Z^a, bias rows 0..m-1
    for (int r = 0; r < m; ++r) {
        const TIn* row = proj + (m * i + r) * ld;
        load8(row + 2 * c + j, z);
        load8(bias + (int64_t)r * c + j, b);
        load8(row + j, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) z[u] += b[u];
        sm.push(z, v);
    }
    // b-window: tokens m*(i-1) .. m*i-1, C^b and Z^b, bias rows m..2m-1;
    // absent for block 0 at the start of a sequence
    if (i > 0 || left != nullptr) {
        for (int r = 0; r < m; ++r) {
            const TIn* row = (i > 0) ? proj + (m * (i - 1) + r) * ld : left + (int64_t)r * ld;
            load8(row + 3 * c + j, z);
            load8(bias + (int64_t)(m + r) * c + j, b);
            load8(row + c + j, v);
#pragma unroll
            for (int u = 0; u < 8; ++u) z[u] += b[u];
            sm.push(z, v);
        }
    }
    float o[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) o[u] = sm.acc[u] / sm.den[u];
    if constexpr (sizeof(TOut) == 2) store8(reinterpret_cast<bf16*>(out + i * c + j), o);
    else store8(reinterpret_cast<float*>(out + i * c + j), o);
}

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(256) hca_compress_kernel(const TIn* __restrict__ proj,
                                                           const float* __restrict__ bias,
                                                           int64_t nb, int c, int mp,
                                                           TOut* __restrict__ out) {
    pdl_wait();
    pdl_launch_next();
    const int groups = c / 8;
    int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= nb * groups) return;
    const int64_t i = gid / groups;
    const int j = (int)(gid % groups) * 8;
    const int64_t ld = 2 * (int64_t)c;

    OnlineSoftmax8 sm;
    sm.init();
    float z[8], b[8], v[8];
#pragma unroll 4
    for (int r = 0; r < mp; ++r) {
        const TIn* row = proj + (mp * i + r) * ld;
        load8(row + c + j, z);
        load8(bias + (int64_t)r * c + j, b);
        load8(row + j, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) z[u] += b[u];
        sm.push(z, v);
    }
    float o[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) o[u] = sm.acc[u] / sm.den[u];
    if constexpr (sizeof(TOut) == 2) store8(reinterpret_cast<bf16*>(out + i * c + j), o);
    else store8(reinterpret_cast<float*>(out + i * c + j), o);
}

// The sum of nsplit fp32 slices of 8 channels, slice s at src + s * pstride,
// added in slice order. The loads of 16 slices issue before their adds (a
// batch past the last slice re-reads the last one and adds nothing).
__device__ __forceinline__ void sum_slices(const float* src, int nsplit, int64_t pstride, float (&v)[8]) {
    load8(src, v);
    for (int k0 = 1; k0 < nsplit; k0 += 16) {
        float u[16][8];
#pragma unroll
        for (int q = 0; q < 16; ++q) load8(src + (int64_t)min(k0 + q, nsplit - 1) * pstride, u[q]);
#pragma unroll
        for (int q = 0; q < 16; ++q)
            if (k0 + q < nsplit) {
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] += u[q][e];
            }
    }
}

// Decode-time compression through the per-sequence state cache [Walk §5
// item 2: CSA keeps the tail tokens that have not yet formed a block; Notes
// §2.6 Fig. 6]. Each sequence keeps the projected rows of its last 2m tokens
// (m' for HCA) in a ring, token tau in slot tau mod 2m. A step stores the
// newest token's row and, when that token closes a block, mixes the block
// from the ring in exactly the order of the chunk kernels above (a-window,
// then b-window), so a sequence compressed token by token gets the same
// entries as one compressed in a chunk. A thread owns 8 channels of one
// sequence and reads only the ring values of those channels, written by the
// same thread slot in this step or an earlier one (an earlier launch has
// completed before pdl_wait returns).
// proj may hold nsplit partial sums of the projection (a split-K GEMM),
// slice s at proj + s * pstride; they are added in slice order. One launch
// serves up to two streams with the same m and positions (the KV and
// index-key compressors of a decode step): blocks [0, blocks0) take stream 0,
// the rest stream 1. A block takes 32 (sequence, 8-channel) pairs; warp w
// sums and stores group w of the four (a-values, b-values, a-logits,
// b-logits), and after a block barrier warp 0 mixes the blocks that close.
// kM > 0: the compression rate is the compile-time kM, so the window loops
// unroll and their loads issue together.
template <typename TOut, int kM>
__global__ void __launch_bounds__(128) csa_compress_step_kernel(const StepStream s0, const StepStream s1,
                                                                const int32_t* __restrict__ pos, int B, int m_rt,
                                                                int64_t Nmax, int blocks0) {
    const int m = kM > 0 ? kM : m_rt;
    pdl_wait();
    pdl_launch_next();
    const bool second = (int)blockIdx.x >= blocks0;
    const int blk = second ? (int)blockIdx.x - blocks0 : (int)blockIdx.x;
    const int c = second ? s1.c : s0.c;
    const float* __restrict__ proj_new = second ? s1.proj : s0.proj;
    float* state = second ? s1.state : s0.state;
    const float* __restrict__ bias = second ? s1.bias : s0.bias;
    const int nsplit = second ? s1.nsplit : s0.nsplit;
    const int64_t pstride = second ? s1.pstride : s0.pstride;
    const int groups = c / 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t pair = (int64_t)blk * 32 + lane;
    const bool live = groups > 0 && pair < (int64_t)B * groups;
    int b = 0, j = 0;
    int64_t p = -1;
    if (live) {
        b = (int)(pair / groups);
        j = (int)(pair % groups) * 8;
        p = pos[b];
    }
    const int64_t ld = 4 * (int64_t)c;
    float* ring = state + (int64_t)b * 2 * m * ld;
    if (live && p >= 0) {
        float v[8];
        sum_slices(proj_new + (int64_t)b * ld + warp * c + j, nsplit, pstride, v);
        store8(ring + (p % (2 * m)) * ld + warp * c + j, v);
    }
    __syncthreads();   // the block's ring stores are visible to its warp 0
    if (warp != 0 || !live || p < 0 || (p + 1) % m != 0) return;
    const int64_t i = (p + 1) / m - 1;   // the block this token closes
    if (i >= Nmax) return;

    OnlineSoftmax8 sm;
    sm.init();
    float z[8], bb[8], v[8];
#pragma unroll(kM > 0 ? kM : 1)
    for (int r = 0; r < m; ++r) {
        const float* row = ring + ((m * i + r) % (2 * m)) * ld;
        load8(row + 2 * c + j, z);
        load8(bias + (int64_t)r * c + j, bb);
        load8(row + j, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) z[u] += bb[u];
        sm.push(z, v);
    }
    if (i > 0) {
#pragma unroll(kM > 0 ? kM : 1)
        for (int r = 0; r < m; ++r) {
            const float* row = ring + ((m * (i - 1) + r) % (2 * m)) * ld;
            load8(row + 3 * c + j, z);
            load8(bias + (int64_t)(m + r) * c + j, bb);
            load8(row + c + j, v);
#pragma unroll
            for (int u = 0; u < 8; ++u) z[u] += bb[u];
            sm.push(z, v);
        }
    }
    float o[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) o[u] = sm.acc[u] / sm.den[u];
    TOut* out = reinterpret_cast<TOut*>(static_cast<char*>(second ? s1.cache : s0.cache) +
                                        row_byte_offset((int64_t)b * Nmax + i, (int64_t)c * sizeof(TOut),
                                                        second ? s1.cb : s0.cb)) + j;
    if constexpr (sizeof(TOut) == 2) store8(reinterpret_cast<bf16*>(out), o);
    else store8(reinterpret_cast<float*>(out), o);
}

// HCA: a ring of m' rows (C | Z), slot tau mod m'; the token that closes a
// block finds the block's rows in slots 0 .. m'-1 in token order.
template <typename TOut>
__global__ void __launch_bounds__(256) hca_compress_step_kernel(const float* __restrict__ proj_new,
                                                                float* __restrict__ state,
                                                                const float* __restrict__ bias,
                                                                const int32_t* __restrict__ pos, int B, int c,
                                                                int mp, int64_t Nmax, TOut* __restrict__ cache,
                                                                int nsplit, int64_t pstride, RowBlocks cb) {
    pdl_wait();
    pdl_launch_next();
    const int groups = c / 8;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (int64_t)B * groups) return;
    const int b = (int)(gid / groups);
    const int j = (int)(gid % groups) * 8;
    const int64_t p = pos[b];
    if (p < 0) return;
    const int64_t ld = 2 * (int64_t)c;
    float* ring = state + (int64_t)b * mp * ld;
    {
        const float* src = proj_new + (int64_t)b * ld;
        float* dst = ring + (p % mp) * ld;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
            float v[8];
            sum_slices(src + h * c + j, nsplit, pstride, v);
            store8(dst + h * c + j, v);
        }
    }
    if ((p + 1) % mp != 0) return;
    const int64_t i = (p + 1) / mp - 1;
    if (i >= Nmax) return;

    OnlineSoftmax8 sm;
    sm.init();
    float z[8], bb[8], v[8];
#pragma unroll 4
    for (int r = 0; r < mp; ++r) {
        const float* row = ring + (int64_t)r * ld;
        load8(row + c + j, z);
        load8(bias + (int64_t)r * c + j, bb);
        load8(row + j, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) z[u] += bb[u];
        sm.push(z, v);
    }
    float o[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) o[u] = sm.acc[u] / sm.den[u];
    TOut* out = reinterpret_cast<TOut*>(reinterpret_cast<char*>(cache) +
                                        row_byte_offset((int64_t)b * Nmax + i, (int64_t)c * sizeof(TOut), cb)) + j;
    if constexpr (sizeof(TOut) == 2) store8(reinterpret_cast<bf16*>(out), o);
    else store8(reinterpret_cast<float*>(out), o);
}

// Chunk compression at any start and length through the state ring [Walk §5
// item 2; Notes §2.6 Fig. 6]: the chunk holds tokens start .. start+n-1 of
// one sequence, projected (fp32, proj row tau - start). It writes the entry
// of every block that ends inside the chunk, i in [i_lo, i_lo + nb), taking
// each window token tau from the chunk when tau >= start and from the ring
// (slot tau mod ring_rows) when the token came earlier: the ring holds the
// projected rows of the sequence's last ring_rows tokens before the chunk
// (2m for CSA, m' for HCA). One thread per (entry, 8 channels), the window
// terms in the chunk kernels' order, so an entry is the same wherever its
// tokens came from. The ring is refreshed afterwards by ring_store_kernel, a
// separate launch, because a new token's slot may hold a row this one reads.
template <typename TOut>
__global__ void __launch_bounds__(256) compress_chunk_state_kernel(const float* __restrict__ proj,
                                                                   const float* __restrict__ ring,
                                                                   const float* __restrict__ bias, int64_t start,
                                                                   int64_t i_lo, int64_t nb, int c, int m,
                                                                   int overlap, TOut* __restrict__ cache) {
    pdl_wait();
    pdl_launch_next();
    const int groups = c / 8;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= nb * groups) return;
    const int64_t i = i_lo + gid / groups;
    const int j = (int)(gid % groups) * 8;
    const int64_t ld = (overlap ? 4 : 2) * (int64_t)c;
    const int ring_rows = overlap ? 2 * m : m;
    auto row_of = [&](int64_t tau) -> const float* {
        return tau >= start ? proj + (tau - start) * ld : ring + (tau % ring_rows) * ld;
    };
    OnlineSoftmax8 sm;
    sm.init();
    float z[8], b[8], v[8];
    // a-window (CSA: C^a, Z^a, bias rows 0..m-1; HCA: C, Z, bias rows 0..m'-1)
    for (int r = 0; r < m; ++r) {
        const float* row = row_of(m * i + r);
        load8(row + (overlap ? 2 * c : c) + j, z);
        load8(bias + (int64_t)r * c + j, b);
        load8(row + j, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) z[u] += b[u];
        sm.push(z, v);
    }
    // CSA b-window: the previous block's tokens, C^b, Z^b, bias rows m..2m-1;
    // none for the first block of the sequence
    if (overlap && i > 0) {
        for (int r = 0; r < m; ++r) {
            const float* row = row_of(m * (i - 1) + r);
            load8(row + 3 * c + j, z);
            load8(bias + (int64_t)(m + r) * c + j, b);
            load8(row + c + j, v);
#pragma unroll
            for (int u = 0; u < 8; ++u) z[u] += b[u];
            sm.push(z, v);
        }
    }
    float o[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) o[u] = sm.acc[u] / sm.den[u];
    TOut* out = cache + i * c + j;
    if constexpr (sizeof(TOut) == 2) store8(reinterpret_cast<bf16*>(out), o);
    else store8(reinterpret_cast<float*>(out), o);
}

// The ring after the chunk: the projected rows of the chunk's last
// min(n, ring_rows) tokens go to their slots (tau mod ring_rows); the other
// slots keep the earlier tokens that are still among the last ring_rows.
__global__ void __launch_bounds__(256) ring_store_kernel(const float* __restrict__ proj, float* __restrict__ ring,
                                                         int64_t start, int64_t n, int ring_rows, int64_t ld) {
    pdl_wait();
    pdl_launch_next();
    const int64_t keep = n < ring_rows ? n : ring_rows;
    const int64_t per_row = ld / 4;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= keep * per_row) return;
    const int64_t tau = start + n - keep + gid / per_row;
    const int64_t col = (gid % per_row) * 4;
    const float4 v = *reinterpret_cast<const float4*>(proj + (tau - start) * ld + col);
    *reinterpret_cast<float4*>(ring + (tau % ring_rows) * ld + col) = v;
}

cudaError_t compress_chunk_state(const float* proj, float* state, const float* bias, int64_t start, int64_t n, int c,
                                 int m, bool overlap, void* cache, ElemType out_t, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const int64_t i_lo = start / m;
    const int64_t nb = (start + n) / m - i_lo;
    const int64_t threads = nb * (c / 8);
    cudaError_t e = cudaSuccess;
    if (threads > 0) {
        const dim3 grid((unsigned)((threads + 255) / 256));
        if (out_t == ElemType::BF16)
            CSA_LAUNCH(st, overlap ? "csa_compress_chunk" : "hca_compress_chunk",
                       e = launch_pdl(compress_chunk_state_kernel<bf16>, grid, dim3(256), 0, st, 0, proj,
                                      (const float*)state, bias, start, i_lo, nb, c, m, overlap ? 1 : 0, (bf16*)cache));
        else
            CSA_LAUNCH(st, overlap ? "csa_compress_chunk" : "hca_compress_chunk",
                       e = launch_pdl(compress_chunk_state_kernel<float>, grid, dim3(256), 0, st, 0, proj,
                                      (const float*)state, bias, start, i_lo, nb, c, m, overlap ? 1 : 0,
                                      (float*)cache));
        if (e != cudaSuccess) return e;
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int ring_rows = overlap ? 2 * m : m;
    const int64_t ld = (overlap ? 4 : 2) * (int64_t)c;
    const int64_t keep = n < ring_rows ? n : ring_rows;
    const int64_t t2 = keep * (ld / 4);
    CSA_LAUNCH(st, "ring_store",
               e = launch_pdl(ring_store_kernel, dim3((unsigned)((t2 + 255) / 256)), dim3(256), 0, st, 0, proj, state,
                              start, n, ring_rows, ld));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename TIn, typename TOut>
cudaError_t launch_csa_compress(const void* proj, const void* left, const float* bias, int64_t n,
                                int c, int m, void* out, cudaStream_t st) {
    int64_t nb = n / m;
    int64_t threads = nb * (c / 8);
    if (threads == 0) return cudaSuccess;
    cudaError_t e = cudaSuccess;
    CSA_LAUNCH(st, "csa_compress",
               e = launch_pdl(csa_compress_kernel<TIn, TOut>, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, st,
                              0, (const TIn*)proj, (const TIn*)left, bias, nb, c, m, (TOut*)out));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename TIn, typename TOut>
cudaError_t launch_hca_compress(const void* proj, const float* bias, int64_t n, int c, int mp,
                                void* out, cudaStream_t st) {
    int64_t nb = n / mp;
    int64_t threads = nb * (c / 8);
    if (threads == 0) return cudaSuccess;
    cudaError_t e = cudaSuccess;
    CSA_LAUNCH(st, "hca_compress",
               e = launch_pdl(hca_compress_kernel<TIn, TOut>, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, st,
                              0, (const TIn*)proj, bias, nb, c, mp, (TOut*)out));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t compress_csa(const void* proj, const void* left, const float* bias, int64_t n, int c,
                         int m, void* out, ElemType in_t, ElemType out_t, cudaStream_t st) {
    if (in_t == ElemType::BF16 && out_t == ElemType::BF16)
        return launch_csa_compress<bf16, bf16>(proj, left, bias, n, c, m, out, st);
    if (in_t == ElemType::F32 && out_t == ElemType::BF16)
        return launch_csa_compress<float, bf16>(proj, left, bias, n, c, m, out, st);
    return launch_csa_compress<float, float>(proj, left, bias, n, c, m, out, st);
}

cudaError_t compress_hca(const void* proj, const float* bias, int64_t n, int c, int mp, void* out,
                         ElemType in_t, ElemType out_t, cudaStream_t st) {
    if (in_t == ElemType::BF16 && out_t == ElemType::BF16)
        return launch_hca_compress<bf16, bf16>(proj, bias, n, c, mp, out, st);
    if (in_t == ElemType::F32 && out_t == ElemType::BF16)
        return launch_hca_compress<float, bf16>(proj, bias, n, c, mp, out, st);
    return launch_hca_compress<float, float>(proj, bias, n, c, mp, out, st);
}

cudaError_t compress_step(const float* proj_new, float* state, const float* bias, const int32_t* pos, int B, int c,
                          int m, bool overlap, int64_t Nmax, void* cache, ElemType out_t, cudaStream_t st, int nsplit,
                          RowBlocks cb) {
    if (overlap) {
        StepStream s{proj_new, state, bias, cache, c, nsplit, (int64_t)B * 4 * c, cb};
        StepStream none{};
        return compress_step_csa2(s, none, pos, B, m, Nmax, out_t, st);
    }
    const int64_t pstride = (int64_t)B * 2 * c;
    const int64_t threads = (int64_t)B * (c / 8);
    if (threads == 0) return cudaSuccess;
    const dim3 grid((unsigned)((threads + 255) / 256));
    cudaError_t e = cudaSuccess;
    if (out_t == ElemType::BF16)
        CSA_LAUNCH(st, "hca_compress_step",
                   e = launch_pdl(hca_compress_step_kernel<bf16>, grid, dim3(256), 0, st, 0, proj_new, state, bias,
                                  pos, B, c, m, Nmax, (bf16*)cache, nsplit, pstride, cb));
    else
        CSA_LAUNCH(st, "hca_compress_step",
                   e = launch_pdl(hca_compress_step_kernel<float>, grid, dim3(256), 0, st, 0, proj_new, state, bias,
                                  pos, B, c, m, Nmax, (float*)cache, nsplit, pstride, cb));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t compress_step_csa2(const StepStream& s0, const StepStream& s1, const int32_t* pos, int B, int m,
                               int64_t Nmax, ElemType out_t, cudaStream_t st) {
    const int64_t pairs0 = (int64_t)B * (s0.c / 8), pairs1 = (int64_t)B * (s1.c / 8);
    const int blocks0 = (int)((pairs0 + 31) / 32);
    const int64_t blocks = blocks0 + (pairs1 + 31) / 32;
    if (blocks == 0) return cudaSuccess;
    const dim3 grid((unsigned)blocks);
    cudaError_t e = cudaSuccess;
    if (out_t == ElemType::BF16)
        CSA_LAUNCH(st, "csa_compress_step",
                   e = launch_pdl(m == 4 ? csa_compress_step_kernel<bf16, 4> : csa_compress_step_kernel<bf16, 0>, grid,
                                  dim3(128), 0, st, 0, s0, s1, pos, B, m, Nmax, blocks0));
    else
        CSA_LAUNCH(st, "csa_compress_step",
                   e = launch_pdl(m == 4 ? csa_compress_step_kernel<float, 4> : csa_compress_step_kernel<float, 0>,
                                  grid, dim3(128), 0, st, 0, s0, s1, pos, B, m, Nmax, blocks0));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace csa
