// Shared-KV multi-query attention [Notes §1.1 last paragraph: each
// compressed entry serves as key and value for all query heads; Walk §2.3.2;
// sink term from Notes §1.3, equation s_{h,i,j}].
// ([Notes] = "DeepSeek-V4: 迈向高效百万级上下文智能" study notes; [Walk] = the
// mlpod.com walk-through of the DeepSeek-V4 report.)
//
// Sparse (CSA: the entries named by idx) and dense (HCA: every entry
// s < floor(p/m')) share one split-KV design:
//   1. mqa_partial: CTA (query, group of 8 heads, split of the entry list)
//      gathers 32 entries at a time into shared memory (fp32), one warp per
//      head computes the 32 logits, updates its running max / sum (online
//      softmax, natural-log domain) and accumulates the unnormalised output
//      for its head; the split writes (O, m, l) to the workspace.
//   2. mqa_combine: per (query, head) merge the splits with their max/sum,
//      add the sink to the denominator, normalise, write out and lse.
// The split boundaries are fixed by (k, nsplit), so results do not depend
// on scheduling.
#include "common.cuh"
#include "kernels.h"

namespace csa {

constexpr int kMqaHeads = 8;     // heads per CTA (one warp each)
constexpr int kMqaTile = 32;     // entries per shared-memory tile

struct MqaPartialArgs {
    const void* q;
    const void* KV;
    const int32_t* idx;   // nullable -> dense
    int k;
    QueryMap qm;
    int n_seq;
    int mp;
    int H, c;
    int64_t Nmax;
    float scale;
    int nsplit;
    int64_t split_len;
    float* part_o;        // [nq][nsplit][H][c]
    float* part_ml;       // [nq][nsplit][H][2]
};

template <typename T>
__global__ void __launch_bounds__(256) mqa_partial_ffma_kernel(MqaPartialArgs a) {
    extern __shared__ float smem[];
    const int c = a.c;
    const int kstride = c + 1;
    float* q_s = smem;                          // [8][c]
    float* kv_s = q_s + kMqaHeads * c;          // [32][c+1]
    float* p_s = kv_s + kMqaTile * kstride;     // [8][32]
    __shared__ int ent[kMqaTile];

    const int t = blockIdx.z;
    const int h0 = blockIdx.y * kMqaHeads;
    const int split = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = h0 + warp;

    const T* qg = (const T*)a.q + (int64_t)t * a.H * c;
    const int seq = a.qm.seq_of(t);
    const bool seq_ok = seq >= 0 && seq < a.n_seq;
    const T* KVb = (const T*)a.KV + (int64_t)(seq_ok ? seq : 0) * a.Nmax * c;
    int64_t n_ent;
    if (!seq_ok) n_ent = 0;
    else if (a.idx) n_ent = a.k;
    else n_ent = visible_entries(a.qm.pos_of(t), a.mp, a.Nmax);
    const int64_t e_beg = (int64_t)split * a.split_len;
    int64_t e_end = e_beg + a.split_len;
    if (e_end > n_ent) e_end = n_ent;

    for (int i = threadIdx.x * 8; i < kMqaHeads * c; i += 256 * 8) {
        int hh = h0 + i / c;
        float v[8];
        if (hh < a.H) load8(qg + (int64_t)h0 * c + i, v);
        else {
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) q_s[i + u] = v[u] * a.scale;
    }

    const int per_lane = c / 32;   // c is a multiple of 32 here
    float o[CSA_MAX_HEAD_DIM / 32];
#pragma unroll
    for (int i = 0; i < CSA_MAX_HEAD_DIM / 32; ++i) o[i] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;

    for (int64_t tb = e_beg; tb < e_end; tb += kMqaTile) {
        __syncthreads();
        if (threadIdx.x < kMqaTile) {
            int64_t e = tb + threadIdx.x;
            int s = -1;
            if (e < e_end) s = a.idx ? a.idx[(int64_t)t * a.k + e] : (int)e;
            if (s >= a.Nmax) s = -1;
            ent[threadIdx.x] = s;
        }
        __syncthreads();
        const int vec_per_row = c / 8;
        for (int i = threadIdx.x; i < kMqaTile * vec_per_row; i += 256) {
            int r = i / vec_per_row, d = (i % vec_per_row) * 8;
            float v[8];
            int s = ent[r];
            if (s >= 0) load8(KVb + (int64_t)s * c + d, v);
            else {
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = 0.f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) kv_s[r * kstride + d + u] = v[u];
        }
        __syncthreads();
        // logits: lane = entry
        const float* qh = q_s + warp * c;
        const float* kr = kv_s + lane * kstride;
        float z = 0.f;
        for (int d = 0; d < c; ++d) z = fmaf(qh[d], kr[d], z);
        if (ent[lane] < 0) z = -INFINITY;
        float tmax = warp_max(z);
        float m_new = fmaxf(m_run, tmax);
        float p = (m_new == -INFINITY) ? 0.f : expf(z - m_new);
        float alpha = (m_new == -INFINITY) ? 1.f : expf(m_run - m_new);
        l_run = l_run * alpha + warp_sum(p);
        m_run = m_new;
        p_s[warp * kMqaTile + lane] = p;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < CSA_MAX_HEAD_DIM / 32; ++i) {
            if (i < per_lane) {
                float acc = o[i] * alpha;
                for (int e = 0; e < kMqaTile; ++e)
                    acc = fmaf(p_s[warp * kMqaTile + e], kv_s[e * kstride + lane + 32 * i], acc);
                o[i] = acc;
            }
        }
    }
    if (h < a.H) {
        float* po = a.part_o + (((int64_t)t * a.nsplit + split) * a.H + h) * c;
#pragma unroll
        for (int i = 0; i < CSA_MAX_HEAD_DIM / 32; ++i)
            if (i < per_lane) po[lane + 32 * i] = o[i];
        if (lane == 0) {
            float* pm = a.part_ml + (((int64_t)t * a.nsplit + split) * a.H + h) * 2;
            pm[0] = m_run;
            pm[1] = l_run;
        }
    }
}

// Merge of split-KV partials: split s holds O_s (fp32, scaled by exp(-m_s)),
// m_s and l_s for every (query, head); the result is
//   out = sum_s e^{m_s - M} O_s / (sum_s e^{m_s - M} l_s + [sink] e^{z' - M})
// with M the largest of the m_s and the sink logit, and lse = M + log(...).
// A block takes kCombineHeads heads of one query and kCombineDims of their
// dims; every thread combines 4 consecutive dims of one head on its own: the
// splits' (m, l) pairs and 16-byte O loads of up to 8 splits are issued
// together, then weighted in split order (one L2 round trip per 8 splits, no
// block barrier); with more than 8 splits the running maximum moves from
// group to group and the sums so far are rescaled (an online merge). A split
// with m = -inf (it saw no entry) staged no O and gets weight 0 by selection,
// never by multiplying its stale rows. One store per 4 results.
constexpr int kCombineHeads = 8;
constexpr int kCombineDims = 128;
template <typename T>
__global__ void __launch_bounds__(kCombineHeads * 32) mqa_combine_kernel(const float* __restrict__ part_o,
                                                                         const float* __restrict__ part_ml,
                                                                         int nsplit, int H, int c,
                                                                         const float* __restrict__ sink,
                                                                         T* __restrict__ out, float* __restrict__ lse) {
    pdl_wait();
    pdl_launch_next();
    const int t = blockIdx.y, h0 = blockIdx.x * kCombineHeads;
    const int nh = H - h0 < kCombineHeads ? H - h0 : kCombineHeads;
    const int d0 = blockIdx.z * kCombineDims;
    const int c4 = (c - d0 < kCombineDims ? c - d0 : kCombineDims) / 4;
    const int64_t sstride = (int64_t)H * c;   // one split to the next
    for (int e = threadIdx.x; e < nh * c4; e += blockDim.x) {
        const int i = e / c4, j4 = e - i * c4, d = d0 + j4 * 4;
        const int h = h0 + i;
        const float* po = part_o + ((int64_t)t * nsplit * H + h) * c + d;
        const float* ml = part_ml + ((int64_t)t * nsplit * H + h) * 2;
        const float z = sink ? __ldg(sink + h) : -INFINITY;
        float M = z, L = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = 0; s0 < nsplit; s0 += 8) {
            float mv[8], lv[8];
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const bool in = s0 + u < nsplit;
                mv[u] = in ? ml[(int64_t)(s0 + u) * H * 2] : -INFINITY;
                lv[u] = in ? ml[(int64_t)(s0 + u) * H * 2 + 1] : 0.f;
                v[u] = in ? *reinterpret_cast<const float4*>(po + (s0 + u) * sstride) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            float Mn = M;
#pragma unroll
            for (int u = 0; u < 8; ++u) Mn = fmaxf(Mn, mv[u]);
            if (Mn == -INFINITY) continue;                 // nothing seen yet
            const float r = M == -INFINITY ? 0.f : expf(M - Mn);
            L *= r;
            acc.x *= r; acc.y *= r; acc.z *= r; acc.w *= r;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (mv[u] == -INFINITY) continue;
                const float wgt = expf(mv[u] - Mn);
                L += wgt * lv[u];
                acc.x += wgt * v[u].x; acc.y += wgt * v[u].y; acc.z += wgt * v[u].z; acc.w += wgt * v[u].w;
            }
            M = Mn;
        }
        if (sink && M != -INFINITY) L += expf(z - M);
        const float inv = (L > 0.f) ? 1.f / L : 0.f;
        store4(out + ((int64_t)t * H + h) * c + d, acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        if (lse && blockIdx.z == 0 && j4 == 0) lse[(int64_t)t * H + h] = (L > 0.f) ? M + logf(L) : -INFINITY;
    }
}

static int mqa_nsplit(int nq, int H, int64_t max_entries) {
    int hg = (H + kMqaHeads - 1) / kMqaHeads;
    int64_t ctas = (int64_t)nq * hg;
    int64_t want = (4 * 148 + ctas - 1) / (ctas > 0 ? ctas : 1);
    int64_t cap = (max_entries + kMqaTile - 1) / kMqaTile;
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    if (want > 64) want = 64;
    return (int)want;
}

static int num_sms_cached() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    }
    return n;
}

static int plan_nsplit(int nq, int H, int64_t max_entries, ElemType t) {
    return t == ElemType::BF16 ? mqa_tc_nsplit(nq, H, max_entries, num_sms_cached())
                               : mqa_nsplit(nq, H, max_entries);
}

size_t mqa_workspace_bytes(int nq, int H, int c, int64_t max_entries, ElemType t) {
    int ns = plan_nsplit(nq, H, max_entries, t);
    // a single split writes the output directly; two merge on chip
    if (t == ElemType::BF16 && (ns == 1 || mqa_tc_pair(ns))) return 0;
    return align256((size_t)nq * ns * H * c * sizeof(float)) +
           align256((size_t)nq * ns * H * 2 * sizeof(float));
}

cudaError_t mqa(const void* q, const void* KV, const int32_t* idx, int k, QuerySpec qs, int mp,
                int nq, int n_seq, int H, int c, int64_t Nmax, float scale, const float* sink, void* out,
                float* lse, void* ws, ElemType t, cudaStream_t st, RowBlocks kvb) {
    if (nq == 0) return cudaSuccess;
    const int64_t max_entries = idx ? k : Nmax;
    if (t == ElemType::BF16) {
        const int ns = plan_nsplit(nq, H, max_entries, t);
        cudaError_t e = mqa_tc(q, KV, idx, k, qs, mp, nq, n_seq, H, c, Nmax, scale, sink, out, lse, ws, ns,
                               device_status(), st, kvb);
        if (e != cudaSuccess || ns == 1 || mqa_tc_pair(ns)) return e;
        float* part_o = (float*)ws;
        float* part_ml = (float*)((char*)ws + align256((size_t)nq * ns * H * c * sizeof(float)));
        CSA_LAUNCH(st, "mqa_combine",
                   e = launch_pdl(mqa_combine_kernel<bf16>,
                                  dim3((H + kCombineHeads - 1) / kCombineHeads, nq, (c + kCombineDims - 1) / kCombineDims),
                                  dim3(kCombineHeads * 32), 0, st, 0, (const float*)part_o,
                                  (const float*)part_ml, ns, H, c, sink, (bf16*)out, lse));
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    const int ns = mqa_nsplit(nq, H, max_entries);
    MqaPartialArgs a{};
    a.q = q; a.KV = KV; a.idx = idx; a.k = k;
    a.qm = QueryMap{qs.seq, qs.pos, qs.pos_base, qs.single_seq};
    a.n_seq = n_seq; a.mp = mp; a.H = H; a.c = c; a.Nmax = Nmax; a.scale = scale; a.nsplit = ns;
    int64_t per = (max_entries + ns - 1) / ns;
    a.split_len = ((per + kMqaTile - 1) / kMqaTile) * kMqaTile;
    if (a.split_len == 0) a.split_len = kMqaTile;
    a.part_o = (float*)ws;
    a.part_ml = (float*)((char*)ws + align256((size_t)nq * ns * H * c * sizeof(float)));
    size_t smem = sizeof(float) * ((size_t)kMqaHeads * c + (size_t)kMqaTile * (c + 1) + kMqaHeads * kMqaTile);
    dim3 grid(ns, (H + kMqaHeads - 1) / kMqaHeads, nq);
    cudaError_t e;
    if (t == ElemType::BF16) {
        auto kern = mqa_partial_ffma_kernel<bf16>;
        e = smem_ceiling(kern);
        if (e != cudaSuccess) return e;
        CSA_LAUNCH(st, "mqa_partial_ffma", kern<<<grid, 256, smem, st>>>(a));
    } else {
        auto kern = mqa_partial_ffma_kernel<float>;
        e = smem_ceiling(kern);
        if (e != cudaSuccess) return e;
        CSA_LAUNCH(st, "mqa_partial_ffma", kern<<<grid, 256, smem, st>>>(a));
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 g2((H + kCombineHeads - 1) / kCombineHeads, nq, (c + kCombineDims - 1) / kCombineDims);
    if (t == ElemType::BF16)
        CSA_LAUNCH(st, "mqa_combine", mqa_combine_kernel<bf16><<<g2, kCombineHeads * 32, 0, st>>>(
                                          a.part_o, a.part_ml, ns, H, c, sink, (bf16*)out, lse));
    else
        CSA_LAUNCH(st, "mqa_combine", mqa_combine_kernel<float><<<g2, kCombineHeads * 32, 0, st>>>(
                                          a.part_o, a.part_ml, ns, H, c, sink, (float*)out, lse));
    return cudaGetLastError();
}

}  // namespace csa
