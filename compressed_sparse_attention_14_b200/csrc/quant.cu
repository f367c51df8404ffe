// Row-wise FP8 (e4m3) storage of indexer operands [Notes §2.4: the indexer
// runs its query-key products in low precision; Notes §1.3: FP8 storage]
// ([Notes] = "DeepSeek-V4: 迈向高效百万级上下文智能", study notes on the
// DeepSeek-V4 report).
//
// Each row of `cols` values gets the scale s = max|row| / 448 (1 for an
// all-zero row), so its largest element maps to the format's largest finite
// magnitude, and every element is stored as the e4m3 value nearest x / s
// (ties to even; magnitudes past 448 saturate: the format has no infinity).
// The scale and the division are taken in fp64, so the stored code is the
// one the exact quotient rounds to; the scale is returned in fp32. With head
// weights w given (one per row), w_out = w * s is written too: the indexer's
// ReLU commutes with the positive query scale, so the scale folds into the
// head weight.
//
// e4m3: sign, 4 exponent bits (bias 7), 3 mantissa bits. Normal values
// 2^-6 .. 448 (exponent field 1..15; the code 0x7F is NaN), subnormals in
// steps of 2^-9 (exponent field 0). One warp per row, four values per lane.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

// 4 consecutive values as fp32 (an 8-byte bf16 load or a 16-byte fp32 one).
__device__ __forceinline__ void load4(const bf16* p, float (&v)[4]) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xFFFF0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xFFFF0000u);
}
__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
    const float4 f = *reinterpret_cast<const float4*>(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}

// The e4m3 code of the value nearest to v (|v| <= 448 assumed after the
// saturation test), written from the format's definition.
__device__ __forceinline__ uint8_t e4m3_code(double v) {
    const uint32_t sign = v < 0.0 ? 0x80u : 0u;
    const double a = fabs(v);
    if (!(a > 0.0)) return (uint8_t)sign;                 // zero (NaN never reaches here)
    if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);       // saturate: 1.75 * 2^8
    // a in [2^e, 2^(e+1)), read from the exponent field: a is a normal double
    // (a quotient of fp32 / bf16 values by their row's max / 448)
    const int e = (int)((__double_as_longlong(a) >> 52) & 0x7ff) - 1023;
    int q = e - 3;                                        // spacing of 4 significant bits
    if (q < -9) q = -9;                                   // subnormal spacing
    // a * 2^-q is exact (a power-of-two scale within range); then nearest,
    // ties to even
    double r = rint(a * __longlong_as_double((long long)(1023 - q) << 52));
    uint32_t code;
    if (q == -9 && r < 8.0) {
        code = (uint32_t)r;                               // subnormal (or zero)
    } else {
        if (r >= 16.0) {                                  // rounded up into the next binade
            r = 8.0;
            ++q;
        }
        const int ef = q + 3 + 7;                         // exponent field of r * 2^q, r in [8, 16)
        code = ((uint32_t)ef << 3) | (uint32_t)(r - 8.0);
        if (code > 0x7Eu) code = 0x7Eu;                   // beyond 448: saturate
    }
    return (uint8_t)(sign | code);
}

// x rows of `ld` values; the first `cols` are quantised. rope (rows of
// rope_dims, the cache dtype) gets the row's values cols .. cols+rope_dims-1
// unchanged when given (the rotary dims of an FP8 KV entry).
template <typename TIn>
__global__ void __launch_bounds__(256) quantize_e4m3_kernel(const TIn* __restrict__ x, int64_t rows, int cols,
                                                            int64_t ld, uint8_t* __restrict__ out,
                                                            float* __restrict__ scale, const float* __restrict__ w,
                                                            float* __restrict__ w_out, TIn* __restrict__ rope,
                                                            int rope_dims) {
    pdl_wait();
    pdl_launch_next();
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (r >= rows) return;
    const TIn* row = x + r * ld;
    // 4 values per lane per step, so that a row of 128 keeps all 32 lanes busy
    float amax = 0.f;
    for (int j = lane * 4; j < cols; j += 128) {
        float v[4];
        load4(row + j, v);
#pragma unroll
        for (int u = 0; u < 4; ++u) amax = fmaxf(amax, fabsf(v[u]));
    }
    // non-negative floats order like their bits
    amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
    const double s = amax > 0.f ? (double)amax / 448.0 : 1.0;
    for (int j = lane * 4; j < cols; j += 128) {
        float v[4];
        load4(row + j, v);
        uint32_t c4 = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) c4 |= (uint32_t)e4m3_code((double)v[u] / s) << (8 * u);
        *reinterpret_cast<uint32_t*>(out + r * cols + j) = c4;
    }
    if (lane == 0) {
        scale[r] = (float)s;
        if (w) w_out[r] = w[r] * (float)s;
    }
    if (rope)
        for (int j = lane * 8; j < rope_dims; j += 256) {
            float v[8];
            load8(row + cols + j, v);
            if constexpr (sizeof(TIn) == 2) store8(reinterpret_cast<bf16*>(rope + r * rope_dims + j), v);
            else store8(reinterpret_cast<float*>(rope + r * rope_dims + j), v);
        }
}

// The value of an e4m3 code, from the format's definition (sign, 4 exponent
// bits with bias 7, 3 mantissa bits; exponent field 0: subnormal).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
    // normal codes (exponent field 1..15): 2^(e-7) * (1 + m/8), assembled
    // as fp32 bits (exponent e - 7 + 127, the 3 mantissa bits on top);
    // subnormals (field 0): m * 2^-9
    const uint32_t ef = (code >> 3) & 15u, mf = code & 7u;
    const float mag = ef ? __uint_as_float(((ef + 120u) << 23) | (mf << 20)) : (float)mf * 0.001953125f;
    return (code & 0x80u) ? -mag : mag;
}

// FP8 KV entries of the selection, dequantised to bf16 rows: out[t][i] =
// entry idx[t][i] of sequence t (bf16(code * scale) for the first c - R
// dims, the bf16 rotary dims after them), idx_out[t][i] = i for a selected
// entry, -1 for an empty slot (its row is zero). A warp takes kGatherSlots
// consecutive slots, 16 dims per lane: all the slots' indices are loaded,
// then all their scales and 16-byte pieces, then converted and stored, so
// that each lane has several loads in flight instead of one.
constexpr int kGatherSlots = 1;

__global__ void __launch_bounds__(256) gather_kv_fp8_kernel(const uint8_t* __restrict__ codes,
                                                            const float* __restrict__ scales,
                                                            const bf16* __restrict__ rope, const int32_t* __restrict__ idx,
                                                            int nq, int k, int64_t Nmax, int c, int rope_dims,
                                                            bf16* __restrict__ out, int32_t* __restrict__ idx_out) {
    pdl_wait();
    pdl_launch_next();
    const int lane = threadIdx.x & 31;
    const int64_t nslots = (int64_t)nq * k;
    const int64_t slot0 = ((int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5)) * kGatherSlots;
    if (slot0 >= nslots) return;
    const int cq = c - rope_dims;
    int64_t R[kGatherSlots];
    bool ok[kGatherSlots];
#pragma unroll
    for (int u = 0; u < kGatherSlots; ++u) {
        const int64_t slot = slot0 + u;
        const bool in = slot < nslots;
        const int e = in ? __ldg(idx + slot) : -1;
        const int64_t t = in ? slot / k : 0;
        ok[u] = e >= 0 && e < Nmax;
        R[u] = t * Nmax + (ok[u] ? e : 0);
        if (in && lane == 0) idx_out[slot] = ok[u] ? (int)(slot - t * k) : -1;
    }
    for (int j = lane * 16; j < c; j += 512) {
        uint4 lo[kGatherSlots], hi[kGatherSlots];
        float s[kGatherSlots];
#pragma unroll
        for (int u = 0; u < kGatherSlots; ++u) {
            lo[u] = hi[u] = make_uint4(0, 0, 0, 0);
            s[u] = 0.f;
            if (!ok[u]) continue;
            if (j < cq) {
                s[u] = __ldg(scales + R[u]);
                lo[u] = __ldg(reinterpret_cast<const uint4*>(codes + R[u] * cq + j));
            } else {
                const uint4* p = reinterpret_cast<const uint4*>(rope + R[u] * rope_dims + (j - cq));
                lo[u] = __ldg(p);
                hi[u] = __ldg(p + 1);
            }
        }
#pragma unroll
        for (int u = 0; u < kGatherSlots; ++u) {
            const int64_t slot = slot0 + u;
            if (slot >= nslots) break;
            bf16* orow = out + slot * c + j;
            if (j < cq) {
                // 16 codes -> 16 bf16 values, written as two 16-byte stores
                const uint32_t wd[4] = {lo[u].x, lo[u].y, lo[u].z, lo[u].w};
                float v[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) v[q] = e4m3_value((wd[q >> 2] >> (8 * (q & 3))) & 255u) * s[u];
                float a[8], b[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) { a[q] = v[q]; b[q] = v[8 + q]; }
                store8(orow, a);
                store8(orow + 8, b);
            } else {
                // the rotary dims are bf16 already (zeros for an empty slot)
                reinterpret_cast<uint4*>(orow)[0] = lo[u];
                reinterpret_cast<uint4*>(orow)[1] = hi[u];
            }
        }
    }
}

}  // namespace

cudaError_t quantize_e4m3(const void* x, int64_t rows, int cols, void* out, float* scale, const float* w, float* w_out,
                          ElemType t, cudaStream_t st, int64_t ld, void* rope, int rope_dims) {
    if (rows == 0) return cudaSuccess;
    if (ld == 0) ld = cols;
    const dim3 grid((unsigned)((rows + 7) / 8));
    cudaError_t e = cudaSuccess;
    if (t == ElemType::BF16)
        CSA_LAUNCH(st, "quantize_e4m3",
                   e = launch_pdl(quantize_e4m3_kernel<bf16>, grid, dim3(256), 0, st, 0, (const bf16*)x, rows, cols, ld,
                                  (uint8_t*)out, scale, w, w_out, (bf16*)rope, rope_dims));
    else
        CSA_LAUNCH(st, "quantize_e4m3",
                   e = launch_pdl(quantize_e4m3_kernel<float>, grid, dim3(256), 0, st, 0, (const float*)x, rows, cols,
                                  ld, (uint8_t*)out, scale, w, w_out, (float*)rope, rope_dims));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t gather_kv_fp8(const uint8_t* codes, const float* scales, const void* rope, const int32_t* idx, int nq,
                          int k, int64_t Nmax, int c, int rope_dims, void* out, int32_t* idx_out, cudaStream_t st) {
    const int64_t slots = (int64_t)nq * k;
    if (slots == 0) return cudaSuccess;
    const dim3 grid((unsigned)((slots + 8 * kGatherSlots - 1) / (8 * kGatherSlots)));
    cudaError_t e = cudaSuccess;
    CSA_LAUNCH(st, "gather_kv_fp8",
               e = launch_pdl(gather_kv_fp8_kernel, grid, dim3(256), 0, st, 0, codes, scales, (const bf16*)rope, idx,
                              nq, k, Nmax, c, rope_dims, (bf16*)out, idx_out));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace csa
