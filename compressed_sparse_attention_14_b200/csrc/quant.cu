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
// steps of 2^-9 (exponent field 0). One warp per row, 16-byte loads.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

// The e4m3 code of the value nearest to v (|v| <= 448 assumed after the
// saturation test), written from the format's definition.
__device__ __forceinline__ uint8_t e4m3_code(double v) {
    const uint32_t sign = v < 0.0 ? 0x80u : 0u;
    const double a = fabs(v);
    if (!(a > 0.0)) return (uint8_t)sign;                 // zero (NaN never reaches here)
    if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);       // saturate: 1.75 * 2^8
    int e = ilogb(a);                                     // a in [2^e, 2^(e+1))
    int q = e - 3;                                        // spacing of 4 significant bits
    if (q < -9) q = -9;                                   // subnormal spacing
    double r = rint(ldexp(a, -q));                        // nearest, ties to even
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

template <typename TIn>
__global__ void __launch_bounds__(256) quantize_e4m3_kernel(const TIn* __restrict__ x, int64_t rows, int cols,
                                                            uint8_t* __restrict__ out, float* __restrict__ scale,
                                                            const float* __restrict__ w, float* __restrict__ w_out) {
    pdl_wait();
    pdl_launch_next();
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (r >= rows) return;
    const TIn* row = x + r * cols;
    double amax = 0.0;
    for (int j = lane * 8; j < cols; j += 256) {
        float v[8];
        load8(row + j, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) amax = fmax(amax, (double)fabsf(v[u]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const double s = amax > 0.0 ? amax / 448.0 : 1.0;
    for (int j = lane * 8; j < cols; j += 256) {
        float v[8];
        load8(row + j, v);
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) lo |= (uint32_t)e4m3_code((double)v[u] / s) << (8 * u);
#pragma unroll
        for (int u = 0; u < 4; ++u) hi |= (uint32_t)e4m3_code((double)v[4 + u] / s) << (8 * u);
        *reinterpret_cast<uint2*>(out + r * cols + j) = make_uint2(lo, hi);
    }
    if (lane == 0) {
        scale[r] = (float)s;
        if (w) w_out[r] = w[r] * (float)s;
    }
}

}  // namespace

cudaError_t quantize_e4m3(const void* x, int64_t rows, int cols, void* out, float* scale, const float* w, float* w_out,
                          ElemType t, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    const dim3 grid((unsigned)((rows + 7) / 8));
    cudaError_t e = cudaSuccess;
    if (t == ElemType::BF16)
        CSA_LAUNCH(st, "quantize_e4m3",
                   e = launch_pdl(quantize_e4m3_kernel<bf16>, grid, dim3(256), 0, st, 0, (const bf16*)x, rows, cols,
                                  (uint8_t*)out, scale, w, w_out));
    else
        CSA_LAUNCH(st, "quantize_e4m3",
                   e = launch_pdl(quantize_e4m3_kernel<float>, grid, dim3(256), 0, st, 0, (const float*)x, rows, cols,
                                  (uint8_t*)out, scale, w, w_out));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace csa
