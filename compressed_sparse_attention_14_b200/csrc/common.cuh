// Shared device helpers for libcsa (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace csa {

using bf16 = __nv_bfloat16;

// Kernels that give up on a bounded wait record an error code in the
// library's device status word (passed to them as a pointer; first writer
// wins) instead of trapping; csa_poll_status() reads it back.
__device__ __forceinline__ void report_device_error(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// ---- programmatic dependent launch
// Kernels launched with launch_pdl() may start while the previous kernel on
// the stream drains. pdl_wait() returns once that kernel has completed and
// its writes are visible (at once when there is none); every CTA calls it
// before its first global memory access, read or write. pdl_launch_next()
// lets the next kernel on the stream begin launching once every CTA of this
// one has called it (or exited).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_next() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- selection order (top-k): score descending, then column ascending
// orderable() maps fp32 to uint32 monotonically (-0.0 folded into +0.0);
// the composite key (orderable(score) << 32) | (0xFFFFFFFF - column) is
// distinct per column and its descending order is the selection order.
__device__ __forceinline__ uint32_t orderable(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;  // -0.0 == +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_orderable(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}
__device__ __forceinline__ uint64_t composite_key(uint32_t key, int64_t col) {
    return ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)col);
}
__device__ __forceinline__ uint64_t composite(float s, int64_t col) { return composite_key(orderable(s), col); }

// ---- element conversion -------------------------------------------------
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

// Load 8 consecutive elements (16-byte aligned for bf16, 32-byte for fp32)
// as fp32.
// four consecutive values, one 16-byte (fp32) or 8-byte (bf16) store
__device__ __forceinline__ void store4(float* p, float a, float b, float c, float d) {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void store4(bf16* p, float a, float b, float c, float d) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&lo);
    u.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p) = u;
}

__device__ __forceinline__ void load8(const bf16* p, float (&v)[8]) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    float4 a = *reinterpret_cast<const float4*>(p);
    float4 b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void store8(bf16* p, const float (&v)[8]) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Query -> sequence and query -> position lookups shared by the attention
// kernels. seq: explicit array, else identity (decode: query b reads
// sequence b), else all queries on sequence 0 (prefill of one sequence).
struct QueryMap {
    const int32_t* seq;    // nullable
    const int32_t* pos;    // nullable: then pos = pos_base + t
    int64_t pos_base;
    int single_seq;        // 1: every query reads sequence 0
    __device__ __forceinline__ int seq_of(int t) const {
        return seq ? seq[t] : (single_seq ? 0 : t);
    }
    __device__ __forceinline__ int64_t pos_of(int t) const {
        return pos ? (int64_t)pos[t] : pos_base + t;
    }
};

__device__ __forceinline__ int64_t visible_entries(int64_t pos, int m, int64_t nmax) {
    int64_t v = pos < 0 ? 0 : pos / m;
    return v < nmax ? v : nmax;
}

}  // namespace csa
