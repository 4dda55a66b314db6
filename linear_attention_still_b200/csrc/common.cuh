// common.cuh -- small device helpers shared by the libstill kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace still {

// Device error word bits (read back by still_get_device_status).
enum : unsigned {
    DEV_ERR_INDEX = 1u,     // an injected kept index lies outside its chunk
    DEV_ERR_POSITION = 2u,  // decode position does not match the state
    DEV_ERR_TIMEOUT = 4u,   // a bounded wait ran out
};

__device__ __forceinline__ void report(unsigned *err, unsigned bit) {
    if (err) atomicOr(err, bit);
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

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

// Load n consecutive elements of a row (n a multiple of 8 for bf16, 4 for f32) into fp32 smem.
template <typename T>
__device__ __forceinline__ void load_row_f32(float *dst, const T *src, int n, int lane, int nlanes) {
    for (int x = lane; x < n; x += nlanes) dst[x] = to_f(src[x]);
}

// softplus(x) = ln(1 + e^x), written to stay accurate for large |x|.
__device__ __forceinline__ float softplus_f(float x) {
    if (x == INFINITY) return INFINITY;
    return x > 0.f ? x + log1pf(expf(-x)) : log1pf(expf(x));
}

// Order-preserving map of an fp32 score to uint32 (larger score -> larger key).
__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace still
