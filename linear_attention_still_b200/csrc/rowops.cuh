// rowops.cuh -- per-row helpers of the SIMT kernels (dot products, NP-Map of one row).
#pragma once

#include "common.cuh"

namespace still {

constexpr int kMaxD = 256;   // head dim limit of the generic path
constexpr int kMaxDf = 256;  // NP-Map width limit

// <q, row> with q staged in fp32 shared memory; row is d elements in global memory.
__device__ __forceinline__ float dot_row(const float *qs, const __nv_bfloat16 *row, int d) {
    float acc = 0.f;
    const uint4 *p = reinterpret_cast<const uint4 *>(row);
    for (int x8 = 0; x8 < d / 8; ++x8) {
        uint4 u = __ldg(p + x8);
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 f = __bfloat1622float2(h2[e]);
            acc = fmaf(qs[8 * x8 + 2 * e], f.x, acc);
            acc = fmaf(qs[8 * x8 + 2 * e + 1], f.y, acc);
        }
    }
    return acc;
}

__device__ __forceinline__ float dot_row(const float *qs, const float *row, int d) {
    float acc = 0.f;
    const float4 *p = reinterpret_cast<const float4 *>(row);
    for (int x4 = 0; x4 < d / 4; ++x4) {
        float4 f = __ldg(p + x4);
        acc = fmaf(qs[4 * x4 + 0], f.x, acc);
        acc = fmaf(qs[4 * x4 + 1], f.y, acc);
        acc = fmaf(qs[4 * x4 + 2], f.z, acc);
        acc = fmaf(qs[4 * x4 + 3], f.w, acc);
    }
    return acc;
}

// NP-Map of one row, computed by one warp: phi = ||x|| * e / ||e||, e_c = exp(y_c - max y), y = x W.
// xs: the row in fp32 shared memory (d values); W: [d, D] in global memory; out: D fp32 values
// (shared or global).  f = softmax(y) = e / sum(e), so f / ||f|| = e / ||e||.
template <typename T>
__device__ void npmap_row_warp(const float *xs, const T *W, int d, int D, float *out, int lane) {
    float y[kMaxDf / 32];
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < kMaxDf / 32; ++u) {
        int c = lane + 32 * u;
        float acc = 0.f;
        if (c < D) {
            for (int a = 0; a < d; ++a) acc = fmaf(xs[a], to_f(W[(size_t)a * D + c]), acc);
            mx = fmaxf(mx, acc);
        }
        y[u] = acc;
    }
    mx = warp_max(mx);
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < kMaxDf / 32; ++u) {
        int c = lane + 32 * u;
        float e = c < D ? expf(y[u] - mx) : 0.f;
        y[u] = e;
        ss = fmaf(e, e, ss);
    }
    ss = warp_sum(ss);
    float nx = 0.f;
    for (int a = lane; a < d; a += 32) nx = fmaf(xs[a], xs[a], nx);
    nx = sqrtf(warp_sum(nx));
    float f = nx / sqrtf(ss);
#pragma unroll
    for (int u = 0; u < kMaxDf / 32; ++u) {
        int c = lane + 32 * u;
        if (c < D) out[c] = y[u] * f;
    }
}

}  // namespace still
