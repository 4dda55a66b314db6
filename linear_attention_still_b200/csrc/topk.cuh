// topk.cuh -- block-wide top-k of one chunk of scores with position tie-break.
#pragma once

#include "common.cuh"

namespace still {

// Barrier after a bitonic compare-exchange stage of `stride` within sorts of `size` (of n entries).
// Work item t pairs entry lo = 2t - (t & (stride-1)) with lo + stride, and a warp's items are always
// the same aligned runs of 32 consecutive t (blockDim.x a multiple of 32), so a stage of stride <= 32
// touches only the warp's own runs of 64 entries: between two such stages a warp barrier suffices.
// A full barrier follows every other stage and the last one.
__device__ __forceinline__ void bitonic_stage_sync(int size, int stride, int n) {
    const int next = stride > 1 ? stride >> 1 : size;  // stride of the next stage
    if (stride <= 32 && next <= 32 && !(stride == 1 && size == n)) __syncwarp();
    else __syncthreads();
}

// Sort the n (<= P, P a power of two) scores sc[0..n) by (score desc, position asc) and leave the
// first k positions, ascending, in pos[0..k).  keys: P u64 of shared memory; pos: Pk u32 (Pk a power
// of two >= k).  Every thread of the block must call this, with blockDim.x a multiple of 32.  The key
// packs the order-preserving score bits over the complemented position, so all keys are distinct and
// a plain descending sort realises the tie-break.
__device__ __forceinline__ void block_topk(const float *sc, int n, int k, unsigned long long *keys, uint32_t *pos,
                                           int P, int Pk) {
    for (int j = threadIdx.x; j < P; j += blockDim.x)
        keys[j] = j < n ? ((unsigned long long)score_key(sc[j]) << 32) | (0xFFFFFFFFu - (uint32_t)j) : 0ull;
    __syncthreads();
    for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = threadIdx.x; t < P / 2; t += blockDim.x) {
                int lo = 2 * t - (t & (stride - 1)), hi = lo + stride;
                bool desc = (lo & size) == 0;
                unsigned long long a = keys[lo], b = keys[hi];
                if ((a < b) == desc) {
                    keys[lo] = b;
                    keys[hi] = a;
                }
            }
            bitonic_stage_sync(size, stride, P);
        }
    }
    for (int t = threadIdx.x; t < Pk; t += blockDim.x)
        pos[t] = t < k ? 0xFFFFFFFFu - (uint32_t)(keys[t] & 0xFFFFFFFFull) : 0xFFFFFFFFu;
    __syncthreads();
    for (int size = 2; size <= Pk; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = threadIdx.x; t < Pk / 2; t += blockDim.x) {
                int lo = 2 * t - (t & (stride - 1)), hi = lo + stride;
                bool asc = (lo & size) == 0;
                uint32_t a = pos[lo], b = pos[hi];
                if ((a > b) == asc) {
                    pos[lo] = b;
                    pos[hi] = a;
                }
            }
            bitonic_stage_sync(size, stride, Pk);
        }
    }
}

inline int pow2_ceil(int x) {
    int p = 1;
    while (p < x) p <<= 1;
    return p;
}

}  // namespace still
