// tc_tile.cuh -- helpers shared by the tcgen05 merge kernels: the exponential phase of one 128-key
// row tile, K-major SW128 descriptors per k-step, warp-uniform decisions, and tensor-map encoding.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace still {
namespace tc {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Lazy rescale threshold of the online softmax (log2 units): a row keeps its reference max m until a
// tile's max exceeds m + kRescaleLog2, so every probability written is at most 2^32.  P is bf16 and O,
// l are fp32 (both with an 8-bit exponent), so the sums stay far from overflow (at most 2^32 x keys x
// max|v|); the relative rounding of P does not depend on the reference.  A large threshold makes the
// O rescale, which must wait for the previous tile's P V, rare: with heavy keys a threshold of 2^8 is
// crossed by some row of a warp in a large share of the tiles.
constexpr float kRescaleLog2 = 32.0f;

// Exponentials of one 128-key row tile: p_c = 2^(s_c tau log2e - m), summed (ls0 + ls1) and written
// as bf16 P to TMEM at tP (four tcgen05.st of 16 columns = 64 columns of packed pairs).  BAND
// additionally sums p_c over the columns [bc_lo, bc_hi) into bsum (the Self-Saliency band of this row
// inside the tile).  EXPV selects where the exponentials run: 0/1 all on the MUFU unit (ex2.approx),
// 2 the last 32-key chunk of each row on the FMA pipe (exp2_poly2), 3 every other 32-key chunk there.
template <int EXPV, bool BAND>
__device__ __forceinline__ void exp_tile(const float (&sv)[128], float scale_log2, float m_run, uint32_t tP,
                                         float &ls0, float &ls1, float &bsum, int bc_lo, int bc_hi) {
    const float2 sc2 = make_float2(scale_log2, scale_log2);
    const float2 neg2 = make_float2(-m_run, -m_run);
    float2 ls = make_float2(0.f, 0.f);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t u[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int c0 = c * 32 + 2 * e;
            const float2 xx = ffma2(make_float2(sv[c0], sv[c0 + 1]), sc2, neg2);
            float2 pp;
            if ((EXPV == 2 && c == 3) || (EXPV == 3 && (c & 1))) {
                pp = exp2_poly2(xx);  // FMA pipe
            } else {
                pp.x = ex2(xx.x);      // MUFU
                pp.y = ex2(xx.y);
            }
            ls = fadd2(ls, pp);
            if (BAND) {
                if (c0 >= bc_lo && c0 < bc_hi) bsum += pp.x;
                if (c0 + 1 >= bc_lo && c0 + 1 < bc_hi) bsum += pp.y;
            }
            u[e] = pack_bf16x2(pp.x, pp.y);
        }
        tmem_st16(tP + c * 16, u);
    }
    ls0 = ls.x;
    ls1 = ls.y;
}

// The same exponentials into registers: u[e] = bf16 pair (p_{2e}, p_{2e+1}) of the row, to be stored
// as P later (store_p).  Lets a softmax warp finish its exponentials before it waits for the MMA that
// still reads the previous P.
template <int EXPV, bool BAND>
__device__ __forceinline__ void exp_row(const float (&sv)[128], float scale_log2, float m_run, uint32_t (&u)[64],
                                        float &ls0, float &ls1, float &bsum, int bc_lo, int bc_hi) {
    const float2 sc2 = make_float2(scale_log2, scale_log2);
    const float2 neg2 = make_float2(-m_run, -m_run);
    // four independent partial sums, so the adds do not serialise the exponentials
    float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
    float bs[2] = {0.f, 0.f};
#pragma unroll
    for (int e = 0; e < 64; ++e) {
        const int c0 = 2 * e;
        const float2 xx = ffma2(make_float2(sv[c0], sv[c0 + 1]), sc2, neg2);
        float2 pp;
        if ((EXPV == 2 && c0 >= 96) || (EXPV == 3 && ((c0 >> 5) & 1))) {
            pp = exp2_poly2(xx);  // FMA pipe
        } else {
            pp.x = ex2(xx.x);      // MUFU
            pp.y = ex2(xx.y);
        }
        ls[e & 3] = fadd2(ls[e & 3], pp);
        if (BAND) {
            if (c0 >= bc_lo && c0 < bc_hi) bs[e & 1] += pp.x;
            if (c0 + 1 >= bc_lo && c0 + 1 < bc_hi) bs[e & 1] += pp.y;
        }
        u[e] = pack_bf16x2(pp.x, pp.y);
    }
    const float2 l01 = fadd2(ls[0], ls[1]), l23 = fadd2(ls[2], ls[3]);
    ls0 = l01.x + l23.x;
    ls1 = l01.y + l23.y;
    if (BAND) bsum += bs[0] + bs[1];
}

// P row (64 packed bf16 pairs = 128 keys) into 64 TMEM columns.
__device__ __forceinline__ void store_p(uint32_t tP, const uint32_t (&u)[64]) {
    tmem_st32(tP, *reinterpret_cast<const uint32_t(*)[32]>(&u[0]));
    tmem_st32(tP + 32, *reinterpret_cast<const uint32_t(*)[32]>(&u[32]));
}

// S row of one key tile from TMEM into registers, masked on the tiles that need it (warp-uniform test):
// LOCAL the causal diagonal tile (columns past the row), PREFIX the ragged last tile of the kept rows.
// On the diagonal tile the row's own raw score is kept in sdiag.
__device__ __forceinline__ void load_s_row(uint32_t tS, float (&sv)[128], bool diag, bool ragged, int limit, int r,
                                           float &sdiag) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t u[32];
        tmem_ld32(tS + c * 32, u);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(u[e]);
    }
    tmem_wait_ld();
    if (diag) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
            if (c == r) sdiag = sv[c];  // unrolled select keeps sv in registers
    }
    if (diag || ragged) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
            if (c >= limit) sv[c] = -INFINITY;
    }
}

// tcgen05.ld/st are warp-collective: every decision that guards them is made warp-uniform.
__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

// Bounded mbarrier wait taken by a whole warp, with one result for all its lanes.
__device__ __forceinline__ bool mbar_wait_w(uint32_t bar, uint32_t parity, volatile int *abort) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
}

// The same two waits with the form chosen per kernel: SUSP = true sleeps in mbarrier.try_wait between
// tests (no issue slots taken while waiting), false spins on the non-suspending test.
template <bool SUSP>
__device__ __forceinline__ bool mbar_wait_t(uint32_t bar, uint32_t parity, volatile int *abort) {
    return SUSP ? mbar_wait_susp(bar, parity, abort) : mbar_wait(bar, parity, abort);
}
template <bool SUSP>
__device__ __forceinline__ bool mbar_wait_wt(uint32_t bar, uint32_t parity, volatile int *abort) {
    return __all_sync(0xffffffffu, mbar_wait_t<SUSP>(bar, parity, abort));
}

// K-major SW128 descriptor of k-step kk (16 elements) of a tile whose rows are split into 64-col
// regions of `region_bytes` each.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int kk, uint32_t region_bytes) {
    return sw128_desc(base + (kk >> 2) * region_bytes + (kk & 3) * 32, 16, 1024);
}

// Row max of a 128-column row tile: four chains of 3-input max over 32 columns each.
__device__ __forceinline__ float row_max128(const float (&sv)[128]) {
    float mxc[4];
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
        float mv = fmax3(sv[32 * k4], sv[32 * k4 + 1], sv[32 * k4 + 2]);
#pragma unroll
        for (int c = 32 * k4 + 3; c + 1 < 32 * k4 + 32; c += 2) mv = fmax3(mv, sv[c], sv[c + 1]);
        mxc[k4] = fmaxf(mv, sv[32 * k4 + 31]);
    }
    return fmax3(mxc[0], mxc[1], fmaxf(mxc[2], mxc[3]));
}

// bf16 tensor [d2][d1][d0] (d0 innermost), box {64, box1, 1}, 128-byte swizzle, zero fill out of
// range.  False when the driver entry point is missing or the base is not 16-byte aligned.
bool make_map(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box1);

}  // namespace tc
}  // namespace still
