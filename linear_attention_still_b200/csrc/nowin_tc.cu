// nowin_tc.cu -- the STILL layer with no softmax window (w = 0): pure causal linear attention with
// the Norm-Preserved Feature Map, chunked, on sm_100a tensor cores (bf16 storage, head dim 64).
// ([p1] jsqmd.com introduction: the tokens that are not kept go to linear attention; "NP-Map":
// phi(x) = ||x|| f(x W) / ||f(x W)||, f = softmax over the D features; [p4] atlas.scime.ai "Approach".)
//
// For query i of chunk t (chunk C, 128-query tiles, C a multiple of 128):
//   o_i = (phi(q_i)^T S_t + sum_{tC <= j <= i} <phi(q_i), phi(k_j)> v_j)
//       / (phi(q_i)^T z_t + sum_{tC <= j <= i} <phi(q_i), phi(k_j)>),
// S_t = sum_{j < tC} phi(k_j) v_j^T and z_t = sum_{j < tC} phi(k_j) from the linear-state kernels
// (inter-chunk state GEMMs on tensor cores); the intra-chunk causal tile runs here, in two launches.
//
// nowin_phik_kernel: phi(k) of every key once, per (KV head, 128 keys): Y = K Wk^T (tcgen05, TMEM
// lane = key) -> NP-Map per key -> bf16 rows [B*Hkv, N, DF] in the workspace.  (Each key tile is read
// by every query head of its group and every later query tile of its chunk: G * C / 256 times on
// average, each of which would otherwise form phi(k) again on its own serial chain.)
//
// nowin_tc_kernel: one CTA = (b, query head h, 128 queries).  Roles: four feature warps (TMEM lane =
// row), a TMA producer warp and an MMA warp.  Prologue: Y = Q Wq^T (tcgen05) -> phi(q) per row -> bf16
// into shared memory (the A operand of every later product) -> O := phi(Q) S_t^T, l := phi(q).z_t.
// Per key tile j of the chunk: A = phi(Q) phi(K_j)^T (tcgen05, phi(K_j) by TMA) -> causal mask on the
// diagonal tile, l += row sum, P = A in bf16 over A's TMEM columns -> O += P V_j (tcgen05, P from TMEM).
// phi(K) and V have stages of their own: a phi(K) stage is free once A has read it, so the next tile's
// phi(K) lands while this tile's P is formed.  Epilogue o = O / l.
// Every mbarrier wait is bounded; on a timeout the CTA records DEV_ERR_TIMEOUT, drains its own copies
// and MMAs, frees TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "still_internal.h"
#include "tc_ptx.cuh"
#include "tc_tile.cuh"

namespace still {

using namespace tc;

namespace {

// D = 64: two CTAs per SM (256 TMEM columns each), so one CTA's serial chain (A -> P -> P V) overlaps
// the other's (1), or one CTA per SM (0).  Measured on B200 (1B-shaped layer, w = 0, 16K tokens, with
// phi(k) still formed per tile inside this kernel): 0.290 -> 0.212 ms.
#ifndef STILL_NOWIN_PAIR
#define STILL_NOWIN_PAIR 1
#endif

template <int DF>
struct NowinCfg {
    static constexpr bool PAIR = STILL_NOWIN_PAIR != 0 && DF == 64;
    static constexpr int MINB = PAIR ? 2 : 1;
    static constexpr int REG = 128 * 128;                // 128 rows x 64 bf16 (one SW128 region)
    static constexpr int Q_BYTES = REG;                  // 128 queries x 64
    static constexpr int W_BYTES = DF * 128;             // Wq^T: DF rows x 64
    static constexpr int ST_BYTES = 64 * DF * 2;         // S_t^T: 64 rows x DF (DF/64 regions of 64 rows)
    static constexpr int PHI_BYTES = 128 * DF * 2;       // 128 rows x DF (DF/64 regions)
    static constexpr int NSK = 2, NSV = PAIR ? 1 : 2;    // phi(K) and V stages
    static constexpr int OFF_Q = 0, OFF_WQ = OFF_Q + Q_BYTES, OFF_ST = OFF_WQ + W_BYTES, OFF_PQ = OFF_ST + ST_BYTES,
                         OFF_PK = OFF_PQ + PHI_BYTES, OFF_V = OFF_PK + NSK * PHI_BYTES, OFF_BAR = OFF_V + NSV * REG;
    static constexpr int BAR_BYTES = 512;
    static constexpr int SMEM = OFF_BAR + BAR_BYTES + 1024;
    static_assert(SMEM <= 232448, "shared memory");
    static_assert(MINB * (SMEM + 1024) <= 233472, "shared memory per SM");
    static constexpr int THREADS = 192;
    static constexpr int PRODUCER_WARP = 4, MMA_WARP = 5;
    static constexpr int A_COL = 0, O_COL = 128, TMEM_COLS = 256;
    static_assert(DF <= 128 && O_COL + 64 <= TMEM_COLS && MINB * TMEM_COLS <= 512, "TMEM columns");
    // barrier slots
    static constexpr int B_QFULL = 0, B_WFULL = 1, B_YQ = 2, B_PHIQ = 3, B_PRO = 4, B_DRAIN = 5, B_A = 6, B_P = 7,
                         B_O = 8, B_KFULL = 9, B_KEMPTY = B_KFULL + NSK, B_VFULL = B_KEMPTY + NSK,
                         B_VEMPTY = B_VFULL + NSV;
    static constexpr int NUM_BARS = B_VEMPTY + NSV;
    static constexpr int TMEM_SLOT_OFF = 8 * NUM_BARS;
    static constexpr int ABORT_OFF = TMEM_SLOT_OFF + 8;
    static_assert(ABORT_OFF + 8 <= BAR_BYTES, "barrier area overflow");
};

// The phi(K) kernel: one 128-key tile and Wk^T, Y in DF TMEM columns.  Shared memory is padded to 48 KB
// so that at most four CTAs share an SM: their TMEM columns (4 x DF <= 512) then always fit and
// tcgen05.alloc never waits for another CTA's columns.  MINB is the register bound (DF = 128 keeps its
// 128 features in registers with two CTAs' worth).
template <int DF>
struct PhikCfg {
    static constexpr int REG = 128 * 128;
    static constexpr int W_BYTES = DF * 128;
    static constexpr int OFF_K = 0, OFF_W = REG, OFF_BAR = OFF_W + W_BYTES;
    static constexpr int B_FULL = 0, B_Y = 1, TMEM_SLOT_OFF = 16, ABORT_OFF = 24;
    static constexpr int USED = OFF_BAR + 64 + 1024;
    static constexpr int SMEM = USED > 48 * 1024 ? USED : 48 * 1024;
    static constexpr int MINB = DF == 64 ? 4 : 2;
    static constexpr int TMEM_COLS = DF;
    static_assert(4 * (SMEM + 1024) <= 233472 && 5 * (SMEM + 1024) > 233472, "at most four CTAs per SM");
    static_assert(4 * TMEM_COLS <= 512, "TMEM columns");
};

struct PhikParams {
    int N, Hkv, n_ktiles;
    __nv_bfloat16 *phik;   // [B*Hkv, N, DF]
    unsigned *err;
};

struct NowinParams {
    int B, H, Hkv, N, C, G, T, n_qtiles;
    const float *z;        // [B*Hkv*(T+1), DF] fp32: z_t of every query chunk
    __nv_bfloat16 *o;      // [B,H,N,64]
    unsigned *err;
};

// phi(x) of one row, in place, from Y = x W (DF values of this thread's TMEM lane) and ||x||^2:
// ||x|| e / ||e||, e = exp(Y - max Y) (fp32, for the caller's dot products and stores).
template <int DF>
__device__ __forceinline__ void npmap_row(float (&y)[DF], float xx) {
    float ymax = -INFINITY;
#pragma unroll
    for (int c = 0; c < DF; ++c) ymax = fmaxf(ymax, y[c]);
    float ee = 0.f;
#pragma unroll
    for (int c = 0; c < DF; ++c) {
        y[c] = ex2((y[c] - ymax) * kLog2e);
        ee = fmaf(y[c], y[c], ee);
    }
    const float f = sqrtf(xx) * rsqrtf(ee);
#pragma unroll
    for (int c = 0; c < DF; ++c) y[c] *= f;
}

template <int DF>
__device__ __forceinline__ void store_row_sw128(uint8_t *tile, int row, const float (&y)[DF]) {
#pragma unroll
    for (int rr = 0; rr < DF / 64; ++rr) {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
            uint4 w;
            const int a0 = rr * 64 + ch * 8;
            w.x = pack_bf16x2(y[a0 + 0], y[a0 + 1]);
            w.y = pack_bf16x2(y[a0 + 2], y[a0 + 3]);
            w.z = pack_bf16x2(y[a0 + 4], y[a0 + 5]);
            w.w = pack_bf16x2(y[a0 + 6], y[a0 + 7]);
            *reinterpret_cast<uint4 *>(tile + rr * (128 * 128) + row * 128 + ((ch ^ (row & 7)) << 4)) = w;
        }
    }
}

// ||x||^2 of row `row` of a swizzled 128 x 64 bf16 tile.
__device__ __forceinline__ float row_sqnorm_sw128(const uint8_t *tile, int row) {
    float acc = 0.f;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        const uint4 u = *reinterpret_cast<const uint4 *>(tile + row * 128 + ((ch ^ (row & 7)) << 4));
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h2[e]);
            acc = fmaf(f.x, f.x, acc);
            acc = fmaf(f.y, f.y, acc);
        }
    }
    return acc;
}

// This thread's TMEM lane of DF fp32 columns starting at t (t carries the warp's lane quarter), as
// floats; warp-collective.
template <int DF>
__device__ __forceinline__ void load_y_row(uint32_t t, float (&y)[DF]) {
#pragma unroll
    for (int c = 0; c < DF / 32; ++c) {
        uint32_t u[32];
        tmem_ld32(t + c * 32, u);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) y[c * 32 + e] = __uint_as_float(u[e]);
    }
}

template <int DF>
__global__ void __launch_bounds__(128, PhikCfg<DF>::MINB)
    nowin_phik_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_wk,
                      const PhikParams p) {
    using Cfg = PhikCfg<DF>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint8_t *bar_area = smem + Cfg::OFF_BAR;
    const uint32_t bFull = smem_u32(bar_area) + 8u * Cfg::B_FULL, bY = smem_u32(bar_area) + 8u * Cfg::B_Y;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_area + Cfg::TMEM_SLOT_OFF);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bar_area + Cfg::ABORT_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bg = blockIdx.x / p.n_ktiles, kt = blockIdx.x % p.n_ktiles;
    const int j0 = kt * 128;

    if (threadIdx.x == 0) {
        mbar_init(bFull, 1);
        mbar_init(bY, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool issued = false;
    if (warp == 0) {
        // K tile and Wk^T by TMA (rows past N read as zero), then Y = K Wk^T; Y is committed only when
        // the MMAs ran, so a failed wait leaves the other warps to see the abort flag
        mbar_arrive_expect_tx_w(bFull, Cfg::REG + Cfg::W_BYTES);
        tma_load_3d_w(sbase + Cfg::OFF_K, &map_k, bFull, 0, j0, bg);
        tma_load_3d_w(sbase + Cfg::OFF_W, &map_wk, bFull, 0, 0, bg % p.Hkv);
        if (mbar_wait_w(bFull, 0, abort_flag)) {
            constexpr uint32_t ID_Y = idesc_bf16(128, DF, 0, 0);
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ss_w(tmem, kmajor_desc(sbase + Cfg::OFF_K, kk, Cfg::REG),
                         kmajor_desc(sbase + Cfg::OFF_W, kk, Cfg::W_BYTES), ID_Y, kk > 0);
            mma_commit_w(bY);
            issued = true;
        } else {
            *abort_flag = 1;
            if (lane == 0) report(p.err, DEV_ERR_TIMEOUT);
            mbar_wait_drain(bFull, 0, 100000000ull);
        }
    }
    // every warp: phi of key row j0 + r (TMEM lane r), stored bf16 when the key exists
    const int r = warp * 32 + lane;
    const bool ok = warp_all(mbar_wait(bY, 0, abort_flag));
    if (ok) {
        tc_fence_after();
        float y[DF];
        load_y_row<DF>(tmem + ((uint32_t)(warp * 32) << 16), y);
        npmap_row<DF>(y, row_sqnorm_sw128(smem + Cfg::OFF_K, r));
        const int key = j0 + r;
        if (key < p.N) {
            uint4 *dst = reinterpret_cast<uint4 *>(p.phik + ((size_t)bg * p.N + key) * DF);
#pragma unroll
            for (int c8 = 0; c8 < DF / 8; ++c8) {
                uint4 w;
                w.x = pack_bf16x2(y[8 * c8 + 0], y[8 * c8 + 1]);
                w.y = pack_bf16x2(y[8 * c8 + 2], y[8 * c8 + 3]);
                w.z = pack_bf16x2(y[8 * c8 + 4], y[8 * c8 + 5]);
                w.w = pack_bf16x2(y[8 * c8 + 6], y[8 * c8 + 7]);
                dst[c8] = w;
            }
        }
    } else if (lane == 0) {
        *abort_flag = 1;
        report(p.err, DEV_ERR_TIMEOUT);
    }
    if (issued && !ok) mbar_wait_drain(bY, 0, 100000000ull);  // MMAs issued but not seen complete
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, Cfg::TMEM_COLS);
}

template <int DF>
__global__ void __launch_bounds__(NowinCfg<DF>::THREADS, NowinCfg<DF>::MINB)
    nowin_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_pk,
                    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_wq,
                    const __grid_constant__ CUtensorMap map_st, const NowinParams p) {
    using Cfg = NowinCfg<DF>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint8_t *bar_area = smem + Cfg::OFF_BAR;
    const uint32_t sBar = smem_u32(bar_area);
    auto BAR = [&](int i) { return sBar + 8u * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_area + Cfg::TMEM_SLOT_OFF);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bar_area + Cfg::ABORT_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // CTA -> (b, h, query tile); later (heavier) query tiles first
    const int per_qt = p.B * p.H;
    const int qt = p.n_qtiles - 1 - (int)(blockIdx.x / per_qt);
    const int bh = blockIdx.x % per_qt;
    const int b = bh / p.H, h = bh % p.H, g = h / p.G;
    const int bg = b * p.Hkv + g;
    const int i0 = qt * 128;
    const int t = i0 / p.C;
    const int kbase = t * p.C;
    const int n_tiles = (i0 - kbase) / 128 + 1;
    const int tslot = bg * (p.T + 1) + t;

    if (threadIdx.x == 0) {
        for (int i = 0; i < Cfg::NUM_BARS; ++i) {
            const bool many = i == Cfg::B_PHIQ || i == Cfg::B_P;
            mbar_init(BAR(i), many ? 128 : 1);
        }
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == Cfg::MMA_WARP) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == Cfg::PRODUCER_WARP) {
        // ================================================================ TMA producer (whole warp)
        bool ok = true;
        int issued_k = 0, issued_v = 0;
        mbar_arrive_expect_tx_w(BAR(Cfg::B_QFULL), Cfg::Q_BYTES);
        tma_load_3d_w(sbase + Cfg::OFF_Q, &map_q, BAR(Cfg::B_QFULL), 0, i0, b * p.H + h);
        mbar_arrive_expect_tx_w(BAR(Cfg::B_WFULL), Cfg::W_BYTES + Cfg::ST_BYTES);
        tma_load_3d_w(sbase + Cfg::OFF_WQ, &map_wq, BAR(Cfg::B_WFULL), 0, 0, h);
        for (int rr = 0; rr < DF / 64; ++rr)
            tma_load_3d_w(sbase + Cfg::OFF_ST + rr * (64 * 128), &map_st, BAR(Cfg::B_WFULL), rr * 64, 0, tslot);
        for (int j = 0; j < n_tiles; ++j) {
            // phi(K_j): its stage is free once A(j - NSK) has read it; rows past N read as zero
            const int sk = j % Cfg::NSK, sv = j % Cfg::NSV;
            if (j >= Cfg::NSK && !(ok = mbar_wait_w(BAR(Cfg::B_KEMPTY + sk), ((j / Cfg::NSK) - 1) & 1, abort_flag)))
                break;
            const uint32_t sPK = sbase + Cfg::OFF_PK + sk * Cfg::PHI_BYTES;
            mbar_arrive_expect_tx_w(BAR(Cfg::B_KFULL + sk), Cfg::PHI_BYTES);
            for (int rr = 0; rr < DF / 64; ++rr)
                tma_load_3d_w(sPK + rr * Cfg::REG, &map_pk, BAR(Cfg::B_KFULL + sk), rr * 64, kbase + j * 128, bg);
            issued_k = j + 1;
            // V_j: its stage is free once P V(j - NSV) has completed
            if (j >= Cfg::NSV && !(ok = mbar_wait_w(BAR(Cfg::B_VEMPTY + sv), ((j / Cfg::NSV) - 1) & 1, abort_flag)))
                break;
            mbar_arrive_expect_tx_w(BAR(Cfg::B_VFULL + sv), Cfg::REG);
            tma_load_3d_w(sbase + Cfg::OFF_V + sv * Cfg::REG, &map_v, BAR(Cfg::B_VFULL + sv), 0, kbase + j * 128, bg);
            issued_v = j + 1;
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) report(p.err, DEV_ERR_TIMEOUT);
            mbar_wait_drain(BAR(Cfg::B_QFULL), 0, 100000000ull);
            mbar_wait_drain(BAR(Cfg::B_WFULL), 0, 100000000ull);
            // only the last NSK (NSV) loads of a kind can be in flight: each earlier one was consumed
            for (int j = max(0, issued_k - Cfg::NSK); j < issued_k; ++j)
                mbar_wait_drain(BAR(Cfg::B_KFULL + j % Cfg::NSK), (j / Cfg::NSK) & 1, 100000000ull);
            for (int j = max(0, issued_v - Cfg::NSV); j < issued_v; ++j)
                mbar_wait_drain(BAR(Cfg::B_VFULL + j % Cfg::NSV), (j / Cfg::NSV) & 1, 100000000ull);
        }
    } else if (warp == Cfg::MMA_WARP) {
        // ================================================================ MMA issuer (whole warp)
        const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
        constexpr uint32_t ID_Y = idesc_bf16(128, DF, 0, 0);
        constexpr uint32_t ID_N64 = idesc_bf16(128, 64, 0, 0);
        constexpr uint32_t ID_N128 = idesc_bf16(128, 128, 0, 0);
        constexpr uint32_t ID_PV = idesc_bf16(128, 64, 0, 1);
        bool ok = mbar_wait_w(BAR(Cfg::B_QFULL), 0, abort_flag) && mbar_wait_w(BAR(Cfg::B_WFULL), 0, abort_flag);
        if (ok) {
            // Y_Q = Q Wq^T
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ss_w(tm + Cfg::A_COL, kmajor_desc(sbase + Cfg::OFF_Q, kk, Cfg::REG),
                         kmajor_desc(sbase + Cfg::OFF_WQ, kk, Cfg::W_BYTES), ID_Y, kk > 0);
            mma_commit_w(BAR(Cfg::B_YQ));
            // O := phi(Q) S_t^T
            ok = mbar_wait_w(BAR(Cfg::B_PHIQ), 0, abort_flag);
        }
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < DF / 16; ++kk)
                mma_ss_w(tm + Cfg::O_COL, kmajor_desc(sbase + Cfg::OFF_PQ, kk, Cfg::REG),
                         kmajor_desc(sbase + Cfg::OFF_ST, kk, 64 * 128), ID_N64, kk > 0);
            mma_commit_w(BAR(Cfg::B_PRO));
        }
        for (int j = 0; ok && j < n_tiles; ++j) {
            const int sk = j % Cfg::NSK, sv = j % Cfg::NSV;
            const uint32_t sPK = sbase + Cfg::OFF_PK + sk * Cfg::PHI_BYTES, sV = sbase + Cfg::OFF_V + sv * Cfg::REG;
            // A = phi(Q) phi(K_j)^T (after P V(j-1) in issue order, so A's columns are free)
            if (!(ok = mbar_wait_w(BAR(Cfg::B_KFULL + sk), (j / Cfg::NSK) & 1, abort_flag))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < DF / 16; ++kk)
                mma_ss_w(tm + Cfg::A_COL, kmajor_desc(sbase + Cfg::OFF_PQ, kk, Cfg::REG), kmajor_desc(sPK, kk, Cfg::REG),
                         ID_N128, kk > 0);
            mma_commit_w(BAR(Cfg::B_A));
            mma_commit_w(BAR(Cfg::B_KEMPTY + sk));
            // O += P V_j, P (bf16) over A's columns
            if (!(ok = mbar_wait_w(BAR(Cfg::B_VFULL + sv), (j / Cfg::NSV) & 1, abort_flag))) break;
            if (!(ok = mbar_wait_w(BAR(Cfg::B_P), j & 1, abort_flag))) break;
            tc_fence_after();
            const uint64_t dv = sw128_desc(sV, Cfg::REG, 1024);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_ts_w(tm + Cfg::O_COL, tm + Cfg::A_COL + kk * 8, dv + (uint64_t)(kk * 128), ID_PV, 1u);
            mma_commit_w(BAR(Cfg::B_O));
            mma_commit_w(BAR(Cfg::B_VEMPTY + sv));
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) report(p.err, DEV_ERR_TIMEOUT);
        }
        mma_commit_w(BAR(Cfg::B_DRAIN));
        mbar_wait_drain(BAR(Cfg::B_DRAIN), 0, 100000000ull);
    } else {
        // ================================================================ feature warps
        const int r = warp * 32 + lane;                 // TMEM lane = query row
        const int i = i0 + r;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint32_t tA = tmem + lane_off + Cfg::A_COL, tO = tmem + lane_off + Cfg::O_COL;
        bool ok = warp_all(mbar_wait(BAR(Cfg::B_QFULL), 0, abort_flag) && mbar_wait(BAR(Cfg::B_YQ), 0, abort_flag));
        float l_run = 0.f;
        {
            float y[DF];
            if (ok) {
                tc_fence_after();
                load_y_row<DF>(tA, y);
            }
            npmap_row<DF>(y, row_sqnorm_sw128(smem + Cfg::OFF_Q, r));
            const float4 *zt = reinterpret_cast<const float4 *>(p.z + (size_t)tslot * DF);
#pragma unroll
            for (int c4 = 0; c4 < DF / 4; ++c4) {
                const float4 zz = __ldg(zt + c4);
                l_run = fmaf(y[4 * c4], zz.x, l_run);
                l_run = fmaf(y[4 * c4 + 1], zz.y, l_run);
                l_run = fmaf(y[4 * c4 + 2], zz.z, l_run);
                l_run = fmaf(y[4 * c4 + 3], zz.w, l_run);
            }
            store_row_sw128<DF>(smem + Cfg::OFF_PQ, r, y);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // phi(Q) -> tensor core
            tc_fence_before();
            mbar_arrive(BAR(Cfg::B_PHIQ));
        }
        for (int j = 0; ok && j < n_tiles; ++j) {
            // A row: mask the diagonal tile causally, sum, P = A (bf16) over A's columns
            ok = warp_all(mbar_wait(BAR(Cfg::B_A), j & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            float sv[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t u[32];
                tmem_ld32(tA + c * 32, u);
#pragma unroll
                for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(u[e]);
            }
            tmem_wait_ld();
            if (j == n_tiles - 1) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c > r) sv[c] = 0.f;
            }
            float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            uint32_t pu[64];
#pragma unroll
            for (int e = 0; e < 64; ++e) {
                const float2 a = make_float2(sv[2 * e], sv[2 * e + 1]);
                acc[e & 3] = fadd2(acc[e & 3], a);
                pu[e] = pack_bf16x2(a.x, a.y);
            }
            const float2 s01 = fadd2(acc[0], acc[1]), s23 = fadd2(acc[2], acc[3]);
            l_run += (s01.x + s23.x) + (s01.y + s23.y);
            // (P V(j-1) read the previous P: it completed before A(j), issued after it)
            store_p(tA, pu);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(BAR(Cfg::B_P));
        }
        // ---- epilogue: o = O / l (the P V of the last tile done; O := phi(Q) S_t^T when n_tiles = 0)
        ok = warp_all(ok && mbar_wait(BAR(Cfg::B_PRO), 0, abort_flag) &&
                      (n_tiles == 0 || mbar_wait(BAR(Cfg::B_O), (n_tiles - 1) & 1, abort_flag)));
        if (ok) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            __nv_bfloat16 *orow = p.o + ((size_t)(b * p.H + h) * p.N + i) * 64;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t u[32];
                tmem_ld32(tO + c * 32, u);
                tmem_wait_ld();
                if (i < p.N) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(u[8 * v4 + 0]) * inv, __uint_as_float(u[8 * v4 + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(u[8 * v4 + 2]) * inv, __uint_as_float(u[8 * v4 + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(u[8 * v4 + 4]) * inv, __uint_as_float(u[8 * v4 + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(u[8 * v4 + 6]) * inv, __uint_as_float(u[8 * v4 + 7]) * inv);
                        dst[v4] = w;
                    }
                }
            }
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) report(p.err, DEV_ERR_TIMEOUT);
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == Cfg::MMA_WARP) tmem_dealloc(tmem, Cfg::TMEM_COLS);
}

template <int DF>
cudaError_t launch_phik_cfg(const Dims &s, const void *k, const void *wkt, void *phik, unsigned *err,
                            cudaStream_t st) {
    using Cfg = PhikCfg<DF>;
    CUtensorMap mk, mwk;
    if (!make_map(&mk, k, 64, s.N, (uint64_t)s.B * s.Hkv, 128) || !make_map(&mwk, wkt, 64, DF, s.Hkv, DF))
        return cudaErrorInvalidValue;
    PhikParams prm;
    prm.N = s.N;
    prm.Hkv = s.Hkv;
    prm.n_ktiles = (s.N + 127) / 128;
    prm.phik = static_cast<__nv_bfloat16 *>(phik);
    prm.err = err;
    auto kern = nowin_phik_kernel<DF>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(prm.n_ktiles * s.B * s.Hkv), 128, Cfg::SMEM, st>>>(mk, mwk, prm);
    return cudaGetLastError();
}

template <int DF>
cudaError_t launch_nowin_cfg(const Dims &s, const void *q, const void *v, const void *wqt, const void *st_t,
                             const float *z, const void *phik, void *o, unsigned *err, cudaStream_t st) {
    using Cfg = NowinCfg<DF>;
    const int T = s.T();
    const int n_qtiles = (s.N + 127) / 128;
    CUtensorMap mq, mpk, mv, mwq, ms;
    bool ok = make_map(&mq, q, 64, s.N, (uint64_t)s.B * s.H, 128) &&
              make_map(&mpk, phik, DF, s.N, (uint64_t)s.B * s.Hkv, 128) &&
              make_map(&mv, v, 64, s.N, (uint64_t)s.B * s.Hkv, 128) && make_map(&mwq, wqt, 64, DF, s.H, DF) &&
              make_map(&ms, st_t, DF, 64, (uint64_t)s.B * s.Hkv * (T + 1), 64);
    if (!ok) return cudaErrorInvalidValue;
    NowinParams prm;
    prm.B = s.B;
    prm.H = s.H;
    prm.Hkv = s.Hkv;
    prm.N = s.N;
    prm.C = s.C;
    prm.G = s.G();
    prm.T = T;
    prm.n_qtiles = n_qtiles;
    prm.z = z;
    prm.o = static_cast<__nv_bfloat16 *>(o);
    prm.err = err;
    auto kern = nowin_tc_kernel<DF>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(n_qtiles * s.B * s.H), Cfg::THREADS, Cfg::SMEM, st>>>(mq, mpk, mv, mwq, ms, prm);
    return cudaGetLastError();
}

}  // namespace

bool tc_nowin_supported(const Dims &s) {
    return s.bf16 && s.w == 0 && s.d == 64 && (s.D == 64 || s.D == 128) && s.C % 128 == 0 && s.C <= 1024 &&
           s.N > 0;
}

// w = 0 with head dimension 64: phi(k) of every key once, bf16 [B*Hkv, N, D] into `phik`.
cudaError_t launch_nowin_phik(const Dims &s, const void *k, const void *wkt, void *phik, unsigned *err,
                              cudaStream_t st) {
    if (s.D == 64) return launch_phik_cfg<64>(s, k, wkt, phik, err, st);
    if (s.D == 128) return launch_phik_cfg<128>(s, k, wkt, phik, err, st);
    return cudaErrorNotSupported;
}

// w = 0 with head dimension 64: every output row (o = (phi(q)^T S_t + intra-chunk causal tile) / (...)),
// with phi(K) from launch_nowin_phik.
cudaError_t launch_nowin_tc(const Dims &s, const void *q, const void *v, const void *wqt, const void *st_t,
                            const float *z, const void *phik, void *o, unsigned *err, cudaStream_t st) {
    if (s.D == 64) return launch_nowin_cfg<64>(s, q, v, wqt, st_t, z, phik, o, err, st);
    if (s.D == 128) return launch_nowin_cfg<128>(s, q, v, wqt, st_t, z, phik, o, err, st);
    return cudaErrorNotSupported;
}

}  // namespace still
