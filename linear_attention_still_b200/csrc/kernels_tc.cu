// kernels_tc.cu -- tcgen05 / TMEM / TMA kernels for sm_100a (bf16 storage, fp32 accumulation):
// the hybrid merge of "STILL: Selecting Tokens for Intra-Layer Hybrid Attention to Linearize LLMs"
// ([p1] jsqmd.com introduction: kept tokens -> softmax attention, the rest -> linear attention, in
// the same layer; "NP-Map": one shared distribution for both branches; [p4] atlas.scime.ai
// "Approach").
//
// One CTA = one (batch b, KV group g) x HP query heads of that group x 128 consecutive queries of
// one chunk t (C is a multiple of 128).  The HP heads see the same keys, so every K/V tile is loaded
// once per CTA.  Per query row i (TMEM lane = row):
//   prologue:  Y = Q Wq^T (tensor cores) -> phi(q) = ||q|| e/||e||, e = exp(Y - max Y)
//              O := phi(q) S_t^T (tensor cores), l := phi(q) . z_t (fp32), running max := 0
//              (or -inf, l := 0 when the linear branch is empty) -- the linear branch enters the
//              online softmax as a pre-accumulated term under the shared normaliser;
//   main loop: key tiles of 128: the kept rows of chunks c <= t-m-1 (compact cache, ragged last
//              tile masked), then the window [max(0,(t-m)C), i0+127] (diagonal tile masked
//              causally); S = Q K^T into TMEM, softmax rows in registers, P (bf16) written back
//              into TMEM over S, O += P V with P as the TMEM operand;
//   epilogue:  o = O / l.
// Warp roles: 4*HP softmax warps (warpgroup x owns head tile x), one TMA producer warp, one MMA
// warp (also allocates TMEM).  Every mbarrier wait is bounded; on a timeout the CTA records
// DEV_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "rowops.cuh"
#include "still_internal.h"
#include "tc_ptx.cuh"
#include "tc_tile.cuh"

namespace still {

using namespace tc;

namespace {

template <int DH, int DF, int HP>
struct MergeCfg {
    static constexpr int BM = 128;                     // query rows per head tile
    static constexpr int BN = 128;                     // keys per tile
    static constexpr int REG = 128 * 128;              // one 128-row x 64-col bf16 region (16 KB)
    static constexpr int TILE_BYTES = 128 * DH * 2;    // 128 x DH bf16 = DH/64 regions
    static constexpr int Q_BYTES = HP * TILE_BYTES;
    static constexpr int NS = DH == 128 ? 2 : 4;       // K/V pipeline stages
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES; // K + V
    static constexpr int WQ_BYTES = DF * DH * 2;       // one Wq^T [DF rows x DH]
    static constexpr int ST_BYTES = DH * DF * 2;       // S_t^T [DH rows x DF]
    static_assert(HP * WQ_BYTES + ST_BYTES <= NS * STAGE_BYTES, "prologue tiles must fit the stage area");
    static constexpr int NUM_BARS = 4 + 3 * NS + 5 * HP;  // see the slot map in the kernel
    static constexpr int TMEM_SLOT_OFF = 8 * NUM_BARS;          // u32 TMEM base address
    static constexpr int ABORT_OFF = TMEM_SLOT_OFF + 8;         // int abort flag
    static constexpr int BAR_BYTES = 256;
    static_assert(ABORT_OFF + 8 <= BAR_BYTES, "barrier area overflow");
    static constexpr int SMEM = Q_BYTES + NS * STAGE_BYTES + BAR_BYTES + 1024;
    // Two heads: three full warpgroups (softmax 0, softmax 1, producer + MMA + 2 idle warps) so the
    // register budget can be moved from the third warpgroup to the softmax ones (setmaxnreg).
    static constexpr int THREADS = HP == 2 ? 384 : 128 * HP + 64;
    static constexpr int PRODUCER_WARP = 4 * HP;
    static constexpr int MMA_WARP = 4 * HP + 1;
    // launch budget 384 x 168 = 64512 registers = 2 x 128 x 208 (softmax) + 128 x 88 (the rest)
    static constexpr int REG_SOFTMAX = 208, REG_OTHER = 88;
    static_assert(HP != 2 || 2 * 128 * REG_SOFTMAX + 128 * REG_OTHER <= THREADS * 168, "register split");
    static constexpr int TMEM_COLS = 512;
    // The budget is full at d = 128 (2 x S + 2 x O = 512 columns): P is written over S, and the next
    // tile's scores wait for P V.  (Head dimension 64 runs the ring-scheduled kernel of merge_ring.cu.)
    __host__ __device__ static constexpr int s_col(int x) { return x * 128; }
    __host__ __device__ static constexpr int p_col(int x) { return x * 128; }
    __host__ __device__ static constexpr int o_col(int x) { return 128 * HP + x * DH; }
    static_assert(128 * HP + HP * DH <= TMEM_COLS, "TMEM budget");
};

struct MergeParams {
    int B, H, Hkv, N, C, k, w, G, T;
    float scale_log2;      // tau * log2(e)
    const float *z;        // [B*Hkv*(T+1), DF] fp32
    __nv_bfloat16 *o;      // [B,H,N,DH]: window part (normalised) after LOCAL, final output after PREFIX
    float *lse;            // [B,H,N]: log2-sum-exp of the window part (LOCAL writes, PREFIX reads and
                           // replaces it with the row's whole log2 normaliser)
    float *sigma;          // [B,H,N]: Self-Saliency Score per query head (LOCAL writes)
    int *fix_list;         // rows whose band sum underflowed against the window max (recomputed later)
    unsigned *fix_count;
    unsigned *err;
    int n_qtiles;          // ceil(N/128)
    int qt_first;          // first query tile of this launch (PREFIX: chunks t > m only)
    int pairs;             // G / HP
};

// EXPV selects the exponential phase: 0 scalar FFMA + MUFU, 1 packed FFMA2/FADD2 + MUFU,
// 2 packed with the last 32-key chunk of each row on the FMA-pipe exp2, 3 with every other 32-key
// chunk there.  Measured on B200 with concurrent softmax warpgroups (1B 16K / 8B B4 16K layers, the
// two merge phases, ms): variant 1 0.612/3.629, 2 0.608/3.646, 3 0.641/3.799 -> variant 1 is built.
#ifndef STILL_MERGE_EXP
#define STILL_MERGE_EXP 1
#endif
constexpr int kMergeExpVariant = STILL_MERGE_EXP;
// Every wait of this kernel sleeps in mbarrier.try_wait instead of spinning (fewer issue slots and
// shared-memory tests taken from the softmax warps).  Measured on B200 (8B B4 16K layer, both phases):
// 3.24 -> 3.13 ms per step; the head-dim-64 ring kernel measured 0.489 -> 0.496 ms and keeps spinning.
constexpr bool kMergeSuspend = true;
// MODE kMergeLocal: keys = the window [max(0,(t-m)C), i]; also the Self-Saliency Score of every row
//   ([p1] "Self-Saliency Score"): the band keys [i-w+1, i-1] are window keys, so the band's
//   log-sum-exp is accumulated from the same exponentials (masked adds on the two partial tiles),
//   and the diagonal logit is read from the diagonal tile.  Writes o_A = window part / its sum,
//   lse_A (log2 units) and sigma.
// MODE kMergePrefix: keys = the kept rows of the decided chunks; the prologue folds the linear
//   branch and the window part into the accumulator under one shared normaliser:
//   M = max(lse_A, log2 b), O = O_lin 2^-M + o_A 2^(lse_A - M), l = 2^(lse_A - M) + b 2^-M.
constexpr int kMergeLocal = 0, kMergePrefix = 1;

template <int DH, int DF, int HP, int EXPV, int MODE>
__global__ void __launch_bounds__(MergeCfg<DH, DF, HP>::THREADS, 1)
    merge_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_kh,
                    const __grid_constant__ CUtensorMap map_vh, const __grid_constant__ CUtensorMap map_wq,
                    const __grid_constant__ CUtensorMap map_st, const MergeParams p) {
    using Cfg = MergeCfg<DH, DF, HP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase;                         // HP tiles
    const uint32_t sStage = sbase + Cfg::Q_BYTES;      // NS x (K tile, V tile); prologue Wq^T / S^T alias it
    uint8_t *bar_area = smem + Cfg::Q_BYTES + Cfg::NS * Cfg::STAGE_BYTES;
    const uint32_t sBar = smem_u32(bar_area);
    // barrier slots (8 bytes each)
    auto BAR = [&](int i) { return sBar + 8u * i; };
    const int B_QFULL = 0, B_WFULL = 1, B_PRO = 2, B_DRAIN = 3;
    const int B_KFULL = 4, B_VFULL = 4 + Cfg::NS, B_KVEMPTY = 4 + 2 * Cfg::NS;
    const int B_Y = 4 + 3 * Cfg::NS, B_PHI = B_Y + HP, B_S = B_PHI + HP, B_P = B_S + HP, B_O = B_P + HP;
    static_assert(Cfg::NUM_BARS == 4 + 3 * Cfg::NS + 5 * HP, "slot map");
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_area + Cfg::TMEM_SLOT_OFF);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bar_area + Cfg::ABORT_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- CTA -> (b, g, head pair, query tile); heavier (later) query tiles first
    const int per_qt = p.B * p.Hkv * p.pairs;
    const int qt = p.n_qtiles - 1 - (int)(blockIdx.x / per_qt);  // >= qt_first by the grid size
    const int rem = blockIdx.x % per_qt;
    const int pair = rem % p.pairs;
    const int bg = rem / p.pairs;
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const int i0 = qt * Cfg::BM;
    const int t = i0 / p.C;
    const int m = p.w / p.C;
    const int nk = p.k * max(0, t - m);                  // kept rows seen by this chunk
    const int lo = max(0, (t - m) * p.C);                // window start
    constexpr bool LOCAL = MODE == kMergeLocal;
    const int n_pre = LOCAL ? 0 : (nk + Cfg::BN - 1) / Cfg::BN;
    const int n_tiles = LOCAL ? (i0 - lo) / Cfg::BN + 1 : n_pre;
    const int tslot = bg * (p.T + 1) + t;                // linear state slot

    if (threadIdx.x == 0) {
        mbar_init(BAR(B_QFULL), 1);
        mbar_init(BAR(B_WFULL), 1);
        mbar_init(BAR(B_PRO), 1);
        mbar_init(BAR(B_DRAIN), 1);
        for (int s = 0; s < Cfg::NS; ++s) {
            mbar_init(BAR(B_KFULL + s), 1);
            mbar_init(BAR(B_VFULL + s), 1);
            mbar_init(BAR(B_KVEMPTY + s), 1);
        }
        for (int x = 0; x < HP; ++x) {
            mbar_init(BAR(B_Y + x), 1);
            mbar_init(BAR(B_PHI + x), 128);
            mbar_init(BAR(B_S + x), 1);
            mbar_init(BAR(B_P + x), 128);
            mbar_init(BAR(B_O + x), 1);
        }
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == Cfg::MMA_WARP) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == Cfg::PRODUCER_WARP && lane == 0) {
        tma_prefetch_desc(&map_q);
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_v);
        tma_prefetch_desc(&map_kh);
        tma_prefetch_desc(&map_vh);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Register budget changes sit at the top of each warpgroup's branch, so every role's code is
    // dominated by its own setmaxnreg.
    if (warp >= 4 * HP) {
    if (HP == 2) setmaxnreg_dec<Cfg::REG_OTHER>();
    if (warp == Cfg::PRODUCER_WARP) {
        // ================================================================ TMA producer
        // (the whole warp runs the issue loop; one elected lane issues each copy)
        {
            bool ok = true;
            int issued = 0;
            mbar_arrive_expect_tx_w(BAR(B_QFULL), Cfg::Q_BYTES);
            for (int x = 0; x < HP; ++x) {
                const int h = g * p.G + pair * HP + x;
                for (int rr = 0; rr < DH / 64; ++rr)
                    tma_load_3d_w(sQ + x * Cfg::TILE_BYTES + rr * Cfg::REG, &map_q, BAR(B_QFULL), rr * 64, i0,
                                b * p.H + h);
            }
            if (!LOCAL) {
                mbar_arrive_expect_tx_w(BAR(B_WFULL), HP * Cfg::WQ_BYTES + Cfg::ST_BYTES);
                for (int x = 0; x < HP; ++x) {
                    const int h = g * p.G + pair * HP + x;
                    for (int rr = 0; rr < DH / 64; ++rr)
                        tma_load_3d_w(sStage + x * Cfg::WQ_BYTES + rr * (DF * 128), &map_wq, BAR(B_WFULL), rr * 64, 0,
                                    h);
                }
                for (int rr = 0; rr < DF / 64; ++rr)
                    tma_load_3d_w(sStage + HP * Cfg::WQ_BYTES + rr * (DH * 128), &map_st, BAR(B_WFULL), rr * 64, 0,
                                tslot);
                ok = mbar_wait_wt<kMergeSuspend>(BAR(B_PRO), 0, abort_flag);  // prologue operands consumed
            }
            for (int j = 0; ok && j < n_tiles; ++j) {
                const int s = j % Cfg::NS;
                if (j >= Cfg::NS) {
                    ok = mbar_wait_wt<kMergeSuspend>(BAR(B_KVEMPTY + s), ((j / Cfg::NS) - 1) & 1, abort_flag);
                    if (!ok) break;
                }
                const uint32_t sK = sStage + s * Cfg::STAGE_BYTES, sV = sK + Cfg::TILE_BYTES;
                const CUtensorMap *mk = LOCAL ? &map_k : &map_kh;
                const CUtensorMap *mv = LOCAL ? &map_v : &map_vh;
                const int row = LOCAL ? lo + j * Cfg::BN : j * Cfg::BN;
                mbar_arrive_expect_tx_w(BAR(B_KFULL + s), Cfg::TILE_BYTES);
                for (int rr = 0; rr < DH / 64; ++rr)
                    tma_load_3d_w(sK + rr * Cfg::REG, mk, BAR(B_KFULL + s), rr * 64, row, bg);
                mbar_arrive_expect_tx_w(BAR(B_VFULL + s), Cfg::TILE_BYTES);
                for (int rr = 0; rr < DH / 64; ++rr)
                    tma_load_3d_w(sV + rr * Cfg::REG, mv, BAR(B_VFULL + s), rr * 64, row, bg);
                issued = j + 1;
            }
            if (!ok) {
                *abort_flag = 1;
                if (lane == 0) report(p.err, DEV_ERR_TIMEOUT);
                // drain this CTA's copies still in flight
                mbar_wait_drain(BAR(B_QFULL), 0, 100000000ull);
                if (!LOCAL) mbar_wait_drain(BAR(B_WFULL), 0, 100000000ull);
                for (int j = max(0, issued - Cfg::NS); j < issued; ++j) {
                    mbar_wait_drain(BAR(B_KFULL + j % Cfg::NS), (j / Cfg::NS) & 1, 100000000ull);
                    mbar_wait_drain(BAR(B_VFULL + j % Cfg::NS), (j / Cfg::NS) & 1, 100000000ull);
                }
            }
        }
    } else if (warp == Cfg::MMA_WARP) {
        // ================================================================ MMA issuer
        // (the whole warp runs the issue loop; one elected lane issues each MMA and commit)
        {
            const uint32_t tmem_w = __shfl_sync(0xffffffffu, tmem, 0);
            constexpr uint32_t ID_Y = idesc_bf16(128, DF, 0, 0);
            constexpr uint32_t ID_LIN = idesc_bf16(128, DH, 0, 0);
            constexpr uint32_t ID_S = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t ID_PV = idesc_bf16(128, DH, 0, 1);
            bool ok = mbar_wait_wt<kMergeSuspend>(BAR(B_QFULL), 0, abort_flag) && (LOCAL || mbar_wait_wt<kMergeSuspend>(BAR(B_WFULL), 0, abort_flag));
            if (ok && !LOCAL) {
                tc_fence_after();
                for (int x = 0; x < HP; ++x) {
                    const uint32_t aq = sQ + x * Cfg::TILE_BYTES, bw = sStage + x * Cfg::WQ_BYTES;
                    for (int kk = 0; kk < DH / 16; ++kk)
                        mma_ss_w(tmem_w + Cfg::s_col(x), kmajor_desc(aq, kk, Cfg::REG), kmajor_desc(bw, kk, DF * 128),
                               ID_Y, kk > 0);
                    mma_commit_w(BAR(B_Y + x));
                }
                for (int x = 0; x < HP && ok; ++x) {
                    ok = mbar_wait_wt<kMergeSuspend>(BAR(B_PHI + x), 0, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t bs = sStage + HP * Cfg::WQ_BYTES;
                    for (int kk = 0; kk < DF / 16; ++kk)
                        mma_ts_w(tmem_w + Cfg::o_col(x), tmem_w + Cfg::s_col(x) + kk * 8, kmajor_desc(bs, kk, DH * 128),
                               ID_LIN, kk > 0);
                }
                if (ok) mma_commit_w(BAR(B_PRO));
            }
            // Descriptors are built once per operand tile and advanced per 16-element k-step by a
            // constant added to the start-address field (addresses stay below 256 KB, so no carry).
            // K-major k-step kk: region kk/4, 32 bytes per step inside the 128-byte row.
            auto kstep = [](int kk) -> uint64_t { return (uint64_t)((((kk >> 2) * Cfg::REG) + ((kk & 3) * 32)) >> 4); };
            uint64_t dq[HP];
#pragma unroll
            for (int x = 0; x < HP; ++x) dq[x] = sw128_desc(sQ + x * Cfg::TILE_BYTES, 16, 1024);
            auto issue_s = [&](int x, uint32_t sK) {
                const uint64_t dk = sw128_desc(sK, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < DH / 16; ++kk)
                    mma_ss_w(tmem_w + Cfg::s_col(x), dq[x] + kstep(kk), dk + kstep(kk), ID_S, kk > 0);
                mma_commit_w(BAR(B_S + x));
            };
            // first score tiles
            if (ok && n_tiles > 0) ok = mbar_wait_wt<kMergeSuspend>(BAR(B_KFULL + 0), 0, abort_flag);
            if (ok && n_tiles > 0) {
                tc_fence_after();
                for (int x = 0; x < HP; ++x) issue_s(x, sStage);
            }
            // In-order issue: per tile, head 0 then head 1 (next scores, then P V).  (An issuer driven by
            // whichever barrier completes first measured 5-10 % slower on B200.)
            for (int j = 0; ok && j < n_tiles; ++j) {
                const int s = j % Cfg::NS;
                const uint64_t dv = sw128_desc(sStage + s * Cfg::STAGE_BYTES + Cfg::TILE_BYTES, Cfg::REG, 1024);
                const int s1 = (j + 1) % Cfg::NS;
                const uint32_t sK1 = sStage + s1 * Cfg::STAGE_BYTES;
                for (int x = 0; x < HP && ok; ++x) {
                    if (x == 0) ok = mbar_wait_wt<kMergeSuspend>(BAR(B_VFULL + s), (j / Cfg::NS) & 1, abort_flag);
                    if (ok) ok = mbar_wait_wt<kMergeSuspend>(BAR(B_P + x), j & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)  // V k-step: 16 keys = 16 rows of 128 bytes
                        mma_ts_w(tmem_w + Cfg::o_col(x), tmem_w + Cfg::p_col(x) + kk * 8, dv + (uint64_t)(kk * 128), ID_PV,
                               (LOCAL && j == 0 && kk == 0) ? 0u : 1u);  // LOCAL: the first PV starts O
                    mma_commit_w(BAR(B_O + x));
                    if (j + 1 < n_tiles) {
                        // P_x(j) lives over S_x: the next scores wait for PV_x(j) (in-order issue)
                        if (x == 0) ok = mbar_wait_wt<kMergeSuspend>(BAR(B_KFULL + s1), ((j + 1) / Cfg::NS) & 1, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        issue_s(x, sK1);
                    }
                }
                if (ok) mma_commit_w(BAR(B_KVEMPTY + s));
            }
            if (!ok) {
                *abort_flag = 1;
                if (lane == 0) report(p.err, DEV_ERR_TIMEOUT);
            }
            // drain every MMA this thread issued before TMEM is released
            mma_commit_w(BAR(B_DRAIN));
            mbar_wait_drain(BAR(B_DRAIN), 0, 100000000ull);
        }
    }
    } else {
        if (HP == 2) setmaxnreg_inc<Cfg::REG_SOFTMAX>();
        // ================================================================ softmax warpgroups
        const int x = warp >> 2;                       // head tile
        const int r = (warp & 3) * 32 + lane;          // row in the tile = TMEM lane
        const int i = i0 + r;
        const int h = g * p.G + pair * HP + x;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + Cfg::s_col(x);
        const uint32_t tO = tmem + lane_off + Cfg::o_col(x);
        const uint32_t tP = tmem + lane_off + Cfg::p_col(x);
        bool ok = true;

        const size_t row = ((size_t)b * p.H + h) * p.N + i;  // this thread's query row
        float m_run = -INFINITY, l_run = 0.f;
        float bs = 0.f, sdiag = 0.f;  // LOCAL: band sum (same reference as l) and raw diagonal score

        if constexpr (!LOCAL) {
            // the window part of this row (o_A, written by the window phase) is read in the fold below:
            // start bringing it into L2 now
            if (i < p.N) {
#pragma unroll
                for (int v = 0; v < DH * 2; v += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.o + row * DH + v / 2));
            }
            // ---- prologue: phi(q) from Y = Q Wq^T
            ok = warp_all(mbar_wait_t<kMergeSuspend>(BAR(B_QFULL), 0, abort_flag) && mbar_wait_t<kMergeSuspend>(BAR(B_Y + x), 0, abort_flag));
            float y[DF];
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < DF / 32; ++c) {
                    uint32_t u[32];
                    tmem_ld32(tS + c * 32, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) y[c * 32 + e] = __uint_as_float(u[e]);
                }
            }
            // ||q||^2 from the swizzled Q tile in shared memory
            float qq = 0.f;
            const uint8_t *qrow = smem + x * Cfg::TILE_BYTES + r * 128;
#pragma unroll
            for (int rr = 0; rr < DH / 64; ++rr) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(qrow + rr * Cfg::REG + ((ch ^ (r & 7)) << 4));
                    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(h2[e]);
                        qq = fmaf(f.x, f.x, qq);
                        qq = fmaf(f.y, f.y, qq);
                    }
                }
            }
            float ymax = -INFINITY;
#pragma unroll
            for (int c = 0; c < DF; ++c) ymax = fmaxf(ymax, y[c]);
            float ee = 0.f;
#pragma unroll
            for (int c = 0; c < DF; ++c) {
                y[c] = ex2((y[c] - ymax) * kLog2e);
                ee = fmaf(y[c], y[c], ee);
            }
            const float f = sqrtf(qq) * rsqrtf(ee);
            const float *zt = p.z + (size_t)tslot * DF;
            float bden = 0.f;
#pragma unroll
            for (int c = 0; c < DF; ++c) {
                y[c] *= f;
                bden = fmaf(y[c], __ldg(zt + c), bden);
            }
            if (ok) {
#pragma unroll
                for (int c = 0; c < DF / 64; ++c) {
                    uint32_t u[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) u[e] = pack_bf16x2(y[c * 64 + 2 * e], y[c * 64 + 2 * e + 1]);
                    tmem_st32(tS + c * 32, u);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(BAR(B_PHI + x));
            // ---- fold the window part (o_A, lse_A) into O = phi(q) S_t^T under one normaliser
            // the window part's row is loaded while phi(q) S_t^T runs
            const bool valid = i < p.N;
            const float lse_a = valid ? p.lse[row] : 0.f;
            uint4 oa[DH / 8];
            {
                const uint4 *orow = reinterpret_cast<const uint4 *>(p.o + row * DH);
#pragma unroll
                for (int v = 0; v < DH / 8; ++v) oa[v] = valid ? orow[v] : make_uint4(0, 0, 0, 0);
            }
            ok = warp_all(ok && mbar_wait_t<kMergeSuspend>(BAR(B_PRO), 0, abort_flag));
            if (ok) {
                tc_fence_after();
                const float M = bden > 0.f ? fmaxf(lse_a, __log2f(bden)) : lse_a;
                const float wa = ex2(lse_a - M), wb = ex2(-M);
#pragma unroll
                for (int c = 0; c < DH / 32; ++c) {
                    uint32_t u[32];
                    tmem_ld32(tO + c * 32, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        const uint4 w = oa[c * 4 + v4];
                        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ww[e]));
                            const int q0 = 8 * v4 + 2 * e;
                            u[q0] = __float_as_uint(fmaf(__uint_as_float(u[q0]), wb, a.x * wa));
                            u[q0 + 1] = __float_as_uint(fmaf(__uint_as_float(u[q0 + 1]), wb, a.y * wa));
                        }
                    }
                    tmem_st32(tO + c * 32, u);
                }
                tmem_wait_st();
                m_run = M;
                l_run = wa + bden * wb;
            }
        }

        // ---- main loop over key tiles
        for (int j = 0; ok && j < n_tiles; ++j) {
            ok = warp_all(mbar_wait_t<kMergeSuspend>(BAR(B_S + x), j & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            const bool diag = LOCAL && j == n_tiles - 1;
            const bool ragged = !LOCAL && nk - j * Cfg::BN < Cfg::BN;
            const int limit = diag ? r + 1 : nk - j * Cfg::BN;
            float sv[128];
            load_s_row(tS, sv, diag, ragged, limit, r, sdiag);
            // O *= a on the rows that move their reference (warp-collective: the warp takes it together
            // when any of its rows needs it).  P V(j-1) has completed: the scores of tile j were issued
            // after it (PREFIX j = 0: the prologue's phi(q) S_t^T).
            auto rescale_o = [&](bool touch, float a) -> bool {
                if (!__any_sync(0xffffffffu, touch)) return true;
                if (!warp_all(j == 0 ? (LOCAL || mbar_wait_t<kMergeSuspend>(BAR(B_PRO), 0, abort_flag))
                                     : mbar_wait_t<kMergeSuspend>(BAR(B_O + x), (j - 1) & 1, abort_flag)))
                    return false;
                tc_fence_after();
                const float f = touch ? a : 1.f;
#pragma unroll
                for (int c = 0; c < DH / 32; ++c) {
                    uint32_t u[32];
                    tmem_ld32(tO + c * 32, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * f);
                    tmem_st32(tO + c * 32, u);
                }
                tmem_wait_st();
                return true;
            };
            // Lazy rescale: a row moves its reference max only when the max grows by more than
            // kRescaleLog2 (see tc_tile.cuh).
            const float mnew = row_max128(sv) * p.scale_log2;
            const bool need = mnew > m_run + kRescaleLog2;
            const float alpha = need ? ex2(m_run - mnew) : 1.f;
            // O holds nothing yet while m_run = -inf
            if (!(ok = rescale_o(need && m_run != -INFINITY, alpha))) break;
            if (need) {
                l_run *= alpha;
                bs *= alpha;
                m_run = mnew;
            }
            // LOCAL band tiles: keys kstart + c; the band of row r is [i-w+1, i-1]
            int btype = 0;  // 0 none, 1 whole tile, 2 columns c > r, 3 columns c < r
            if (LOCAL) {
                const int kstart = lo + j * Cfg::BN;
                if (diag) btype = 3;
                else if (i0 >= p.w && kstart == i0 - p.w) btype = 2;
                else if (i0 >= p.w && kstart < i0 - p.w) btype = 0;
                else btype = 1;
            }
            // exponentials stored to P (over S) as they are formed
            float ls0, ls1, bsum = 0.f;
            if (btype >= 2) {
                const int bc_lo = btype == 2 ? r + 1 : 0, bc_hi = btype == 2 ? 128 : r;
                exp_tile<EXPV, true>(sv, p.scale_log2, m_run, tP, ls0, ls1, bsum, bc_lo, bc_hi);
            } else {
                exp_tile<EXPV, false>(sv, p.scale_log2, m_run, tP, ls0, ls1, bsum, 0, 0);
            }
            l_run += ls0 + ls1;
            if (btype == 1) bs += ls0 + ls1;
            else if (btype >= 2) bs += bsum;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(BAR(B_P + x));
        }
        // ---- epilogue: o = O / l
        ok = warp_all(ok && (n_tiles > 0 ? mbar_wait_t<kMergeSuspend>(BAR(B_O + x), (n_tiles - 1) & 1, abort_flag) : true));
        if (ok) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            __nv_bfloat16 *orow = p.o + row * DH;
#pragma unroll
            for (int c = 0; c < DH / 32; ++c) {
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
            // lse: LOCAL the window part's log2-sum-exp (read back by the prefix phase); PREFIX the
            // row's whole normaliser (both branches), left for the backward pass
            if (!LOCAL && i < p.N) p.lse[row] = m_run + __log2f(l_run);
            if (LOCAL && i < p.N) {
                p.lse[row] = m_run + __log2f(l_run);
                // sigma = softplus(s_ii - LSE_{band}) in natural units; +inf for an empty band (i = 0)
                float sig = INFINITY;
                if (i > 0) {
                    if (bs > 0x1p-90f) {
                        const float lse_band = (m_run + __log2f(bs)) * kLn2;
                        sig = softplus_f(sdiag * (p.scale_log2 * kLn2) - lse_band);
                    } else {
                        // every band key sits > 90 binary orders below the window maximum: the shared
                        // reference has underflowed the band sum; the row is rescored with its own max
                        p.fix_list[atomicAdd(p.fix_count, 1u)] = (int)row;
                        sig = 0.f;
                    }
                }
                p.sigma[row] = sig;
            }
        }
        if (!ok) {
            *abort_flag = 1;
            report(p.err, DEV_ERR_TIMEOUT);
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == Cfg::MMA_WARP) tmem_dealloc(tmem, Cfg::TMEM_COLS);
}

// ------------------------------------------------------------------ banded saliency
// Self-Saliency Score ([p1] "Self-Saliency Score"; [p4] "Approach"): for query row i of head h,
// sigma = softplus(s_ii - LSE_{j in [i-w+1, i-1]} s_ij) = -ln(1 - p_ii), +inf for an empty band.
// One CTA = (b, g, HP heads, 128 queries).  Key tiles cover [max(0, i0-w), i0+127] (w is a multiple
// of 128): the first tile of a full window masks c <= r (key i0-w+c is below row r's band), the
// diagonal tile masks c >= r and takes c == r as s_ii.  S = Q K^T in TMEM, double-buffered per head so
// the next tile's MMA overlaps this tile's exponentials; per row an online log-sum-exp in registers.
// Writes sigma per query head; the group mean is taken by mean_heads_kernel.
template <int DH, int HP>
struct SalCfg {
    static constexpr int REG = 128 * 128;
    static constexpr int TILE_BYTES = 128 * DH * 2;
    static constexpr int Q_BYTES = HP * TILE_BYTES;
    static constexpr int NS = DH == 128 ? 4 : 6;
    static constexpr int NUM_BARS = 2 + 2 * NS + 4 * HP;
    static constexpr int TMEM_SLOT_OFF = 8 * NUM_BARS;
    static constexpr int ABORT_OFF = TMEM_SLOT_OFF + 8;
    static constexpr int BAR_BYTES = 256;
    static_assert(ABORT_OFF + 8 <= BAR_BYTES, "barrier area overflow");
    static constexpr int SIG_BYTES = HP * 128 * 4;  // per-row sigma of each head (group mean)
    static constexpr int SMEM = Q_BYTES + NS * TILE_BYTES + BAR_BYTES + SIG_BYTES + 1024;
    static constexpr int THREADS = 128 * HP + 64;
    static constexpr int PRODUCER_WARP = 4 * HP;
    static constexpr int MMA_WARP = 4 * HP + 1;
    static constexpr int TMEM_COLS = HP == 2 ? 512 : 256;
    __host__ __device__ static constexpr int s_col(int x, int buf) { return (x * 2 + buf) * 128; }
};

struct SalParams {
    int B, H, Hkv, N, w, G, pairs, n_qtiles;
    float scale_log2;
    float *sigma;      // [B,H,N] or nullptr
    float *r_kv;       // [B,Hkv,N], written here when the CTA holds the whole group (pairs == 1)
    unsigned *err;
};

template <int DH, int HP>
__global__ void __launch_bounds__(SalCfg<DH, HP>::THREADS, 1)
    saliency_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                       const SalParams p) {
    using Cfg = SalCfg<DH, HP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase, sK = sbase + Cfg::Q_BYTES;
    uint8_t *bar_area = smem + Cfg::Q_BYTES + Cfg::NS * Cfg::TILE_BYTES;
    const uint32_t sBar = smem_u32(bar_area);
    auto BAR = [&](int i) { return sBar + 8u * i; };
    const int B_QFULL = 0, B_DRAIN = 1, B_KFULL = 2, B_KEMPTY = 2 + Cfg::NS;
    const int B_SFULL = 2 + 2 * Cfg::NS, B_SEMPTY = B_SFULL + 2 * HP;  // [x*2 + buf]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_area + Cfg::TMEM_SLOT_OFF);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bar_area + Cfg::ABORT_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const int per_qt = p.B * p.Hkv * p.pairs;
    const int qt = p.n_qtiles - 1 - (int)(blockIdx.x / per_qt);  // >= qt_first by the grid size
    const int rem = blockIdx.x % per_qt;
    const int pair = rem % p.pairs;
    const int bg = rem / p.pairs;
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const int i0 = qt * 128;
    const int kbase = max(0, i0 - p.w);
    const int n_tiles = (i0 - kbase) / 128 + 1;
    const bool low_mask_first = i0 >= p.w;  // first tile starts at i0 - w

    if (threadIdx.x == 0) {
        mbar_init(BAR(B_QFULL), 1);
        mbar_init(BAR(B_DRAIN), 1);
        for (int s = 0; s < Cfg::NS; ++s) {
            mbar_init(BAR(B_KFULL + s), 1);
            mbar_init(BAR(B_KEMPTY + s), 1);
        }
        for (int e = 0; e < 2 * HP; ++e) {
            mbar_init(BAR(B_SFULL + e), 1);
            mbar_init(BAR(B_SEMPTY + e), 128);
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
        if (lane == 0) {
            bool ok = true;
            int issued = 0;
            mbar_arrive_expect_tx(BAR(B_QFULL), Cfg::Q_BYTES);
            for (int x = 0; x < HP; ++x) {
                const int h = g * p.G + pair * HP + x;
                for (int rr = 0; rr < DH / 64; ++rr)
                    tma_load_3d(sQ + x * Cfg::TILE_BYTES + rr * Cfg::REG, &map_q, BAR(B_QFULL), rr * 64, i0,
                                b * p.H + h);
            }
            for (int j = 0; j < n_tiles; ++j) {
                const int s = j % Cfg::NS;
                if (j >= Cfg::NS) {
                    ok = mbar_wait(BAR(B_KEMPTY + s), ((j / Cfg::NS) - 1) & 1, abort_flag);
                    if (!ok) break;
                }
                mbar_arrive_expect_tx(BAR(B_KFULL + s), Cfg::TILE_BYTES);
                for (int rr = 0; rr < DH / 64; ++rr)
                    tma_load_3d(sK + s * Cfg::TILE_BYTES + rr * Cfg::REG, &map_k, BAR(B_KFULL + s), rr * 64,
                                kbase + j * 128, bg);
                issued = j + 1;
            }
            if (!ok) {
                *abort_flag = 1;
                report(p.err, DEV_ERR_TIMEOUT);
                mbar_wait_drain(BAR(B_QFULL), 0, 100000000ull);
                for (int j = max(0, issued - Cfg::NS); j < issued; ++j)
                    mbar_wait_drain(BAR(B_KFULL + j % Cfg::NS), (j / Cfg::NS) & 1, 100000000ull);
            }
        }
    } else if (warp == Cfg::MMA_WARP) {
        if (lane == 0) {
            constexpr uint32_t ID_S = idesc_bf16(128, 128, 0, 0);
            bool ok = mbar_wait(BAR(B_QFULL), 0, abort_flag);
            for (int j = 0; ok && j < n_tiles; ++j) {
                const int s = j % Cfg::NS, buf = j & 1;
                ok = mbar_wait(BAR(B_KFULL + s), (j / Cfg::NS) & 1, abort_flag);
                for (int x = 0; x < HP && ok; ++x) {
                    if (j >= 2) ok = mbar_wait(BAR(B_SEMPTY + 2 * x + buf), ((j >> 1) - 1) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    #pragma unroll 1
                    for (int kk = 0; kk < DH / 16; ++kk)
                        mma_ss(tmem + Cfg::s_col(x, buf), kmajor_desc(sQ + x * Cfg::TILE_BYTES, kk, Cfg::REG),
                               kmajor_desc(sK + s * Cfg::TILE_BYTES, kk, Cfg::REG), ID_S, kk > 0);
                    mma_commit(BAR(B_SFULL + 2 * x + buf));
                }
                if (ok) mma_commit(BAR(B_KEMPTY + s));
            }
            if (!ok) {
                *abort_flag = 1;
                report(p.err, DEV_ERR_TIMEOUT);
            }
            mma_commit(BAR(B_DRAIN));
            mbar_wait_drain(BAR(B_DRAIN), 0, 100000000ull);
        }
    } else {
        const int x = warp >> 2;
        const int r = (warp & 3) * 32 + lane;
        const int i = i0 + r;
        const int h = g * p.G + pair * HP + x;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        float m2 = -INFINITY, l = 0.f, sdiag = 0.f;
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            const int buf = j & 1;
            ok = warp_all(mbar_wait(BAR(B_SFULL + 2 * x + buf), (j >> 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            float sv[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t u[32];
                tmem_ld32(tmem + lane_off + Cfg::s_col(x, buf) + c * 32, u);
#pragma unroll
                for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(u[e]);
            }
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(BAR(B_SEMPTY + 2 * x + buf));  // the buffer can take tile j+2
            // band [lo_c, hi_c): keys kbase + j*128 + c
            int lo_c = 0, hi_c = 128;
            if (j == 0 && low_mask_first) lo_c = r + 1;
            if (j == n_tiles - 1) {
                hi_c = r;
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c == r) sdiag = sv[c];  // unrolled select keeps sv in registers
            }
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                const bool in = c >= lo_c && c < hi_c;
                sv[c] = in ? sv[c] * p.scale_log2 : -INFINITY;
                mx = fmaxf(mx, sv[c]);
            }
            if (mx > m2) {
                l *= ex2(m2 - mx);
                m2 = mx;
            }
            if (m2 != -INFINITY) {
                float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                for (int c = 0; c < 128; c += 4) {
                    a0 += ex2(sv[c] - m2);
                    a1 += ex2(sv[c + 1] - m2);
                    a2 += ex2(sv[c + 2] - m2);
                    a3 += ex2(sv[c + 3] - m2);
                }
                l += (a0 + a1) + (a2 + a3);
            }
        }
        // ln-domain: LSE = (m2 + log2 l) ln 2, s_ii = sdiag * tau
        float sigma = INFINITY;
        if (m2 != -INFINITY) {
            const float lse = (m2 + __log2f(l)) * 0.6931471805599453f;
            sigma = softplus_f(sdiag * (p.scale_log2 * 0.6931471805599453f) - lse);
        }
        if (!ok) {
            *abort_flag = 1;
            report(p.err, DEV_ERR_TIMEOUT);
        }
        if (ok && p.sigma && i < p.N) p.sigma[((size_t)b * p.H + h) * p.N + i] = sigma;
        if (p.pairs == 1) {
            // the CTA holds every head of the group: mean over heads, in head order
            float *ssig = reinterpret_cast<float *>(bar_area + Cfg::BAR_BYTES);
            ssig[x * 128 + r] = sigma;
            asm volatile("bar.sync 1, %0;" ::"r"(128 * HP) : "memory");
            if (ok && x == 0 && i < p.N) {
                float acc = 0.f;
#pragma unroll
                for (int xx = 0; xx < HP; ++xx) acc += ssig[xx * 128 + r];
                p.r_kv[(size_t)bg * p.N + i] = acc / (float)HP;
            }
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == Cfg::MMA_WARP) tmem_dealloc(tmem, Cfg::TMEM_COLS);
}

// r[b,g,i] = mean over the G heads of g of sigma[b,h,i], summed in head order.
__global__ void mean_heads_kernel(const float *__restrict__ sigma, float *__restrict__ r, int B, int H, int Hkv,
                                  int N) {
    const int G = H / Hkv;
    const size_t total = (size_t)B * Hkv * N;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
        const size_t bg = e / N;
        const int i = (int)(e % N);
        const size_t b = bg / Hkv, g = bg % Hkv;
        float acc = 0.f;
        for (int hh = 0; hh < G; ++hh) acc += sigma[((b * H) + g * G + hh) * N + i];
        r[e] = acc / (float)G;
    }
}

// ------------------------------------------------------------------ linear state (NP-Map fused)
// Linear branch state ([p1] introduction: the unselected tokens are aggregated linearly; "NP-Map":
// phi(x) = ||x|| f(x Wk) / ||f(x Wk)||): for each (b, g) and each chunk c <= T-m-1 that some query
// chunk sees, Delta S_c = sum over the unkept tokens j of c of phi(k_j) v_j^T [D, d] and
// Delta z_c = sum phi(k_j), written to slot c+m+1 of S / z (the prefix kernel then sums the slots).
// One CTA per (b, g, c); per 128-token subtile: Y = K Wk^T (tcgen05, TMEM, double-buffered) ->
// four warps turn their token's row into phi (zero for kept tokens) and store it bf16 into shared
// memory in the 128-byte-swizzled layout -> Delta S += Phi^T V and Delta z += Phi^T 1 (tcgen05,
// Phi^T and V as MN-major operands, fp32 accumulators in TMEM).  The feature dimension is padded
// to 128 rows of the MMA (D = 64 leaves the upper half zero).
#ifndef STILL_LIN_PAIR
#define STILL_LIN_PAIR 1
#endif
constexpr bool kLinPair = STILL_LIN_PAIR != 0;

template <int DH, int DF>
struct LinCfg {
    static constexpr int REG = 128 * 128;                 // 128 rows x 64 bf16
    static constexpr int TILE_BYTES = 128 * DH * 2;       // 128 tokens x DH
    static constexpr int NS = 2;
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;    // K + V
    static constexpr int WK_BYTES = DF * DH * 2;          // Wk^T [DF rows x DH]
    static constexpr int PHI_BYTES = 2 * REG;             // [128 tokens x 128 features] (2 regions)
    static constexpr int ONES_BYTES = 2 * 16 * 128;       // [16 rows x 128 tokens] of ones (2 regions)
    static constexpr int NUM_BARS = 9 + 3 * NS;
    static constexpr int TMEM_SLOT_OFF = 8 * NUM_BARS;
    static constexpr int ABORT_OFF = TMEM_SLOT_OFF + 8;
    static constexpr int BAR_BYTES = 256;
    static_assert(ABORT_OFF + 8 <= BAR_BYTES, "barrier area overflow");
    static constexpr int SMEM = WK_BYTES + NS * STAGE_BYTES + PHI_BYTES + ONES_BYTES + BAR_BYTES + 1024;
    static constexpr int THREADS = 128 + 64;
    static constexpr int PRODUCER_WARP = 4, MMA_WARP = 5;
    // d = D = 64: two CTAs per SM (the two Y buffers, S and z fit in 256 TMEM columns), so the chunk
    // CTAs of a layer run in one wave instead of two
    static constexpr bool PAIR = kLinPair && DH == 64 && DF == 64;
    static constexpr int MINB = PAIR ? 2 : 1;
    static constexpr int YB = PAIR ? DF : 128;  // columns between the two Y buffers
    static constexpr int Y_COL = 0, S_COL = PAIR ? 2 * DF : 256, Z_COL = S_COL + (PAIR ? DH : 128),
                         TMEM_COLS = PAIR ? 256 : 512;
    static_assert(Z_COL + 16 <= TMEM_COLS && Y_COL + YB + DF <= S_COL, "TMEM columns");
    static_assert(MINB * (SMEM + 1024) <= 233472, "shared memory per SM");
};

struct LinParams {
    int B, Hkv, N, C, k, m, T;
    const int32_t *idx;   // [B,Hkv,T,k] kept positions
    float *S;             // [B,Hkv,T+1,D,d]
    float *z;             // [B,Hkv,T+1,D]
    unsigned *err;
};

template <int DH, int DF>
__global__ void __launch_bounds__(LinCfg<DH, DF>::THREADS, LinCfg<DH, DF>::MINB)
    linear_state_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                           const __grid_constant__ CUtensorMap map_wk, const LinParams p) {
    using Cfg = LinCfg<DH, DF>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sWk = sbase;
    const uint32_t sStage = sWk + Cfg::WK_BYTES;
    const uint32_t sPhi = sStage + Cfg::NS * Cfg::STAGE_BYTES;
    const uint32_t sOnes = sPhi + Cfg::PHI_BYTES;
    uint8_t *phi_ptr = smem + (sPhi - sbase);
    uint8_t *bar_area = smem + (sOnes - sbase) + Cfg::ONES_BYTES;
    const uint32_t sBar = smem_u32(bar_area);
    auto BAR = [&](int i) { return sBar + 8u * i; };
    // slots: 0 WK full, 1 drain, 2/3 Y full [buf], 4/5 Y empty [buf], 6 Phi full, 7 Phi empty,
    //        8.. K full[s], 8+NS.. V full[s], 8+2NS.. KV empty[s], 8+3NS done
    const int B_WK = 0, B_DRAIN = 1, B_YFULL = 2, B_YEMPTY = 4, B_PFULL = 6, B_PEMPTY = 7, B_KFULL = 8,
              B_VFULL = 8 + Cfg::NS, B_KVEMPTY = 8 + 2 * Cfg::NS, B_DONE = 8 + 3 * Cfg::NS;
    static_assert(8 + 3 * Cfg::NS + 1 == Cfg::NUM_BARS, "slot map");
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_area + Cfg::TMEM_SLOT_OFF);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bar_area + Cfg::ABORT_OFF);
    __shared__ unsigned char kept[1024];  // per-subtile scratch is enough: C <= 1024 checked on the host
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nc = p.T - p.m;
    const int c = blockIdx.x % nc;
    const int bg = blockIdx.x / nc;
    const int g = bg % p.Hkv;
    const int nsub = p.C / 128;

    if (threadIdx.x == 0) {
        for (int i = 0; i < Cfg::NUM_BARS; ++i) mbar_init(BAR(i), (i == B_PFULL || i == B_YEMPTY || i == B_YEMPTY + 1) ? 128 : 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    for (int j = threadIdx.x; j < p.C; j += blockDim.x) kept[j] = 0;
    // constant tile of ones (any layout: every element is 1) and zero Phi (the padded features stay 0)
    for (int e = threadIdx.x; e < Cfg::ONES_BYTES / 4; e += blockDim.x)
        reinterpret_cast<uint32_t *>(smem + (sOnes - sbase))[e] = 0x3F803F80u;
    for (int e = threadIdx.x; e < Cfg::PHI_BYTES / 16; e += blockDim.x)
        reinterpret_cast<uint4 *>(phi_ptr)[e] = make_uint4(0, 0, 0, 0);
    if (warp == Cfg::MMA_WARP) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    __syncthreads();
    for (int n = threadIdx.x; n < p.k; n += blockDim.x) {
        const int j = p.idx[((size_t)bg * p.T + c) * p.k + n] - c * p.C;
        if (j >= 0 && j < p.C) kept[j] = 1;
        else report(p.err, DEV_ERR_INDEX);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // ones / zero Phi -> tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == Cfg::PRODUCER_WARP) {
        if (lane == 0) {
            bool ok = true;
            int issued = 0;
            mbar_arrive_expect_tx(BAR(B_WK), Cfg::WK_BYTES);
            for (int rr = 0; rr < DH / 64; ++rr) tma_load_3d(sWk + rr * (DF * 128), &map_wk, BAR(B_WK), rr * 64, 0, g);
            for (int u = 0; u < nsub; ++u) {
                const int s = u % Cfg::NS;
                if (u >= Cfg::NS) {
                    ok = mbar_wait(BAR(B_KVEMPTY + s), ((u / Cfg::NS) - 1) & 1, abort_flag);
                    if (!ok) break;
                }
                const uint32_t sK = sStage + s * Cfg::STAGE_BYTES, sV = sK + Cfg::TILE_BYTES;
                const int row = c * p.C + u * 128;
                mbar_arrive_expect_tx(BAR(B_KFULL + s), Cfg::TILE_BYTES);
                for (int rr = 0; rr < DH / 64; ++rr) tma_load_3d(sK + rr * Cfg::REG, &map_k, BAR(B_KFULL + s), rr * 64, row, bg);
                mbar_arrive_expect_tx(BAR(B_VFULL + s), Cfg::TILE_BYTES);
                for (int rr = 0; rr < DH / 64; ++rr) tma_load_3d(sV + rr * Cfg::REG, &map_v, BAR(B_VFULL + s), rr * 64, row, bg);
                issued = u + 1;
            }
            if (!ok) {
                *abort_flag = 1;
                report(p.err, DEV_ERR_TIMEOUT);
                mbar_wait_drain(BAR(B_WK), 0, 100000000ull);
                for (int u = max(0, issued - Cfg::NS); u < issued; ++u) {
                    mbar_wait_drain(BAR(B_KFULL + u % Cfg::NS), (u / Cfg::NS) & 1, 100000000ull);
                    mbar_wait_drain(BAR(B_VFULL + u % Cfg::NS), (u / Cfg::NS) & 1, 100000000ull);
                }
            }
        }
    } else if (warp == Cfg::MMA_WARP) {
        if (lane == 0) {
            constexpr uint32_t ID_Y = idesc_bf16(128, DF, 0, 0);
            constexpr uint32_t ID_S = idesc_bf16(128, DH, 1, 1);   // A = Phi^T (MN-major), B = V (MN-major)
            constexpr uint32_t ID_Z = idesc_bf16(128, 16, 1, 0);   // B = ones (K-major)
            bool ok = mbar_wait(BAR(B_WK), 0, abort_flag);
            // Y for subtile u goes to buffer u&1; the next Y is issued as soon as its K tile is in
            auto issue_y = [&](int u) -> bool {
                const int s = u % Cfg::NS, yb = u & 1;
                if (!mbar_wait(BAR(B_KFULL + s), (u / Cfg::NS) & 1, abort_flag)) return false;
                if (u >= 2 && !mbar_wait(BAR(B_YEMPTY + yb), ((u >> 1) - 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t sK = sStage + s * Cfg::STAGE_BYTES;
                #pragma unroll 1
                for (int kk = 0; kk < DH / 16; ++kk)
                    mma_ss(tmem + Cfg::Y_COL + yb * Cfg::YB, kmajor_desc(sK, kk, Cfg::REG), kmajor_desc(sWk, kk, DF * 128),
                           ID_Y, kk > 0);
                mma_commit(BAR(B_YFULL + yb));
                return true;
            };
            if (ok) ok = issue_y(0);
            for (int u = 0; ok && u < nsub; ++u) {
                const int s = u % Cfg::NS;
                if (u + 1 < nsub) ok = issue_y(u + 1);
                if (ok) ok = mbar_wait(BAR(B_VFULL + s), (u / Cfg::NS) & 1, abort_flag);
                if (ok) ok = mbar_wait(BAR(B_PFULL), u & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t sV = sStage + s * Cfg::STAGE_BYTES + Cfg::TILE_BYTES;
                #pragma unroll 1
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t adesc = sw128_desc(sPhi + kk * 2048, Cfg::REG, 1024);
                    mma_ss(tmem + Cfg::S_COL, adesc, sw128_desc(sV + kk * 2048, Cfg::REG, 1024), ID_S,
                           (u > 0 || kk > 0) ? 1u : 0u);
                    mma_ss(tmem + Cfg::Z_COL, adesc, kmajor_desc(sOnes, kk, 16 * 128), ID_Z, (u > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(BAR(B_PEMPTY));
                mma_commit(BAR(B_KVEMPTY + s));
            }
            if (ok) mma_commit(BAR(B_DONE));
            if (!ok) {
                *abort_flag = 1;
                report(p.err, DEV_ERR_TIMEOUT);
            }
            mma_commit(BAR(B_DRAIN));
            mbar_wait_drain(BAR(B_DRAIN), 0, 100000000ull);
        }
    } else {
        // epilogue warps: row r = token of the subtile (featurise), then row r = feature (write out)
        const int r = warp * 32 + lane;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        bool ok = true;
        for (int u = 0; u < nsub; ++u) {
            const int s = u % Cfg::NS, yb = u & 1;
            ok = warp_all(mbar_wait(BAR(B_YFULL + yb), (u >> 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
            float y[DF];
#pragma unroll
            for (int cc = 0; cc < DF / 32; ++cc) {
                uint32_t uu[32];
                tmem_ld32(tmem + lane_off + Cfg::Y_COL + yb * Cfg::YB + cc * 32, uu);
#pragma unroll
                for (int e = 0; e < 32; ++e) y[cc * 32 + e] = __uint_as_float(uu[e]);
            }
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(BAR(B_YEMPTY + yb));
            // ||k||^2 from the swizzled K tile (still resident: released only after this subtile's MMAs)
            float kk2 = 0.f;
            const uint8_t *krow = smem + (sStage - sbase) + s * Cfg::STAGE_BYTES + r * 128;
#pragma unroll
            for (int rr = 0; rr < DH / 64; ++rr) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint4 v4 = *reinterpret_cast<const uint4 *>(krow + rr * Cfg::REG + ((ch ^ (r & 7)) << 4));
                    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&v4);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(h2[e]);
                        kk2 = fmaf(f.x, f.x, kk2);
                        kk2 = fmaf(f.y, f.y, kk2);
                    }
                }
            }
            float ymax = -INFINITY;
#pragma unroll
            for (int a = 0; a < DF; ++a) ymax = fmaxf(ymax, y[a]);
            float ee = 0.f;
#pragma unroll
            for (int a = 0; a < DF; ++a) {
                y[a] = ex2((y[a] - ymax) * kLog2e);
                ee = fmaf(y[a], y[a], ee);
            }
            const float f = kept[u * 128 + r] ? 0.f : sqrtf(kk2) * rsqrtf(ee);
            // Phi buffer free again (previous subtile's MMAs done)?
            if (u > 0) {
                ok = warp_all(mbar_wait(BAR(B_PEMPTY), (u - 1) & 1, abort_flag));
                if (!ok) break;
            }
#pragma unroll
            for (int rr = 0; rr < DF / 64; ++rr) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    uint4 w;
                    const int a0 = rr * 64 + ch * 8;
                    w.x = pack_bf16x2(y[a0 + 0] * f, y[a0 + 1] * f);
                    w.y = pack_bf16x2(y[a0 + 2] * f, y[a0 + 3] * f);
                    w.z = pack_bf16x2(y[a0 + 4] * f, y[a0 + 5] * f);
                    w.w = pack_bf16x2(y[a0 + 6] * f, y[a0 + 7] * f);
                    *reinterpret_cast<uint4 *>(phi_ptr + rr * Cfg::REG + r * 128 + ((ch ^ (r & 7)) << 4)) = w;
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(BAR(B_PFULL));
        }
        if (ok) ok = warp_all(mbar_wait(BAR(B_DONE), 0, abort_flag));
        if (ok) {
            tc_fence_after();
            // lane = feature a; columns = x (S) and column 0 (z)
            const size_t slot = (size_t)bg * (p.T + 1) + c + p.m + 1;
            float *Srow = p.S + (slot * DF + r) * DH;
#pragma unroll
            for (int cc = 0; cc < DH / 32; ++cc) {
                uint32_t uu[32];
                tmem_ld32(tmem + lane_off + Cfg::S_COL + cc * 32, uu);
                tmem_wait_ld();
                if (r < DF) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4 *>(Srow + cc * 32 + e) =
                            make_float4(__uint_as_float(uu[e]), __uint_as_float(uu[e + 1]), __uint_as_float(uu[e + 2]),
                                        __uint_as_float(uu[e + 3]));
                }
            }
            uint32_t zz[32];
            tmem_ld32(tmem + lane_off + Cfg::Z_COL, zz);
            tmem_wait_ld();
            if (r < DF) p.z[slot * DF + r] = __uint_as_float(zz[0]);
        }
        if (!ok) {
            *abort_flag = 1;
            report(p.err, DEV_ERR_TIMEOUT);
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == Cfg::MMA_WARP) tmem_dealloc(tmem, Cfg::TMEM_COLS);
}

// ------------------------------------------------------------------ small helper kernels
// Wq [H, d, D] -> Wq^T [H, D, d] (bf16), the K-major operand of Y = Q Wq.
__global__ void transpose_wq_kernel(const __nv_bfloat16 *__restrict__ wq, __nv_bfloat16 *__restrict__ wqt, int H,
                                    int d, int D) {
    const size_t n = (size_t)H * d * D;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x) {
        const int h = (int)(e / ((size_t)d * D));
        const int rem = (int)(e % ((size_t)d * D));
        const int c = rem / d, a = rem % d;  // output [h][c][a]
        wqt[e] = wq[((size_t)h * d + a) * D + c];
    }
}

}  // namespace

// ------------------------------------------------------------------ host side
namespace tc {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// bf16 tensor [d2][d1][d0] (d0 innermost), box {64, box1, 1}, 128-byte swizzle, zero fill out of range.
bool make_map(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box1) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || ((uintptr_t)base & 15)) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    cuuint32_t box[3] = {64, box1, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

namespace {

template <int DH, int DF, int HP>
cudaError_t launch_merge_cfg(int mode, const Dims &s, const MergeOperands &a, unsigned *err, cudaStream_t st) {
    using Cfg = MergeCfg<DH, DF, HP>;
    const int T = s.T();
    const int n_qtiles = (s.N + 127) / 128;
    // PREFIX: only the query chunks t > m see a kept prefix or a linear state
    const int qt_first = mode == kMergeLocal ? 0 : std::min(n_qtiles, (s.m() + 1) * s.C / 128);
    if (qt_first >= n_qtiles) return cudaSuccess;
    CUtensorMap mq, mk, mv, mkh, mvh, mw, ms;
    const uint64_t khrows = (uint64_t)T * s.k > 0 ? (uint64_t)T * s.k : 1;
    bool ok = make_map(&mq, a.q, DH, s.N, (uint64_t)s.B * s.H, 128) &&
              make_map(&mk, a.k, DH, s.N, (uint64_t)s.B * s.Hkv, 128) &&
              make_map(&mv, a.v, DH, s.N, (uint64_t)s.B * s.Hkv, 128) &&
              make_map(&mkh, a.khat, DH, khrows, (uint64_t)s.B * s.Hkv, 128) &&
              make_map(&mvh, a.vhat, DH, khrows, (uint64_t)s.B * s.Hkv, 128) &&
              make_map(&mw, a.wqt, DH, DF, s.H, DF) &&
              make_map(&ms, a.st_t, DF, DH, (uint64_t)s.B * s.Hkv * (T + 1), DH);
    if (!ok) return cudaErrorInvalidValue;
    MergeParams prm;
    prm.B = s.B;
    prm.H = s.H;
    prm.Hkv = s.Hkv;
    prm.N = s.N;
    prm.C = s.C;
    prm.k = s.k;
    prm.w = s.w;
    prm.G = s.G();
    prm.T = T;
    prm.scale_log2 = s.scale * kLog2e;
    prm.z = a.z;
    prm.o = static_cast<__nv_bfloat16 *>(a.o);
    prm.lse = a.lse;
    prm.sigma = a.sigma;
    prm.fix_list = a.fix_list;
    prm.fix_count = a.fix_count;
    prm.err = err;
    prm.n_qtiles = n_qtiles;
    prm.qt_first = qt_first;
    prm.pairs = s.G() / HP;
    auto kern = mode == kMergeLocal ? merge_tc_kernel<DH, DF, HP, kMergeExpVariant, kMergeLocal>
                                    : merge_tc_kernel<DH, DF, HP, kMergeExpVariant, kMergePrefix>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)(n_qtiles - qt_first) * s.B * s.Hkv * prm.pairs;
    kern<<<grid, Cfg::THREADS, Cfg::SMEM, st>>>(mq, mk, mv, mkh, mvh, mw, ms, prm);
    return cudaGetLastError();
}

}  // namespace


bool tc_merge_supported(const Dims &s) {
    return s.bf16 && s.w > 0 && (s.d == 64 || s.d == 128) && (s.D == 64 || s.D == 128) && s.C % 128 == 0 &&
           s.N > 0 && encode_fn() != nullptr;
}

// W [Hx, d, D] -> W^T [Hx, D, d] (bf16).
cudaError_t launch_w_transpose(int Hx, int d, int D, const void *w, void *wt, cudaStream_t st) {
    const size_t n = (size_t)Hx * d * D;
    const unsigned blocks = (unsigned)std::min<size_t>((n + 255) / 256, 4096);
    transpose_wq_kernel<<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16 *>(w), static_cast<__nv_bfloat16 *>(wt),
                                                 Hx, d, D);
    return cudaGetLastError();
}

bool tc_linear_supported(const Dims &s) {
    return s.bf16 && s.w > 0 && (s.d == 64 || s.d == 128) && (s.D == 64 || s.D == 128) && s.C % 128 == 0 &&
           s.C <= 1024 && encode_fn() != nullptr;
}

template <int DH, int DF>
static cudaError_t launch_linear_cfg(const Dims &s, const void *k, const void *v, const void *wkt,
                                     const int32_t *idx, float *S, float *z, unsigned *err, cudaStream_t st) {
    using Cfg = LinCfg<DH, DF>;
    const int nc = s.T() - s.m();
    if (nc <= 0 || s.B * s.Hkv == 0) return cudaSuccess;
    CUtensorMap mk, mv, mw;
    if (!make_map(&mk, k, DH, s.N, (uint64_t)s.B * s.Hkv, 128) || !make_map(&mv, v, DH, s.N, (uint64_t)s.B * s.Hkv, 128) ||
        !make_map(&mw, wkt, DH, DF, s.Hkv, DF))
        return cudaErrorInvalidValue;
    LinParams prm;
    prm.B = s.B;
    prm.Hkv = s.Hkv;
    prm.N = s.N;
    prm.C = s.C;
    prm.k = s.k;
    prm.m = s.m();
    prm.T = s.T();
    prm.idx = idx;
    prm.S = S;
    prm.z = z;
    prm.err = err;
    auto kern = linear_state_tc_kernel<DH, DF>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(s.B * s.Hkv * nc), Cfg::THREADS, Cfg::SMEM, st>>>(mk, mv, mw, prm);
    return cudaGetLastError();
}

// Delta S / Delta z of every chunk into slot c+m+1 (the prefix kernel finishes S_t, z_t).
cudaError_t launch_linear_tc(const Dims &s, const void *k, const void *v, const void *wkt, const int32_t *idx,
                             float *S, float *z, unsigned *err, cudaStream_t st) {
#define STILL_LIN_CASE(DH, DF) \
    if (s.d == DH && s.D == DF) return launch_linear_cfg<DH, DF>(s, k, v, wkt, idx, S, z, err, st);
    STILL_LIN_CASE(64, 64)
    STILL_LIN_CASE(128, 128)
    STILL_LIN_CASE(64, 128)
    STILL_LIN_CASE(128, 64)
#undef STILL_LIN_CASE
    return cudaErrorNotSupported;
}

cudaError_t launch_merge_ring(int mode, const Dims &s, const MergeOperands &a, unsigned *err, cudaStream_t st);

// mode 0: window part + Self-Saliency Score (writes o_A, lse_A, sigma); mode 1: kept prefix + linear
// branch folded with the window part (writes o).  Head dimension 64 runs the persistent ring-scheduled
// kernel (merge_ring.cu), 128 the kernel above.
cudaError_t launch_merge_tc(int mode, const Dims &s, const MergeOperands &a, unsigned *err, cudaStream_t st) {
    if (s.d == 64) return launch_merge_ring(mode, s, a, err, st);
    const bool pair = s.G() % 2 == 0;
    if (s.d == 128 && s.D == 128)
        return pair ? launch_merge_cfg<128, 128, 2>(mode, s, a, err, st) : launch_merge_cfg<128, 128, 1>(mode, s, a, err, st);
    if (s.d == 128 && s.D == 64)
        return pair ? launch_merge_cfg<128, 64, 2>(mode, s, a, err, st) : launch_merge_cfg<128, 64, 1>(mode, s, a, err, st);
    return cudaErrorNotSupported;
}

bool tc_saliency_supported(const Dims &s) {
    return s.bf16 && s.w > 0 && (s.d == 64 || s.d == 128) && s.w % 128 == 0 && s.N > 0 && encode_fn() != nullptr;
}

template <int DH, int HP>
static cudaError_t launch_saliency_cfg(const Dims &s, const void *q, const void *k, float *r_kv, float *sigma,
                                       unsigned *err, cudaStream_t st) {
    using Cfg = SalCfg<DH, HP>;
    CUtensorMap mq, mk;
    if (!make_map(&mq, q, DH, s.N, (uint64_t)s.B * s.H, 128) || !make_map(&mk, k, DH, s.N, (uint64_t)s.B * s.Hkv, 128))
        return cudaErrorInvalidValue;
    SalParams prm;
    prm.B = s.B;
    prm.H = s.H;
    prm.Hkv = s.Hkv;
    prm.N = s.N;
    prm.w = s.w;
    prm.G = s.G();
    prm.pairs = s.G() / HP;
    prm.n_qtiles = (s.N + 127) / 128;
    prm.scale_log2 = s.scale * kLog2e;
    prm.sigma = sigma;
    prm.r_kv = r_kv;
    prm.err = err;
    auto kern = saliency_tc_kernel<DH, HP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)prm.n_qtiles * s.B * s.Hkv * prm.pairs;
    kern<<<grid, Cfg::THREADS, Cfg::SMEM, st>>>(mq, mk, prm);
    return cudaGetLastError();
}

// Self-Saliency Score of the rows listed by the window kernel, recomputed with the band's own maximum
// (one warp per row, lanes split the band keys; same definition as the window kernel:
// sigma = softplus(s_ii - LSE_{j in [i-w+1, i-1]} s_ij)).
template <int DH>
__global__ void __launch_bounds__(128) saliency_fixup_kernel(const __nv_bfloat16 *__restrict__ q,
                                                             const __nv_bfloat16 *__restrict__ k,
                                                             const int *__restrict__ list,
                                                             const unsigned *__restrict__ count, float *sigma, int H,
                                                             int Hkv, int N, int w, float scale) {
    __shared__ __align__(16) float qs[4][DH];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned n = *count;
    for (unsigned e = blockIdx.x * 4 + warp; e < n; e += gridDim.x * 4) {
        const size_t row = (size_t)list[e];
        const int i = (int)(row % N);
        const size_t bh = row / N;
        const int h = (int)(bh % H), b = (int)(bh / H), g = h / (H / Hkv);
        const __nv_bfloat16 *kg = k + ((size_t)b * Hkv + g) * N * DH;
        for (int x = lane; x < DH; x += 32) qs[warp][x] = __bfloat162float(q[row * DH + x]);
        __syncwarp();
        const int lo = max(0, i - w + 1);
        float mx = -INFINITY, sm = 0.f;
        // one band key per lane and step; the key row's DH/8 loads are all issued before its dot product
#pragma unroll 2
        for (int j = lo + lane; j < i; j += 32) {
            const uint4 *kr = reinterpret_cast<const uint4 *>(kg + (size_t)j * DH);
            uint4 u[DH / 8];
#pragma unroll
            for (int x8 = 0; x8 < DH / 8; ++x8) u[x8] = __ldg(kr + x8);
            float acc = 0.f;
#pragma unroll
            for (int x8 = 0; x8 < DH / 8; ++x8) {
                const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u[x8]);
#pragma unroll
                for (int e2 = 0; e2 < 4; ++e2) {
                    const float2 f = __bfloat1622float2(h2[e2]);
                    acc = fmaf(qs[warp][8 * x8 + 2 * e2], f.x, acc);
                    acc = fmaf(qs[warp][8 * x8 + 2 * e2 + 1], f.y, acc);
                }
            }
            const float l = scale * acc;
            if (l > mx) {
                sm = sm * expf(mx - l) + 1.f;
                mx = l;
            } else {
                sm += expf(l - mx);
            }
        }
        const float M = warp_max(mx);
        const float Z = warp_sum(mx == -INFINITY ? 0.f : sm * expf(mx - M));
        float dp = 0.f;
        for (int x = lane; x < DH; x += 32) dp = fmaf(qs[warp][x], __bfloat162float(kg[(size_t)i * DH + x]), dp);
        const float sii = scale * warp_sum(dp);
        if (lane == 0) sigma[row] = (i == lo) ? INFINITY : softplus_f(sii - (M + logf(Z)));
        __syncwarp();
    }
}

cudaError_t launch_saliency_fixup(const Dims &s, const void *q, const void *k, const int *list, const unsigned *count,
                                  float *sigma, cudaStream_t st) {
    const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(q), *kb = static_cast<const __nv_bfloat16 *>(k);
    if (s.d == 64)
        saliency_fixup_kernel<64><<<148, 128, 0, st>>>(qb, kb, list, count, sigma, s.H, s.Hkv, s.N, s.w, s.scale);
    else if (s.d == 128)
        saliency_fixup_kernel<128><<<148, 128, 0, st>>>(qb, kb, list, count, sigma, s.H, s.Hkv, s.N, s.w, s.scale);
    else
        return cudaErrorNotSupported;
    return cudaGetLastError();
}

cudaError_t launch_mean_heads(const Dims &s, const float *sigma, float *r, cudaStream_t st) {
    const size_t total = (size_t)s.B * s.Hkv * s.N;
    if (total == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)std::min<size_t>((total + 255) / 256, 8192);
    mean_heads_kernel<<<blocks, 256, 0, st>>>(sigma, r, s.B, s.H, s.Hkv, s.N);
    return cudaGetLastError();
}

// r_kv: [B,Hkv,N]; sigma: [B,H,N] per-head scores (may be nullptr only when G <= 2, where one CTA
// holds the whole group and writes the mean itself).
cudaError_t launch_saliency_tc(const Dims &s, const void *q, const void *k, float *r_kv, float *sigma, unsigned *err,
                               cudaStream_t st) {
    const bool pair = s.G() % 2 == 0;
    if (!sigma && s.G() > 2) return cudaErrorInvalidValue;
    cudaError_t e;
    if (s.d == 64)
        e = pair ? launch_saliency_cfg<64, 2>(s, q, k, r_kv, sigma, err, st)
                 : launch_saliency_cfg<64, 1>(s, q, k, r_kv, sigma, err, st);
    else
        e = pair ? launch_saliency_cfg<128, 2>(s, q, k, r_kv, sigma, err, st)
                 : launch_saliency_cfg<128, 1>(s, q, k, r_kv, sigma, err, st);
    if (e != cudaSuccess) return e;
    if (s.G() <= 2) return cudaSuccess;  // the kernel wrote the group mean
    const size_t total = (size_t)s.B * s.Hkv * s.N;
    const unsigned blocks = (unsigned)std::min<size_t>((total + 255) / 256, 8192);
    mean_heads_kernel<<<blocks, 256, 0, st>>>(sigma, r_kv, s.B, s.H, s.Hkv, s.N);
    return cudaGetLastError();
}

}  // namespace still
