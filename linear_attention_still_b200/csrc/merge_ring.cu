// merge_ring.cu -- the hybrid merge of "STILL: Selecting Tokens for Intra-Layer Hybrid Attention to
// Linearize LLMs" at head dimension 64 on sm_100a ([p1] jsqmd.com introduction: kept tokens go to
// softmax attention and the rest to linear attention in the same layer, under one shared distribution;
// [p4] atlas.scime.ai "Approach").  Same arithmetic and the same two phases as the head-dim-128 merge
// in kernels_tc.cu; what differs is the schedule:
//
// * Persistent CTAs.  The grid holds one CTA per SM; each walks work items (b, g, head pair, 128
//   queries of one chunk), heaviest query tiles first, CTA c taking items c, c + grid, ...  The producer
//   loads the next item's query tiles (double-buffered) while the current item computes, and the MMA
//   warp issues the next item's first score tile while the softmax warps run the current epilogue.
// * Scores, probabilities and output in separate TMEM columns per head: S (128 fp32 columns, one
//   N = 128 MMA per k-step at a 128-column boundary), P (128 keys as bf16 pairs, 64 columns) and O (64):
//   2 x (128 + 64 + 64) = 512 columns.  The next tile's scores are issued as soon as the softmax has
//   read S; the softmax computes a tile's exponentials into registers and only then waits for the P V
//   product that still reads the previous P (issued a whole exponential phase earlier, so normally
//   done), rescales O if its max moved, and stores P.
// * The two softmax warpgroups take turns on the exponential phase, handing it over through named CTA
//   barriers (bar.sync / bar.arrive), so a waiting warpgroup sleeps in hardware instead of spinning on
//   an mbarrier next to the warps that hold the MUFU unit.  A named barrier has no time limit: a warp
//   that leaves on a timeout sets the abort flag and arrives once on each hand-over barrier, and every
//   warp tests the flag before it sleeps, so no warp is left waiting for a partner that has gone.
//
// Per row (TMEM lane = query row), as in the head-dim-128 kernel:
//   window phase (kMergeLocal): keys [max(0,(t-m)C), i]; also the Self-Saliency Score of every row
//     ([p1] "Self-Saliency Score") from the same exponentials; writes o_A, lse_A (log2) and sigma;
//   prefix phase (kMergePrefix): prologue Y = Q Wq^T -> phi(q) = ||q|| e/||e||, O := phi(q) S_t^T,
//     b := phi(q).z_t, folded with o_A under one normaliser ([p1] "NP-Map"); then the kept rows of the
//     decided chunks ([p1] "Chunk-Wise parallel + delayed selection").
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

template <int DF, int HP, int NH>
struct RingCfg {
    // NH = 2: two independent single-head pipelines (halves) in one CTA, each with its own item stream,
    // query / key / value buffers, barriers and 256 TMEM columns (see the file comment)
    static_assert(NH == 1 || (NH == 2 && HP == 1 && DF == 64), "two halves run one head each, D = 64");
    static constexpr int DH = 64;
    static constexpr int BN = 128;                       // keys per tile
    static constexpr int TILE_BYTES = 128 * 128;         // 128 rows x 64 bf16: one SW128 region
    static constexpr int Q_BYTES = HP * TILE_BYTES;      // one item's query tiles
    static constexpr int NQ = 2;                         // query buffers
    static constexpr int NS = NH == 2 ? 2 : (DF == 64 ? 4 : 3);  // K/V stages
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;   // K + V
    static constexpr int WQ_BYTES = DF * DH * 2;         // Wq^T of one head: DF rows x 64
    static constexpr int ST_BYTES = DH * DF * 2;         // S_t^T: 64 rows x DF
    static constexpr int W_BYTES = HP * WQ_BYTES + ST_BYTES;
    static constexpr int BAR_BYTES = NH == 2 ? 256 : 512;  // per half
    static constexpr int HALF_BYTES = NQ * Q_BYTES + NS * STAGE_BYTES + W_BYTES;  // one half's operands
    static_assert(HALF_BYTES % 1024 == 0, "tiles stay on 1024-byte boundaries");
    static constexpr int SMEM = NH * HALF_BYTES + NH * BAR_BYTES + 1024;
    static_assert(SMEM <= 232448, "shared memory");
    static constexpr int SOFTMAX_WARPS = 4 * HP * NH;
    static constexpr int THREADS = SOFTMAX_WARPS == 8 ? 384 : 192;
    // warps after the softmax warps: per half a TMA producer warp and an MMA warp (half 0's below)
    static constexpr int PRODUCER_WARP = SOFTMAX_WARPS, MMA_WARP = SOFTMAX_WARPS + 1;
    // launch budget 384 x 168 = 64512 registers = 2 x 128 x 208 (softmax) + 128 x 88 (the rest)
    static constexpr int REG_SOFTMAX = 208, REG_OTHER = 88;
    static_assert(THREADS != 384 || 2 * 128 * REG_SOFTMAX + 128 * REG_OTHER <= THREADS * 168, "register split");
    static constexpr int TMEM_COLS = THREADS == 384 ? 512 : 256;
    static constexpr uint32_t HALF_COLS = 256u * HP;  // TMEM columns of one half
    __host__ __device__ static constexpr uint32_t s_col(int x) { return 128u * x; }
    __host__ __device__ static constexpr uint32_t p_col(int x) { return 128u * HP + 64u * x; }
    __host__ __device__ static constexpr uint32_t o_col(int x) { return 192u * HP + 64u * x; }
    static_assert(NH * 256 * HP <= TMEM_COLS, "TMEM budget");
    // barrier slots
    static constexpr int B_QFULL = 0, B_QEMPTY = 2, B_WFULL = 4, B_WEMPTY = 5, B_PRO = 6, B_DRAIN = 7;
    static constexpr int B_KFULL = 8, B_VFULL = 8 + NS, B_KVEMPTY = 8 + 2 * NS;
    static constexpr int B_Y = 8 + 3 * NS, B_PHI = B_Y + HP, B_S = B_PHI + HP, B_SFREE = B_S + HP,
                         B_O = B_SFREE + HP, B_P = B_O + HP;  // B_P: [2 * HP], tile parity fastest
    static constexpr int B_TURN = B_P + 2 * HP;                      // [2]: exponential-phase turns
    static constexpr int NUM_BARS = B_TURN + 2;
    static constexpr int TMEM_SLOT_OFF = 8 * NUM_BARS;
    static constexpr int ABORT_OFF = TMEM_SLOT_OFF + 8;
    static_assert(ABORT_OFF + 8 <= BAR_BYTES, "barrier area overflow");
};

struct RingParams {
    int B, H, Hkv, N, C, k, w, G, T;
    float scale_log2;      // tau * log2(e)
    const float *z;        // [B*Hkv*(T+1), DF] fp32
    __nv_bfloat16 *o;      // [B,H,N,64]: window part (normalised) after LOCAL, final output after PREFIX
    float *lse;            // [B,H,N]: log2-sum-exp of the window part (LOCAL writes, PREFIX reads and
                           // replaces it with the row's whole log2 normaliser)
    float *sigma;          // [B,H,N]: Self-Saliency Score per query head (LOCAL writes)
    int *fix_list;         // rows whose band sum underflowed against the window max (recomputed later)
    unsigned *fix_count;
    unsigned *err;
    int n_qtiles;          // ceil(N/128)
    int n_items;           // (n_qtiles - qt_first) x B x Hkv x pairs
    int pairs;             // G / HP
    int stall;             // test hook: CTA 0's producer issues no key/value tile (its consumers time out)
};

// Work item `it` (heaviest query tiles first).
struct Item {
    int b, bg, h0, i0, t, lo, nk, n_tiles, tslot;
};

template <int HP, bool LOCAL>
__device__ __forceinline__ Item item_of(int it, const RingParams &p) {
    Item I;
    const int per_qt = p.B * p.Hkv * p.pairs;
    const int qt = p.n_qtiles - 1 - it / per_qt;
    const int rem = it % per_qt;
    const int pair = rem % p.pairs;
    I.bg = rem / p.pairs;
    I.b = I.bg / p.Hkv;
    const int g = I.bg % p.Hkv;
    I.h0 = g * p.G + pair * HP;
    I.i0 = qt * 128;
    I.t = I.i0 / p.C;
    const int m = p.w / p.C;
    I.nk = p.k * max(0, I.t - m);                 // kept rows seen by this chunk
    I.lo = max(0, (I.t - m) * p.C);               // window start
    I.n_tiles = LOCAL ? (I.i0 - I.lo) / 128 + 1 : (I.nk + 127) / 128;
    I.tslot = I.bg * (p.T + 1) + I.t;             // linear state slot
    return I;
}

// Where the exponentials run (see exp_row): the window phase keeps every exponential on the MUFU unit;
// the kept-prefix phase sends the last 32 keys of each row to the FMA pipe.  Measured on B200 (1B 16K
// layer, ms per phase, window / prefix): all on MUFU 0.232 / 0.291, a quarter on FMA 0.243 / 0.273.
#ifndef STILL_RING_EXP_LOCAL
#define STILL_RING_EXP_LOCAL 1
#endif
#ifndef STILL_RING_EXP_PREFIX
#define STILL_RING_EXP_PREFIX 2
#endif
constexpr int kRingExpLocal = STILL_RING_EXP_LOCAL, kRingExpPrefix = STILL_RING_EXP_PREFIX;
// Two heads per CTA: the softmax warpgroups take turns on the exponential phase of each tile (head 0,
// head 1, head 0, ...), so one warpgroup's row bookkeeping (TMEM read of S, row max, P store) overlaps
// the other's exponentials instead of both leaving the MUFU unit idle at the same time.  Hand-over
// forms: 0 none (both exponentiate at once), 1 an mbarrier tested in a spin loop, 3 named CTA barriers
// (bar.sync / bar.arrive: the waiting warps sleep in hardware and take no issue slots).  Measured on
// B200 (1B 16K layer, both phases): 1 -> 3 0.492 -> 0.475 ms; 0 was 5 % slower than 1.
#ifndef STILL_RING_TURNS
#define STILL_RING_TURNS 3
#endif
constexpr int kRingTurns = STILL_RING_TURNS;
// D = 64: two independent single-head halves per CTA (1) or one two-head pipeline (0).
#ifndef STILL_RING_HALVES
#define STILL_RING_HALVES 0
#endif
constexpr bool kRingHalves = STILL_RING_HALVES != 0;
static_assert(kRingTurns == 0 || kRingTurns == 1 || kRingTurns == 3, "hand-over form");


template <int DF, int HP, int NH, int EXPV, int MODE>
__global__ void __launch_bounds__(RingCfg<DF, HP, NH>::THREADS, 1)
    merge_ring_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_kh,
                      const __grid_constant__ CUtensorMap map_vh, const __grid_constant__ CUtensorMap map_wq,
                      const __grid_constant__ CUtensorMap map_st, const RingParams p) {
    using Cfg = RingCfg<DF, HP, NH>;
    constexpr bool LOCAL = MODE == 0;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem0 = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the half this warp serves: softmax warps by warpgroup, then (producer, MMA) pairs per half
    const int half = warp < Cfg::SOFTMAX_WARPS ? warp / (4 * HP) : min((warp - Cfg::SOFTMAX_WARPS) >> 1, NH - 1);
    uint8_t *smem = smem0 + half * Cfg::HALF_BYTES;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase;                                      // NQ x HP query tiles
    const uint32_t sStage = sQ + Cfg::NQ * Cfg::Q_BYTES;            // NS x (K tile, V tile)
    const uint32_t sW = sStage + Cfg::NS * Cfg::STAGE_BYTES;        // HP x Wq^T, then S_t^T
    uint8_t *bar_area0 = smem0 + NH * Cfg::HALF_BYTES;  // half 0's barriers, the TMEM slot and abort flag
    const uint32_t sBar = smem_u32(bar_area0 + half * Cfg::BAR_BYTES);
    auto BAR = [&](int i) { return sBar + 8u * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_area0 + Cfg::TMEM_SLOT_OFF);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bar_area0 + Cfg::ABORT_OFF);
    // work items of this half: ifirst, ifirst + istep, ...
    const int ifirst = (int)blockIdx.x * NH + half, istep = (int)gridDim.x * NH;

    if (threadIdx.x == 0) {
        for (int hh = 0; hh < NH; ++hh) {
            const uint32_t hb = smem_u32(bar_area0 + hh * Cfg::BAR_BYTES);
            auto BAR = [&](int i) { return hb + 8u * i; };
            for (int e = 0; e < 2; ++e) {
                mbar_init(BAR(Cfg::B_QFULL + e), 1);
                mbar_init(BAR(Cfg::B_QEMPTY + e), LOCAL ? 1 : 1 + 128 * HP);  // MMA commit (+ the softmax's ||q|| read)
            }
            mbar_init(BAR(Cfg::B_WFULL), 1);
            mbar_init(BAR(Cfg::B_WEMPTY), 1);
            mbar_init(BAR(Cfg::B_PRO), 1);
            mbar_init(BAR(Cfg::B_DRAIN), 1);
            for (int s = 0; s < Cfg::NS; ++s) {
                mbar_init(BAR(Cfg::B_KFULL + s), 1);
                mbar_init(BAR(Cfg::B_VFULL + s), 1);
                mbar_init(BAR(Cfg::B_KVEMPTY + s), 1);
            }
            for (int x = 0; x < HP; ++x) {
                mbar_init(BAR(Cfg::B_Y + x), 1);
                mbar_init(BAR(Cfg::B_PHI + x), 128);
                mbar_init(BAR(Cfg::B_S + x), 1);
                mbar_init(BAR(Cfg::B_SFREE + x), 128);
                mbar_init(BAR(Cfg::B_O + x), 1);
                mbar_init(BAR(Cfg::B_P + 2 * x), 128);
                mbar_init(BAR(Cfg::B_P + 2 * x + 1), 128);
            }
            mbar_init(BAR(Cfg::B_TURN + 0), 128);
            mbar_init(BAR(Cfg::B_TURN + 1), 128);
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
        tma_prefetch_desc(LOCAL ? &map_k : &map_kh);
        tma_prefetch_desc(LOCAL ? &map_v : &map_vh);
        if (!LOCAL) {
            tma_prefetch_desc(&map_wq);
            tma_prefetch_desc(&map_st);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem0 = *tmem_slot;
    const uint32_t tmem = tmem0 + half * Cfg::HALF_COLS;  // this half's columns

    if (warp >= Cfg::SOFTMAX_WARPS) {
        if (Cfg::THREADS == 384) setmaxnreg_dec<Cfg::REG_OTHER>();
        const int role = warp - Cfg::SOFTMAX_WARPS - 2 * half;  // 0 producer, 1 MMA issuer, else idle
        if (role == 0) {
            // (the whole warp runs the issue loop; one elected lane issues each copy)
            // ================================================================ TMA producer
            bool ok = true, stalled = false;
            int G = 0, n = 0, nq = 0, nw = 0;  // K/V tiles, items, query loads, W loads issued
            for (int it = ifirst; ok && !stalled && it < p.n_items; it += istep, ++n) {
                const Item I = item_of<HP, LOCAL>(it, p);
                const int qb = n & 1;
                if (n >= 2 && !(ok = mbar_wait_w(BAR(Cfg::B_QEMPTY + qb), ((n >> 1) - 1) & 1, abort_flag))) break;
                mbar_arrive_expect_tx_w(BAR(Cfg::B_QFULL + qb), Cfg::Q_BYTES);
                for (int x = 0; x < HP; ++x)
                    tma_load_3d_w(sQ + qb * Cfg::Q_BYTES + x * Cfg::TILE_BYTES, &map_q, BAR(Cfg::B_QFULL + qb), 0, I.i0,
                                I.b * p.H + I.h0 + x);
                nq = n + 1;
                if (!LOCAL) {
                    if (n >= 1 && !(ok = mbar_wait_w(BAR(Cfg::B_WEMPTY), (n - 1) & 1, abort_flag))) break;
                    mbar_arrive_expect_tx_w(BAR(Cfg::B_WFULL), Cfg::W_BYTES);
                    for (int x = 0; x < HP; ++x)
                        tma_load_3d_w(sW + x * Cfg::WQ_BYTES, &map_wq, BAR(Cfg::B_WFULL), 0, 0, I.h0 + x);
                    for (int rr = 0; rr < DF / 64; ++rr)
                        tma_load_3d_w(sW + HP * Cfg::WQ_BYTES + rr * (64 * 128), &map_st, BAR(Cfg::B_WFULL), rr * 64, 0,
                                    I.tslot);
                    nw = n + 1;
                }
                if (p.stall && blockIdx.x == 0) {
                    stalled = true;  // no key/value tile: the MMA warp's bounded wait runs out
                    break;
                }
                for (int jj = 0; jj < I.n_tiles; ++jj, ++G) {
                    const int s = G % Cfg::NS;
                    if (G >= Cfg::NS && !(ok = mbar_wait_w(BAR(Cfg::B_KVEMPTY + s), ((G / Cfg::NS) - 1) & 1, abort_flag)))
                        break;
                    const uint32_t sK = sStage + s * Cfg::STAGE_BYTES, sV = sK + Cfg::TILE_BYTES;
                    const int row = LOCAL ? I.lo + jj * Cfg::BN : jj * Cfg::BN;
                    mbar_arrive_expect_tx_w(BAR(Cfg::B_KFULL + s), Cfg::TILE_BYTES);
                    tma_load_3d_w(sK, LOCAL ? &map_k : &map_kh, BAR(Cfg::B_KFULL + s), 0, row, I.bg);
                    mbar_arrive_expect_tx_w(BAR(Cfg::B_VFULL + s), Cfg::TILE_BYTES);
                    tma_load_3d_w(sV, LOCAL ? &map_v : &map_vh, BAR(Cfg::B_VFULL + s), 0, row, I.bg);
                }
            }
            if (!ok) {
                *abort_flag = 1;
                if (lane == 0) report(p.err, DEV_ERR_TIMEOUT);
            }
            if (!ok || stalled) {
                // drain this CTA's copies still in flight
                for (int u = max(0, nq - 2); u < nq; ++u)
                    mbar_wait_drain(BAR(Cfg::B_QFULL + (u & 1)), (u >> 1) & 1, 100000000ull);
                if (nw > 0) mbar_wait_drain(BAR(Cfg::B_WFULL), (nw - 1) & 1, 100000000ull);
                for (int u = max(0, G - Cfg::NS); u < G; ++u) {
                    mbar_wait_drain(BAR(Cfg::B_KFULL + u % Cfg::NS), (u / Cfg::NS) & 1, 100000000ull);
                    mbar_wait_drain(BAR(Cfg::B_VFULL + u % Cfg::NS), (u / Cfg::NS) & 1, 100000000ull);
                }
            }
        } else if (role == 1) {
            // (the whole warp runs the issue loop; one elected lane issues each MMA and commit)
            const uint32_t tmem_w = __shfl_sync(0xffffffffu, tmem, 0);
            // ================================================================ MMA issuer
            constexpr uint32_t ID_N128 = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t ID_N64 = idesc_bf16(128, 64, 0, 0);
            constexpr uint32_t ID_PV = idesc_bf16(128, 64, 0, 1);
            bool ok = true;
            int J = 0, G = 0, n = 0;
            // K-major k-step kk of a 64-column tile: 32 bytes per step inside the 128-byte row
            auto kstep = [](int kk) -> uint64_t { return (uint64_t)((kk * 32) >> 4); };
            // D[128 x nrows] = A[128 x 64] B[nrows x 64]^T into the score columns of head x (nrows = 128:
            // scores of a key tile; nrows = DF: Y = Q Wq^T of the prologue)
            auto issue_qk = [&](int x, uint64_t da, uint32_t sB, int nrows) {
                const uint64_t db = sw128_desc(sB, 16, 1024);
                const uint32_t id = nrows == 64 ? ID_N64 : ID_N128;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) mma_ss_w(tmem_w + Cfg::s_col(x), da + kstep(kk), db + kstep(kk), id, kk > 0);
            };
            // The first MMA of an item that writes the score columns (LOCAL: the scores of its first key
            // tile; PREFIX: Y = Q Wq^T) is issued during the previous item's last tile, right after the
            // softmax has read that tile's scores, so it is ready when the softmax leaves the epilogue.
            // `pre` marks an item whose first MMA was issued that way.
            auto issue_head = [&](const Item &In, int nn, int Jn, int Gn) -> bool {
                const int qbn = nn & 1;
                if (!mbar_wait_w(BAR(Cfg::B_QFULL + qbn), (nn >> 1) & 1, abort_flag)) return false;
                if (!LOCAL && !mbar_wait_w(BAR(Cfg::B_WFULL), nn & 1, abort_flag)) return false;
                if (LOCAL && !mbar_wait_w(BAR(Cfg::B_KFULL + Gn % Cfg::NS), (Gn / Cfg::NS) & 1, abort_flag)) return false;
                for (int x = 0; x < HP; ++x) {
                    // the score columns: the softmax has read tile Jn-1
                    if (Jn > 0 && !mbar_wait_w(BAR(Cfg::B_SFREE + x), (Jn - 1) & 1, abort_flag)) return false;
                    tc_fence_after();
                    const uint64_t dqn = sw128_desc(sQ + qbn * Cfg::Q_BYTES + x * Cfg::TILE_BYTES, 16, 1024);
                    if (LOCAL) {
                        issue_qk(x, dqn, sStage + (Gn % Cfg::NS) * Cfg::STAGE_BYTES, 128);
                        mma_commit_w(BAR(Cfg::B_S + x));
                    } else {
                        issue_qk(x, dqn, sW + x * Cfg::WQ_BYTES, DF);
                        mma_commit_w(BAR(Cfg::B_Y + x));
                    }
                }
                return true;
            };
            bool pre = false;
            for (int it = ifirst; ok && it < p.n_items; it += istep, ++n) {
                const Item I = item_of<HP, LOCAL>(it, p);
                const int qb = n & 1;
                uint64_t dq[HP];
#pragma unroll
                for (int x = 0; x < HP; ++x) dq[x] = sw128_desc(sQ + qb * Cfg::Q_BYTES + x * Cfg::TILE_BYTES, 16, 1024);
                if (!pre && (LOCAL ? I.n_tiles > 0 : true) && !(ok = issue_head(I, n, J, G))) break;
                pre = false;
                if (!LOCAL) {
                    // prologue: Y (issued above or ahead) -> phi(q) (bf16) over the score columns ->
                    // O := phi(q) S_t^T -> the scores of the first kept tile
                    const uint32_t sST = sW + HP * Cfg::WQ_BYTES;
                    for (int x = 0; ok && x < HP; ++x) {
                        if (!(ok = mbar_wait_w(BAR(Cfg::B_PHI + x), n & 1, abort_flag))) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < DF / 16; ++kk)
                            mma_ts_w(tmem_w + Cfg::o_col(x), tmem_w + Cfg::s_col(x) + kk * 8,
                                   kmajor_desc(sST, kk, 64 * 128), ID_N64, kk > 0);
                    }
                    if (!ok) break;
                    mma_commit_w(BAR(Cfg::B_PRO));
                    mma_commit_w(BAR(Cfg::B_WEMPTY));
                    if (I.n_tiles > 0) {
                        if (!(ok = mbar_wait_w(BAR(Cfg::B_KFULL + G % Cfg::NS), (G / Cfg::NS) & 1, abort_flag))) break;
                        tc_fence_after();
                        for (int x = 0; x < HP; ++x) {
                            issue_qk(x, dq[x], sStage + (G % Cfg::NS) * Cfg::STAGE_BYTES, 128);
                            mma_commit_w(BAR(Cfg::B_S + x));
                        }
                    }
                }
                const bool has_next = it + istep < p.n_items;
                for (int jj = 0; ok && jj < I.n_tiles; ++jj, ++G) {
                    const int Jt = J + jj, s = G % Cfg::NS, s1 = (G + 1) % Cfg::NS;
                    // next scores first: they only need the softmax to have read S(Jt)
                    if (jj + 1 < I.n_tiles) {
                        for (int x = 0; x < HP; ++x) {
                            if (x == 0 && !(ok = mbar_wait_w(BAR(Cfg::B_KFULL + s1), ((G + 1) / Cfg::NS) & 1, abort_flag)))
                                break;
                            if (!(ok = mbar_wait_w(BAR(Cfg::B_SFREE + x), Jt & 1, abort_flag))) break;
                            tc_fence_after();
                            issue_qk(x, dq[x], sStage + s1 * Cfg::STAGE_BYTES, 128);
                            mma_commit_w(BAR(Cfg::B_S + x));
                        }
                        if (!ok) break;
                    } else if (has_next) {
                        // last tile: the next item's first score-column MMA goes ahead of this P V
                        const Item In = item_of<HP, LOCAL>(it + istep, p);
                        if (!(ok = issue_head(In, n + 1, Jt + 1, G + 1))) break;
                        pre = true;
                    }
                    const uint64_t dv = sw128_desc(sStage + s * Cfg::STAGE_BYTES + Cfg::TILE_BYTES, Cfg::TILE_BYTES, 1024);
                    for (int x = 0; x < HP; ++x) {
                        if (x == 0 && !(ok = mbar_wait_w(BAR(Cfg::B_VFULL + s), (G / Cfg::NS) & 1, abort_flag))) break;
                        if (!(ok = mbar_wait_w(BAR(Cfg::B_P + 2 * x + (Jt & 1)), (Jt >> 1) & 1, abort_flag))) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)  // 16 keys = 16 rows of V per k-step
                            mma_ts_w(tmem_w + Cfg::o_col(x), tmem_w + Cfg::p_col(x) + kk * 8,
                                   dv + (uint64_t)(kk * 128), ID_PV, (LOCAL && jj == 0 && kk == 0) ? 0u : 1u);
                        mma_commit_w(BAR(Cfg::B_O + x));
                    }
                    if (!ok) break;
                    mma_commit_w(BAR(Cfg::B_KVEMPTY + s));
                }
                if (!ok) break;
                mma_commit_w(BAR(Cfg::B_QEMPTY + qb));
                J += I.n_tiles;
            }
            if (!ok) {
                *abort_flag = 1;
                if (lane == 0) report(p.err, DEV_ERR_TIMEOUT);
            }
            // drain every MMA this thread issued before TMEM is released
            mma_commit_w(BAR(Cfg::B_DRAIN));
            mbar_wait_drain(BAR(Cfg::B_DRAIN), 0, 100000000ull);
        }
    } else {
        if (Cfg::THREADS == 384) setmaxnreg_inc<Cfg::REG_SOFTMAX>();
        // ================================================================ softmax warpgroups
        const int x = (warp >> 2) - half * HP;         // head of the pair
        const int r = (warp & 3) * 32 + lane;          // row in the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + Cfg::s_col(x);
        const uint32_t tP = tmem + lane_off + Cfg::p_col(x);
        const uint32_t tO = tmem + lane_off + Cfg::o_col(x);
        bool ok = true;
        int J = 0, n = 0;
        for (int it = ifirst; ok && it < p.n_items; it += istep, ++n) {
            const Item I = item_of<HP, LOCAL>(it, p);
            const int i = I.i0 + r;
            const size_t row = ((size_t)I.b * p.H + I.h0 + x) * p.N + i;  // this thread's query row
            const bool valid = i < p.N;
            float m_run = -INFINITY, l_run = 0.f;
            float bs = 0.f, sdiag = 0.f;  // LOCAL: band sum (same reference as l) and raw diagonal score

            if constexpr (!LOCAL) {
                // the window part of this row (o_A, written by the window phase) is read in the fold
                if (valid) asm volatile("prefetch.global.L2 [%0];" ::"l"(p.o + row * 64));
                const int qb = n & 1;
                ok = warp_all(mbar_wait(BAR(Cfg::B_QFULL + qb), (n >> 1) & 1, abort_flag) &&
                              mbar_wait(BAR(Cfg::B_Y + x), n & 1, abort_flag));
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
                // ||q||^2 from the swizzled query tile in shared memory
                float qq = 0.f;
                const uint8_t *qrow = smem + qb * Cfg::Q_BYTES + x * Cfg::TILE_BYTES + r * 128;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(qrow + ((ch ^ (r & 7)) << 4));
                    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(h2[e]);
                        qq = fmaf(f.x, f.x, qq);
                        qq = fmaf(f.y, f.y, qq);
                    }
                }
                mbar_arrive(BAR(Cfg::B_QEMPTY + qb));  // this thread is done with the query tile
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
                const float4 *zt = reinterpret_cast<const float4 *>(p.z + (size_t)I.tslot * DF);
                float bden = 0.f;
#pragma unroll
                for (int c4 = 0; c4 < DF / 4; ++c4) {
                    const float4 zz = __ldg(zt + c4);
                    y[4 * c4] *= f;
                    y[4 * c4 + 1] *= f;
                    y[4 * c4 + 2] *= f;
                    y[4 * c4 + 3] *= f;
                    bden = fmaf(y[4 * c4], zz.x, bden);
                    bden = fmaf(y[4 * c4 + 1], zz.y, bden);
                    bden = fmaf(y[4 * c4 + 2], zz.z, bden);
                    bden = fmaf(y[4 * c4 + 3], zz.w, bden);
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
                mbar_arrive(BAR(Cfg::B_PHI + x));
                // fold the window part (o_A, lse_A) into O = phi(q) S_t^T under one normaliser; the
                // window part's row is loaded while phi(q) S_t^T runs
                const float lse_a = valid ? p.lse[row] : 0.f;
                uint4 oa[8];
                {
                    const uint4 *orow = reinterpret_cast<const uint4 *>(p.o + row * 64);
#pragma unroll
                    for (int v = 0; v < 8; ++v) oa[v] = valid ? orow[v] : make_uint4(0, 0, 0, 0);
                }
                ok = warp_all(ok && mbar_wait(BAR(Cfg::B_PRO), n & 1, abort_flag));
                if (ok) {
                    tc_fence_after();
                    const float M = bden > 0.f ? fmaxf(lse_a, __log2f(bden)) : lse_a;
                    const float wa = ex2(lse_a - M), wb = ex2(-M);
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
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

            // ---- key tiles
            for (int jj = 0; ok && jj < I.n_tiles; ++jj) {
                const int Jt = J + jj;
                ok = warp_all(mbar_wait(BAR(Cfg::B_S + x), Jt & 1, abort_flag));
                if (!ok) break;
                tc_fence_after();
                const bool diag = LOCAL && jj == I.n_tiles - 1;
                const bool ragged = !LOCAL && I.nk - jj * Cfg::BN < Cfg::BN;
                const int limit = diag ? r + 1 : I.nk - jj * Cfg::BN;
                float sv[128];
                load_s_row(tS, sv, diag, ragged, limit, r, sdiag);
                tc_fence_before();
                mbar_arrive(BAR(Cfg::B_SFREE + x));  // S may now take the next tile's scores
                // Lazy rescale: a row moves its reference max only when the max grows by more than
                // kRescaleLog2 (see tc_tile.cuh).  The O rescale uses warp-collective tcgen05.ld/st, so the
                // warp takes it together when any of its rows needs it (rows that do not keep alpha = 1).
                const float mnew = row_max128(sv) * p.scale_log2;
                const bool need = mnew > m_run + kRescaleLog2;
                const float alpha = need ? ex2(m_run - mnew) : 1.f;
                const bool touch_o = need && m_run != -INFINITY;  // O holds nothing yet while m_run = -inf
                if (need) {
                    l_run *= alpha;
                    bs *= alpha;
                    m_run = mnew;
                }
                // LOCAL band tiles: keys kstart + c; the band of row r is [i-w+1, i-1]
                int btype = 0;  // 0 none, 1 whole tile, 2 columns c > r, 3 columns c < r
                if (LOCAL) {
                    const int kstart = I.lo + jj * Cfg::BN;
                    if (diag) btype = 3;
                    else if (I.i0 >= p.w && kstart == I.i0 - p.w) btype = 2;
                    else if (I.i0 >= p.w && kstart < I.i0 - p.w) btype = 0;
                    else btype = 1;
                }
                const int bc_lo = btype == 2 ? r + 1 : 0, bc_hi = btype == 2 ? 128 : r;
                float ls0, ls1, bsum = 0.f;
                uint32_t pu[64];
                // head 1 takes its turn after head 0's exponentials of this tile, head 0 after head 1's
                // of the previous one (barrier phase = global tile index)
                if (HP == 2 && kRingTurns != 0 && (x == 1 || Jt > 0)) {
                    if (kRingTurns == 3) {
                        ok = warp_all(*abort_flag == 0);
                        if (!ok) break;
                        nbar_sync(1 + x, 256);
                    } else {
                        ok = warp_all(mbar_wait(BAR(Cfg::B_TURN + x), (x == 1 ? Jt : Jt - 1) & 1, abort_flag));
                        if (!ok) break;
                    }
                }
                if (btype >= 2) exp_row<EXPV, true>(sv, p.scale_log2, m_run, pu, ls0, ls1, bsum, bc_lo, bc_hi);
                else exp_row<EXPV, false>(sv, p.scale_log2, m_run, pu, ls0, ls1, bsum, 0, 0);
                if (HP == 2 && kRingTurns != 0) {
                    if (kRingTurns == 3) nbar_arrive(1 + (x ^ 1), 256);
                    else mbar_arrive(BAR(Cfg::B_TURN + (x ^ 1)));
                }
                l_run += ls0 + ls1;
                if (btype == 1) bs += ls0 + ls1;
                else if (btype >= 2) bs += bsum;
                // P V(Jt-1) still reads P and adds into O: wait for it before P is rewritten or O rescaled.
                // (It was issued a whole exponential phase ago.  The first tile of an item has none in
                // flight: the previous item's epilogue waited for its last P V, and the prologue's fold
                // waited for the only MMA that wrote O since.)  The wait is for phase Jt-1 of the O
                // barrier, whose phase Jt-2 this warp already waited for at the previous tile, so the
                // parity test cannot be fooled by a barrier two phases behind.
                if (jj > 0) {
                    ok = warp_all(mbar_wait(BAR(Cfg::B_O + x), (Jt - 1) & 1, abort_flag));
                    if (!ok) break;
                    tc_fence_after();
                }
                if (__any_sync(0xffffffffu, touch_o)) {
                    const float fa = touch_o ? alpha : 1.f;
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint32_t u[32];
                        tmem_ld32(tO + c * 32, u);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * fa);
                        tmem_st32(tO + c * 32, u);
                    }
                }
                store_p(tP, pu);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(BAR(Cfg::B_P + 2 * x + (Jt & 1)));
            }
            // ---- epilogue: o = O / l
            ok = warp_all(ok && (I.n_tiles > 0 ? mbar_wait(BAR(Cfg::B_O + x), (J + I.n_tiles - 1) & 1, abort_flag)
                                               : true));
            if (ok) {
                tc_fence_after();
                const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
                __nv_bfloat16 *orow = p.o + row * 64;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t u[32];
                    tmem_ld32(tO + c * 32, u);
                    tmem_wait_ld();
                    if (valid) {
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
                if (!LOCAL && valid) p.lse[row] = m_run + __log2f(l_run);
                if (LOCAL && valid) {
                    p.lse[row] = m_run + __log2f(l_run);
                    // sigma = softplus(s_ii - LSE_{band}) in natural units; +inf for an empty band (i = 0)
                    float sig = INFINITY;
                    if (i > 0) {
                        if (bs > 0x1p-90f) {
                            const float lse_band = (m_run + __log2f(bs)) * kLn2;
                            sig = softplus_f(sdiag * (p.scale_log2 * kLn2) - lse_band);
                        } else {
                            // every band key sits > 90 binary orders below the window maximum: the
                            // shared reference has underflowed the band sum; the row is rescored with
                            // its own max
                            p.fix_list[atomicAdd(p.fix_count, 1u)] = (int)row;
                            sig = 0.f;
                        }
                    }
                    p.sigma[row] = sig;
                }
            }
            J += I.n_tiles;
        }
        if (!ok) {
            *abort_flag = 1;
            report(p.err, DEV_ERR_TIMEOUT);
            if (HP == 2 && kRingTurns == 3) {
                // the other warpgroup may sleep on a hand-over this warp will not make: one arrival on
                // each barrier releases it (it then sees the abort flag before its next wait)
                __threadfence_block();
                nbar_arrive(1, 256);
                nbar_arrive(2, 256);
            }
        } else if (HP == 2 && kRingTurns == 3 && x == 0 && J > 0) {
            // head 1's hand-over after the last tile has no later wait of head 0: take it here
            if (warp_all(*abort_flag == 0)) nbar_sync(1, 256);
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == Cfg::MMA_WARP) tmem_dealloc(tmem0, Cfg::TMEM_COLS);
}

int sm_count() {
    static int cached[128] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

int g_stall = 0, g_max_ctas = 0;

template <int DF, int HP, int NH>
cudaError_t launch_ring_cfg(int mode, const Dims &s, const MergeOperands &a, unsigned *err, cudaStream_t st) {
    using Cfg = RingCfg<DF, HP, NH>;
    const int T = s.T();
    const int n_qtiles = (s.N + 127) / 128;
    // PREFIX: only the query chunks t > m see a kept prefix or a linear state
    const int qt_first = mode == 0 ? 0 : std::min(n_qtiles, (s.m() + 1) * s.C / 128);
    if (qt_first >= n_qtiles) return cudaSuccess;
    CUtensorMap mq, mk, mv, mkh, mvh, mw, ms;
    const uint64_t khrows = (uint64_t)T * s.k > 0 ? (uint64_t)T * s.k : 1;
    bool ok = make_map(&mq, a.q, 64, s.N, (uint64_t)s.B * s.H, 128) &&
              make_map(&mk, a.k, 64, s.N, (uint64_t)s.B * s.Hkv, 128) &&
              make_map(&mv, a.v, 64, s.N, (uint64_t)s.B * s.Hkv, 128) &&
              make_map(&mkh, a.khat, 64, khrows, (uint64_t)s.B * s.Hkv, 128) &&
              make_map(&mvh, a.vhat, 64, khrows, (uint64_t)s.B * s.Hkv, 128) &&
              make_map(&mw, a.wqt, 64, DF, s.H, DF) &&
              make_map(&ms, a.st_t, DF, 64, (uint64_t)s.B * s.Hkv * (T + 1), 64);
    if (!ok) return cudaErrorInvalidValue;
    RingParams prm;
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
    prm.pairs = s.G() / HP;
    prm.n_items = (n_qtiles - qt_first) * s.B * s.Hkv * prm.pairs;
    prm.stall = g_stall;
    auto kern = mode == 0 ? merge_ring_kernel<DF, HP, NH, kRingExpLocal, 0>
                          : merge_ring_kernel<DF, HP, NH, kRingExpPrefix, 1>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    int ctas = std::min((prm.n_items + NH - 1) / NH, sm_count());
    if (g_max_ctas > 0) ctas = std::min(ctas, g_max_ctas);
    const unsigned grid = (unsigned)ctas;
    kern<<<grid, Cfg::THREADS, Cfg::SMEM, st>>>(mq, mk, mv, mkh, mvh, mw, ms, prm);
    return cudaGetLastError();
}

}  // namespace

// Head dimension 64: mode 0 window part + Self-Saliency Score (writes o_A, lse_A, sigma); mode 1 kept
// prefix + linear branch folded with the window part (writes o).
cudaError_t launch_merge_ring(int mode, const Dims &s, const MergeOperands &a, unsigned *err, cudaStream_t st) {
    if (s.d != 64) return cudaErrorNotSupported;
    const bool pair = s.G() % 2 == 0;
    if (s.D == 64) {
        if (kRingHalves) return launch_ring_cfg<64, 1, 2>(mode, s, a, err, st);
        return pair ? launch_ring_cfg<64, 2, 1>(mode, s, a, err, st) : launch_ring_cfg<64, 1, 1>(mode, s, a, err, st);
    }
    if (s.D == 128)
        return pair ? launch_ring_cfg<128, 2, 1>(mode, s, a, err, st) : launch_ring_cfg<128, 1, 1>(mode, s, a, err, st);
    return cudaErrorNotSupported;
}

void set_merge_debug(int stall, int max_ctas) {
    g_stall = stall;
    g_max_ctas = max_ctas > 0 ? max_ctas : 0;
}

}  // namespace still
