// backward_tc.cu -- the softmax branch of the STILL layer's backward pass on sm_100a tensor cores
// (bf16 storage, fp32 accumulation in TMEM).  "STILL: Selecting Tokens for Intra-Layer Hybrid
// Attention to Linearize LLMs": [p1] jsqmd.com introduction and "Chunk-Wise" (one chunk-parallel
// implementation serves training and inference); [p4] atlas.scime.ai "Approach".
//
// For query row i (head h of group g, chunk t) the softmax set is Soft(i) = the kept rows of chunks
// 0..t-m-1 (the compact kept cache) ++ the window [max(0,(t-m)C), i]; the linear branch enters the
// shared normaliser.  In log2 units (x_ij = tau log2(e) <q_i, k_j>):
//   M = max_j x_ij,  l = sum_j 2^(x_ij - M),  u = sum_j 2^(x_ij - M) <dO_i, v_j>,
//   Ms = max(M, log2 lden_i),  Z = l 2^(M - Ms) + lden_i 2^-Ms,  L_i = Ms + log2 Z,
//   D_i = <dO_i, o_i> = (u 2^(M - Ms) + dl_i 2^-Ms) / Z,
// with lden_i = phi(q_i).z_t and dl_i = <phi(q_i)^T S_t, dO_i> from the linear pre-pass.  Then
//   P_ij = 2^(x_ij - L_i),  dS_ij = P_ij (<dO_i, v_j> - D_i),
//   dq_i = tau sum_j dS_ij k_j,  dk_j = tau sum_i dS_ij q_i,  dv_j = sum_i P_ij dO_i.
//
// bwd_dq_tc_kernel: one CTA per (b, h, 128 query rows).  Two sweeps over the row tile's keys in tiles
// of 64: sweep 1 forms S = Q K^T and dP = dO V^T (tcgen05, TMEM lane = row) and accumulates M, l, u in
// registers; the row's L_i and D_i follow (written for the key pass); sweep 2 forms S and dP again,
// dS (bf16) over dP's TMEM columns, and dQ += dS K with dS as the TMEM operand.
// bwd_dkv_tc_kernel: one CTA per (b, g, 128 keys) [kept keys: per 128 kept-cache entries and one
// segment of query rows].  For each head of the group and each 64-row query tile that sees the keys:
// S^T = K Q^T and dP^T = V dO^T (TMEM lane = key), P^T and dS^T (bf16) over their own columns, then
// dV += P^T dO and dK += dS^T Q with P^T / dS^T as TMEM operands; the accumulators stay in TMEM for
// the whole CTA.  Window keys write dk, dv; kept keys add into the rows their entries name.
//
// Roles in both kernels: two warpgroups of row warps (TMEM lane = row; each warpgroup takes half of a
// tile's 64 columns), one TMA producer warp, one MMA warp (which also allocates TMEM).  Every mbarrier wait is bounded; on a timeout the CTA records
// DEV_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "still_internal.h"
#include "tc_ptx.cuh"
#include "tc_tile.cuh"

namespace still {

using namespace tc;

namespace {

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

struct BwdParams {
    int B, H, Hkv, N, C, k, w, G, T;
    float scale, scale_log2;  // tau, tau log2(e)
    const float *lden, *dl;   // [B,H,N] from the linear pre-pass (dq kernel without its own prologue)
    const float *z;           // [B*Hkv*(T+1), D] z_t (dq kernel prologue)
    float *Phi, *SG;          // [B,H,N,D] phi(q) and S_t dO (fp32), written by the dq kernel prologue; its
                              // epilogue then replaces them with a = 2^-L phi(q) and dY = dL/d(q Wq)
    float *L, *Dv;            // [B,H,N] log2 normaliser and D_i (dq kernel writes, key kernel reads)
    const float *lse_in;      // [B,H,N] the forward's log2 normaliser, or null (the dq kernel forms it)
    const __nv_bfloat16 *o_in;  // [B,H,N,d] the forward's output (with lse_in: D_i = <dO_i, o_i>)
    float *dq, *dk, *dv;      // fp32 gradients
    const int32_t *idx;       // [B,Hkv,T,k] (kept keys)
    int n_qtiles;             // dq kernel: ceil(N / 128)
    int n_ktiles;             // key kernel: 128-key tiles per (b, g)
    int seg_rows;             // kept keys: query rows per segment
    unsigned *err;
};

// ================================================================================ dq kernel
// DF = 0: the rows' linear terms (phi(q).z_t, <phi(q)^T S_t, dO>) come from the pre-pass in global
// memory.  DF in {64, 128}: the kernel forms them itself in a prologue on the tensor cores:
// Y = Q Wq^T, phi(q) per row (stored fp32 for the linear branch's later kernels and in bf16 over
// Y's TMEM columns), lin = phi(q) S_t^T and sg = dO S_t (bf16 S_t^T; sg stored fp32), as the forward
// merge's prologue does.
template <int DH, int DF>
struct BwdQCfg {
    static constexpr bool PRO = DF > 0;
    static constexpr int Q_REG = 128 * 128;          // 128 rows x 64 bf16 (one SW128 region)
    static constexpr int K_REG = 64 * 128;           // 64 rows x 64 bf16
    static constexpr int Q_BYTES = 128 * DH * 2;     // Q / dO tile (DH/64 regions)
    static constexpr int K_BYTES = 64 * DH * 2;      // K / V tile of 64 keys
    static constexpr int WQ_BYTES = PRO ? DF * DH * 2 : 0;  // Wq^T [DF rows x DH] (DH/64 regions of DF rows)
    static constexpr int ST_BYTES = PRO ? DH * DF * 2 : 0;  // S_t^T [DH rows x DF] (DF/64 regions of DH rows)
    static constexpr int NS = DH == 64 ? (DF == 128 ? 2 : PRO ? 3 : 4) : 2;  // K/V stages
    static constexpr int STAGE_BYTES = 2 * K_BYTES;
    static constexpr int OFF_Q = 0, OFF_DO = Q_BYTES, OFF_WQ = 2 * Q_BYTES, OFF_ST = OFF_WQ + WQ_BYTES,
                         OFF_STAGE = OFF_ST + ST_BYTES, OFF_BAR = OFF_STAGE + NS * STAGE_BYTES;
    // B_SDONE: the row warps hold S, dP of a tile in registers; B_DSFULL + (n & 1): they wrote the dS
    // of sweep-2 tile n (two barriers taking turns, so neither runs two phases ahead of its waiter)
    // prologue: B_WFULL (Wq^T, S_t^T tiles), B_Y (Y done), B_PHI (phi(q) written, warpgroup 0),
    // B_LIN (lin and sg done), B_PRO (warpgroup 0 has read them)
    // epilogue (with the prologue): B_W2FULL (the Wq tile), B_DY (dY / tau written, both warpgroups)
    static constexpr int B_QFULL = 0, B_S = 1, B_SDONE = 2, B_DQ = 3, B_DRAIN = 4, B_WG = 5, B_DSFULL = 6,
                         B_WFULL = 8, B_Y = 9, B_PHI = 10, B_LIN = 11, B_PRO = 12, B_W2FULL = 13, B_DY = 14,
                         B_KFULL = 15, B_VFULL = 15 + NS, B_KVEMPTY = 15 + 2 * NS, NUM_BARS = 15 + 3 * NS;
    static constexpr int TMEM_SLOT_OFF = 8 * NUM_BARS, ABORT_OFF = TMEM_SLOT_OFF + 8, BAR_BYTES = 256;
    static_assert(ABORT_OFF + 8 <= BAR_BYTES, "barrier area overflow");
    static constexpr int OFF_XCH = OFF_BAR + BAR_BYTES;   // [2][128][3] row statistics of each half
    static constexpr int OFF_LXC = OFF_XCH + 2 * 128 * 3 * 4;  // [128][3] lden, dl, ||q||^2 (prologue, for warpgroup 1)
    static constexpr int SMEM = OFF_LXC + 128 * 3 * 4 + 1024;
    // Two warpgroups of row warps: warpgroup x takes key columns [32x, 32x + 32) of every tile.
    static constexpr int THREADS = 320, PRODUCER_WARP = 8, MMA_WARP = 9, ROW_THREADS = 256;
    // S (64 keys), dP (64 keys), dQ (DH), dS of alternate tiles (bf16, 64 keys = 32 columns each);
    // prologue: Y then phi (bf16) at column 0, lin at DQ_COL, then sg at column 0
    static constexpr int S_COL = 0, DP_COL = 64, DQ_COL = 128, DS_COL = 128 + DH, TMEM_COLS = DH == 64 ? 256 : 512;
    static constexpr int Y_COL = 0, LIN_COL = DQ_COL;
    static_assert(DS_COL + 64 <= TMEM_COLS && DF <= 128, "TMEM budget");
    static constexpr int MIN_BLOCKS = DH == 64 ? 2 : 1;  // two CTAs per SM overlap each other's phases
    static_assert(MIN_BLOCKS * (SMEM + 1024) <= 233472, "shared memory per SM");
};

template <int DH, int DF>
__global__ void __launch_bounds__(BwdQCfg<DH, DF>::THREADS, BwdQCfg<DH, DF>::MIN_BLOCKS)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_do,
                     const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                     const __grid_constant__ CUtensorMap map_kh, const __grid_constant__ CUtensorMap map_vh,
                     const __grid_constant__ CUtensorMap map_wq, const __grid_constant__ CUtensorMap map_st,
                     const __grid_constant__ CUtensorMap map_w, const BwdParams p) {
    using Cfg = BwdQCfg<DH, DF>;
    constexpr bool PRO = Cfg::PRO;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint8_t *bar_area = smem + Cfg::OFF_BAR;
    const uint32_t sBar = smem_u32(bar_area);
    auto BAR = [&](int i) { return sBar + 8u * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_area + Cfg::TMEM_SLOT_OFF);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bar_area + Cfg::ABORT_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // CTA -> (b, h, query tile); later query tiles (more kept keys) first
    const int per_qt = p.B * p.H;
    const int qt = p.n_qtiles - 1 - (int)(blockIdx.x / per_qt);
    const int bh = blockIdx.x % per_qt;
    const int b = bh / p.H, h = bh % p.H, g = h / p.G;
    const int bg = b * p.Hkv + g;
    const int i0 = qt * 128;
    const int t = i0 / p.C, m = p.w / p.C;
    const int nk = p.k * max(0, t - m);                 // kept rows seen by this chunk
    const int lo = max(0, (t - m) * p.C);               // window start
    const int nkt = (nk + 63) / 64;                     // kept tiles
    const int nt = nkt + (i0 + 128 - lo) / 64;          // key tiles per sweep
    const int ntot = 2 * nt;
    const int tslot = bg * (p.T + 1) + t;               // linear state slot of the chunk
    // with the forward's normaliser and output the statistics sweep is skipped: tiles first .. ntot - 1
    // (pipeline slot and barrier phase of tile jj: jj - first)
    const int first = p.lse_in ? nt : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < Cfg::NUM_BARS; ++i)
            mbar_init(BAR(i), i == Cfg::B_SDONE || i == Cfg::B_WG || i == Cfg::B_DSFULL || i == Cfg::B_DSFULL + 1 ||
                                      i == Cfg::B_DY
                                  ? Cfg::ROW_THREADS
                                  : (i == Cfg::B_PHI || i == Cfg::B_PRO) ? 128 : 1);
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
        int issued = 0;
        mbar_arrive_expect_tx_w(BAR(Cfg::B_QFULL), 2 * Cfg::Q_BYTES);
        for (int rr = 0; rr < DH / 64; ++rr) {
            tma_load_3d_w(sbase + Cfg::OFF_Q + rr * Cfg::Q_REG, &map_q, BAR(Cfg::B_QFULL), rr * 64, i0, bh);
            tma_load_3d_w(sbase + Cfg::OFF_DO + rr * Cfg::Q_REG, &map_do, BAR(Cfg::B_QFULL), rr * 64, i0, bh);
        }
        if constexpr (PRO) {
            mbar_arrive_expect_tx_w(BAR(Cfg::B_WFULL), Cfg::WQ_BYTES + Cfg::ST_BYTES);
            for (int rr = 0; rr < DH / 64; ++rr)
                tma_load_3d_w(sbase + Cfg::OFF_WQ + rr * (DF * 128), &map_wq, BAR(Cfg::B_WFULL), rr * 64, 0, h);
            for (int rr = 0; rr < DF / 64; ++rr)
                tma_load_3d_w(sbase + Cfg::OFF_ST + rr * (DH * 128), &map_st, BAR(Cfg::B_WFULL), rr * 64, 0, tslot);
        }
        for (int pj = 0; pj < ntot - first; ++pj) {
            const int jj = pj + first, s = pj % Cfg::NS;
            if (pj >= Cfg::NS && !(ok = mbar_wait_w(BAR(Cfg::B_KVEMPTY + s), ((pj / Cfg::NS) - 1) & 1, abort_flag)))
                break;
            const int j = jj < nt ? jj : jj - nt;
            const bool kept = j < nkt;
            const int row = kept ? 64 * j : lo + 64 * (j - nkt);
            const CUtensorMap *mk = kept ? &map_kh : &map_k;
            const CUtensorMap *mv = kept ? &map_vh : &map_v;
            const uint32_t sK = sbase + Cfg::OFF_STAGE + s * Cfg::STAGE_BYTES, sV = sK + Cfg::K_BYTES;
            mbar_arrive_expect_tx_w(BAR(Cfg::B_KFULL + s), Cfg::K_BYTES);
            for (int rr = 0; rr < DH / 64; ++rr)
                tma_load_3d_w(sK + rr * Cfg::K_REG, mk, BAR(Cfg::B_KFULL + s), rr * 64, row, bg);
            mbar_arrive_expect_tx_w(BAR(Cfg::B_VFULL + s), Cfg::K_BYTES);
            for (int rr = 0; rr < DH / 64; ++rr)
                tma_load_3d_w(sV + rr * Cfg::K_REG, mv, BAR(Cfg::B_VFULL + s), rr * 64, row, bg);
            issued = pj + 1;
        }
        bool w2 = false;
        if (PRO && ok && (ok = mbar_wait_w(BAR(Cfg::B_PRO), 0, abort_flag))) {
            // Wq [DH rows x DF] for dq += dY Wq^T, over the Wq^T tile the prologue has finished with
            mbar_arrive_expect_tx_w(BAR(Cfg::B_W2FULL), Cfg::WQ_BYTES);
            for (int rr = 0; rr < DF / 64; ++rr)
                tma_load_3d_w(sbase + Cfg::OFF_WQ + rr * (DH * 128), &map_w, BAR(Cfg::B_W2FULL), rr * 64, 0, h);
            w2 = true;
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) report(p.err, DEV_ERR_TIMEOUT);
            mbar_wait_drain(BAR(Cfg::B_QFULL), 0, 100000000ull);
            if (PRO) mbar_wait_drain(BAR(Cfg::B_WFULL), 0, 100000000ull);
            if (w2) mbar_wait_drain(BAR(Cfg::B_W2FULL), 0, 100000000ull);
            for (int pj = max(0, issued - Cfg::NS); pj < issued; ++pj) {
                mbar_wait_drain(BAR(Cfg::B_KFULL + pj % Cfg::NS), (pj / Cfg::NS) & 1, 100000000ull);
                mbar_wait_drain(BAR(Cfg::B_VFULL + pj % Cfg::NS), (pj / Cfg::NS) & 1, 100000000ull);
            }
        }
    } else if (warp == Cfg::MMA_WARP) {
        // ================================================================ MMA issuer (whole warp)
        const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
        constexpr uint32_t ID_S = idesc_bf16(128, 64, 0, 0);
        constexpr uint32_t ID_DQ = idesc_bf16(128, DH, 0, 1);
        const uint32_t sQ = sbase + Cfg::OFF_Q, sDO = sbase + Cfg::OFF_DO;
        // dQ += dS K for tile jj (sweep 2): dS (bf16, 64 keys = 32 columns, buffer jj & 1) from TMEM, K
        // as the MN-major B operand (N = DH, K = 64 keys; 16 keys = 16 rows of 128 bytes per k-step).
        // The row warps reuse a dS buffer only after B_S of the tile two later, whose commit covers
        // this MMA.
        auto issue_dq = [&](int jj) {
            const int st = (jj - first) % Cfg::NS;
            const uint64_t dk = sw128_desc(sbase + Cfg::OFF_STAGE + st * Cfg::STAGE_BYTES, Cfg::K_REG, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ts_w(tm + Cfg::DQ_COL, tm + Cfg::DS_COL + 32 * (jj & 1) + kk * 8, dk + (uint64_t)(kk * 128), ID_DQ,
                         (jj > nt || kk > 0) ? 1u : 0u);
            mma_commit_w(BAR(Cfg::B_KVEMPTY + st));
        };
        bool ok = mbar_wait_w(BAR(Cfg::B_QFULL), 0, abort_flag);
        if (PRO && ok && (ok = mbar_wait_w(BAR(Cfg::B_WFULL), 0, abort_flag))) {
            // Y = Q Wq^T (K-major Wq^T rows of DH)
            constexpr uint32_t ID_Y = idesc_bf16(128, PRO ? DF : 64, 0, 0);
            constexpr uint32_t ID_LIN = idesc_bf16(128, DH, 0, 0);
            constexpr uint32_t ID_SG = idesc_bf16(128, PRO ? DF : 64, 0, 1);
            const uint32_t sWQ = sbase + Cfg::OFF_WQ, sST = sbase + Cfg::OFF_ST;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < DH / 16; ++kk)
                mma_ss_w(tm + Cfg::Y_COL, kmajor_desc(sQ, kk, Cfg::Q_REG), kmajor_desc(sWQ, kk, DF * 128), ID_Y, kk > 0);
            mma_commit_w(BAR(Cfg::B_Y));
            if ((ok = mbar_wait_w(BAR(Cfg::B_PHI), 0, abort_flag))) {
                tc_fence_after();
                // lin = phi(q) S_t^T: phi (bf16) from TMEM, S_t^T rows of DF (K-major)
#pragma unroll
                for (int kk = 0; kk < DF / 16; ++kk)
                    mma_ts_w(tm + Cfg::LIN_COL, tm + Cfg::Y_COL + kk * 8, kmajor_desc(sST, kk, DH * 128), ID_LIN, kk > 0);
                // sg = dO S_t: the S_t^T tile as an MN-major operand (N = DF features, K = DH rows), over
                // Y's columns (the MMA above, issued first, has read phi)
                const uint64_t dst = sw128_desc(sST, DH * 128, 1024);
#pragma unroll
                for (int kk = 0; kk < DH / 16; ++kk)
                    mma_ss_w(tm + Cfg::Y_COL, kmajor_desc(sDO, kk, Cfg::Q_REG), dst + (uint64_t)(kk * 128), ID_SG,
                             kk > 0);
                mma_commit_w(BAR(Cfg::B_LIN));
                ok = mbar_wait_w(BAR(Cfg::B_PRO), 0, abort_flag);  // warpgroup 0 has read lin and sg
            }
        }
        for (int jj = first; ok && jj < ntot; ++jj) {
            const int pj = jj - first, s = pj % Cfg::NS;
            const uint32_t sK = sbase + Cfg::OFF_STAGE + s * Cfg::STAGE_BYTES, sV = sK + Cfg::K_BYTES;
            if (!(ok = mbar_wait_w(BAR(Cfg::B_KFULL + s), (pj / Cfg::NS) & 1, abort_flag))) break;
            if (!(ok = mbar_wait_w(BAR(Cfg::B_VFULL + s), (pj / Cfg::NS) & 1, abort_flag))) break;
            // the row warps hold S, dP of tile jj-1 in registers: the columns are free
            if (pj > 0 && !(ok = mbar_wait_w(BAR(Cfg::B_SDONE), (pj - 1) & 1, abort_flag))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < DH / 16; ++kk)
                mma_ss_w(tm + Cfg::S_COL, kmajor_desc(sQ, kk, Cfg::Q_REG), kmajor_desc(sK, kk, Cfg::K_REG), ID_S, kk > 0);
#pragma unroll
            for (int kk = 0; kk < DH / 16; ++kk)
                mma_ss_w(tm + Cfg::DP_COL, kmajor_desc(sDO, kk, Cfg::Q_REG), kmajor_desc(sV, kk, Cfg::K_REG), ID_S, kk > 0);
            mma_commit_w(BAR(Cfg::B_S));
            if (jj < nt) mma_commit_w(BAR(Cfg::B_KVEMPTY + s));  // sweep 1: the stage is done with
            if (jj - 1 >= nt) {
                // dS of tile jj-1 written: dQ += dS K (overlaps the row warps' work on tile jj)
                const int n = jj - 1 - nt;
                if (!(ok = mbar_wait_w(BAR(Cfg::B_DSFULL + (n & 1)), (n >> 1) & 1, abort_flag))) break;
                tc_fence_after();
                issue_dq(jj - 1);
            }
        }
        if (ok && (ok = mbar_wait_w(BAR(Cfg::B_DSFULL + ((nt - 1) & 1)), ((nt - 1) >> 1) & 1, abort_flag))) {
            tc_fence_after();
            issue_dq(ntot - 1);
            if (PRO && (ok = mbar_wait_w(BAR(Cfg::B_W2FULL), 0, abort_flag) && mbar_wait_w(BAR(Cfg::B_DY), 0, abort_flag))) {
                // dQ += (dY / tau) Wq^T: dY (bf16, DF features = DF/2 columns) from TMEM over S, Wq rows of DF
                constexpr uint32_t ID_W = idesc_bf16(128, DH, 0, 0);
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < DF / 16; ++kk)
                    mma_ts_w(tm + Cfg::DQ_COL, tm + Cfg::S_COL + kk * 8, kmajor_desc(sbase + Cfg::OFF_WQ, kk, DH * 128), ID_W,
                             1u);
            }
            if (ok) mma_commit_w(BAR(Cfg::B_DQ));
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) report(p.err, DEV_ERR_TIMEOUT);
        }
        mma_commit_w(BAR(Cfg::B_DRAIN));
        mbar_wait_drain(BAR(Cfg::B_DRAIN), 0, 100000000ull);
    } else {
        // ================================================================ row warps (TMEM lane = query row)
        // warpgroup x takes key columns [32x, 32x + 32) of each tile; the two halves of a row combine
        // their running statistics once, after sweep 1
        const int x = warp >> 2, quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int i = i0 + r;
        const bool live = i < p.N;
        const size_t row = (size_t)bh * p.N + i;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_off + Cfg::S_COL + 32 * x, tDP = tmem + lane_off + Cfg::DP_COL + 32 * x,
                       tDS = tmem + lane_off + Cfg::DS_COL + 16 * x;
        float lden = 0.f, dl = 0.f, qn2 = 0.f;  // qn2 = ||q||^2 = ||phi(q)||^2 (prologue)
        bool ok = true;
        if constexpr (!PRO) {
            lden = live ? p.lden[row] : 0.f;
            dl = live ? p.dl[row] : 0.f;
        } else if (x == 0) {
            // ---- prologue (warpgroup 0, row r): phi(q) from Y, lden = phi.z_t, dl = <lin, dO>, sg
            const uint32_t tY = tmem + lane_off + Cfg::Y_COL;
            ok = warp_all(mbar_wait(BAR(Cfg::B_QFULL), 0, abort_flag) && mbar_wait(BAR(Cfg::B_Y), 0, abort_flag));
            if (ok) {
                tc_fence_after();
                // ||q||^2 from the swizzled Q tile
                float qq = 0.f;
#pragma unroll
                for (int rr = 0; rr < DH / 64; ++rr)
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        const uint4 w4 = *reinterpret_cast<const uint4 *>(smem + Cfg::OFF_Q + rr * Cfg::Q_REG + r * 128 +
                                                                          ((ch ^ (r & 7)) << 4));
                        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&w4);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f2 = __bfloat1622float2(h2[e]);
                            qq = fmaf(f2.x, f2.x, fmaf(f2.y, f2.y, qq));
                        }
                    }
                // three passes over Y in TMEM (32 columns at a time): max, sum of e^2, then phi
                float ymax = -INFINITY;
#pragma unroll
                for (int c = 0; c < DF / 32; ++c) {
                    uint32_t w[32];
                    tmem_ld32(tY + 32 * c, w);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) ymax = fmaxf(ymax, __uint_as_float(w[e]));
                }
                float ee = 0.f;
#pragma unroll
                for (int c = 0; c < DF / 32; ++c) {
                    uint32_t w[32];
                    tmem_ld32(tY + 32 * c, w);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float ex = ex2((__uint_as_float(w[e]) - ymax) * kLog2e);
                        ee = fmaf(ex, ex, ee);
                    }
                }
                const float fscale = sqrtf(qq) * rsqrtf(ee);
                qn2 = qq;
                const float *zt = p.z + (size_t)tslot * DF;
                float *phig = p.Phi + row * DF;
#pragma unroll
                for (int c = 0; c < DF / 32; ++c) {
                    uint32_t w[32], pk[16];
                    tmem_ld32(tY + 32 * c, w);
                    tmem_wait_ld();
                    float ph[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        ph[e] = ex2((__uint_as_float(w[e]) - ymax) * kLog2e) * fscale;
                        lden = fmaf(ph[e], __ldg(zt + 32 * c + e), lden);
                    }
                    if (live) {
#pragma unroll
                        for (int v4 = 0; v4 < 8; ++v4)
                            reinterpret_cast<float4 *>(phig + 32 * c)[v4] =
                                make_float4(ph[4 * v4], ph[4 * v4 + 1], ph[4 * v4 + 2], ph[4 * v4 + 3]);
                    }
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(ph[2 * e], ph[2 * e + 1]);
                    // phi (bf16) of columns 32c.. lands on columns [16c, 16c + 16), already read
                    tmem_st16(tY + 16 * c, pk);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(BAR(Cfg::B_PHI));
            ok = warp_all(ok && mbar_wait(BAR(Cfg::B_LIN), 0, abort_flag));
            if (ok) {
                tc_fence_after();
                // dl = <phi(q)^T S_t, dO> with dO from the swizzled dO tile
#pragma unroll
                for (int c = 0; c < DH / 32; ++c) {
                    uint32_t w[32];
                    tmem_ld32(tmem + lane_off + Cfg::LIN_COL + 32 * c, w);
                    tmem_wait_ld();
                    const int rr = c >> 1;
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        const int chunk = (c & 1) * 4 + ch;  // 16-byte chunk of the 128-byte row
                        const uint4 w4 = *reinterpret_cast<const uint4 *>(smem + Cfg::OFF_DO + rr * Cfg::Q_REG + r * 128 +
                                                                          ((chunk ^ (r & 7)) << 4));
                        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&w4);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f2 = __bfloat1622float2(h2[e]);
                            dl = fmaf(__uint_as_float(w[ch * 8 + 2 * e]), f2.x, dl);
                            dl = fmaf(__uint_as_float(w[ch * 8 + 2 * e + 1]), f2.y, dl);
                        }
                    }
                }
                // sg = dO S_t (fp32) for the linear branch's query side
                float *sgg = p.SG + row * DF;
#pragma unroll
                for (int c = 0; c < DF / 32; ++c) {
                    uint32_t w[32];
                    tmem_ld32(tY + 32 * c, w);
                    tmem_wait_ld();
                    if (live) {
#pragma unroll
                        for (int v4 = 0; v4 < 8; ++v4)
                            reinterpret_cast<float4 *>(sgg + 32 * c)[v4] =
                                make_float4(__uint_as_float(w[4 * v4]), __uint_as_float(w[4 * v4 + 1]),
                                            __uint_as_float(w[4 * v4 + 2]), __uint_as_float(w[4 * v4 + 3]));
                    }
                }
            }
            float *lx = reinterpret_cast<float *>(smem + Cfg::OFF_LXC);
            lx[3 * r] = lden;
            lx[3 * r + 1] = dl;
            lx[3 * r + 2] = qn2;
            tc_fence_before();
            mbar_arrive(BAR(Cfg::B_PRO));
        }
        const float sl2 = p.scale_log2;
        float M = -INFINITY, l = 0.f, u = 0.f, Lr = 0.f, Di = 0.f;
        if (p.lse_in) {
            // the forward's normaliser of the row and D_i = <dO_i, o_i> (dO from the swizzled tile)
            ok = warp_all(ok && mbar_wait(BAR(Cfg::B_QFULL), 0, abort_flag));
            if (ok && live) {
                Lr = p.lse_in[row];
                const uint4 *orow = reinterpret_cast<const uint4 *>(p.o_in + row * DH);
#pragma unroll
                for (int c = 0; c < DH / 8; ++c) {
                    const uint4 ov = orow[c];
                    const uint4 gv = *reinterpret_cast<const uint4 *>(smem + Cfg::OFF_DO + (c >> 3) * Cfg::Q_REG + r * 128 +
                                                                      (((c & 7) ^ (r & 7)) << 4));
                    const __nv_bfloat162 *oh = reinterpret_cast<const __nv_bfloat162 *>(&ov);
                    const __nv_bfloat162 *gh = reinterpret_cast<const __nv_bfloat162 *>(&gv);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 of = __bfloat1622float2(oh[e]), gf = __bfloat1622float2(gh[e]);
                        Di = fmaf(of.x, gf.x, fmaf(of.y, gf.y, Di));
                    }
                }
                if (x == 0) {
                    p.L[row] = Lr;
                    p.Dv[row] = Di;
                }
            }
            if (PRO && x == 1) {  // the prologue's linear terms of this row (warpgroup 0)
                ok = warp_all(ok && mbar_wait(BAR(Cfg::B_PRO), 0, abort_flag));
                if (ok) {
                    const float *lx = reinterpret_cast<const float *>(smem + Cfg::OFF_LXC);
                    lden = lx[3 * r];
                    dl = lx[3 * r + 1];
                    qn2 = lx[3 * r + 2];
                }
            }
        }
        for (int jj = first; ok && jj < ntot; ++jj) {
            if (!(ok = warp_all(mbar_wait(BAR(Cfg::B_S), (jj - first) & 1, abort_flag)))) break;
            tc_fence_after();
            const int j = jj < nt ? jj : jj - nt;
            // columns c < lim are in Soft(i): kept entries below nk, window keys at or before i
            const int lim = (j < nkt ? nk - 64 * j : i - (lo + 64 * (j - nkt)) + 1) - 32 * x;
            if (jj < nt) {
                // ---- sweep 1: running max, sum and sum of exp * <dO, v> over this half's columns
                // (raw scores; tau log2(e) > 0 is applied to the max and inside the exponent's FFMA)
                float sv[32];
                {
                    uint32_t w[32];
                    tmem_ld32(tS, w);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) sv[e] = __uint_as_float(w[e]);
                }
                if (!warp_all(lim >= 32)) {  // a ragged or diagonal tile: masked columns never win
#pragma unroll
                    for (int e = 0; e < 32; ++e) sv[e] = e < lim ? sv[e] : -INFINITY;
                }
                float m3[3] = {sv[0], sv[1], sv[2]};
#pragma unroll
                for (int e = 3; e + 2 < 32; e += 3) {
                    m3[0] = fmaxf(m3[0], sv[e]);
                    m3[1] = fmaxf(m3[1], sv[e + 1]);
                    m3[2] = fmaxf(m3[2], sv[e + 2]);
                }
                const float mt = fmax3(fmax3(m3[0], m3[1], m3[2]), sv[30], sv[31]) * sl2;
                const float mn = fmaxf(M, mt);
                const float mref = mn == -INFINITY ? 0.f : mn;
                const float sc = M == -INFINITY ? 0.f : ex2(M - mref);
                const float2 sl2v = make_float2(sl2, sl2), nm = make_float2(-mref, -mref);
                float2 l2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                float2 u2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                {
                    uint32_t w[32];
                    tmem_ld32(tDP, w);
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(BAR(Cfg::B_SDONE));  // S and dP of this tile are in registers
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const float2 xx = ffma2(make_float2(sv[e], sv[e + 1]), sl2v, nm);
                        const float2 pp = make_float2(ex2(xx.x), ex2(xx.y));
                        l2[(e >> 1) & 1] = fadd2(l2[(e >> 1) & 1], pp);
                        u2[(e >> 1) & 1] = ffma2(pp, make_float2(__uint_as_float(w[e]), __uint_as_float(w[e + 1])),
                                                 u2[(e >> 1) & 1]);
                    }
                }
                const float2 ls = fadd2(l2[0], l2[1]), us = fadd2(u2[0], u2[1]);
                l = fmaf(l, sc, ls.x + ls.y);
                u = fmaf(u, sc, us.x + us.y);
                M = mn;
                if (jj == nt - 1) {
                    // ---- combine the two halves, then the row's normaliser with the linear branch and D_i
                    float *xch = reinterpret_cast<float *>(smem + Cfg::OFF_XCH);
                    xch[(x * 128 + r) * 3 + 0] = M;
                    xch[(x * 128 + r) * 3 + 1] = l;
                    xch[(x * 128 + r) * 3 + 2] = u;
                    mbar_arrive(BAR(Cfg::B_WG));
                    if (!(ok = warp_all(mbar_wait(BAR(Cfg::B_WG), 0, abort_flag)))) break;
                    const float Mo = xch[((x ^ 1) * 128 + r) * 3 + 0], lo_ = xch[((x ^ 1) * 128 + r) * 3 + 1],
                                uo = xch[((x ^ 1) * 128 + r) * 3 + 2];
                    if (PRO && x == 1) {  // the prologue's linear terms of this row (warpgroup 0)
                        const float *lx = reinterpret_cast<const float *>(smem + Cfg::OFF_LXC);
                        lden = lx[3 * r];
                        dl = lx[3 * r + 1];
                        qn2 = lx[3 * r + 2];
                    }
                    const float Mc = fmaxf(M, Mo);
                    const float f0 = M == -INFINITY ? 0.f : ex2(M - Mc), f1 = Mo == -INFINITY ? 0.f : ex2(Mo - Mc);
                    l = l * f0 + lo_ * f1;
                    u = u * f0 + uo * f1;
                    M = Mc;
                    const float Ms = lden > 0.f ? fmaxf(M, __log2f(lden)) : M;
                    const float a_soft = ex2(M - Ms), a_lin = lden > 0.f ? ex2(-Ms) : 0.f;
                    const float Z = fmaf(l, a_soft, lden * a_lin);
                    Lr = Ms + __log2f(Z);
                    Di = fmaf(u, a_soft, dl * a_lin) / Z;
                    if (live && x == 0) {
                        p.L[row] = Lr;
                        p.Dv[row] = Di;
                    }
                }
            } else {
                // ---- sweep 2: P = 2^(x - L), dS = P (dP - D) in bf16 into this half of the dS columns
                const float2 sc2 = make_float2(sl2, sl2), nl2 = make_float2(-Lr, -Lr), nd2 = make_float2(-Di, -Di);
                uint32_t ws[32], wd[32], pk[16];
                tmem_ld32(tS, ws);
                tmem_ld32(tDP, wd);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(BAR(Cfg::B_SDONE));  // S and dP of this tile are in registers
                const bool full = warp_all(lim >= 32);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 xx = ffma2(make_float2(__uint_as_float(ws[2 * e]), __uint_as_float(ws[2 * e + 1])),
                                            sc2, nl2);
                    float2 pp = make_float2(ex2(xx.x), ex2(xx.y));
                    if (!full) {
                        pp.x = 2 * e < lim ? pp.x : 0.f;
                        pp.y = 2 * e + 1 < lim ? pp.y : 0.f;
                    }
                    const float2 dd = fmul2(pp, fadd2(make_float2(__uint_as_float(wd[2 * e]), __uint_as_float(wd[2 * e + 1])),
                                                      nd2));
                    pk[e] = pack_bf16x2(dd.x, dd.y);
                }
                tmem_st16(tDS + 32 * (jj & 1), pk);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(BAR(Cfg::B_DSFULL + ((jj - nt) & 1)));
            }
        }
        float kappa = 0.f;  // with the prologue: the x-coefficient of the NP-Map backward, dL/dq += kappa q
        if constexpr (PRO) {
            // ---- the linear branch's query side (warpgroup x: features [x DF/2, (x + 1) DF/2) of the row):
            // dphi = 2^-L (S_t dO - D z_t); NP-Map backward from phi itself: with kappa = <phi, dphi> / |phi|^2,
            // dY = phi (dphi - kappa phi) and dL/dq = dY Wq^T + kappa q (the f.df term vanishes: df is
            // orthogonal to f).  Both sums are known: |phi|^2 = |q|^2 and <phi, dphi> = 2^-L (<phi, S_t dO>
            // - D <phi, z_t>) = 2^-L (dl - D lden).  a = 2^-L phi and dY replace phi and S_t dO in memory.
            constexpr int HF = DF / 2;
            const float cl = ex2(-Lr);
            const float *zt = p.z + (size_t)tslot * DF + x * HF;
            float *phg = p.Phi + row * DF + x * HF, *sgg = p.SG + row * DF + x * HF;
            kappa = qn2 > 0.f ? cl * (dl - Di * lden) / qn2 : 0.f;
            const float itau = 1.f / p.scale;
            const uint32_t tDY = tmem + lane_off + Cfg::S_COL + x * (HF / 2);
#pragma unroll
            for (int c = 0; c < HF / 32; ++c) {
                uint32_t pk[16];
#pragma unroll
                for (int a4 = 0; a4 < 8; ++a4) {
                    float4 ph = make_float4(0.f, 0.f, 0.f, 0.f), dy = ph;
                    if (ok && live) {
                        ph = reinterpret_cast<const float4 *>(phg)[8 * c + a4];
                        const float4 sg = reinterpret_cast<const float4 *>(sgg)[8 * c + a4];
                        const float4 zz = __ldg(reinterpret_cast<const float4 *>(zt) + 8 * c + a4);
                        dy.x = ph.x * (cl * (sg.x - Di * zz.x) - kappa * ph.x);
                        dy.y = ph.y * (cl * (sg.y - Di * zz.y) - kappa * ph.y);
                        dy.z = ph.z * (cl * (sg.z - Di * zz.z) - kappa * ph.z);
                        dy.w = ph.w * (cl * (sg.w - Di * zz.w) - kappa * ph.w);
                        reinterpret_cast<float4 *>(phg)[8 * c + a4] = make_float4(cl * ph.x, cl * ph.y, cl * ph.z, cl * ph.w);
                        reinterpret_cast<float4 *>(sgg)[8 * c + a4] = dy;
                    }
                    pk[2 * a4] = pack_bf16x2(dy.x * itau, dy.y * itau);
                    pk[2 * a4 + 1] = pack_bf16x2(dy.z * itau, dy.w * itau);
                }
                // dY / tau (bf16) of features x HF + 32c.. into columns [x HF/2 + 16c, +16) over S (free:
                // every tile's S has been read)
                tmem_st16(tDY + 16 * c, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(BAR(Cfg::B_DY));
        }
        // ---- epilogue: dq = tau dQ (+ kappa q) (fp32); warpgroup x writes columns [x DH/2, (x + 1) DH/2)
        ok = warp_all(ok && mbar_wait(BAR(Cfg::B_DQ), 0, abort_flag));
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < DH / 64; ++c) {
                const int col = x * (DH / 2) + c * 32;
                uint32_t w[32];
                tmem_ld32(tmem + lane_off + Cfg::DQ_COL + col, w);
                tmem_wait_ld();
                if (live) {
                    float qv[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) qv[e] = 0.f;
                    if (PRO) {  // q of columns col.. from the swizzled Q tile
#pragma unroll
                        for (int ch = 0; ch < 4; ++ch) {
                            const int chunk = ((col & 63) >> 3) + ch;
                            const uint4 w4 = *reinterpret_cast<const uint4 *>(smem + Cfg::OFF_Q + (col >> 6) * Cfg::Q_REG +
                                                                              r * 128 + ((chunk ^ (r & 7)) << 4));
                            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&w4);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 f2 = __bfloat1622float2(h2[e]);
                                qv[ch * 8 + 2 * e] = f2.x;
                                qv[ch * 8 + 2 * e + 1] = f2.y;
                            }
                        }
                    }
                    float4 *dst = reinterpret_cast<float4 *>(p.dq + row * DH + col);
#pragma unroll
                    for (int v4 = 0; v4 < 8; ++v4)
                        dst[v4] = make_float4(fmaf(__uint_as_float(w[4 * v4]), p.scale, kappa * qv[4 * v4]),
                                              fmaf(__uint_as_float(w[4 * v4 + 1]), p.scale, kappa * qv[4 * v4 + 1]),
                                              fmaf(__uint_as_float(w[4 * v4 + 2]), p.scale, kappa * qv[4 * v4 + 2]),
                                              fmaf(__uint_as_float(w[4 * v4 + 3]), p.scale, kappa * qv[4 * v4 + 3]));
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

// ================================================================================ key kernel
template <int DH>
struct BwdKVCfg {
    static constexpr int K_REG = 128 * 128;          // 128 rows x 64 bf16
    static constexpr int Q_REG = 64 * 128;           // 64 rows x 64 bf16
    static constexpr int K_BYTES = 128 * DH * 2;     // K / V tile of 128 keys
    static constexpr int Q_BYTES = 64 * DH * 2;      // Q / dO tile of 64 query rows
    static constexpr int NS = DH == 64 ? 8 : 4;      // query stages
    static constexpr int STAGE_BYTES = 2 * Q_BYTES + 1024;  // Q, dO, then L and D of the 64 rows
    static constexpr int OFF_K = 0, OFF_V = K_BYTES, OFF_STAGE = 2 * K_BYTES,
                         OFF_BAR = OFF_STAGE + NS * STAGE_BYTES;
    // Two S^T / dP^T buffers: tile u uses buffer u & 1 and warpgroup u & 1 of the row warps, so the
    // MMAs of tile u + 1 run while the other warpgroup works on tile u.  B_S + b: S^T, dP^T of a tile
    // in buffer b are ready; B_PDONE + b: P^T, dS^T of that tile are written.
    static constexpr int B_KVFULL = 0, B_ACC = 1, B_DRAIN = 2, B_S = 3, B_PDONE = 5, B_QFULL = 7,
                         B_STFULL = 7 + NS, B_QEMPTY = 7 + 2 * NS, NUM_BARS = 7 + 3 * NS;
    static constexpr int TMEM_SLOT_OFF = 8 * NUM_BARS, ABORT_OFF = TMEM_SLOT_OFF + 8, BAR_BYTES = 512;
    static_assert(ABORT_OFF + 8 <= BAR_BYTES, "barrier area overflow");
    static constexpr int SMEM = OFF_BAR + BAR_BYTES + 1024;
    static_assert(SMEM <= 232448, "shared memory");
    static constexpr int THREADS = 320, PRODUCER_WARP = 8, MMA_WARP = 9;
    // per buffer b: S^T (64 queries; P^T in bf16 over its first 32 columns), dP^T (dS^T likewise);
    // then dV, dK
    __host__ __device__ static constexpr int s_col(int b) { return 128 * b; }
    __host__ __device__ static constexpr int dp_col(int b) { return 128 * b + 64; }
    static constexpr int DV_COL = 256, DK_COL = 256 + DH, TMEM_COLS = 512;
    static_assert(DK_COL + DH <= TMEM_COLS, "TMEM budget");
};

template <int DH, bool KEPT>
__global__ void __launch_bounds__(BwdKVCfg<DH>::THREADS, 1)
    bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                      const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_do,
                      const BwdParams p) {
    using Cfg = BwdKVCfg<DH>;
    const int BK = p.B * p.Hkv;
    const int bg = blockIdx.x % BK, b = bg / p.Hkv, g = bg % p.Hkv;
    const int kt = (blockIdx.x / BK) % p.n_ktiles;
    const int m = p.w / p.C;
    const int j0 = kt * 128;  // first key (window) or kept-cache entry (kept) of the tile
    int qbeg, qend;
    if (!KEPT) {
        qbeg = j0;
        qend = min(p.N, (j0 / p.C + m + 1) * p.C);
    } else {
        const int seg = (int)(blockIdx.x / BK) / p.n_ktiles;
        qbeg = (j0 / p.k + m + 1) * p.C + seg * p.seg_rows;  // queries that see the tile's first chunk
        qend = min(p.N, qbeg + p.seg_rows);
        if (qbeg >= p.N) return;  // (uniform over the CTA, before any barrier or TMEM use)
    }
    const int nqt = (qend - qbeg + 63) / 64;
    const int tiles = p.G * nqt;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint8_t *bar_area = smem + Cfg::OFF_BAR;
    const uint32_t sBar = smem_u32(bar_area);
    auto BAR = [&](int i) { return sBar + 8u * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_area + Cfg::TMEM_SLOT_OFF);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bar_area + Cfg::ABORT_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < Cfg::NUM_BARS; ++i) {
            const bool stats = i >= Cfg::B_STFULL && i < Cfg::B_STFULL + Cfg::NS;
            mbar_init(BAR(i), i == Cfg::B_PDONE || i == Cfg::B_PDONE + 1 ? 128 : stats ? 32 : 1);
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
        int issued = 0;
        mbar_arrive_expect_tx_w(BAR(Cfg::B_KVFULL), 2 * Cfg::K_BYTES);
        for (int rr = 0; rr < DH / 64; ++rr) {
            tma_load_3d_w(sbase + Cfg::OFF_K + rr * Cfg::K_REG, &map_k, BAR(Cfg::B_KVFULL), rr * 64, j0, bg);
            tma_load_3d_w(sbase + Cfg::OFF_V + rr * Cfg::K_REG, &map_v, BAR(Cfg::B_KVFULL), rr * 64, j0, bg);
        }
        // L and D of a tile's 64 rows (zero past the sequence end; those columns are masked), two per
        // lane, loaded into registers one tile ahead of their stores so the loads' latency overlaps
        const float *__restrict__ gL = p.L;
        const float *__restrict__ gD = p.Dv;
        float nL[2], nD[2];
        auto load_stats = [&](int u) {
            const int hh = u / nqt, iq0 = qbeg + 64 * (u % nqt);
            const size_t rb = (size_t)(b * p.H + g * p.G + hh) * p.N;
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int i = iq0 + lane + 32 * k2;
                nL[k2] = i < p.N ? __ldg(gL + rb + i) : 0.f;
                nD[k2] = i < p.N ? __ldg(gD + rb + i) : 0.f;
            }
        };
        if (tiles > 0) load_stats(0);
        for (int u = 0; u < tiles; ++u) {
            const int s = u % Cfg::NS;
            if (u >= Cfg::NS && !(ok = mbar_wait_w(BAR(Cfg::B_QEMPTY + s), ((u / Cfg::NS) - 1) & 1, abort_flag))) break;
            const int hh = u / nqt, iq0 = qbeg + 64 * (u % nqt);
            const int bh = b * p.H + g * p.G + hh;
            const uint32_t sQ = sbase + Cfg::OFF_STAGE + s * Cfg::STAGE_BYTES, sDO = sQ + Cfg::Q_BYTES;
            mbar_arrive_expect_tx_w(BAR(Cfg::B_QFULL + s), 2 * Cfg::Q_BYTES);
            for (int rr = 0; rr < DH / 64; ++rr) {
                tma_load_3d_w(sQ + rr * Cfg::Q_REG, &map_q, BAR(Cfg::B_QFULL + s), rr * 64, iq0, bh);
                tma_load_3d_w(sDO + rr * Cfg::Q_REG, &map_do, BAR(Cfg::B_QFULL + s), rr * 64, iq0, bh);
            }
            const float cL0 = nL[0], cL1 = nL[1], cD0 = nD[0], cD1 = nD[1];
            if (u + 1 < tiles) load_stats(u + 1);
            float *st = reinterpret_cast<float *>(smem + Cfg::OFF_STAGE + s * Cfg::STAGE_BYTES + 2 * Cfg::Q_BYTES);
            st[lane] = cL0;
            st[lane + 32] = cL1;
            st[64 + lane] = cD0;
            st[96 + lane] = cD1;
            mbar_arrive(BAR(Cfg::B_STFULL + s));
            issued = u + 1;
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) report(p.err, DEV_ERR_TIMEOUT);
            mbar_wait_drain(BAR(Cfg::B_KVFULL), 0, 100000000ull);
            for (int u = max(0, issued - Cfg::NS); u < issued; ++u)
                mbar_wait_drain(BAR(Cfg::B_QFULL + u % Cfg::NS), (u / Cfg::NS) & 1, 100000000ull);
        }
    } else if (warp == Cfg::MMA_WARP) {
        // ================================================================ MMA issuer (whole warp)
        const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
        constexpr uint32_t ID_S = idesc_bf16(128, 64, 0, 0);
        constexpr uint32_t ID_ACC = idesc_bf16(128, DH, 0, 1);
        const uint32_t sK = sbase + Cfg::OFF_K, sV = sbase + Cfg::OFF_V;
        // dV += P^T dO and dK += dS^T Q for tile u: P^T / dS^T (bf16, 64 queries = 32 columns) from
        // buffer u & 1 of TMEM, dO / Q as MN-major B operands (N = DH, K = 64 query rows; 16 rows per
        // k-step).  Issued before the scores of tile u + 2, which overwrite that buffer.
        auto issue_acc = [&](int u) {
            const int b = u & 1;
            const uint32_t sQ = sbase + Cfg::OFF_STAGE + (u % Cfg::NS) * Cfg::STAGE_BYTES, sDO = sQ + Cfg::Q_BYTES;
            const uint64_t ddo = sw128_desc(sDO, Cfg::Q_REG, 1024), dqq = sw128_desc(sQ, Cfg::Q_REG, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ts_w(tm + Cfg::DV_COL, tm + Cfg::s_col(b) + kk * 8, ddo + (uint64_t)(kk * 128), ID_ACC,
                         (u > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_ts_w(tm + Cfg::DK_COL, tm + Cfg::dp_col(b) + kk * 8, dqq + (uint64_t)(kk * 128), ID_ACC,
                         (u > 0 || kk > 0) ? 1u : 0u);
            mma_commit_w(BAR(Cfg::B_QEMPTY + u % Cfg::NS));
        };
        bool ok = mbar_wait_w(BAR(Cfg::B_KVFULL), 0, abort_flag);
        for (int u = 0; ok && u < tiles; ++u) {
            const int s = u % Cfg::NS, b = u & 1;
            const uint32_t sQ = sbase + Cfg::OFF_STAGE + s * Cfg::STAGE_BYTES, sDO = sQ + Cfg::Q_BYTES;
            if (!(ok = mbar_wait_w(BAR(Cfg::B_QFULL + s), (u / Cfg::NS) & 1, abort_flag))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < DH / 16; ++kk)
                mma_ss_w(tm + Cfg::s_col(b), kmajor_desc(sK, kk, Cfg::K_REG), kmajor_desc(sQ, kk, Cfg::Q_REG), ID_S,
                         kk > 0);
#pragma unroll
            for (int kk = 0; kk < DH / 16; ++kk)
                mma_ss_w(tm + Cfg::dp_col(b), kmajor_desc(sV, kk, Cfg::K_REG), kmajor_desc(sDO, kk, Cfg::Q_REG), ID_S,
                         kk > 0);
            mma_commit_w(BAR(Cfg::B_S + b));
            if (u > 0) {
                // P^T, dS^T of tile u-1 written by the other warpgroup (overlaps S^T, dP^T of tile u)
                const int v = u - 1;
                if (!(ok = mbar_wait_w(BAR(Cfg::B_PDONE + (v & 1)), (v >> 1) & 1, abort_flag))) break;
                tc_fence_after();
                issue_acc(v);
            }
        }
        if (ok && (ok = mbar_wait_w(BAR(Cfg::B_PDONE + ((tiles - 1) & 1)), ((tiles - 1) >> 1) & 1, abort_flag))) {
            tc_fence_after();
            issue_acc(tiles - 1);
            mma_commit_w(BAR(Cfg::B_ACC));
        }
        if (!ok) {
            *abort_flag = 1;
            if (lane == 0) report(p.err, DEV_ERR_TIMEOUT);
        }
        mma_commit_w(BAR(Cfg::B_DRAIN));
        mbar_wait_drain(BAR(Cfg::B_DRAIN), 0, 100000000ull);
    } else {
        // ================================================================ row warps (TMEM lane = key)
        // warpgroup x takes the tiles u = x, x + 2, ... (TMEM buffer x)
        const int x = warp >> 2, quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int TK = p.T * p.k;
        // query rows i >= thr see this key: the key itself (window), or the chunk after the window
        // that follows the entry's chunk (kept)
        int thr;
        if (!KEPT) thr = j0 + r;
        else thr = j0 + r < TK ? ((j0 + r) / p.k + m + 1) * p.C : 0x7fffffff;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_off + Cfg::s_col(x), tDP = tmem + lane_off + Cfg::dp_col(x);
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        bool ok = true;
        for (int u = x; u < tiles; u += 2) {
            const int s = u % Cfg::NS;
            if (!(ok = warp_all(mbar_wait(BAR(Cfg::B_S + x), (u >> 1) & 1, abort_flag) &&
                                mbar_wait(BAR(Cfg::B_STFULL + s), (u / Cfg::NS) & 1, abort_flag))))
                break;
            tc_fence_after();
            const int iq0 = qbeg + 64 * (u % nqt);
            const int c_lo = thr - iq0, c_hi = p.N - iq0;  // columns c_lo <= c < c_hi count
            const bool full = warp_all(c_lo <= 0 && c_hi >= 64);
            const float *st = reinterpret_cast<const float *>(smem + Cfg::OFF_STAGE + s * Cfg::STAGE_BYTES +
                                                              2 * Cfg::Q_BYTES);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t ws[32], wd[32], pp[16], dd[16];
                tmem_ld32(tS + 32 * c, ws);
                tmem_ld32(tDP + 32 * c, wd);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int c0 = 32 * c + 2 * e;
                    const float2 Lc = *reinterpret_cast<const float2 *>(st + c0);
                    const float2 Dc = *reinterpret_cast<const float2 *>(st + 64 + c0);
                    const float2 xx = ffma2(make_float2(__uint_as_float(ws[2 * e]), __uint_as_float(ws[2 * e + 1])), sc2,
                                            make_float2(-Lc.x, -Lc.y));
                    float2 pv = make_float2(ex2(xx.x), ex2(xx.y));
                    if (!full) {  // (the stats of masked columns may be garbage: select, never multiply)
                        pv.x = c0 >= c_lo && c0 < c_hi ? pv.x : 0.f;
                        pv.y = c0 + 1 >= c_lo && c0 + 1 < c_hi ? pv.y : 0.f;
                    }
                    float2 dv2 = fmul2(pv, fadd2(make_float2(__uint_as_float(wd[2 * e]), __uint_as_float(wd[2 * e + 1])),
                                                 make_float2(-Dc.x, -Dc.y)));
                    if (!full) {
                        dv2.x = pv.x != 0.f ? dv2.x : 0.f;
                        dv2.y = pv.y != 0.f ? dv2.y : 0.f;
                    }
                    pp[e] = pack_bf16x2(pv.x, pv.y);
                    dd[e] = pack_bf16x2(dv2.x, dv2.y);
                }
                // columns [16c, 16c + 16) were read above (chunk c loaded columns 32c..32c+31)
                tmem_st16(tS + 16 * c, pp);
                tmem_st16(tDP + 16 * c, dd);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(BAR(Cfg::B_PDONE + x));
        }
        // ---- epilogue: warpgroup 0 writes dv = dV, warpgroup 1 dk = tau dK (window: written; kept:
        //      added into the entry's row)
        ok = warp_all(ok && mbar_wait(BAR(Cfg::B_ACC), 0, abort_flag));
        if (ok) {
            tc_fence_after();
            int dst_row = -1;
            if (!KEPT) {
                if (j0 + r < p.N) dst_row = j0 + r;
            } else if (j0 + r < TK && thr < p.N) {
                const int e = j0 + r, c = e / p.k;
                const int jr = p.idx[(size_t)bg * TK + e];
                if (jr >= c * p.C && jr < (c + 1) * p.C) dst_row = jr;
            }
            const uint32_t tA = tmem + lane_off + (x ? Cfg::DK_COL : Cfg::DV_COL);
            float *out = x ? p.dk : p.dv;
            const float f = x ? p.scale : 1.f;
#pragma unroll
            for (int c = 0; c < DH / 32; ++c) {
                uint32_t w[32];
                tmem_ld32(tA + c * 32, w);
                tmem_wait_ld();
                if (dst_row >= 0) {
                    float4 *dst = reinterpret_cast<float4 *>(out + ((size_t)bg * p.N + dst_row) * DH + c * 32);
#pragma unroll
                    for (int v4 = 0; v4 < 8; ++v4) {
                        const float4 val = make_float4(__uint_as_float(w[4 * v4]) * f, __uint_as_float(w[4 * v4 + 1]) * f,
                                                       __uint_as_float(w[4 * v4 + 2]) * f,
                                                       __uint_as_float(w[4 * v4 + 3]) * f);
                        if (KEPT) atomicAdd(dst + v4, val);
                        else dst[v4] = val;
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

// The dq kernel with its own linear prologue (DF = D) or with the pre-pass's terms (DF = 0).
template <int DH, int DF>
cudaError_t launch_dq(const Dims &s, const CUtensorMap *maps, const void *wqt, const void *st_t, const void *Wq,
                      const BwdParams &prm, cudaStream_t st) {
    using Cfg = BwdQCfg<DH, DF>;
    CUtensorMap mwq = maps[0], mst = maps[0], mw = maps[0];
    if (DF > 0 && (!make_map(&mwq, wqt, DH, DF, s.H, DF) ||
                   !make_map(&mst, st_t, DF, DH, (uint64_t)s.B * s.Hkv * (s.T() + 1), DH) ||
                   !make_map(&mw, Wq, DF, DH, s.H, DH)))
        return cudaErrorInvalidValue;
    auto kern = bwd_dq_tc_kernel<DH, DF>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(prm.n_qtiles * (uint64_t)s.B * s.H), Cfg::THREADS, Cfg::SMEM, st>>>(
        maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], mwq, mst, mw, prm);
    return cudaGetLastError();
}

template <int DH>
cudaError_t launch_bwd_cfg(const Dims &s, const void *q, const void *k, const void *v, const void *khat,
                           const void *vhat, const void *dO, const void *wqt, const void *st_t, const void *Wq,
                           const BwdParams &prm_in, cudaStream_t st, int *launches) {
    const int T = s.T();
    const uint64_t BH = (uint64_t)s.B * s.H, BK = (uint64_t)s.B * s.Hkv;
    const bool has_kept = s.k > 0 && T > 0;
    BwdParams prm = prm_in;
    // dq kernel: 128-row query / dO boxes, 64-row key boxes
    CUtensorMap mq128, mdo128, mk64, mv64, mkh64, mvh64;
    bool ok = make_map(&mq128, q, DH, s.N, BH, 128) && make_map(&mdo128, dO, DH, s.N, BH, 128) &&
              make_map(&mk64, k, DH, s.N, BK, 64) && make_map(&mv64, v, DH, s.N, BK, 64);
    if (has_kept)
        ok = ok && make_map(&mkh64, khat, DH, (uint64_t)T * s.k, BK, 64) &&
             make_map(&mvh64, vhat, DH, (uint64_t)T * s.k, BK, 64);
    else
        mkh64 = mk64, mvh64 = mv64;
    if (!ok) return cudaErrorInvalidValue;
    {
        prm.n_qtiles = (s.N + 127) / 128;
        const CUtensorMap maps[6] = {mq128, mdo128, mk64, mv64, mkh64, mvh64};
        const int ts = timing_begin(kTimeBwdDq, st);
        cudaError_t e;
        if (!wqt) e = launch_dq<DH, 0>(s, maps, nullptr, nullptr, nullptr, prm, st);
        else if (s.D == 64) e = launch_dq<DH, 64>(s, maps, wqt, st_t, Wq, prm, st);
        else if (s.D == 128) e = launch_dq<DH, 128>(s, maps, wqt, st_t, Wq, prm, st);
        else e = cudaErrorNotSupported;
        timing_end(ts, st);
        if (e != cudaSuccess) return e;
        ++*launches;
    }
    // key kernels: 128-row key boxes, 64-row query / dO boxes
    CUtensorMap mk128, mv128, mq64, mdo64, mkh128, mvh128;
    ok = make_map(&mk128, k, DH, s.N, BK, 128) && make_map(&mv128, v, DH, s.N, BK, 128) &&
         make_map(&mq64, q, DH, s.N, BH, 64) && make_map(&mdo64, dO, DH, s.N, BH, 64);
    if (has_kept)
        ok = ok && make_map(&mkh128, khat, DH, (uint64_t)T * s.k, BK, 128) &&
             make_map(&mvh128, vhat, DH, (uint64_t)T * s.k, BK, 128);
    if (!ok) return cudaErrorInvalidValue;
    using Cfg = BwdKVCfg<DH>;
    {
        prm.n_ktiles = (s.N + 127) / 128;
        auto kern = bwd_dkv_tc_kernel<DH, false>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
        if (e != cudaSuccess) return e;
        const int ts = timing_begin(kTimeBwdDkv, st);
        kern<<<(unsigned)(prm.n_ktiles * BK), Cfg::THREADS, Cfg::SMEM, st>>>(mk128, mv128, mq64, mdo64, prm);
        timing_end(ts, st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        ++*launches;
    }
    if (has_kept && (s.m() + 1) * s.C < s.N) {  // some query chunk decides chunk 0
        // kept entries of chunks c with some deciding query chunk (c + m + 1 <= last chunk); the
        // query rows of each 128-entry tile are split into segments so the long early tiles spread
        prm.n_ktiles = (T * s.k + 127) / 128;
        prm.seg_rows = 1024;
        const int n_segs = (s.N + prm.seg_rows - 1) / prm.seg_rows;
        auto kern = bwd_dkv_tc_kernel<DH, true>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
        if (e != cudaSuccess) return e;
        const int ts = timing_begin(kTimeBwdDkv, st);
        kern<<<(unsigned)((uint64_t)n_segs * prm.n_ktiles * BK), Cfg::THREADS, Cfg::SMEM, st>>>(mkh128, mvh128, mq64,
                                                                                                mdo64, prm);
        timing_end(ts, st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        ++*launches;
    }
    return cudaSuccess;
}

}  // namespace

bool tc_backward_supported(const Dims &s) {
    return s.bf16 && s.w > 0 && (s.d == 64 || s.d == 128) && s.C % 128 == 0 && s.N > 0;
}

// Softmax branch of the backward pass on tensor cores: dq (written), the rows' L and D, then dk, dv
// (window keys written, kept keys added).  The rows' linear terms come from the pre-pass (lden, dl)
// or, with pro.wqt set (D in {64, 128}), from the dq kernel's own prologue, which also writes
// phi(q) and S_t dO (pro.Phi, pro.SG) for the linear branch.
cudaError_t launch_backward_tc(const Dims &s, const void *q, const void *k, const void *v, const void *khat,
                               const void *vhat, const int32_t *idx, const void *dO, const float *lden,
                               const float *dl, const BwdPrologue &pro, float *L, float *Dv, float *dq, float *dk,
                               float *dv, unsigned *err, cudaStream_t st, int *launches) {
    BwdParams prm{};
    prm.B = s.B;
    prm.H = s.H;
    prm.Hkv = s.Hkv;
    prm.N = s.N;
    prm.C = s.C;
    prm.k = s.k;
    prm.w = s.w;
    prm.G = s.G();
    prm.T = s.T();
    prm.scale = s.scale;
    prm.scale_log2 = s.scale * kLog2e;
    prm.lden = lden;
    prm.dl = dl;
    prm.z = pro.z;
    prm.Phi = pro.Phi;
    prm.SG = pro.SG;
    prm.L = L;
    prm.Dv = Dv;
    prm.lse_in = pro.lse_fwd;
    prm.o_in = static_cast<const __nv_bfloat16 *>(pro.o_fwd);
    prm.dq = dq;
    prm.dk = dk;
    prm.dv = dv;
    prm.idx = idx;
    prm.err = err;
    if (s.d == 64) return launch_bwd_cfg<64>(s, q, k, v, khat, vhat, dO, pro.wqt, pro.st_t, pro.Wq, prm, st, launches);
    if (s.d == 128)
        return launch_bwd_cfg<128>(s, q, k, v, khat, vhat, dO, pro.wqt, pro.st_t, pro.Wq, prm, st, launches);
    return cudaErrorNotSupported;
}

}  // namespace still
