// backward_lin.cu -- the linear branch of the STILL layer's backward pass as tiled fp32 kernels
// (head dimension d and feature width D in {64, 128}; bf16 or fp32 storage).  "STILL: Selecting
// Tokens for Intra-Layer Hybrid Attention to Linearize LLMs": [p1] jsqmd.com introduction (the
// unselected tokens go to linear attention in the same layer) and "NP-Map" (phi(x) = ||x|| f(x W) /
// ||f(x W)||, f = softmax over the D features); [p4] atlas.scime.ai "Approach".
//
// Every kernel works on a 64-row tile of one (b, head) that lies inside one chunk, so the tile shares
// one linear state; its small products (64 x d x D) run from shared memory on a 16 x 16 thread grid
// with 4 x 4 register tiles (smem_mm), the per-row NP-Map steps on one warp per row.
//   bwd_lin_pre_tile:  phi(q) (-> Phi), lden = phi(q).z_t, sg = S_t dO (-> SG), dl = phi(q).sg
//   bwd_lin_post_tile: with L_i, D_i of the softmax pass: c = 2^-L, dphi = c (sg - D z_t),
//                      a = c phi(q) (-> A, in place of Phi), the NP-Map backward dy (from phi alone),
//                      then dq += dy Wq^T + (dn / ||q||) q, dWq += q^T dy, and the chunk sums of the
//                      key side R_t += a^T dO, r_t += a^T D over the tile's rows (atomics)
//   bwd_key_tile:      unselected keys of a decided chunk c: phi(k) from k Wk; with R, r the suffix
//                      sums from chunk c + m + 1, dv += R^T phi(k), dphi(k) = R v - r, the NP-Map
//                      backward of k, dk += dy Wk^T + (dn / ||k||) k and dWk += k^T dy (atomics)
#include "common.cuh"
#include "still_internal.h"

namespace still {

namespace {

constexpr int kTileThreads = 256;

// acc[mu][nu][i][j] += sum_k AT[k][r] B[k][c] for rows r = 4 ty + 64 mu + i and columns
// c = 4 tx + 64 nu + j, (ty, tx) = (tid / 16, tid % 16): the product A B with A stored transposed
// (row k of AT holds column k of A).  AT and B in shared memory with row strides lda and ldb
// (multiples of 4 floats).
template <int MU, int NU>
__device__ __forceinline__ void smem_mm(const float *AT, int lda, const float *B, int ldb, int K,
                                        float (&acc)[MU][NU][4][4]) {
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll 2
    for (int k = 0; k < K; ++k) {
        float4 a[MU], b[NU];
#pragma unroll
        for (int mu = 0; mu < MU; ++mu) a[mu] = *reinterpret_cast<const float4 *>(AT + k * lda + ty * 4 + 64 * mu);
#pragma unroll
        for (int nu = 0; nu < NU; ++nu) b[nu] = *reinterpret_cast<const float4 *>(B + k * ldb + tx * 4 + 64 * nu);
#pragma unroll
        for (int mu = 0; mu < MU; ++mu)
#pragma unroll
            for (int nu = 0; nu < NU; ++nu) {
                const float av[4] = {a[mu].x, a[mu].y, a[mu].z, a[mu].w};
                const float bv[4] = {b[nu].x, b[nu].y, b[nu].z, b[nu].w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[mu][nu][i][j] = fmaf(av[i], bv[j], acc[mu][nu][i][j]);
            }
    }
}

template <int MU, int NU>
__device__ __forceinline__ void zero_acc(float (&acc)[MU][NU][4][4]) {
#pragma unroll
    for (int mu = 0; mu < MU; ++mu)
#pragma unroll
        for (int nu = 0; nu < NU; ++nu)
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[mu][nu][i][j] = 0.f;
}

// 16 bytes of a row: 8 bf16 or 4 fp32 values, widened to fp32.
__device__ __forceinline__ void load16(const __nv_bfloat16 *p, float (&f)[8]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 t = __bfloat1622float2(h2[e]);
        f[2 * e] = t.x;
        f[2 * e + 1] = t.y;
    }
}
__device__ __forceinline__ void load16(const float *p, float (&f)[4]) {
    const float4 u = *reinterpret_cast<const float4 *>(p);
    f[0] = u.x;
    f[1] = u.y;
    f[2] = u.z;
    f[3] = u.w;
}

// dst[r][c] (row stride ld) = src[r][c] for r < ROWS (zero for r >= valid), c < COLS; rows of src
// start on 16-byte boundaries (sld elements apart).  One 16-byte load per thread and step.
template <int ROWS, int COLS, typename T>
__device__ __forceinline__ void load_rows(float *dst, int ld, const T *src, size_t sld, int valid) {
    constexpr int V = 16 / (int)sizeof(T), VPR = COLS / V;
    static_assert(COLS % V == 0, "whole 16-byte vectors per row");
#pragma unroll 2
    for (int e = threadIdx.x; e < ROWS * VPR; e += kTileThreads) {
        const int r = e / VPR, cv = e % VPR;
        float f[V];
        if (r < valid) {
            load16(src + (size_t)r * sld + cv * V, f);
        } else {
#pragma unroll
            for (int j = 0; j < V; ++j) f[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < V; j += 4)
            *reinterpret_cast<float4 *>(dst + r * ld + cv * V + j) = make_float4(f[j], f[j + 1], f[j + 2], f[j + 3]);
    }
}

// dst[c][r] (row stride ld) = src[r][c], the transpose of the same block.  Consecutive threads take
// consecutive rows, so the transposed shared-memory stores fall in consecutive banks.
template <int ROWS, int COLS, typename T>
__device__ __forceinline__ void load_rows_t(float *dst, int ld, const T *src, size_t sld, int valid) {
    constexpr int V = 16 / (int)sizeof(T), VPR = COLS / V;
    static_assert(COLS % V == 0 && ROWS % 32 == 0, "whole vectors, whole warps per column strip");
#pragma unroll 2
    for (int e = threadIdx.x; e < ROWS * VPR; e += kTileThreads) {
        const int r = e % ROWS, cv = e / ROWS;
        float f[V];
        if (r < valid) {
            load16(src + (size_t)r * sld + cv * V, f);
        } else {
#pragma unroll
            for (int j = 0; j < V; ++j) f[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < V; ++j) dst[(cv * V + j) * ld + r] = f[j];
    }
}

// Writes the register tile acc (64 x N rows x columns) into shared memory dst[r][c] (stride ld).
template <int MU, int NU>
__device__ __forceinline__ void store_tile(float *dst, int ld, const float (&acc)[MU][NU][4][4]) {
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
    for (int mu = 0; mu < MU; ++mu)
#pragma unroll
        for (int nu = 0; nu < NU; ++nu)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                *reinterpret_cast<float4 *>(dst + (ty * 4 + 64 * mu + i) * ld + tx * 4 + 64 * nu) =
                    make_float4(acc[mu][nu][i][0], acc[mu][nu][i][1], acc[mu][nu][i][2], acc[mu][nu][i][3]);
}

// NP-Map backward of one row from phi itself (one warp; lane owns features lane + 32u): phi is a
// positive multiple of f = softmax(y), so f = phi / sum(phi), ||x|| = ||phi|| and phi / ||x|| =
// f / ||f||; x = 0 (phi = 0) has zero gradient.  Returns dn / ||x||, dy into dy.
template <int DF>
__device__ __forceinline__ float npmap_bwd_from_phi(const float (&ph)[DF / 32], const float (&dphi)[DF / 32],
                                                    float (&dy)[DF / 32]) {
    float sp = 0.f, pp = 0.f;
#pragma unroll
    for (int u = 0; u < DF / 32; ++u) {
        sp += ph[u];
        pp = fmaf(ph[u], ph[u], pp);
    }
    sp = warp_sum(sp);
    const float n = sqrtf(warp_sum(pp));
    if (!(n > 0.f)) {
#pragma unroll
        for (int u = 0; u < DF / 32; ++u) dy[u] = 0.f;
        return 0.f;
    }
    const float isp = 1.f / sp, in = 1.f / n, inf_ = sp * in;  // 1 / ||f|| = sum(phi) / ||phi||
    float dn = 0.f, udu = 0.f, du[DF / 32];
#pragma unroll
    for (int u = 0; u < DF / 32; ++u) {
        const float uu = ph[u] * in;  // u = f / ||f|| = phi / ||phi||
        dn = fmaf(dphi[u], uu, dn);
        du[u] = n * dphi[u];
        udu = fmaf(uu, du[u], udu);
    }
    dn = warp_sum(dn);
    udu = warp_sum(udu);
    float fdf = 0.f;
#pragma unroll
    for (int u = 0; u < DF / 32; ++u) {
        du[u] = (du[u] - ph[u] * in * udu) * inf_;  // df
        fdf = fmaf(ph[u] * isp, du[u], fdf);
    }
    fdf = warp_sum(fdf);
#pragma unroll
    for (int u = 0; u < DF / 32; ++u) dy[u] = ph[u] * isp * (du[u] - fdf);  // dy = f (df - <f, df>)
    return dn * in;
}

// phi(x) of one row (one warp) from y = x W (shared, DF values) and ||x||^2: ||x|| e / ||e||,
// e = exp(y - max y); the lane's features into ph.
template <int DF>
__device__ __forceinline__ void npmap_fwd_row(const float *y, float xx, float (&ph)[DF / 32], int lane) {
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < DF / 32; ++u) mx = fmaxf(mx, y[lane + 32 * u]);
    mx = warp_max(mx);
    float ee = 0.f;
#pragma unroll
    for (int u = 0; u < DF / 32; ++u) {
        ph[u] = expf(y[lane + 32 * u] - mx);
        ee = fmaf(ph[u], ph[u], ee);
    }
    const float f = sqrtf(xx) / sqrtf(warp_sum(ee));
#pragma unroll
    for (int u = 0; u < DF / 32; ++u) ph[u] *= f;
}

// ||x||^2 of row r of a transposed tile XT[x][r] (stride ld), DH values, by one warp.
template <int DH>
__device__ __forceinline__ float col_sqnorm(const float *XT, int ld, int r, int lane) {
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < DH / 32; ++u) {
        const float v = XT[(lane + 32 * u) * ld + r];
        acc = fmaf(v, v, acc);
    }
    return warp_sum(acc);
}

constexpr int kLd64 = 64 + 4;  // stride of a [.][64-row] transposed tile

template <int DH, int DF>
struct LinTile {
    static constexpr int LDH = DH + 4, LDF = DF + 4;
    // pre:  XT/GT [DH][68], W/ST [DH][LDF], Y [64][LDF]
    static constexpr int PRE_FLOATS = DH * kLd64 + DH * LDF + 64 * LDF;
    // post: q rows [64][LDH], Wq^T [DF][LDH] (then dO rows), dY^T [DF][68] (then A rows),
    // dY [64][LDF], coef [64], D [64]
    static constexpr int WBUF = DH * LDF > DF * LDH ? DH * LDF : DF * LDH;
    static constexpr int POST_FLOATS = 64 * LDH + WBUF + DF * kLd64 + 64 * LDF + 128;
    // sums: q rows [64][LDH], dY rows [64][LDF], dO rows [64][LDH], a rows [64][LDF], D [64]
    static constexpr int SUMS_FLOATS = 2 * 64 * LDH + 2 * 64 * LDF + 64;
    // key: KT [DH][68] (K^T, V^T, K^T), Wk / R / R^T / Wk^T / K rows, Y [64][LDF] (Y_k, phi(k), dY),
    // PT [DF][68] (phi(k)^T, dphi rows, dY^T), coef [64], kept mask [64]
    static constexpr int RBUF = WBUF;
    static constexpr int KEY_FLOATS = DH * kLd64 + RBUF + 64 * LDF + DF * kLd64 + 128;
    // three CTAs per SM where the shared memory allows it (d = D = 64: at most 70 KB each)
    static constexpr int MIN_BLOCKS = DH == 64 && DF == 64 ? 3 : 1;
};

template <typename T, int DH, int DF>
__global__ void __launch_bounds__(kTileThreads, LinTile<DH, DF>::MIN_BLOCKS) bwd_lin_pre_tile(Dims s, const T *__restrict__ q,
                                                                 const T *__restrict__ Wq, const float *__restrict__ S,
                                                                 const float *__restrict__ z, const T *__restrict__ dO,
                                                                 float *__restrict__ Phi, float *__restrict__ SG,
                                                                 float *__restrict__ lden, float *__restrict__ dl) {
    using Cfg = LinTile<DH, DF>;
    extern __shared__ __align__(16) float sm[];
    float *XT = sm, *W = XT + DH * kLd64, *Y = W + DH * Cfg::LDF;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntile = (s.N + 63) / 64;
    const int bh = blockIdx.x / ntile, i0 = (blockIdx.x % ntile) * 64;
    const int h = bh % s.H, b = bh / s.H, bg = b * s.Hkv + h / s.G();
    const int t = i0 / s.C;
    const int valid = min(64, s.N - i0);
    const size_t row0 = (size_t)bh * s.N + i0;
    const size_t tslot = (size_t)bg * (s.T() + 1) + t;
    load_rows_t<64, DH>(XT, kLd64, q + row0 * DH, DH, valid);
    load_rows<DH, DF>(W, Cfg::LDF, Wq + (size_t)h * DH * DF, DF, DH);
    __syncthreads();
    {
        float acc[1][DF / 64][4][4];
        zero_acc(acc);
        smem_mm<1, DF / 64>(XT, kLd64, W, Cfg::LDF, DH, acc);  // Y = X Wq
        store_tile(Y, Cfg::LDF, acc);
    }
    __syncthreads();
    // phi(q) per row (in place of Y), lden; the sq-norms read the q tile before it is replaced
    const float *zt = z + tslot * DF;
    for (int r = warp; r < 64; r += 8) {
        float ph[DF / 32];
        npmap_fwd_row<DF>(Y + r * Cfg::LDF, col_sqnorm<DH>(XT, kLd64, r, lane), ph, lane);
        float ld = 0.f;
#pragma unroll
        for (int u = 0; u < DF / 32; ++u) {
            Y[r * Cfg::LDF + lane + 32 * u] = ph[u];
            ld = fmaf(ph[u], zt[lane + 32 * u], ld);
            if (r < valid) Phi[(row0 + r) * DF + lane + 32 * u] = ph[u];
        }
        ld = warp_sum(ld);
        if (lane == 0 && r < valid) lden[row0 + r] = ld;
    }
    __syncthreads();
    // sg = dO S_t^T: dO^T over the q tile, S_t^T over Wq
    load_rows_t<64, DH>(XT, kLd64, dO + row0 * DH, DH, valid);
    load_rows_t<DF, DH>(W, Cfg::LDF, S + tslot * DF * DH, DH, DF);  // W[x][a] = S[a][x]
    __syncthreads();
    float acc[1][DF / 64][4][4];
    zero_acc(acc);
    smem_mm<1, DF / 64>(XT, kLd64, W, Cfg::LDF, DH, acc);
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty * 4 + i;
        float part = 0.f;
#pragma unroll
        for (int nu = 0; nu < DF / 64; ++nu) {
            const int c = tx * 4 + 64 * nu;
            const float4 ph = *reinterpret_cast<const float4 *>(Y + r * Cfg::LDF + c);
            part += ph.x * acc[0][nu][i][0] + ph.y * acc[0][nu][i][1] + ph.z * acc[0][nu][i][2] + ph.w * acc[0][nu][i][3];
            if (r < valid)
                *reinterpret_cast<float4 *>(SG + (row0 + r) * DF + c) =
                    make_float4(acc[0][nu][i][0], acc[0][nu][i][1], acc[0][nu][i][2], acc[0][nu][i][3]);
        }
        // the 16 threads of a row tile are one half-warp
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (tx == 0 && r < valid) dl[row0 + r] = part;
    }
}

template <typename T, int DH, int DF>
__global__ void __launch_bounds__(kTileThreads, LinTile<DH, DF>::MIN_BLOCKS) bwd_lin_post_tile(Dims s, const T *__restrict__ q,
                                                                  const T *__restrict__ Wq, const T *__restrict__ dO,
                                                                  const float *__restrict__ z,
                                                                  const float *__restrict__ L,
                                                                  const float *__restrict__ Dv, float *__restrict__ PhiA,
                                                                  const float *__restrict__ SG, float *__restrict__ dq,
                                                                  float *__restrict__ dWq, float *__restrict__ R,
                                                                  float *__restrict__ rr) {
    using Cfg = LinTile<DH, DF>;
    extern __shared__ __align__(16) float sm[];
    float *Xr = sm, *WT = Xr + 64 * Cfg::LDH, *dYT = WT + Cfg::WBUF, *dY = dYT + DF * kLd64, *coef = dY + 64 * Cfg::LDF,
          *Ds = coef + 64;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntile = (s.N + 63) / 64;
    const int bh = blockIdx.x / ntile, i0 = (blockIdx.x % ntile) * 64;
    const int h = bh % s.H, b = bh / s.H, bg = b * s.Hkv + h / s.G();
    const int t = i0 / s.C;
    const int valid = min(64, s.N - i0);
    const size_t row0 = (size_t)bh * s.N + i0;
    const size_t tslot = (size_t)bg * (s.T() + 1) + t;
    const T *Wh = Wq + (size_t)h * DH * DF;
    load_rows<64, DH>(Xr, Cfg::LDH, q + row0 * DH, DH, valid);
    load_rows_t<DH, DF>(WT, Cfg::LDH, Wh, DF, DH);  // Wq^T [DF][DH]
    // per row: c = 2^-L, dphi = c (sg - D z_t), a = c phi (global, read back below), NP-Map backward
    // from phi itself (f = phi / sum(phi), ||q|| = ||phi||)
    const float *zt = z + tslot * DF;
    for (int r = warp; r < 64; r += 8) {
        const size_t row = row0 + r;
        const bool live = r < valid;
        const float c = live ? exp2f(-L[row]) : 0.f, Di = live ? Dv[row] : 0.f;
        float ph[DF / 32], dphi[DF / 32], dy[DF / 32];
#pragma unroll
        for (int u = 0; u < DF / 32; ++u) {
            const int a = lane + 32 * u;
            ph[u] = live ? PhiA[row * DF + a] : 0.f;
            dphi[u] = live ? c * (SG[row * DF + a] - Di * zt[a]) : 0.f;
            if (live) PhiA[row * DF + a] = c * ph[u];
        }
        const float cf = npmap_bwd_from_phi<DF>(ph, dphi, dy);
#pragma unroll
        for (int u = 0; u < DF / 32; ++u) {
            dY[r * Cfg::LDF + lane + 32 * u] = dy[u];
            dYT[(lane + 32 * u) * kLd64 + r] = dy[u];
        }
        if (lane == 0) {
            coef[r] = cf;
            Ds[r] = Di;
        }
    }
    __syncthreads();
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
    {
        // dq += dY Wq^T + coef q
        float acc[1][DH / 64][4][4];
        zero_acc(acc);
        smem_mm<1, DH / 64>(dYT, kLd64, WT, Cfg::LDH, DF, acc);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ty * 4 + i;
            if (r >= valid) continue;
#pragma unroll
            for (int nu = 0; nu < DH / 64; ++nu) {
                const int x = tx * 4 + 64 * nu;
                const float4 xq = *reinterpret_cast<const float4 *>(Xr + r * Cfg::LDH + x);
                float4 *dst = reinterpret_cast<float4 *>(dq + (row0 + r) * DH + x);
                float4 v = *dst;
                v.x += acc[0][nu][i][0] + coef[r] * xq.x;
                v.y += acc[0][nu][i][1] + coef[r] * xq.y;
                v.z += acc[0][nu][i][2] + coef[r] * xq.z;
                v.w += acc[0][nu][i][3] + coef[r] * xq.w;
                *dst = v;
            }
        }
    }
    {
        // dWq += X^T dY (the q rows, the dY rows)
        float acc[DH / 64][DF / 64][4][4];
        zero_acc(acc);
        smem_mm<DH / 64, DF / 64>(Xr, Cfg::LDH, dY, Cfg::LDF, 64, acc);
        float *dW = dWq + (size_t)h * DH * DF;
#pragma unroll
        for (int mu = 0; mu < DH / 64; ++mu)
#pragma unroll
            for (int nu = 0; nu < DF / 64; ++nu)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    atomicAdd(reinterpret_cast<float4 *>(dW + (size_t)(ty * 4 + 64 * mu + i) * DF + tx * 4 + 64 * nu),
                              make_float4(acc[mu][nu][i][0], acc[mu][nu][i][1], acc[mu][nu][i][2], acc[mu][nu][i][3]));
    }
    __syncthreads();
    {
        // the chunk sums of the key side: R_t += A^T dO, r_t += A^T D over the tile's rows (a = c phi
        // rows over dYT's buffer, dO rows over Wq^T's)
        float *Ar = dYT, *Go = WT;
        static_assert(64 * (DF + 4) <= DF * kLd64, "A rows fit the dY^T buffer");
        load_rows<64, DF>(Ar, Cfg::LDF, PhiA + row0 * DF, DF, valid);
        load_rows<64, DH>(Go, Cfg::LDH, dO + row0 * DH, DH, valid);
        __syncthreads();
        float acc[DF / 64][DH / 64][4][4];
        zero_acc(acc);
        smem_mm<DF / 64, DH / 64>(Ar, Cfg::LDF, Go, Cfg::LDH, 64, acc);
        float *Rt = R + tslot * DF * DH;
#pragma unroll
        for (int mu = 0; mu < DF / 64; ++mu)
#pragma unroll
            for (int nu = 0; nu < DH / 64; ++nu)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    atomicAdd(reinterpret_cast<float4 *>(Rt + (size_t)(ty * 4 + 64 * mu + i) * DH + tx * 4 + 64 * nu),
                              make_float4(acc[mu][nu][i][0], acc[mu][nu][i][1], acc[mu][nu][i][2], acc[mu][nu][i][3]));
        if (threadIdx.x < DF) {
            float racc = 0.f;
            for (int r = 0; r < 64; ++r) racc = fmaf(Ar[r * Cfg::LDF + threadIdx.x], Ds[r], racc);
            atomicAdd(rr + tslot * DF + threadIdx.x, racc);
        }
    }
}

// The query side's sums once the dq kernel has formed dY and a (its epilogue): dWq += q^T dY and the
// key side's chunk sums R_t += a^T dO, r_t += a^T D over the tile's 64 rows (atomics).
template <typename T, int DH, int DF>
__global__ void __launch_bounds__(kTileThreads, LinTile<DH, DF>::MIN_BLOCKS) bwd_lin_sums_tile(
    Dims s, const T *__restrict__ q, const T *__restrict__ dO, const float *__restrict__ Dv,
    const float *__restrict__ A, const float *__restrict__ dY, float *__restrict__ dWq, float *__restrict__ R,
    float *__restrict__ rr) {
    using Cfg = LinTile<DH, DF>;
    extern __shared__ __align__(16) float sm[];
    float *Xr = sm, *Yr = Xr + 64 * Cfg::LDH, *Go = Yr + 64 * Cfg::LDF, *Ar = Go + 64 * Cfg::LDH,
          *Ds = Ar + 64 * Cfg::LDF;
    const int ntile = (s.N + 63) / 64;
    const int bh = blockIdx.x / ntile, i0 = (blockIdx.x % ntile) * 64;
    const int h = bh % s.H, b = bh / s.H, bg = b * s.Hkv + h / s.G();
    const int t = i0 / s.C;
    const int valid = min(64, s.N - i0);
    const size_t row0 = (size_t)bh * s.N + i0;
    const size_t tslot = (size_t)bg * (s.T() + 1) + t;
    load_rows<64, DH>(Xr, Cfg::LDH, q + row0 * DH, DH, valid);
    load_rows<64, DF>(Yr, Cfg::LDF, dY + row0 * DF, DF, valid);
    load_rows<64, DH>(Go, Cfg::LDH, dO + row0 * DH, DH, valid);
    load_rows<64, DF>(Ar, Cfg::LDF, A + row0 * DF, DF, valid);
    if (threadIdx.x < 64) Ds[threadIdx.x] = (int)threadIdx.x < valid ? Dv[row0 + threadIdx.x] : 0.f;
    __syncthreads();
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
    {
        float acc[DH / 64][DF / 64][4][4];
        zero_acc(acc);
        smem_mm<DH / 64, DF / 64>(Xr, Cfg::LDH, Yr, Cfg::LDF, 64, acc);
        float *dW = dWq + (size_t)h * DH * DF;
#pragma unroll
        for (int mu = 0; mu < DH / 64; ++mu)
#pragma unroll
            for (int nu = 0; nu < DF / 64; ++nu)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    atomicAdd(reinterpret_cast<float4 *>(dW + (size_t)(ty * 4 + 64 * mu + i) * DF + tx * 4 + 64 * nu),
                              make_float4(acc[mu][nu][i][0], acc[mu][nu][i][1], acc[mu][nu][i][2], acc[mu][nu][i][3]));
    }
    {
        float acc[DF / 64][DH / 64][4][4];
        zero_acc(acc);
        smem_mm<DF / 64, DH / 64>(Ar, Cfg::LDF, Go, Cfg::LDH, 64, acc);
        float *Rt = R + tslot * DF * DH;
#pragma unroll
        for (int mu = 0; mu < DF / 64; ++mu)
#pragma unroll
            for (int nu = 0; nu < DH / 64; ++nu)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    atomicAdd(reinterpret_cast<float4 *>(Rt + (size_t)(ty * 4 + 64 * mu + i) * DH + tx * 4 + 64 * nu),
                              make_float4(acc[mu][nu][i][0], acc[mu][nu][i][1], acc[mu][nu][i][2], acc[mu][nu][i][3]));
        if (threadIdx.x < DF) {
            float racc = 0.f;
            for (int r = 0; r < 64; ++r) racc = fmaf(Ar[r * Cfg::LDF + threadIdx.x], Ds[r], racc);
            atomicAdd(rr + tslot * DF + threadIdx.x, racc);
        }
    }
}

// Unselected keys of 64-key tiles of decided chunks: phi(k) from K Wk, dv += phi(k) R,
// dphi(k) = V R^T - r, the NP-Map backward from phi(k): dk += dy Wk^T + coef k, dWk += k^T dy.
template <typename T, int DH, int DF>
__global__ void __launch_bounds__(kTileThreads, LinTile<DH, DF>::MIN_BLOCKS) bwd_key_tile(Dims s, const T *__restrict__ k, const T *__restrict__ v,
                                                             const T *__restrict__ Wk, const int32_t *__restrict__ idx,
                                                             const float *__restrict__ R, const float *__restrict__ rr,
                                                             float *__restrict__ dk, float *__restrict__ dv,
                                                             float *__restrict__ dWk) {
    using Cfg = LinTile<DH, DF>;
    extern __shared__ __align__(16) float sm[];
    float *KT = sm, *Wb = KT + DH * kLd64, *Y = Wb + Cfg::RBUF, *PT = Y + 64 * Cfg::LDF, *coef = PT + DF * kLd64;
    int *keep = reinterpret_cast<int *>(coef + 64);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T_ = s.T(), m = s.m();
    const int per = T_ * s.C / 64;  // 64-key tiles of the full chunks
    const int bg = blockIdx.x / per, j0 = (blockIdx.x % per) * 64;
    const int g = bg % s.Hkv;
    const int c = j0 / s.C;
    if (c + m + 1 > T_) return;  // no query chunk decides this chunk (uniform over the CTA)
    const size_t row0 = (size_t)bg * s.N + j0;
    const size_t slot = (size_t)bg * (T_ + 1) + c + m + 1;
    const float *Rs = R + slot * DF * DH, *rs = rr + slot * DF;
    const T *Wg = Wk + (size_t)g * DH * DF;
    // kept rows of the tile (their linear-branch gradient is zero)
    if (threadIdx.x < 64) keep[threadIdx.x] = 0;
    __syncthreads();
    if (s.k > 0)
        for (int n = threadIdx.x; n < s.k; n += kTileThreads) {
            const int j = idx[((size_t)bg * T_ + c) * s.k + n] - j0;
            if (j >= 0 && j < 64) keep[j] = 1;
        }
    // Y_k = K Wk, then phi(k) per row (row-major over Y, transposed into PT)
    load_rows_t<64, DH>(KT, kLd64, k + row0 * DH, DH, 64);
    load_rows<DH, DF>(Wb, Cfg::LDF, Wg, DF, DH);
    __syncthreads();
    {
        float acc[1][DF / 64][4][4];
        zero_acc(acc);
        smem_mm<1, DF / 64>(KT, kLd64, Wb, Cfg::LDF, DH, acc);
        store_tile(Y, Cfg::LDF, acc);
    }
    __syncthreads();
    for (int r = warp; r < 64; r += 8) {
        float ph[DF / 32];
        npmap_fwd_row<DF>(Y + r * Cfg::LDF, col_sqnorm<DH>(KT, kLd64, r, lane), ph, lane);
        __syncwarp();
#pragma unroll
        for (int u = 0; u < DF / 32; ++u) {
            Y[r * Cfg::LDF + lane + 32 * u] = ph[u];
            PT[(lane + 32 * u) * kLd64 + r] = ph[u];
        }
    }
    // dv += phi(k) R (R [a][x] over Wb)
    load_rows<DF, DH>(Wb, Cfg::LDH, Rs, DH, DF);
    __syncthreads();
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
    {
        float acc[1][DH / 64][4][4];
        zero_acc(acc);
        smem_mm<1, DH / 64>(PT, kLd64, Wb, Cfg::LDH, DF, acc);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ty * 4 + i;
            if (keep[r]) continue;
#pragma unroll
            for (int nu = 0; nu < DH / 64; ++nu) {
                float4 *dst = reinterpret_cast<float4 *>(dv + (row0 + r) * DH + tx * 4 + 64 * nu);
                float4 w = *dst;
                w.x += acc[0][nu][i][0];
                w.y += acc[0][nu][i][1];
                w.z += acc[0][nu][i][2];
                w.w += acc[0][nu][i][3];
                *dst = w;
            }
        }
    }
    __syncthreads();
    // dphi = V R^T (row-major over PT; r subtracted per row below): V^T over KT, R^T [x][a] over Wb
    float *dP = PT;
    static_assert(64 * (DF + 4) <= DF * kLd64, "dphi rows fit PT");
    load_rows_t<64, DH>(KT, kLd64, v + row0 * DH, DH, 64);
    load_rows_t<DF, DH>(Wb, Cfg::LDF, Rs, DH, DF);
    __syncthreads();
    {
        float acc[1][DF / 64][4][4];
        zero_acc(acc);
        smem_mm<1, DF / 64>(KT, kLd64, Wb, Cfg::LDF, DH, acc);
        store_tile(dP, Cfg::LDF, acc);
    }
    __syncthreads();
    // per key row: the NP-Map backward from phi(k) (row of Y), dy over the same row of Y
    for (int r = warp; r < 64; r += 8) {
        float ph[DF / 32], dphi[DF / 32], dy[DF / 32];
        const bool on = !keep[r];
#pragma unroll
        for (int u = 0; u < DF / 32; ++u) {
            const int a = lane + 32 * u;
            ph[u] = Y[r * Cfg::LDF + a];
            dphi[u] = on ? dP[r * Cfg::LDF + a] - rs[a] : 0.f;
        }
        const float cf = npmap_bwd_from_phi<DF>(ph, dphi, dy);
#pragma unroll
        for (int u = 0; u < DF / 32; ++u) Y[r * Cfg::LDF + lane + 32 * u] = dy[u];
        if (lane == 0) coef[r] = on ? cf : 0.f;
    }
    __syncthreads();
    // dk += dY Wk^T + coef k: dY^T over PT, Wk^T over Wb, K^T (for coef k) back over KT
    load_rows_t<64, DF>(PT, kLd64, Y, Cfg::LDF, 64);
    load_rows_t<DH, DF>(Wb, Cfg::LDH, Wg, DF, DH);
    load_rows_t<64, DH>(KT, kLd64, k + row0 * DH, DH, 64);
    __syncthreads();
    {
        float acc[1][DH / 64][4][4];
        zero_acc(acc);
        smem_mm<1, DH / 64>(PT, kLd64, Wb, Cfg::LDH, DF, acc);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ty * 4 + i;
            if (keep[r]) continue;
#pragma unroll
            for (int nu = 0; nu < DH / 64; ++nu) {
                const int x = tx * 4 + 64 * nu;
                float4 *dst = reinterpret_cast<float4 *>(dk + (row0 + r) * DH + x);
                float4 w = *dst;
                w.x += acc[0][nu][i][0] + coef[r] * KT[(x + 0) * kLd64 + r];
                w.y += acc[0][nu][i][1] + coef[r] * KT[(x + 1) * kLd64 + r];
                w.z += acc[0][nu][i][2] + coef[r] * KT[(x + 2) * kLd64 + r];
                w.w += acc[0][nu][i][3] + coef[r] * KT[(x + 3) * kLd64 + r];
                *dst = w;
            }
        }
    }
    __syncthreads();
    {
        // dWk += K^T dY: K rows over Wb, dY [row][a] in Y (kept rows are zero there: dphi = 0)
        load_rows<64, DH>(Wb, Cfg::LDH, k + row0 * DH, DH, 64);
        __syncthreads();
        float acc[DH / 64][DF / 64][4][4];
        zero_acc(acc);
        smem_mm<DH / 64, DF / 64>(Wb, Cfg::LDH, Y, Cfg::LDF, 64, acc);
        float *dW = dWk + (size_t)g * DH * DF;
#pragma unroll
        for (int mu = 0; mu < DH / 64; ++mu)
#pragma unroll
            for (int nu = 0; nu < DF / 64; ++nu)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    atomicAdd(reinterpret_cast<float4 *>(dW + (size_t)(ty * 4 + 64 * mu + i) * DF + tx * 4 + 64 * nu),
                              make_float4(acc[mu][nu][i][0], acc[mu][nu][i][1], acc[mu][nu][i][2], acc[mu][nu][i][3]));
    }
}

template <int DH, int DF, typename T>
cudaError_t launch_lin_cfg(int which, const Dims &s, const void *q, const void *k, const void *v, const void *Wq,
                           const void *Wk, const void *dO, const int32_t *idx, const BackwardScratch &w, float *dq,
                           float *dk, float *dv, float *dWq, float *dWk, cudaStream_t st) {
    using Cfg = LinTile<DH, DF>;
    const int ntile = (s.N + 63) / 64;
    const unsigned qgrid = (unsigned)((size_t)s.B * s.H * ntile);
    cudaError_t e;
    auto prep = [&](const void *kern, int floats) {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, floats * 4);
    };
    if (which == 0) {
        if ((e = prep((const void *)bwd_lin_pre_tile<T, DH, DF>, Cfg::PRE_FLOATS)) != cudaSuccess) return e;
        bwd_lin_pre_tile<T, DH, DF><<<qgrid, kTileThreads, Cfg::PRE_FLOATS * 4, st>>>(
            s, (const T *)q, (const T *)Wq, w.S, w.z, (const T *)dO, w.A, w.dYq, w.Ms, w.iZ);
        return cudaGetLastError();
    }
    // which == 1: query side after the softmax pass (with the chunk sums), their suffix, the key side;
    // which == 2: the same when the dq kernel has already formed dq, dY and a
    const int T_ = s.T();
    const size_t BK = (size_t)s.B * s.Hkv;
    if ((e = cudaMemsetAsync(dWq, 0, sizeof(float) * (size_t)s.H * DH * DF, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dWk, 0, sizeof(float) * (size_t)s.Hkv * DH * DF, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(w.R, 0, sizeof(float) * BK * (T_ + 1) * DF * DH, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(w.r, 0, sizeof(float) * BK * (T_ + 1) * DF, st)) != cudaSuccess) return e;
    if (which == 2) {
        // the dq kernel has formed dY and a (and dq): only the sums remain on the query side
        if ((e = prep((const void *)bwd_lin_sums_tile<T, DH, DF>, Cfg::SUMS_FLOATS)) != cudaSuccess) return e;
        bwd_lin_sums_tile<T, DH, DF><<<qgrid, kTileThreads, Cfg::SUMS_FLOATS * 4, st>>>(
            s, (const T *)q, (const T *)dO, w.Dv, w.A, w.dYq, dWq, w.R, w.r);
    } else {
        if ((e = prep((const void *)bwd_lin_post_tile<T, DH, DF>, Cfg::POST_FLOATS)) != cudaSuccess) return e;
        bwd_lin_post_tile<T, DH, DF><<<qgrid, kTileThreads, Cfg::POST_FLOATS * 4, st>>>(
            s, (const T *)q, (const T *)Wq, (const T *)dO, w.z, w.L, w.Dv, w.A, w.dYq, dq, dWq, w.R, w.r);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_bwd_suffix(s, w.R, w.r, st)) != cudaSuccess) return e;
    if (T_ > 0) {
        if ((e = prep((const void *)bwd_key_tile<T, DH, DF>, Cfg::KEY_FLOATS)) != cudaSuccess) return e;
        bwd_key_tile<T, DH, DF><<<(unsigned)(BK * (T_ * s.C / 64)), kTileThreads, Cfg::KEY_FLOATS * 4, st>>>(
            s, (const T *)k, (const T *)v, (const T *)Wk, idx, w.R, w.r, dk, dv, dWk);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <typename T>
cudaError_t launch_lin_t(int which, const Dims &s, const void *q, const void *k, const void *v, const void *Wq,
                         const void *Wk, const void *dO, const int32_t *idx, const BackwardScratch &w, float *dq,
                         float *dk, float *dv, float *dWq, float *dWk, cudaStream_t st) {
#define STILL_LIN(DH, DF)                                                                                   \
    if (s.d == DH && s.D == DF) return launch_lin_cfg<DH, DF, T>(which, s, q, k, v, Wq, Wk, dO, idx, w, dq, dk, dv, \
                                                                 dWq, dWk, st)
    STILL_LIN(64, 64);
    STILL_LIN(64, 128);
    STILL_LIN(128, 64);
    STILL_LIN(128, 128);
#undef STILL_LIN
    return cudaErrorNotSupported;
}

}  // namespace

bool tiled_linear_backward_supported(const Dims &s) {
    return (s.d == 64 || s.d == 128) && (s.D == 64 || s.D == 128) && s.C % 64 == 0;
}

// which = 0: the linear pre-pass (Phi, SG, lden, dl); which = 1: everything of the linear branch that
// follows the softmax pass (dq, dWq, R_t, r_t, their suffix sums, dk, dv, dWk of the unselected keys);
// which = 2: as 1 after a dq kernel with the linear prologue and epilogue (dq, dY and a formed there).
cudaError_t launch_linear_backward_tiled(int which, const Dims &s, const void *q, const void *k, const void *v,
                                         const void *Wq, const void *Wk, const void *dO, const int32_t *idx,
                                         const BackwardScratch &w, float *dq, float *dk, float *dv, float *dWq,
                                         float *dWk, cudaStream_t st) {
    if (s.bf16)
        return launch_lin_t<__nv_bfloat16>(which, s, q, k, v, Wq, Wk, dO, idx, w, dq, dk, dv, dWq, dWk, st);
    return launch_lin_t<float>(which, s, q, k, v, Wq, Wk, dO, idx, w, dq, dk, dv, dWq, dWk, st);
}

}  // namespace still
