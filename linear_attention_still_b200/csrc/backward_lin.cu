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
//                      a = c phi(q) (-> A, in place of Phi), the NP-Map backward dy, then
//                      dq += dy Wq^T + (dn / ||q||) q and dWq += q^T dy (atomics)
//   bwd_chunk_tile:    R_t = sum over the rows of query chunk t (all heads of the group) of a_i dO_i^T,
//                      r_t = sum of a_i D_i
//   bwd_key_tile:      unselected keys of a decided chunk c: with R, r the suffix sums from chunk
//                      c + m + 1, dphi(k) = R v - r, dv += R^T phi(k), the NP-Map backward of k,
//                      dk += dy Wk^T + (dn / ||k||) k and dWk += k^T dy (atomics)
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

// dst[r][c] (row stride ld) = src[r][c] for r < rows (zero for r >= valid), c < cols.
template <typename T>
__device__ __forceinline__ void load_rows(float *dst, int ld, const T *src, size_t sld, int rows, int cols, int valid) {
    for (int e = threadIdx.x; e < rows * cols; e += kTileThreads) {
        const int r = e / cols, c = e % cols;
        dst[r * ld + c] = r < valid ? to_f(src[(size_t)r * sld + c]) : 0.f;
    }
}

// dst[c][r] (row stride ld) = src[r][c], the transpose of the same block.
template <typename T>
__device__ __forceinline__ void load_rows_t(float *dst, int ld, const T *src, size_t sld, int rows, int cols,
                                            int valid) {
    for (int e = threadIdx.x; e < rows * cols; e += kTileThreads) {
        const int r = e / cols, c = e % cols;
        dst[c * ld + r] = r < valid ? to_f(src[(size_t)r * sld + c]) : 0.f;
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

// NP-Map backward of one row (one warp; DF features, lane owns features lane + 32u): y = x W (fp32,
// shared), ||x||^2, the upstream dphi -> dy = dL/dy written to dy_out (shared, stride-1), returns
// dn / ||x|| (the coefficient of x in dL/dx; 0 when x = 0).
template <int DF>
__device__ __forceinline__ float npmap_bwd_row(const float *y, float xx, const float (&dphi)[DF / 32], float *dy_out,
                                               int lane) {
    float f[DF / 32];
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < DF / 32; ++u) mx = fmaxf(mx, y[lane + 32 * u]);
    mx = warp_max(mx);
    float se = 0.f;
#pragma unroll
    for (int u = 0; u < DF / 32; ++u) {
        f[u] = expf(y[lane + 32 * u] - mx);
        se += f[u];
    }
    se = warp_sum(se);
    const float ise = 1.f / se;
    float ff = 0.f;
#pragma unroll
    for (int u = 0; u < DF / 32; ++u) {
        f[u] *= ise;  // f = softmax(y)
        ff = fmaf(f[u], f[u], ff);
    }
    const float nf = sqrtf(warp_sum(ff)), inf_ = 1.f / nf;
    const float n = sqrtf(xx);
    // phi = n u, u = f / ||f||
    float dn = 0.f, udu = 0.f, du[DF / 32];
#pragma unroll
    for (int u = 0; u < DF / 32; ++u) {
        const float uu = f[u] * inf_;
        dn = fmaf(dphi[u], uu, dn);
        du[u] = n * dphi[u];
        udu = fmaf(uu, du[u], udu);
    }
    dn = warp_sum(dn);
    udu = warp_sum(udu);
    float fdf = 0.f;
#pragma unroll
    for (int u = 0; u < DF / 32; ++u) {
        du[u] = (du[u] - f[u] * inf_ * udu) * inf_;  // df
        fdf = fmaf(f[u], du[u], fdf);
    }
    fdf = warp_sum(fdf);
#pragma unroll
    for (int u = 0; u < DF / 32; ++u) dy_out[lane + 32 * u] = f[u] * (du[u] - fdf);  // dy = f (df - <f, df>)
    return n > 0.f ? dn / n : 0.f;
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
    // post: XT [DH][68], W then W^T ([DH][LDF] / [DF][LDH]), Y then dY [64][LDF], dYT [DF][68], coef [64]
    static constexpr int WBUF = DH * LDF > DF * LDH ? DH * LDF : DF * LDH;
    static constexpr int POST_FLOATS = DH * kLd64 + WBUF + 64 * LDF + DF * kLd64 + 64;
    // key: KT [DH][68] (then VT), W / W^T / R^T / R, Y [64][LDF] (then dphi, dY), PT [DF][68]
    // (phi(k)^T, then dY^T), coef [64], kept mask [64]
    static constexpr int RBUF = WBUF;
    static constexpr int KEY_FLOATS = DH * kLd64 + RBUF + 64 * LDF + DF * kLd64 + 128;
};

template <typename T, int DH, int DF>
__global__ void __launch_bounds__(kTileThreads) bwd_lin_pre_tile(Dims s, const T *__restrict__ q,
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
    load_rows_t(XT, kLd64, q + row0 * DH, DH, 64, DH, valid);
    load_rows(W, Cfg::LDF, Wq + (size_t)h * DH * DF, DF, DH, DF, DH);
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
    load_rows_t(XT, kLd64, dO + row0 * DH, DH, 64, DH, valid);
    load_rows_t(W, Cfg::LDF, S + tslot * DF * DH, DH, DF, DH, DF);  // W[x][a] = S[a][x]
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
__global__ void __launch_bounds__(kTileThreads) bwd_lin_post_tile(Dims s, const T *__restrict__ q,
                                                                  const T *__restrict__ Wq, const float *__restrict__ z,
                                                                  const float *__restrict__ L,
                                                                  const float *__restrict__ Dv, float *__restrict__ PhiA,
                                                                  const float *__restrict__ SG, float *__restrict__ dq,
                                                                  float *__restrict__ dWq) {
    using Cfg = LinTile<DH, DF>;
    extern __shared__ __align__(16) float sm[];
    float *XT = sm, *W = XT + DH * kLd64, *Y = W + Cfg::WBUF, *dYT = Y + 64 * Cfg::LDF, *coef = dYT + DF * kLd64;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntile = (s.N + 63) / 64;
    const int bh = blockIdx.x / ntile, i0 = (blockIdx.x % ntile) * 64;
    const int h = bh % s.H, b = bh / s.H, bg = b * s.Hkv + h / s.G();
    const int t = i0 / s.C;
    const int valid = min(64, s.N - i0);
    const size_t row0 = (size_t)bh * s.N + i0;
    const T *Wh = Wq + (size_t)h * DH * DF;
    load_rows_t(XT, kLd64, q + row0 * DH, DH, 64, DH, valid);
    load_rows(W, Cfg::LDF, Wh, DF, DH, DF, DH);
    __syncthreads();
    {
        float acc[1][DF / 64][4][4];
        zero_acc(acc);
        smem_mm<1, DF / 64>(XT, kLd64, W, Cfg::LDF, DH, acc);  // Y = X Wq
        store_tile(Y, Cfg::LDF, acc);
    }
    __syncthreads();
    load_rows_t(W, Cfg::LDH, Wh, DF, DH, DF, DH);  // W^T [DF][DH] for dX = dY Wq^T
    const float *zt = z + ((size_t)bg * (s.T() + 1) + t) * DF;
    for (int r = warp; r < 64; r += 8) {
        float dphi[DF / 32];
        const size_t row = row0 + r;
        const bool live = r < valid;
        const float c = live ? exp2f(-L[row]) : 0.f, Di = live ? Dv[row] : 0.f;
#pragma unroll
        for (int u = 0; u < DF / 32; ++u) {
            const int a = lane + 32 * u;
            dphi[u] = live ? c * (SG[row * DF + a] - Di * zt[a]) : 0.f;
            if (live) PhiA[row * DF + a] *= c;
        }
        // dy over y (row r of Y), then into dYT[c][r]
        float *yr = Y + r * Cfg::LDF;
        const float cf = npmap_bwd_row<DF>(yr, col_sqnorm<DH>(XT, kLd64, r, lane), dphi, yr, lane);
        __syncwarp();
#pragma unroll
        for (int u = 0; u < DF / 32; ++u) dYT[(lane + 32 * u) * kLd64 + r] = yr[lane + 32 * u];
        if (lane == 0) coef[r] = cf;
    }
    __syncthreads();
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
    {
        // dq += dY Wq^T + coef q
        float acc[1][DH / 64][4][4];
        zero_acc(acc);
        smem_mm<1, DH / 64>(dYT, kLd64, W, Cfg::LDH, DF, acc);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ty * 4 + i;
            if (r >= valid) continue;
#pragma unroll
            for (int nu = 0; nu < DH / 64; ++nu) {
                const int x = tx * 4 + 64 * nu;
                float4 *dst = reinterpret_cast<float4 *>(dq + (row0 + r) * DH + x);
                float4 v = *dst;
                v.x += acc[0][nu][i][0] + coef[r] * XT[(x + 0) * kLd64 + r];
                v.y += acc[0][nu][i][1] + coef[r] * XT[(x + 1) * kLd64 + r];
                v.z += acc[0][nu][i][2] + coef[r] * XT[(x + 2) * kLd64 + r];
                v.w += acc[0][nu][i][3] + coef[r] * XT[(x + 3) * kLd64 + r];
                *dst = v;
            }
        }
    }
    __syncthreads();
    {
        // dWq += X^T dY: AT[k = row][x] = q rows (re-read into W's buffer), B = dY [row][c] (in Y)
        float *Xr = W;
        load_rows(Xr, Cfg::LDH, q + row0 * DH, DH, 64, DH, valid);
        __syncthreads();
        float acc[DH / 64][DF / 64][4][4];
        zero_acc(acc);
        smem_mm<DH / 64, DF / 64>(Xr, Cfg::LDH, Y, Cfg::LDF, 64, acc);
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
}

// R_t (D x d) and r_t (D) of query chunk t for (b, g): sum over the chunk's rows of all G heads.
template <typename T, int DH, int DF>
__global__ void __launch_bounds__(kTileThreads) bwd_chunk_tile(Dims s, const float *__restrict__ A,
                                                               const float *__restrict__ Dv, const T *__restrict__ dO,
                                                               float *__restrict__ R, float *__restrict__ rr) {
    extern __shared__ __align__(16) float sm[];
    // R_t[a][x] = sum_i A[i][a] dO[i][x]: the reduction runs over the rows, so both tiles stay row-major
    float *Ar = sm, *Gt = Ar + 64 * (DF + 4), *Ds = Gt + 64 * (DH + 4);
    const int T_ = s.T(), G = s.G();
    const int bg = blockIdx.x / (T_ + 1), t = blockIdx.x % (T_ + 1);
    const int b = bg / s.Hkv, g = bg % s.Hkv;
    const int i_lo = t * s.C, i_hi = min(s.N, i_lo + s.C);
    float acc[DF / 64][DH / 64][4][4];
    zero_acc(acc);
    float racc = 0.f;
    for (int hh = 0; hh < G; ++hh) {
        const size_t rb = ((size_t)b * s.H + g * G + hh) * s.N;
        for (int i0 = i_lo; i0 < i_hi; i0 += 64) {
            const int valid = min(64, i_hi - i0);
            __syncthreads();
            load_rows(Ar, DF + 4, A + (rb + i0) * DF, DF, 64, DF, valid);
            load_rows(Gt, DH + 4, dO + (rb + i0) * DH, DH, 64, DH, valid);
            if (threadIdx.x < 64) Ds[threadIdx.x] = (int)threadIdx.x < valid ? Dv[rb + i0 + threadIdx.x] : 0.f;
            __syncthreads();
            smem_mm<DF / 64, DH / 64>(Ar, DF + 4, Gt, DH + 4, 64, acc);
            if (threadIdx.x < DF)
                for (int r = 0; r < 64; ++r) racc = fmaf(Ar[r * (DF + 4) + threadIdx.x], Ds[r], racc);
        }
    }
    const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
    const size_t slot = (size_t)bg * (T_ + 1) + t;
#pragma unroll
    for (int mu = 0; mu < DF / 64; ++mu)
#pragma unroll
        for (int nu = 0; nu < DH / 64; ++nu)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                *reinterpret_cast<float4 *>(R + (slot * DF + ty * 4 + 64 * mu + i) * DH + tx * 4 + 64 * nu) =
                    make_float4(acc[mu][nu][i][0], acc[mu][nu][i][1], acc[mu][nu][i][2], acc[mu][nu][i][3]);
    if (threadIdx.x < DF) rr[slot * DF + threadIdx.x] = racc;
}

// Unselected keys of 64-key tiles of decided chunks: dphi(k) = R v - r, dv += R^T phi(k),
// NP-Map backward of k: dk += dy Wk^T + coef k, dWk += k^T dy.
template <typename T, int DH, int DF>
__global__ void __launch_bounds__(kTileThreads) bwd_key_tile(Dims s, const T *__restrict__ k, const T *__restrict__ v,
                                                             const T *__restrict__ Wk, const int32_t *__restrict__ idx,
                                                             const float *__restrict__ phik,
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
    // dphi = V R^T - r: V^T over KT, R^T [x][a] over Wb
    load_rows_t(KT, kLd64, v + row0 * DH, DH, 64, DH, 64);
    load_rows_t(Wb, Cfg::LDF, Rs, DH, DF, DH, DF);
    __syncthreads();
    {
        float acc[1][DF / 64][4][4];
        zero_acc(acc);
        smem_mm<1, DF / 64>(KT, kLd64, Wb, Cfg::LDF, DH, acc);
        store_tile(Y, Cfg::LDF, acc);  // Y <- V R^T (r subtracted below)
    }
    __syncthreads();
    // dv += phi(k) R: phi(k)^T over PT, R [a][x] over Wb
    load_rows_t(PT, kLd64, phik + row0 * DF, DF, 64, DF, 64);
    load_rows(Wb, Cfg::LDH, Rs, DH, DF, DH, DF);
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
    // Y_k = K Wk (into PT's buffer, row-major [64][LDF]; PT is free) with K^T over KT, Wk over Wb
    float *Yk = PT;
    static_assert(64 * (DF + 4) <= DF * kLd64, "Yk fits PT");
    load_rows_t(KT, kLd64, k + row0 * DH, DH, 64, DH, 64);
    load_rows(Wb, Cfg::LDF, Wg, DF, DH, DF, DH);
    __syncthreads();
    {
        float acc[1][DF / 64][4][4];
        zero_acc(acc);
        smem_mm<1, DF / 64>(KT, kLd64, Wb, Cfg::LDF, DH, acc);
        store_tile(Yk, Cfg::LDF, acc);
    }
    __syncthreads();
    // per key row: dy of the NP-Map (over Y's row: dphi there is consumed first), coef
    for (int r = warp; r < 64; r += 8) {
        float dphi[DF / 32];
        const bool on = !keep[r];
#pragma unroll
        for (int u = 0; u < DF / 32; ++u) {
            const int a = lane + 32 * u;
            dphi[u] = on ? Y[r * Cfg::LDF + a] - rs[a] : 0.f;
        }
        __syncwarp();
        const float cf = npmap_bwd_row<DF>(Yk + r * Cfg::LDF, col_sqnorm<DH>(KT, kLd64, r, lane), dphi,
                                           Y + r * Cfg::LDF, lane);
        if (lane == 0) coef[r] = on ? cf : 0.f;
    }
    __syncthreads();
    // dk += dY Wk^T + coef k: dY^T over PT (Yk no longer needed), Wk^T over Wb
    load_rows_t(PT, kLd64, Y, Cfg::LDF, 64, DF, 64);
    load_rows_t(Wb, Cfg::LDH, Wg, DF, DH, DF, DH);
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
        load_rows(Wb, Cfg::LDH, k + row0 * DH, DH, 64, DH, 64);
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
    // which == 1: query side after the softmax pass, the chunk sums, their suffix, the key side
    if ((e = cudaMemsetAsync(dWq, 0, sizeof(float) * (size_t)s.H * DH * DF, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dWk, 0, sizeof(float) * (size_t)s.Hkv * DH * DF, st)) != cudaSuccess) return e;
    if ((e = prep((const void *)bwd_lin_post_tile<T, DH, DF>, Cfg::POST_FLOATS)) != cudaSuccess) return e;
    bwd_lin_post_tile<T, DH, DF><<<qgrid, kTileThreads, Cfg::POST_FLOATS * 4, st>>>(
        s, (const T *)q, (const T *)Wq, w.z, w.L, w.Dv, w.A, w.dYq, dq, dWq);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int T_ = s.T();
    const int chunk_floats = 64 * (DF + 4) + 64 * (DH + 4) + 64;
    if ((e = prep((const void *)bwd_chunk_tile<T, DH, DF>, chunk_floats)) != cudaSuccess) return e;
    bwd_chunk_tile<T, DH, DF><<<(unsigned)((size_t)s.B * s.Hkv * (T_ + 1)), kTileThreads, chunk_floats * 4, st>>>(
        s, w.A, w.Dv, (const T *)dO, w.R, w.r);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_bwd_suffix(s, w.R, w.r, st)) != cudaSuccess) return e;
    if (T_ > 0) {
        if ((e = prep((const void *)bwd_key_tile<T, DH, DF>, Cfg::KEY_FLOATS)) != cudaSuccess) return e;
        bwd_key_tile<T, DH, DF><<<(unsigned)((size_t)s.B * s.Hkv * (T_ * s.C / 64)), kTileThreads,
                                  Cfg::KEY_FLOATS * 4, st>>>(s, (const T *)k, (const T *)v, (const T *)Wk, idx, w.phik,
                                                             w.R, w.r, dk, dv, dWk);
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
// follows the softmax pass (dq, dWq, R_t, r_t, their suffix sums, dk, dv, dWk of the unselected keys).
cudaError_t launch_linear_backward_tiled(int which, const Dims &s, const void *q, const void *k, const void *v,
                                         const void *Wq, const void *Wk, const void *dO, const int32_t *idx,
                                         const BackwardScratch &w, float *dq, float *dk, float *dv, float *dWq,
                                         float *dWk, cudaStream_t st) {
    if (s.bf16)
        return launch_lin_t<__nv_bfloat16>(which, s, q, k, v, Wq, Wk, dO, idx, w, dq, dk, dv, dWq, dWk, st);
    return launch_lin_t<float>(which, s, q, k, v, Wq, Wk, dO, idx, w, dq, dk, dv, dWq, dWk, st);
}

}  // namespace still
