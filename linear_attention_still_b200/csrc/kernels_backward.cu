// kernels_backward.cu -- backward pass of the STILL hybrid-attention layer ("STILL: Selecting Tokens
// for Intra-Layer Hybrid Attention to Linearize LLMs": [p1] jsqmd.com introduction and "Chunk-Wise"
// describe one chunk-parallel implementation for training and inference).  Gradients of
// L = <dO, o> with respect to q, k, v, Wq, Wk, with the per-chunk selection held fixed (a discrete
// choice with no gradient).  SIMT, fp32 arithmetic; written for correctness first.
//
// For query row i (head h of group g): softmax set Soft(i) = kept rows of the decided chunks ++ the
// local window, linear set Lin(i) = the other rows of the decided chunks; with the joint shift Ms,
//   P_ij = exp(s_ij - Ms) / Z   (j in Soft),   Z = sum_Soft exp(s_ij - Ms) + exp(-Ms) phi(q_i).z_t,
//   o_i = (sum_Soft exp(s_ij - Ms) v_j + exp(-Ms) phi(q_i)^T S_t) / Z,   D_i = <dO_i, o_i>.
// Then
//   dL/ds_ij = P_ij (<dO_i, v_j> - D_i)                  -> dq_i, dk_j (tau), dv_j += P_ij dO_i
//   dL/dphi(q_i) = c_i (S_t dO_i - D_i z_t), c_i = exp(-Ms)/Z
//   dL/dphi(k_j) = R_c v_j - r_c,  dv_j += R_c^T phi(k_j)    (j unselected in decided chunk c)
// with a_i = c_i phi(q_i), R_c = sum of a_i dO_i^T and r_c = sum of a_i D_i over the query rows of
// chunks t >= c+m+1 (a suffix sum over query chunks, the mirror of the forward linear state), and
// the NP-Map backward takes dphi to dx and dW.
#include "common.cuh"
#include "rowops.cuh"
#include "still_internal.h"

namespace still {
namespace {

constexpr int kBwdWarps = 4;

// Key number li of row i's softmax list: kept rows of chunks 0..t-m-1 (chunk order), then the
// window [lo, i].
// A kept index outside its chunk is reported and replaced by the chunk's first row (reads stay in
// bounds; the result is then not meaningful, as the error word says).
__device__ __forceinline__ int soft_key(const Dims &s, const int32_t *idx, int bg, int nk, int lo, int li,
                                        unsigned *err) {
    if (li < nk) {
        const int c = li / s.k;
        const int j = idx[((size_t)bg * s.T() + c) * s.k + li % s.k];
        if (j < c * s.C || j >= (c + 1) * s.C) {
            report(err, DEV_ERR_INDEX);
            return c * s.C;
        }
        return j;
    }
    return lo + (li - nk);
}

// NP-Map backward of one row by one warp: given x (fp32, smem, d values), W [d, D] (global) and
// dphi (smem, D values): writes dy = dL/d(xW) to dys (smem, D values) and returns through dx the
// lane's share of dL/dx (elements x = lane + 32u).
template <typename T>
__device__ void npmap_backward_warp(const float *xs, const T *__restrict__ W, int d, int D, const float *dphi,
                                    float *dys, float (&dx)[kMaxD / 32], int lane) {
    float y[kMaxDf / 32];
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < kMaxDf / 32; ++u) {
        const int c = lane + 32 * u;
        float acc = 0.f;
        if (c < D) {
            for (int a = 0; a < d; ++a) acc = fmaf(xs[a], to_f(W[(size_t)a * D + c]), acc);
            mx = fmaxf(mx, acc);
        }
        y[u] = acc;
    }
    mx = warp_max(mx);
    float se = 0.f;
#pragma unroll
    for (int u = 0; u < kMaxDf / 32; ++u) {
        const int c = lane + 32 * u;
        y[u] = c < D ? expf(y[u] - mx) : 0.f;
        se += y[u];
    }
    se = warp_sum(se);
    float ff = 0.f;  // ||f||^2
#pragma unroll
    for (int u = 0; u < kMaxDf / 32; ++u) {
        y[u] /= se;  // f
        ff = fmaf(y[u], y[u], ff);
    }
    const float nf = sqrtf(warp_sum(ff));
    float nx2 = 0.f;
    for (int a = lane; a < d; a += 32) nx2 = fmaf(xs[a], xs[a], nx2);
    const float n = sqrtf(warp_sum(nx2));
    // phi = n u, u = f / ||f||
    float dn = 0.f, udu = 0.f;
    float du[kMaxDf / 32];
#pragma unroll
    for (int u = 0; u < kMaxDf / 32; ++u) {
        const int c = lane + 32 * u;
        const float dp = c < D ? dphi[c] : 0.f;
        const float uu = y[u] / nf;
        dn = fmaf(dp, uu, dn);
        du[u] = n * dp;
        udu = fmaf(uu, du[u], udu);
    }
    dn = warp_sum(dn);
    udu = warp_sum(udu);
    float fdf = 0.f;
#pragma unroll
    for (int u = 0; u < kMaxDf / 32; ++u) {
        du[u] = (du[u] - (y[u] / nf) * udu) / nf;  // df
        fdf = fmaf(y[u], du[u], fdf);
    }
    fdf = warp_sum(fdf);
#pragma unroll
    for (int u = 0; u < kMaxDf / 32; ++u) {
        const int c = lane + 32 * u;
        if (c < D) dys[c] = y[u] * (du[u] - fdf);  // dy = f (df - <f, df>)
    }
    __syncwarp();
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) {
        const int a = lane + 32 * u;
        float acc = 0.f;
        if (a < d) {
            const T *wr = W + (size_t)a * D;
            for (int c = 0; c < D; ++c) acc = fmaf(to_f(wr[c]), dys[c], acc);
            if (n > 0.f) acc = fmaf(dn, xs[a] / n, acc);
        }
        dx[u] = acc;
    }
}

// One warp per query row (b, h, i): recomputes the row's forward, then dq_i (all of it), the
// softmax branch's contributions to dk and dv (atomics), a_i, D_i and dL/d(q_i Wq).
template <typename T, bool ATOMIC_KV>
__global__ void __launch_bounds__(32 * kBwdWarps) bwd_row_kernel(Dims s, const T *__restrict__ q,
                                                                 const T *__restrict__ k, const T *__restrict__ v,
                                                                 const T *__restrict__ Wq,
                                                                 const int32_t *__restrict__ idx,
                                                                 const float *__restrict__ S,
                                                                 const float *__restrict__ z,
                                                                 const T *__restrict__ dO, float *__restrict__ dq,
                                                                 float *__restrict__ dk, float *__restrict__ dv,
                                                                 float *__restrict__ Abuf, float *__restrict__ Dbuf,
                                                                 float *__restrict__ Msb, float *__restrict__ iZb,
                                                                 float *__restrict__ dYq, unsigned *err) {
    __shared__ __align__(16) float qs[kBwdWarps][kMaxD];
    __shared__ __align__(16) float gs[kBwdWarps][kMaxD];
    __shared__ __align__(16) float ps[kBwdWarps][kMaxDf];
    __shared__ __align__(16) float dps[kBwdWarps][kMaxDf];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kBwdWarps + warp;  // over B * H * N
    if (row >= (long long)s.B * s.H * s.N) return;
    const int d = s.d, D = s.D, G = s.G(), m = s.m(), T_ = s.T();
    const int i = (int)(row % s.N), h = (int)((row / s.N) % s.H), b = (int)(row / ((long long)s.N * s.H));
    const int g = h / G, bg = b * s.Hkv + g;
    const int t = i / s.C;
    const int nk = s.k * max(0, min(t - m, T_));
    const int lo = max(0, (t - m) * s.C);
    const int nsoft = nk + (i - lo + 1);
    const T *K = k + (size_t)bg * s.N * d, *Vv = v + (size_t)bg * s.N * d;
    for (int x = lane; x < d; x += 32) {
        qs[warp][x] = to_f(q[(size_t)row * d + x]);
        gs[warp][x] = to_f(dO[(size_t)row * d + x]);
    }
    __syncwarp();
    // ---- forward of the row: softmax part (online), linear part, shared normaliser
    float M = -INFINITY, Ls = 0.f;
    float acc[kMaxD / 32];
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) acc[u] = 0.f;
    for (int base = 0; base < nsoft; base += 32) {
        const int li = base + lane;
        int j = 0;
        float sc = -INFINITY;
        if (li < nsoft) {
            j = soft_key(s, idx, bg, nk, lo, li, err);
            sc = s.scale * dot_row(qs[warp], K + (size_t)j * d, d);
        }
        const float nm = fmaxf(M, warp_max(sc));
        const float so = M == -INFINITY ? 0.f : expf(M - nm);
        const float p = li < nsoft ? expf(sc - nm) : 0.f;
        Ls = Ls * so + warp_sum(p);
#pragma unroll
        for (int u = 0; u < kMaxD / 32; ++u) acc[u] *= so;
        const int cnt = min(32, nsoft - base);
        for (int jj = 0; jj < cnt; ++jj) {
            const float pj = __shfl_sync(0xffffffffu, p, jj);
            const int jr = __shfl_sync(0xffffffffu, j, jj);
#pragma unroll
            for (int u = 0; u < kMaxD / 32; ++u) {
                const int x = lane + 32 * u;
                if (x < d) acc[u] = fmaf(pj, to_f(Vv[(size_t)jr * d + x]), acc[u]);
            }
        }
        M = nm;
    }
    npmap_row_warp<T>(qs[warp], Wq + (size_t)h * d * D, d, D, ps[warp], lane);
    __syncwarp();
    const size_t tslot = (size_t)bg * (T_ + 1) + t;
    const float *St = S + tslot * D * d, *zt = z + tslot * D;
    float lden = 0.f;
    for (int a = lane; a < D; a += 32) lden = fmaf(ps[warp][a], zt[a], lden);
    lden = warp_sum(lden);
    float lin[kMaxD / 32];
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) {
        const int x = lane + 32 * u;
        float a_ = 0.f;
        if (x < d)
            for (int a = 0; a < D; ++a) a_ = fmaf(ps[warp][a], St[(size_t)a * d + x], a_);
        lin[u] = a_;
    }
    const float Ms = lden > 0.f ? fmaxf(M, logf(lden)) : M;
    const float a_soft = M == -INFINITY ? 0.f : expf(M - Ms);
    const float a_lin = expf(-Ms);
    const float Z = Ls * a_soft + lden * a_lin;
    const float invZ = Z > 0.f ? 1.f / Z : 0.f;
    float Di = 0.f;
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) {
        const int x = lane + 32 * u;
        if (x < d) Di = fmaf(gs[warp][x], (acc[u] * a_soft + lin[u] * a_lin) * invZ, Di);
    }
    Di = warp_sum(Di);
    if (lane == 0) {
        Msb[row] = Ms;
        iZb[row] = invZ;
    }
    // ---- softmax branch backward: dq here; dk and dv by atomics (ATOMIC_KV) or, from the stored
    //      Ms, 1/Z and D_i, in bwd_kv_block_kernel
    float dqa[kMaxD / 32];
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) dqa[u] = 0.f;
    float *dK = dk + (size_t)bg * s.N * d, *dV = dv + (size_t)bg * s.N * d;
    for (int base = 0; base < nsoft; base += 32) {
        const int li = base + lane;
        int j = 0;
        float P = 0.f, dS = 0.f;
        if (li < nsoft) {
            j = soft_key(s, idx, bg, nk, lo, li, err);
            const float sc = s.scale * dot_row(qs[warp], K + (size_t)j * d, d);
            const float gv = dot_row(gs[warp], Vv + (size_t)j * d, d);
            P = expf(sc - Ms) * invZ;
            dS = P * (gv - Di);
        }
        const int cnt = min(32, nsoft - base);
        for (int jj = 0; jj < cnt; ++jj) {
            const float Pj = __shfl_sync(0xffffffffu, P, jj);
            const float dSj = __shfl_sync(0xffffffffu, dS, jj) * s.scale;
            const int jr = __shfl_sync(0xffffffffu, j, jj);
#pragma unroll
            for (int u = 0; u < kMaxD / 32; ++u) {
                const int x = lane + 32 * u;
                if (x < d) {
                    dqa[u] = fmaf(dSj, to_f(K[(size_t)jr * d + x]), dqa[u]);
                    if (ATOMIC_KV) {
                        atomicAdd(dK + (size_t)jr * d + x, dSj * qs[warp][x]);
                        atomicAdd(dV + (size_t)jr * d + x, Pj * gs[warp][x]);
                    }
                }
            }
        }
    }
    // ---- linear branch backward on the query side: dphi(q) = c (S_t dO - D_i z_t), a_i = c phi(q)
    const float cl = a_lin * invZ;
    for (int a = lane; a < D; a += 32) {
        const float *sr = St + (size_t)a * d;
        float sg = 0.f;
        for (int x = 0; x < d; ++x) sg = fmaf(sr[x], gs[warp][x], sg);
        dps[warp][a] = cl * (sg - Di * zt[a]);
        Abuf[(size_t)row * D + a] = cl * ps[warp][a];
    }
    if (lane == 0) Dbuf[row] = Di;
    __syncwarp();
    float dxa[kMaxD / 32];
    npmap_backward_warp<T>(qs[warp], Wq + (size_t)h * d * D, d, D, dps[warp], ps[warp], dxa, lane);
    for (int c = lane; c < D; c += 32) dYq[(size_t)row * D + c] = ps[warp][c];
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) {
        const int x = lane + 32 * u;
        if (x < d) dq[(size_t)row * d + x] = dqa[u] + dxa[u];
    }
}

// Softmax branch, key side, by blocks of 32 keys of one (b, g) (d <= 128): the CTA streams the
// query rows that attend to its keys through shared memory 32 at a time (q, dO and the row's Ms,
// 1/Z, D_i), and thread (key kk, quarter sl of the head dim) accumulates its quarter of dk_j and
// dv_j in registers:  P_ij = exp(tau <q_i, k_j> - Ms_i) / Z_i,  dS_ij = tau P_ij (<dO_i, v_j> - D_i),
// dk_j += dS_ij q_i,  dv_j += P_ij dO_i  (dot products reduced over the 4 threads of a key).
//   KEPT = false: keys j0..j0+31 of the sequence, queries from j0 to the end of the last key's window
//   reach (chunks c .. c+m), each pair masked by i >= j and t(i) <= c(j) + m; writes dk, dv.
//   KEPT = true: 32 kept keys of chunk c (entries of idx), queries of chunks t >= c+m+1 (every pair
//   counts); adds to dk, dv.
template <typename T, int DH, bool KEPT>
__global__ void __launch_bounds__(128) bwd_kv_block_kernel(Dims s, const T *__restrict__ q,
                                                           const T *__restrict__ k, const T *__restrict__ v,
                                                           const int32_t *__restrict__ idx,
                                                           const T *__restrict__ dO, const float *__restrict__ Msb,
                                                           const float *__restrict__ iZb,
                                                           const float *__restrict__ Dbuf, float *__restrict__ dk,
                                                           float *__restrict__ dv) {
    constexpr int QT = 32, SL = DH / 4;
    __shared__ __align__(16) float qt[QT][DH];
    __shared__ __align__(16) float gt[QT][DH];
    __shared__ float st[QT][4];  // Ms, 1/Z, D, chunk of the row
    const int tid = threadIdx.x, kk = tid >> 2, sl = tid & 3;
    const int bg = blockIdx.y, b = bg / s.Hkv, g = bg % s.Hkv, G = s.G(), m = s.m(), T_ = s.T();
    int j = -1, cj = 0;
    int i0, i1;
    if (!KEPT) {
        const int j0 = blockIdx.x * QT;
        if (j0 + kk < s.N) j = j0 + kk;
        const int jl = min(s.N, j0 + QT) - 1;
        i0 = j0;
        i1 = min(s.N, (jl / s.C + m + 1) * s.C);
        cj = j >= 0 ? j / s.C : 0;
    } else {
        const int c = blockIdx.x / ((s.k + QT - 1) / QT), n0 = (blockIdx.x % ((s.k + QT - 1) / QT)) * QT;
        if (n0 + kk < s.k) j = idx[((size_t)bg * T_ + c) * s.k + n0 + kk];
        if (j >= 0 && (j < c * s.C || j >= (c + 1) * s.C)) j = -1;  // outside its chunk: skipped
        i0 = (c + m + 1) * s.C;
        i1 = s.N;
        cj = c;
    }
    float kr[SL], vr[SL], dka[SL], dva[SL];
#pragma unroll
    for (int e = 0; e < SL; ++e) {
        kr[e] = j >= 0 ? to_f(k[((size_t)bg * s.N + j) * DH + sl * SL + e]) : 0.f;
        vr[e] = j >= 0 ? to_f(v[((size_t)bg * s.N + j) * DH + sl * SL + e]) : 0.f;
        dka[e] = dva[e] = 0.f;
    }
    for (int hh = 0; hh < G; ++hh) {
        const size_t rb = ((size_t)b * s.H + (size_t)g * G + hh) * s.N;
        for (int ib = i0; ib < i1; ib += QT) {
            const int nq = min(QT, i1 - ib);
            __syncthreads();  // the previous tile is consumed
            for (int e = tid; e < QT * DH; e += 128) {
                const int r = e / DH, x = e % DH;
                qt[r][x] = r < nq ? to_f(q[(rb + ib + r) * DH + x]) : 0.f;
                gt[r][x] = r < nq ? to_f(dO[(rb + ib + r) * DH + x]) : 0.f;
            }
            if (tid < QT) {
                const int i = ib + tid;
                st[tid][0] = tid < nq ? Msb[rb + i] : 0.f;
                st[tid][1] = tid < nq ? iZb[rb + i] : 0.f;
                st[tid][2] = tid < nq ? Dbuf[rb + i] : 0.f;
                st[tid][3] = (float)(i / s.C);
            }
            __syncthreads();
            for (int r = 0; r < nq; ++r) {
                float sp = 0.f, gp = 0.f;
#pragma unroll
                for (int e = 0; e < SL; ++e) {
                    sp = fmaf(qt[r][sl * SL + e], kr[e], sp);
                    gp = fmaf(gt[r][sl * SL + e], vr[e], gp);
                }
                sp += __shfl_xor_sync(0xffffffffu, sp, 1);
                sp += __shfl_xor_sync(0xffffffffu, sp, 2);
                gp += __shfl_xor_sync(0xffffffffu, gp, 1);
                gp += __shfl_xor_sync(0xffffffffu, gp, 2);
                const int i = ib + r;
                bool on = j >= 0;
                if (!KEPT) on = on && i >= j && (int)st[r][3] <= cj + m;
                const float P = on ? expf(s.scale * sp - st[r][0]) * st[r][1] : 0.f;
                const float dS = s.scale * P * (gp - st[r][2]);
#pragma unroll
                for (int e = 0; e < SL; ++e) {
                    dka[e] = fmaf(dS, qt[r][sl * SL + e], dka[e]);
                    dva[e] = fmaf(P, gt[r][sl * SL + e], dva[e]);
                }
            }
        }
    }
    if (j >= 0) {
        float *dkr = dk + ((size_t)bg * s.N + j) * DH + sl * SL, *dvr = dv + ((size_t)bg * s.N + j) * DH + sl * SL;
#pragma unroll
        for (int e = 0; e < SL; ++e) {
            if (KEPT) {
                dkr[e] += dka[e];
                dvr[e] += dva[e];
            } else {
                dkr[e] = dka[e];
                dvr[e] = dva[e];
            }
        }
    }
}

template <typename T, int DH>
cudaError_t launch_kv_blocks(const Dims &s, const T *Q, const T *K, const T *V, const int32_t *idx, const T *GO,
                             const BackwardScratch &w, float *dk, float *dv, cudaStream_t st) {
    bwd_kv_block_kernel<T, DH, false><<<dim3((s.N + 31) / 32, s.B * s.Hkv), 128, 0, st>>>(
        s, Q, K, V, idx, GO, w.Ms, w.iZ, w.Dv, dk, dv);
    const int nc = s.T() - s.m() - 1 >= 0 ? s.T() - s.m() : 0;  // chunks c with c + m + 1 <= T
    if (s.k > 0 && nc > 0)
        bwd_kv_block_kernel<T, DH, true><<<dim3(nc * ((s.k + 31) / 32), s.B * s.Hkv), 128, 0, st>>>(
            s, Q, K, V, idx, GO, w.Ms, w.iZ, w.Dv, dk, dv);
    return cudaGetLastError();
}

// Per (b, g, query chunk t): R_t = sum over the chunk's rows of all G heads of a_i dO_i^T (D x d)
// and r_t = sum a_i D_i (D).  Slots t = 0..T (T holds the trailing partial chunk).
template <typename T>
__global__ void __launch_bounds__(256) bwd_chunk_kernel(Dims s, const float *__restrict__ Abuf,
                                                        const float *__restrict__ Dbuf, const T *__restrict__ dO,
                                                        float *__restrict__ R, float *__restrict__ r) {
    const int bg = blockIdx.y, t = blockIdx.x, b = bg / s.Hkv, g = bg % s.Hkv, G = s.G();
    const int d = s.d, D = s.D, T_ = s.T();
    const int i0 = t * s.C, i1 = min(s.N, i0 + s.C);
    const size_t slot = (size_t)bg * (T_ + 1) + t;
    for (int e = blockIdx.z * blockDim.x + threadIdx.x; e < D * d + D; e += gridDim.z * blockDim.x) {
        float acc = 0.f;
        for (int hh = 0; hh < G; ++hh) {
            const size_t rb = ((size_t)b * s.H + g * G + hh) * s.N;
            if (e < D * d) {
                const int a = e / d, x = e % d;
                for (int i = i0; i < i1; ++i) acc = fmaf(Abuf[(rb + i) * D + a], to_f(dO[(rb + i) * d + x]), acc);
            } else {
                const int a = e - D * d;
                for (int i = i0; i < i1; ++i) acc = fmaf(Abuf[(rb + i) * D + a], Dbuf[rb + i], acc);
            }
        }
        if (e < D * d) R[slot * D * d + e] = acc;
        else r[slot * D + (e - D * d)] = acc;
    }
}

// In place: R_t <- sum over t' >= t of R_t' (and r), for every (b, g) entry.
__global__ void bwd_suffix_kernel(Dims s, float *__restrict__ R, float *__restrict__ r) {
    const int T_ = s.T(), Dd = s.D * s.d, per = Dd + s.D;
    const size_t gid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (size_t)s.B * s.Hkv * per) return;
    const size_t bg = gid / per;
    const int e = (int)(gid % per);
    float run = 0.f;
    for (int t = T_; t >= 0; --t) {
        float *p = e < Dd ? &R[(bg * (T_ + 1) + t) * Dd + e] : &r[(bg * (T_ + 1) + t) * s.D + (e - Dd)];
        run += *p;
        *p = run;
    }
}

// One warp per key row j of a full chunk c that some query chunk decides (c + m + 1 <= T) and that
// was not kept: the linear branch's dphi(k_j) = R v_j - r and dv_j += R^T phi(k_j) with
// R = suffix(c + m + 1), then the NP-Map backward of k_j.
template <typename T>
__global__ void __launch_bounds__(32 * kBwdWarps) bwd_key_kernel(Dims s, const T *__restrict__ k,
                                                                 const T *__restrict__ v, const T *__restrict__ Wk,
                                                                 const int32_t *__restrict__ idx,
                                                                 const float *__restrict__ phik,
                                                                 const float *__restrict__ R,
                                                                 const float *__restrict__ r, float *__restrict__ dk,
                                                                 float *__restrict__ dv, float *__restrict__ dYk) {
    __shared__ __align__(16) float ks[kBwdWarps][kMaxD];
    __shared__ __align__(16) float vs[kBwdWarps][kMaxD];
    __shared__ __align__(16) float dps[kBwdWarps][kMaxDf];
    __shared__ __align__(16) float dys[kBwdWarps][kMaxDf];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kBwdWarps + warp;  // over B * Hkv * T * C
    const int T_ = s.T(), m = s.m(), d = s.d, D = s.D;
    if (row >= (long long)s.B * s.Hkv * T_ * s.C) return;
    const int j = (int)(row % ((long long)T_ * s.C));
    const int bg = (int)(row / ((long long)T_ * s.C)), g = bg % s.Hkv;
    const int c = j / s.C;
    if (c + m + 1 > T_) return;
    if (s.k > 0) {
        bool kept = false;
        for (int n = lane; n < s.k; n += 32) kept |= idx[((size_t)bg * T_ + c) * s.k + n] == j;
        if (__any_sync(0xffffffffu, kept)) return;
    }
    const size_t krow = (size_t)bg * s.N + j;
    for (int x = lane; x < d; x += 32) {
        ks[warp][x] = to_f(k[krow * d + x]);
        vs[warp][x] = to_f(v[krow * d + x]);
    }
    __syncwarp();
    const size_t slot = (size_t)bg * (T_ + 1) + (c + m + 1);
    const float *Rs = R + slot * D * d, *rs = r + slot * D;
    const float *ph = phik + krow * D;
    for (int a = lane; a < D; a += 32) {
        const float *rr = Rs + (size_t)a * d;
        float acc = 0.f;
        for (int x = 0; x < d; ++x) acc = fmaf(rr[x], vs[warp][x], acc);
        dps[warp][a] = acc - rs[a];
    }
    for (int x = lane; x < d; x += 32) {
        float acc = 0.f;
        for (int a = 0; a < D; ++a) acc = fmaf(Rs[(size_t)a * d + x], ph[a], acc);
        dv[krow * d + x] += acc;
    }
    __syncwarp();
    float dxa[kMaxD / 32];
    npmap_backward_warp<T>(ks[warp], Wk + (size_t)g * d * D, d, D, dps[warp], dys[warp], dxa, lane);
    for (int cc = lane; cc < D; cc += 32) dYk[krow * D + cc] = dys[warp][cc];
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) {
        const int x = lane + 32 * u;
        if (x < d) dk[krow * d + x] += dxa[u];
    }
}

// dW[hx][x][c] = sum over batch and rows of X[b, hx, row, x] * dY[b, hx, row, c].
template <typename T>
__global__ void __launch_bounds__(256) bwd_weight_kernel(int B, int Hx, int N, int d, int D, const T *__restrict__ X,
                                                         const float *__restrict__ dY, float *__restrict__ dW) {
    const int hx = blockIdx.y, x = blockIdx.x;
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
        float acc = 0.f;
        for (int b = 0; b < B; ++b) {
            const size_t base = ((size_t)b * Hx + hx) * N;
            for (int i = 0; i < N; ++i) acc = fmaf(to_f(X[(base + i) * d + x]), dY[(base + i) * D + c], acc);
        }
        dW[((size_t)hx * d + x) * D + c] = acc;
    }
}

// Linear branch of one query row before the tensor-core softmax passes (one warp per row):
// phi(q_i) -> Phi, sg_i = S_t dO_i -> SG, lden_i = phi(q_i).z_t and dl_i = <phi(q_i)^T S_t, dO_i> =
// phi(q_i).sg_i (the two linear terms of the row's normaliser and of D_i).
template <typename T>
__global__ void __launch_bounds__(32 * kBwdWarps) bwd_lin_pre_kernel(Dims s, const T *__restrict__ q,
                                                                     const T *__restrict__ Wq,
                                                                     const float *__restrict__ S,
                                                                     const float *__restrict__ z,
                                                                     const T *__restrict__ dO, float *__restrict__ Phi,
                                                                     float *__restrict__ SG, float *__restrict__ lden,
                                                                     float *__restrict__ dl) {
    __shared__ __align__(16) float qs[kBwdWarps][kMaxD];
    __shared__ __align__(16) float gs[kBwdWarps][kMaxD];
    __shared__ __align__(16) float ps[kBwdWarps][kMaxDf];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kBwdWarps + warp;  // over B * H * N
    if (row >= (long long)s.B * s.H * s.N) return;
    const int d = s.d, D = s.D, G = s.G(), T_ = s.T();
    const int i = (int)(row % s.N), h = (int)((row / s.N) % s.H), b = (int)(row / ((long long)s.N * s.H));
    const int bg = b * s.Hkv + h / G, t = i / s.C;
    for (int x = lane; x < d; x += 32) {
        qs[warp][x] = to_f(q[(size_t)row * d + x]);
        gs[warp][x] = to_f(dO[(size_t)row * d + x]);
    }
    __syncwarp();
    npmap_row_warp<T>(qs[warp], Wq + (size_t)h * d * D, d, D, ps[warp], lane);
    __syncwarp();
    const size_t tslot = (size_t)bg * (T_ + 1) + t;
    const float *St = S + tslot * D * d, *zt = z + tslot * D;
    float ld = 0.f, dd = 0.f;
    for (int a = lane; a < D; a += 32) {
        const float sg = dot_row(gs[warp], St + (size_t)a * d, d);
        const float ph = ps[warp][a];
        ld = fmaf(ph, zt[a], ld);
        dd = fmaf(ph, sg, dd);
        Phi[(size_t)row * D + a] = ph;
        SG[(size_t)row * D + a] = sg;
    }
    ld = warp_sum(ld);
    dd = warp_sum(dd);
    if (lane == 0) {
        lden[row] = ld;
        dl[row] = dd;
    }
}

// Linear branch of one query row after the softmax passes (one warp per row), from the row's log2
// normaliser L_i and D_i: c_i = 2^-L_i = exp(-Ms)/Z, dphi(q_i) = c_i (S_t dO_i - D_i z_t), then the
// NP-Map backward (dq += dL/dq, dY -> dYq) and a_i = c_i phi(q_i) (in place of Phi) for the key side.
template <typename T>
__global__ void __launch_bounds__(32 * kBwdWarps) bwd_lin_post_kernel(Dims s, const T *__restrict__ q,
                                                                      const T *__restrict__ Wq,
                                                                      const float *__restrict__ z,
                                                                      const float *__restrict__ L,
                                                                      const float *__restrict__ Dv,
                                                                      float *__restrict__ PhiA,
                                                                      float *__restrict__ SGdY, float *__restrict__ dq) {
    __shared__ __align__(16) float qs[kBwdWarps][kMaxD];
    __shared__ __align__(16) float dps[kBwdWarps][kMaxDf];
    __shared__ __align__(16) float dys[kBwdWarps][kMaxDf];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kBwdWarps + warp;  // over B * H * N
    if (row >= (long long)s.B * s.H * s.N) return;
    const int d = s.d, D = s.D, G = s.G(), T_ = s.T();
    const int i = (int)(row % s.N), h = (int)((row / s.N) % s.H), b = (int)(row / ((long long)s.N * s.H));
    const int bg = b * s.Hkv + h / G, t = i / s.C;
    for (int x = lane; x < d; x += 32) qs[warp][x] = to_f(q[(size_t)row * d + x]);
    const float c = exp2f(-L[row]), Di = Dv[row];
    const float *zt = z + ((size_t)bg * (T_ + 1) + t) * D;
    for (int a = lane; a < D; a += 32) {
        dps[warp][a] = c * (SGdY[(size_t)row * D + a] - Di * zt[a]);
        PhiA[(size_t)row * D + a] *= c;
    }
    __syncwarp();
    float dxa[kMaxD / 32];
    npmap_backward_warp<T>(qs[warp], Wq + (size_t)h * d * D, d, D, dps[warp], dys[warp], dxa, lane);
    for (int cc = lane; cc < D; cc += 32) SGdY[(size_t)row * D + cc] = dys[warp][cc];
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) {
        const int x = lane + 32 * u;
        if (x < d) dq[(size_t)row * d + x] += dxa[u];
    }
}

// ------------------------------------------------------------------ w = 0 (no softmax window)
// Every key j <= i is in the linear set of row i (pure causal linear attention with the NP-Map):
// with w_ij = <phi(q_i), phi(k_j)>, Z_i = sum_{j<=i} w_ij, o_i = sum_{j<=i} w_ij v_j / Z_i,
// D_i = <dO_i, o_i> and a_i = phi(q_i) / Z_i,
//   dphi(q_i) = (sum_{j<=i} phi(k_j) (<v_j, dO_i> - D_i)) / Z_i,
//   dphi(k_j) = sum_{i>=j} a_i (<dO_i, v_j> - D_i),   dv_j = sum_{i>=j} <a_i, phi(k_j)> dO_i.
// The sums over earlier chunks come from the chunk states S_t, z_t (prefix) and R_t, r_t (suffix);
// the rows of a key's own chunk are summed explicitly.  SIMT, fp32, correct-first.

// One warp per query row: o_i, D_i, a_i, the NP-Map backward of q (dq written, dYq).
template <typename T>
__global__ void __launch_bounds__(32 * kBwdWarps) bwd_nowin_row_kernel(Dims s, const T *__restrict__ q,
                                                                       const T *__restrict__ v,
                                                                       const T *__restrict__ Wq,
                                                                       const float *__restrict__ phik,
                                                                       const float *__restrict__ S,
                                                                       const float *__restrict__ z,
                                                                       const T *__restrict__ dO, float *__restrict__ dq,
                                                                       float *__restrict__ Abuf, float *__restrict__ Dbuf,
                                                                       float *__restrict__ dYq) {
    __shared__ __align__(16) float qs[kBwdWarps][kMaxD];
    __shared__ __align__(16) float gs[kBwdWarps][kMaxD];
    __shared__ __align__(16) float ps[kBwdWarps][kMaxDf];
    __shared__ __align__(16) float dps[kBwdWarps][kMaxDf];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * kBwdWarps + warp;  // over B * H * N
    if (row >= (long long)s.B * s.H * s.N) return;
    const int d = s.d, D = s.D, G = s.G(), T_ = s.T();
    const int i = (int)(row % s.N), h = (int)((row / s.N) % s.H), b = (int)(row / ((long long)s.N * s.H));
    const int bg = b * s.Hkv + h / G, t = i / s.C, c0 = t * s.C;
    for (int x = lane; x < d; x += 32) {
        qs[warp][x] = to_f(q[(size_t)row * d + x]);
        gs[warp][x] = to_f(dO[(size_t)row * d + x]);
    }
    __syncwarp();
    npmap_row_warp<T>(qs[warp], Wq + (size_t)h * d * D, d, D, ps[warp], lane);
    __syncwarp();
    const size_t tslot = (size_t)bg * (T_ + 1) + t;
    const float *St = S + tslot * D * d, *zt = z + tslot * D;
    const T *Vb = v + (size_t)bg * s.N * d;
    const float *Pk = phik + (size_t)bg * s.N * D;
    // pass 1: Z and the numerator (lane holds elements x = lane + 32u)
    float Z = 0.f;
    for (int a = lane; a < D; a += 32) Z = fmaf(ps[warp][a], zt[a], Z);
    Z = warp_sum(Z);
    float num[kMaxD / 32];
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) {
        const int x = lane + 32 * u;
        float acc = 0.f;
        if (x < d)
            for (int a = 0; a < D; ++a) acc = fmaf(ps[warp][a], St[(size_t)a * d + x], acc);
        num[u] = acc;
    }
    for (int j = c0; j <= i; ++j) {
        float wj = 0.f;
        for (int a = lane; a < D; a += 32) wj = fmaf(ps[warp][a], Pk[(size_t)j * D + a], wj);
        wj = warp_sum(wj);
        Z += wj;
#pragma unroll
        for (int u = 0; u < kMaxD / 32; ++u) {
            const int x = lane + 32 * u;
            if (x < d) num[u] = fmaf(wj, to_f(Vb[(size_t)j * d + x]), num[u]);
        }
    }
    const float iZ = Z > 0.f ? 1.f / Z : 0.f;
    float Di = 0.f;
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) {
        const int x = lane + 32 * u;
        if (x < d) Di = fmaf(gs[warp][x], num[u] * iZ, Di);
    }
    Di = warp_sum(Di);
    // pass 2: dphi(q) = (S_t dO - D z_t + sum_j phi(k_j) (<v_j, dO> - D)) / Z
    for (int a = lane; a < D; a += 32) {
        const float *sr = St + (size_t)a * d;
        float sg = 0.f;
        for (int x = 0; x < d; ++x) sg = fmaf(sr[x], gs[warp][x], sg);
        dps[warp][a] = sg - Di * zt[a];
    }
    __syncwarp();
    for (int j = c0; j <= i; ++j) {
        float vg = 0.f;
        for (int x = lane; x < d; x += 32) vg = fmaf(to_f(Vb[(size_t)j * d + x]), gs[warp][x], vg);
        const float cf = warp_sum(vg) - Di;
        for (int a = lane; a < D; a += 32) dps[warp][a] = fmaf(cf, Pk[(size_t)j * D + a], dps[warp][a]);
    }
    for (int a = lane; a < D; a += 32) {
        dps[warp][a] *= iZ;
        Abuf[(size_t)row * D + a] = ps[warp][a] * iZ;
    }
    if (lane == 0) Dbuf[row] = Di;
    __syncwarp();
    float dxa[kMaxD / 32];
    npmap_backward_warp<T>(qs[warp], Wq + (size_t)h * d * D, d, D, dps[warp], ps[warp], dxa, lane);
    for (int c = lane; c < D; c += 32) dYq[(size_t)row * D + c] = ps[warp][c];
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) {
        const int x = lane + 32 * u;
        if (x < d) dq[(size_t)row * d + x] = dxa[u];
    }
}

// One warp per key row j (chunk c): dphi(k_j), dv_j from the later chunks (R, r of slot c + 1 after
// the suffix sums) and from the rows i >= j of chunk c (all heads of the group); then the NP-Map
// backward of k (dk written, dYk).
template <typename T>
__global__ void __launch_bounds__(32 * kBwdWarps) bwd_nowin_key_kernel(Dims s, const T *__restrict__ k,
                                                                       const T *__restrict__ v,
                                                                       const T *__restrict__ Wk,
                                                                       const float *__restrict__ phik,
                                                                       const float *__restrict__ Abuf,
                                                                       const float *__restrict__ Dbuf,
                                                                       const T *__restrict__ dO,
                                                                       const float *__restrict__ R,
                                                                       const float *__restrict__ r, float *__restrict__ dk,
                                                                       float *__restrict__ dv, float *__restrict__ dYk) {
    __shared__ __align__(16) float ks[kBwdWarps][kMaxD];
    __shared__ __align__(16) float vs[kBwdWarps][kMaxD];
    __shared__ __align__(16) float dps[kBwdWarps][kMaxDf];
    __shared__ __align__(16) float dys[kBwdWarps][kMaxDf];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long krow = (long long)blockIdx.x * kBwdWarps + warp;  // over B * Hkv * N
    if (krow >= (long long)s.B * s.Hkv * s.N) return;
    const int d = s.d, D = s.D, G = s.G(), T_ = s.T();
    const int j = (int)(krow % s.N), bg = (int)(krow / s.N), b = bg / s.Hkv, g = bg % s.Hkv;
    const int c = j / s.C, c1 = min(s.N, (c + 1) * s.C);
    for (int x = lane; x < d; x += 32) {
        ks[warp][x] = to_f(k[(size_t)krow * d + x]);
        vs[warp][x] = to_f(v[(size_t)krow * d + x]);
    }
    __syncwarp();
    const float *ph = phik + (size_t)krow * D;
    const bool later = c + 1 <= T_;  // slot c + 1 exists (it is empty when no row lies past chunk c)
    const size_t slot = (size_t)bg * (T_ + 1) + c + 1;
    for (int a = lane; a < D; a += 32) {
        float acc = 0.f;
        if (later) {
            const float *rr = R + slot * D * d + (size_t)a * d;
            for (int x = 0; x < d; ++x) acc = fmaf(rr[x], vs[warp][x], acc);
            acc -= r[slot * D + a];
        }
        dps[warp][a] = acc;
    }
    float dva[kMaxD / 32];
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) {
        const int x = lane + 32 * u;
        float acc = 0.f;
        if (x < d && later)
            for (int a = 0; a < D; ++a) acc = fmaf(R[slot * D * d + (size_t)a * d + x], ph[a], acc);
        dva[u] = acc;
    }
    __syncwarp();
    for (int hh = 0; hh < G; ++hh) {
        const size_t rb = ((size_t)b * s.H + g * G + hh) * s.N;
        for (int i = j; i < c1; ++i) {
            const T *gi = dO + (rb + i) * d;
            const float *ai = Abuf + (rb + i) * D;
            float gv = 0.f, aw = 0.f;
            for (int x = lane; x < d; x += 32) gv = fmaf(to_f(gi[x]), vs[warp][x], gv);
            for (int a = lane; a < D; a += 32) aw = fmaf(ai[a], ph[a], aw);
            const float cf = warp_sum(gv) - Dbuf[rb + i];
            aw = warp_sum(aw);
            for (int a = lane; a < D; a += 32) dps[warp][a] = fmaf(cf, ai[a], dps[warp][a]);
#pragma unroll
            for (int u = 0; u < kMaxD / 32; ++u) {
                const int x = lane + 32 * u;
                if (x < d) dva[u] = fmaf(aw, to_f(gi[x]), dva[u]);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) {
        const int x = lane + 32 * u;
        if (x < d) dv[(size_t)krow * d + x] = dva[u];
    }
    __syncwarp();
    float dxa[kMaxD / 32];
    npmap_backward_warp<T>(ks[warp], Wk + (size_t)g * d * D, d, D, dps[warp], dys[warp], dxa, lane);
    for (int cc = lane; cc < D; cc += 32) dYk[(size_t)krow * D + cc] = dys[warp][cc];
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) {
        const int x = lane + 32 * u;
        if (x < d) dk[(size_t)krow * d + x] = dxa[u];
    }
}

template <typename T>
cudaError_t backward_nowin_t(const Dims &s, const void *q, const void *k, const void *v, const void *Wq,
                             const void *Wk, const void *dO, float *dq, float *dk, float *dv, float *dWq, float *dWk,
                             const BackwardScratch &w, unsigned *err, cudaStream_t st, int *launches) {
    const T *Q = (const T *)q, *K = (const T *)k, *V = (const T *)v, *WQ = (const T *)Wq, *WK = (const T *)Wk;
    const T *GO = (const T *)dO;
    const int T_ = s.T();
    Dims s0 = s;
    s0.k = 0;  // w = 0: nothing is kept; every earlier chunk enters the linear state whole
    cudaError_t e = launch_npmap(s.B * s.Hkv * s.N, s.Hkv, s.N, s.d, s.D, s.bf16, k, Wk, w.phik, st);
    if (e != cudaSuccess) return e;
    if ((e = launch_linear_state(s0, w.phik, v, nullptr, w.S, w.z, nullptr, err, st)) != cudaSuccess) return e;
    *launches += 3;
    const long long rows = (long long)s.B * s.H * s.N;
    bwd_nowin_row_kernel<T><<<(unsigned)((rows + kBwdWarps - 1) / kBwdWarps), 32 * kBwdWarps, 0, st>>>(
        s, Q, V, WQ, w.phik, w.S, w.z, GO, dq, w.A, w.Dv, w.dYq);
    bwd_chunk_kernel<T><<<dim3(T_ + 1, s.B * s.Hkv, (s.D * s.d + s.D + 255) / 256), 256, 0, st>>>(s, w.A, w.Dv, GO,
                                                                                               w.R, w.r);
    if ((e = launch_bwd_suffix(s, w.R, w.r, st)) != cudaSuccess) return e;
    const long long krows = (long long)s.B * s.Hkv * s.N;
    bwd_nowin_key_kernel<T><<<(unsigned)((krows + kBwdWarps - 1) / kBwdWarps), 32 * kBwdWarps, 0, st>>>(
        s, K, V, WK, w.phik, w.A, w.Dv, GO, w.R, w.r, dk, dv, w.dYk);
    bwd_weight_kernel<T><<<dim3(s.d, s.H), 256, 0, st>>>(s.B, s.H, s.N, s.d, s.D, Q, w.dYq, dWq);
    bwd_weight_kernel<T><<<dim3(s.d, s.Hkv), 256, 0, st>>>(s.B, s.Hkv, s.N, s.d, s.D, K, w.dYk, dWk);
    *launches += 6;
    return cudaGetLastError();
}

template <typename T>
cudaError_t backward_t(const Dims &s, const void *q, const void *k, const void *v, const void *Wq, const void *Wk,
                       const int32_t *idx, const void *dO, float *dq, float *dk, float *dv, float *dWq,
                       float *dWk, const BackwardScratch &w, unsigned *err, cudaStream_t st, int *launches,
                       const void *o_fwd, const float *lse_fwd) {
    const T *Q = (const T *)q, *K = (const T *)k, *V = (const T *)v, *WQ = (const T *)Wq, *WK = (const T *)Wk;
    const T *GO = (const T *)dO;
    const int T_ = s.T();
    cudaError_t e;
    // linear state of the forward (S_t, z_t per query chunk): on tensor cores where the tiled linear
    // backward runs (it forms phi(k) itself), else from phi(k) of every key
    const bool tiled_state = tc_backward_supported(s) && tiled_linear_backward_supported(s) && tc_linear_supported(s);
    if (tiled_state) {
        const int ts = timing_begin(kTimeBwdLinear, st);
        if ((e = launch_w_transpose(s.Hkv, s.d, s.D, Wk, w.wkt, st)) != cudaSuccess) return e;
        if ((e = launch_linear_tc(s, k, v, w.wkt, idx, w.S, w.z, err, st)) != cudaSuccess) return e;
        if ((e = launch_linear_prefix(s, w.S, w.z, w.st_t, st)) != cudaSuccess) return e;  // + S_t^T (bf16)
        if ((e = launch_w_transpose(s.H, s.d, s.D, Wq, w.wqt, st)) != cudaSuccess) return e;
        timing_end(ts, st);
        *launches += 4;
    } else {
        e = launch_npmap(s.B * s.Hkv * s.N, s.Hkv, s.N, s.d, s.D, s.bf16, k, Wk, w.phik, st);
        if (e != cudaSuccess) return e;
        ++*launches;
        e = launch_linear_state(s, w.phik, v, idx, w.S, w.z, nullptr, err, st);
        if (e != cudaSuccess) return e;
        *launches += 2;
    }
    if ((e = cudaMemsetAsync(w.dYk, 0, sizeof(float) * (size_t)s.B * s.Hkv * s.N * s.D, st)) != cudaSuccess) return e;
    const long long rows = (long long)s.B * s.H * s.N;
    const unsigned rgrid = (unsigned)((rows + kBwdWarps - 1) / kBwdWarps);
    if (tc_backward_supported(s)) {
        // softmax branch on tensor cores: linear pre-pass (phi(q), S_t dO, lden, dl), then dq with
        // the rows' normalisers, dk and dv by key tiles, then the linear branch's query and key sides
        const bool tiled = tiled_linear_backward_supported(s);
        if (s.k > 0 && T_ > 0) {
            if ((e = launch_gather(s, idx, k, v, w.khat, w.vhat, err, st)) != cudaSuccess) return e;
            ++*launches;
        }
        // tiled linear branch with the tensor-core linear state: the dq kernel forms the rows' linear
        // terms itself (its prologue writes phi(q) and S_t dO for the later linear kernels)
        BwdPrologue pro{nullptr, Wq, nullptr, w.z, w.A, w.dYq};
        pro.o_fwd = o_fwd;      // the forward's output and normaliser (null: the dq kernel forms L, D)
        pro.lse_fwd = lse_fwd;
        if (tiled && tiled_state) {
            pro.wqt = w.wqt;
            pro.st_t = w.st_t;
        } else if (tiled) {
            const int ts = timing_begin(kTimeBwdLinear, st);
            e = launch_linear_backward_tiled(0, s, q, k, v, Wq, Wk, dO, idx, w, dq, dk, dv, dWq, dWk, st);
            timing_end(ts, st);
            if (e != cudaSuccess) return e;
            ++*launches;
        } else {
            bwd_lin_pre_kernel<T><<<rgrid, 32 * kBwdWarps, 0, st>>>(s, Q, WQ, w.S, w.z, GO, w.A, w.dYq, w.Ms, w.iZ);
            ++*launches;
        }
        e = launch_backward_tc(s, q, k, v, w.khat, w.vhat, idx, dO, w.Ms, w.iZ, pro, w.L, w.Dv, dq, dk, dv, err, st,
                               launches);
        if (e != cudaSuccess) return e;
        if (tiled) {
            // query side (dq, dWq), chunk sums, suffix, key side (dk, dv, dWk) of the linear branch (the
            // dq kernel with the prologue has formed dq, dY and a itself)
            const int ts = timing_begin(kTimeBwdLinear, st);
            e = launch_linear_backward_tiled(pro.wqt ? 2 : 1, s, q, k, v, Wq, Wk, dO, idx, w, dq, dk, dv, dWq, dWk, st);
            timing_end(ts, st);
            if (e != cudaSuccess) return e;
            *launches += T_ > 0 ? 3 : 2;
            return cudaSuccess;
        }
        bwd_lin_post_kernel<T><<<rgrid, 32 * kBwdWarps, 0, st>>>(s, Q, WQ, w.z, w.L, w.Dv, w.A, w.dYq, dq);
        ++*launches;
    } else if (s.d == 64 || s.d == 128) {
        // dk, dv by key blocks (written there; no atomics)
        bwd_row_kernel<T, false><<<rgrid, 32 * kBwdWarps, 0, st>>>(s, Q, K, V, WQ, idx, w.S, w.z, GO, dq, dk, dv,
                                                                    w.A, w.Dv, w.Ms, w.iZ, w.dYq, err);
        e = s.d == 64 ? launch_kv_blocks<T, 64>(s, Q, K, V, idx, GO, w, dk, dv, st)
                      : launch_kv_blocks<T, 128>(s, Q, K, V, idx, GO, w, dk, dv, st);
        if (e != cudaSuccess) return e;
        *launches += 3;
    } else {
        if ((e = cudaMemsetAsync(dk, 0, sizeof(float) * (size_t)s.B * s.Hkv * s.N * s.d, st)) != cudaSuccess) return e;
        if ((e = cudaMemsetAsync(dv, 0, sizeof(float) * (size_t)s.B * s.Hkv * s.N * s.d, st)) != cudaSuccess) return e;
        bwd_row_kernel<T, true><<<rgrid, 32 * kBwdWarps, 0, st>>>(s, Q, K, V, WQ, idx, w.S, w.z, GO, dq, dk, dv,
                                                                   w.A, w.Dv, w.Ms, w.iZ, w.dYq, err);
        ++*launches;
    }
    bwd_chunk_kernel<T><<<dim3(T_ + 1, s.B * s.Hkv, (s.D * s.d + s.D + 255) / 256), 256, 0, st>>>(s, w.A, w.Dv, GO,
                                                                                               w.R, w.r);
    ++*launches;
    const size_t ent = (size_t)s.B * s.Hkv * ((size_t)s.D * s.d + s.D);
    bwd_suffix_kernel<<<(unsigned)((ent + 255) / 256), 256, 0, st>>>(s, w.R, w.r);
    ++*launches;
    const long long krows = (long long)s.B * s.Hkv * T_ * s.C;
    if (krows > 0) {
        bwd_key_kernel<T><<<(unsigned)((krows + kBwdWarps - 1) / kBwdWarps), 32 * kBwdWarps, 0, st>>>(
            s, K, V, WK, idx, w.phik, w.R, w.r, dk, dv, w.dYk);
        ++*launches;
    }
    bwd_weight_kernel<T><<<dim3(s.d, s.H), 256, 0, st>>>(s.B, s.H, s.N, s.d, s.D, Q, w.dYq, dWq);
    bwd_weight_kernel<T><<<dim3(s.d, s.Hkv), 256, 0, st>>>(s.B, s.Hkv, s.N, s.d, s.D, K, w.dYk, dWk);
    *launches += 2;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_suffix(const Dims &s, float *R, float *r, cudaStream_t st) {
    const size_t ent = (size_t)s.B * s.Hkv * ((size_t)s.D * s.d + s.D);
    if (ent == 0) return cudaSuccess;
    bwd_suffix_kernel<<<(unsigned)((ent + 255) / 256), 256, 0, st>>>(s, R, r);
    return cudaGetLastError();
}

cudaError_t launch_backward(const Dims &s, const void *q, const void *k, const void *v, const void *Wq,
                            const void *Wk, const int32_t *idx, const void *dO, float *dq, float *dk, float *dv,
                            float *dWq, float *dWk, const BackwardScratch &w, unsigned *err, cudaStream_t st,
                            int *launches, const void *o_fwd, const float *lse_fwd) {
    if (s.w == 0) {
        if (s.bf16)
            return backward_nowin_t<__nv_bfloat16>(s, q, k, v, Wq, Wk, dO, dq, dk, dv, dWq, dWk, w, err, st, launches);
        return backward_nowin_t<float>(s, q, k, v, Wq, Wk, dO, dq, dk, dv, dWq, dWk, w, err, st, launches);
    }
    if (s.bf16)
        return backward_t<__nv_bfloat16>(s, q, k, v, Wq, Wk, idx, dO, dq, dk, dv, dWq, dWk, w, err, st, launches, o_fwd,
                                         lse_fwd);
    return backward_t<float>(s, q, k, v, Wq, Wk, idx, dO, dq, dk, dv, dWq, dWk, w, err, st, launches, nullptr, nullptr);
}

}  // namespace still
