// kernels_generic.cu -- SIMT kernels for every step of the STILL layer.
//
// These take fp32 or bf16 storage and compute in fp32 with the accurate
// libm-style functions (expf, logf, log1pf).  They serve the fp32 workloads,
// shapes the tensor-core kernels do not cover, the w = 0 (pure linear) mode,
// and the small steps (top-k, gather, NP-Map, linear state) of every path.
//
// Method: "STILL: Selecting Tokens for Intra-Layer Hybrid Attention to
// Linearize LLMs" ([p1] jsqmd.com: introduction, "Self-Saliency Score",
// "NP-Map", "Chunk-Wise"; [p4] atlas.scime.ai: "Approach").
#include "common.cuh"
#include "rowops.cuh"
#include "still_internal.h"
#include "topk.cuh"

namespace still {
namespace {

// ------------------------------------------------------------------ saliency
// Self-Saliency Score ([p1] "Self-Saliency Score"; [p4] "Approach"):
// sigma = softplus(s_ii - LSE_{j in [i-w+1, i-1]} s_ij) = -ln(1 - p_ii); +inf for an empty band.
// One CTA: 8 query positions x all G heads of one KV group; one warp per (head, position),
// lanes split the band keys.  The group score is the mean over heads, summed in head order.
constexpr int kSalRows = 8;

template <typename T>
__global__ void __launch_bounds__(128) saliency_generic_kernel(Dims s, const T *__restrict__ q,
                                                               const T *__restrict__ k, float *__restrict__ r_kv,
                                                               float *__restrict__ r_q) {
    __shared__ float sig[32 * kSalRows];
    __shared__ __align__(16) float qs[4][kMaxD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = s.G(), bg = blockIdx.y, b = bg / s.Hkv, g = bg % s.Hkv;
    const int i0 = blockIdx.x * kSalRows;
    const T *kg = k + (size_t)bg * s.N * s.d;
    for (int pair = warp; pair < G * kSalRows; pair += 4) {
        const int hh = pair / kSalRows, ii = pair % kSalRows, i = i0 + ii;
        if (i >= s.N) continue;
        const int h = g * G + hh;
        const T *qrow = q + (((size_t)b * s.H + h) * s.N + i) * s.d;
        for (int x = lane; x < s.d; x += 32) qs[warp][x] = to_f(qrow[x]);
        __syncwarp();
        const int lo = max(0, i - s.w + 1);
        float mx = -INFINITY, sm = 0.f;
        for (int j = lo + lane; j < i; j += 32) {
            float l = s.scale * dot_row(qs[warp], kg + (size_t)j * s.d, s.d);
            if (l > mx) {
                sm = sm * expf(mx - l) + 1.f;
                mx = l;
            } else {
                sm += expf(l - mx);
            }
        }
        float M = warp_max(mx);
        float part = (mx == -INFINITY) ? 0.f : sm * expf(mx - M);
        float Z = warp_sum(part);
        float dpart = 0.f;
        for (int x = lane; x < s.d; x += 32) dpart = fmaf(qs[warp][x], to_f(kg[(size_t)i * s.d + x]), dpart);
        float sii = s.scale * warp_sum(dpart);
        float sigma = (i == lo) ? INFINITY : softplus_f(sii - (M + logf(Z)));
        if (lane == 0) {
            sig[hh * kSalRows + ii] = sigma;
            if (r_q) r_q[((size_t)b * s.H + h) * s.N + i] = sigma;
        }
        __syncwarp();
    }
    __syncthreads();
    if (threadIdx.x < kSalRows) {
        const int i = i0 + threadIdx.x;
        if (i < s.N) {
            float acc = 0.f;
            for (int hh = 0; hh < G; ++hh) acc += sig[hh * kSalRows + threadIdx.x];
            r_kv[(size_t)bg * s.N + i] = acc / (float)G;
        }
    }
}

// ------------------------------------------------------------------ top-k + gather
// Per-chunk top-k ([p1] "Chunk-Wise"; [p4] "Approach"): key = (order-preserving score bits, ~position),
// unique per element, so a descending bitonic sort gives (score desc, position asc); the first k
// positions are then sorted ascending and written.  The kept K/V rows are copied into the compact
// chunk-ordered cache at rows c*k .. c*k+k-1 of (b, g).
template <typename T>
__global__ void __launch_bounds__(1024) topk_gather_kernel(Dims s, const float *__restrict__ r,
                                                           int32_t *__restrict__ idx, const T *__restrict__ k,
                                                           const T *__restrict__ v, T *__restrict__ khat,
                                                           T *__restrict__ vhat, int P, int Pk) {
    extern __shared__ unsigned long long keys[];  // P entries, then Pk uint32 positions
    uint32_t *pos = reinterpret_cast<uint32_t *>(keys + P);
    const int T_ = s.T(), c = blockIdx.x % T_, bg = blockIdx.x / T_;
    block_topk(r + (size_t)bg * s.N + (size_t)c * s.C, s.C, s.k, keys, pos, P, Pk);
    int32_t *out = idx + ((size_t)bg * T_ + c) * s.k;
    for (int t = threadIdx.x; t < s.k; t += blockDim.x) out[t] = c * s.C + (int32_t)pos[t];
    if (khat) {
        const size_t rowbase = (size_t)bg * T_ * s.k + (size_t)c * s.k;
        const int vec = sizeof(T) == 2 ? 8 : 4;  // elements per 16-byte vector
        const int nv = s.d / vec;
        for (int t = threadIdx.x; t < s.k * nv; t += blockDim.x) {
            int rr = t / nv, x = t % nv;
            size_t src = ((size_t)bg * s.N + (size_t)c * s.C + pos[rr]) * s.d;
            size_t dst = (rowbase + rr) * s.d;
            reinterpret_cast<uint4 *>(khat + dst)[x] = reinterpret_cast<const uint4 *>(k + src)[x];
            reinterpret_cast<uint4 *>(vhat + dst)[x] = reinterpret_cast<const uint4 *>(v + src)[x];
        }
    }
}

// Gather of an injected selection: rows idx[b,g,c,:] of K and V into the compact cache; an index
// outside its chunk is reported through the device error word and its row is zero-filled.
template <typename T>
__global__ void __launch_bounds__(256) gather_kernel(Dims s, const int32_t *__restrict__ idx, const T *__restrict__ k,
                                                     const T *__restrict__ v, T *__restrict__ khat,
                                                     T *__restrict__ vhat, unsigned *err) {
    const int T_ = s.T(), c = blockIdx.x % T_, bg = blockIdx.x / T_;
    const int nv = s.d / (sizeof(T) == 2 ? 8 : 4);
    const size_t rowbase = (size_t)bg * T_ * s.k + (size_t)c * s.k;
    for (int t = threadIdx.x; t < s.k * nv; t += blockDim.x) {
        const int rr = t / nv, x = t % nv;
        const int j = idx[((size_t)bg * T_ + c) * s.k + rr];
        const size_t dst = (rowbase + rr) * s.d;
        uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
        if (j >= c * s.C && j < (c + 1) * s.C) {
            const size_t src = ((size_t)bg * s.N + j) * s.d;
            kv = reinterpret_cast<const uint4 *>(k + src)[x];
            vv = reinterpret_cast<const uint4 *>(v + src)[x];
        } else if (x == 0) {
            report(err, DEV_ERR_INDEX);
        }
        reinterpret_cast<uint4 *>(khat + dst)[x] = kv;
        reinterpret_cast<uint4 *>(vhat + dst)[x] = vv;
    }
}

// ------------------------------------------------------------------ NP-Map
template <typename T>
__global__ void __launch_bounds__(128) npmap_kernel(int rows, int Hx, int N, int d, int D, const T *__restrict__ x,
                                                    const T *__restrict__ W, float *__restrict__ phi) {
    __shared__ __align__(16) float xs[4][kMaxD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * 4 + warp;
    if (row >= rows) return;
    const int hx = (row / N) % Hx;
    for (int a = lane; a < d; a += 32) xs[warp][a] = to_f(x[(size_t)row * d + a]);
    __syncwarp();
    npmap_row_warp<T>(xs[warp], W + (size_t)hx * d * D, d, D, phi + (size_t)row * D, lane);
}

// ------------------------------------------------------------------ linear state
// Delta S_c = sum over the unkept tokens j of chunk c of phi(k_j) v_j^T  [D,d], Delta z_c = sum phi(k_j),
// for the chunks c <= T-m-1 that some query chunk sees; written to slot c+m+1 of S [B,Hkv,T+1,D,d]
// so that the inclusive prefix over slots gives S_t = sum_{c <= t-m-1} Delta S_c ([p1] introduction:
// the unselected tokens are aggregated linearly).  w = 0: m = 0 and nothing is kept.
constexpr int kLinTok = 32;   // tokens staged per step
constexpr int kLinEnt = 32;   // state entries per thread

template <typename T>
__global__ void __launch_bounds__(256) linear_delta_kernel(Dims s, const float *__restrict__ phik,
                                                           const T *__restrict__ v, const int32_t *__restrict__ idx,
                                                           float *__restrict__ S, float *__restrict__ z,
                                                           unsigned *err) {
    extern __shared__ float lsm[];  // ph[kLinTok][D], vs[kLinTok][d], then C flag bytes
    float *ph = lsm;
    float *vs = ph + kLinTok * s.D;
    unsigned char *kept = reinterpret_cast<unsigned char *>(vs + kLinTok * s.d);
    const int c = blockIdx.x, bg = blockIdx.y, T_ = s.T(), m = s.m();
    const int Dd = s.D * s.d;
    for (int j = threadIdx.x; j < s.C; j += blockDim.x) kept[j] = 0;
    __syncthreads();
    if (s.k > 0) {
        for (int n = threadIdx.x; n < s.k; n += blockDim.x) {
            int j = idx[((size_t)bg * T_ + c) * s.k + n] - c * s.C;
            if (j >= 0 && j < s.C) kept[j] = 1;
            else report(err, DEV_ERR_INDEX);
        }
    }
    __syncthreads();
    float acc[kLinEnt];
#pragma unroll
    for (int u = 0; u < kLinEnt; ++u) acc[u] = 0.f;
    float zacc = 0.f;
    const int ebase = blockIdx.z * blockDim.x * kLinEnt;
    for (int jb = 0; jb < s.C; jb += kLinTok) {
        for (int t = threadIdx.x; t < kLinTok * s.D; t += blockDim.x) {
            int rr = t / s.D, a = t % s.D, j = jb + rr;
            float val = 0.f;
            if (j < s.C && !kept[j]) val = phik[((size_t)bg * s.N + (size_t)c * s.C + j) * s.D + a];
            ph[t] = val;
        }
        for (int t = threadIdx.x; t < kLinTok * s.d; t += blockDim.x) {
            int rr = t / s.d, x = t % s.d, j = jb + rr;
            vs[t] = j < s.C ? to_f(v[((size_t)bg * s.N + (size_t)c * s.C + j) * s.d + x]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kLinEnt; ++u) {
            int e = ebase + threadIdx.x + u * blockDim.x;
            if (e < Dd) {
                int a = e / s.d, x = e % s.d;
                float sacc = acc[u];
                for (int rr = 0; rr < kLinTok; ++rr) sacc = fmaf(ph[rr * s.D + a], vs[rr * s.d + x], sacc);
                acc[u] = sacc;
            }
        }
        if (blockIdx.z == 0 && threadIdx.x < s.D)
            for (int rr = 0; rr < kLinTok; ++rr) zacc += ph[rr * s.D + threadIdx.x];
        __syncthreads();
    }
    const size_t slot = (size_t)bg * (T_ + 1) + c + m + 1;
#pragma unroll
    for (int u = 0; u < kLinEnt; ++u) {
        int e = ebase + threadIdx.x + u * blockDim.x;
        if (e < Dd) S[slot * Dd + e] = acc[u];
    }
    if (blockIdx.z == 0 && threadIdx.x < s.D) z[slot * s.D + threadIdx.x] = zacc;
}

// Inclusive prefix over slots 0..T: slots 0..m are zero (no chunk has been decided for them).
// st_t (optional): a bf16 copy of every S_t, transposed to [d, D] (K-major operand of phi(q) S_t).
// One CTA per (b, g) and tile of kPfxRows rows (a) x 32 columns (x) of S's [D, d] elements, two per
// thread; z goes with the tiles of column 0.  Slots are read eight at a time (the loads of a batch in
// flight together; the sum over slots is sequential, in slot order).  The transposed copy passes
// through shared memory, so that its stores, like the loads, cover whole 32-byte sectors: written
// straight from the [D, d] order, each of them was a lone 2-byte store.
constexpr int kPfxRows = 16, kPfxSlots = 8, kPfxThreads = 256;
constexpr int kPfxPer = kPfxRows * 32 / kPfxThreads;  // elements per thread
static_assert(kPfxPer * kPfxThreads == kPfxRows * 32 && kPfxThreads % kPfxRows == 0, "prefix tile");

__global__ void __launch_bounds__(kPfxThreads) linear_prefix_kernel(Dims s, float *__restrict__ S,
                                                                   float *__restrict__ z,
                                                                   __nv_bfloat16 *__restrict__ st_t) {
    __shared__ float tile[kPfxRows][33];
    const int T_ = s.T(), m = s.m(), D = s.D, d = s.d;
    const size_t Dd = (size_t)D * d;
    const int bg = blockIdx.z, a0 = blockIdx.y * kPfxRows, x0 = blockIdx.x * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    float *Sb = S + (size_t)bg * (T_ + 1) * Dd;
    float *zb = z + (size_t)bg * (T_ + 1) * D;
    bool live[kPfxPer];
    size_t off[kPfxPer];
#pragma unroll
    for (int u = 0; u < kPfxPer; ++u) {
        const int a = a0 + ty + 8 * u;
        live[u] = a < D && x0 + tx < d;
        off[u] = live[u] ? (size_t)a * d + x0 + tx : 0;
    }
    const bool has_z = blockIdx.x == 0 && ty == 0 && tx < kPfxRows && a0 + tx < D;
    // transposed store of this thread: row x0 + xo (+ 32 / kPfxPer per element), column a0 + ao
    const int ao = threadIdx.x % kPfxRows, xo = threadIdx.x / kPfxRows;
    float run[kPfxPer], zrun = 0.f;
#pragma unroll
    for (int u = 0; u < kPfxPer; ++u) run[u] = 0.f;
    for (int t0 = 0; t0 <= T_; t0 += kPfxSlots) {
        float v[kPfxSlots][kPfxPer], vz[kPfxSlots];
#pragma unroll
        for (int q = 0; q < kPfxSlots; ++q) {
            const int t = t0 + q;
            const bool add = t <= T_ && t >= m + 1;
#pragma unroll
            for (int u = 0; u < kPfxPer; ++u) v[q][u] = add && live[u] ? Sb[(size_t)t * Dd + off[u]] : 0.f;
            vz[q] = add && has_z ? zb[(size_t)t * D + a0 + tx] : 0.f;
        }
#pragma unroll
        for (int q = 0; q < kPfxSlots; ++q) {
            const int t = t0 + q;
            if (t > T_) break;  // the same for every thread of the CTA
#pragma unroll
            for (int u = 0; u < kPfxPer; ++u) {
                run[u] += v[q][u];
                if (live[u]) Sb[(size_t)t * Dd + off[u]] = run[u];
            }
            zrun += vz[q];
            if (has_z) zb[(size_t)t * D + a0 + tx] = zrun;
            if (st_t) {
#pragma unroll
                for (int u = 0; u < kPfxPer; ++u) tile[ty + 8 * u][tx] = run[u];
                __syncthreads();
#pragma unroll
                for (int u = 0; u < kPfxPer; ++u) {
                    const int xr = xo + u * (kPfxThreads / kPfxRows);
                    const int x = x0 + xr, a = a0 + ao;
                    if (x < d && a < D)
                        st_t[((size_t)(bg * (T_ + 1) + t) * d + x) * D + a] = __float2bfloat16_rn(tile[ao][xr]);
                }
                __syncthreads();
            }
        }
    }
}

// ------------------------------------------------------------------ hybrid merge
// One warp per query row i of head h ([p1] introduction: both branches in one layer; "NP-Map":
// the branches share one distribution):
//   softmax keys: kept rows of chunks c <= t-m-1 (compact cache rows [0, k(t-m))) then the local
//   window [max(0,(t-m)C), i]; lanes take 32 keys at a time, online max/sum across the warp;
//   linear: phi(q)^T S_t and phi(q)^T z_t (+ the chunk-local linear keys when w = 0);
//   merge under one normaliser, with the joint shift M* = max(m, ln(linear denominator)).
template <typename T>
__device__ __forceinline__ void soft_keys(const float *qs, const T *K, const T *V, int n, float scale, int d,
                                          int lane, float &M, float &L, float *acc) {
    for (int base = 0; base < n; base += 32) {
        const int j = base + lane;
        float l = j < n ? scale * dot_row(qs, K + (size_t)j * d, d) : -INFINITY;
        float gm = warp_max(l);
        float nm = fmaxf(M, gm);
        float so = (M == -INFINITY) ? 0.f : expf(M - nm);
        float p = j < n ? expf(l - nm) : 0.f;
        L = L * so + warp_sum(p);
#pragma unroll
        for (int u = 0; u < kMaxD / 32; ++u) acc[u] *= so;
        const int cnt = min(32, n - base);
        for (int jj = 0; jj < cnt; ++jj) {
            float pj = __shfl_sync(0xffffffffu, p, jj);
            const T *vr = V + (size_t)(base + jj) * d;
#pragma unroll
            for (int u = 0; u < kMaxD / 32; ++u) {
                int x = lane + 32 * u;
                if (x < d) acc[u] = fmaf(pj, to_f(vr[x]), acc[u]);
            }
        }
        M = nm;
    }
}

template <typename T>
__global__ void __launch_bounds__(128) merge_generic_kernel(Dims s, const T *__restrict__ q, const T *__restrict__ k,
                                                            const T *__restrict__ v, const T *__restrict__ Wq,
                                                            const T *__restrict__ khat, const T *__restrict__ vhat,
                                                            const float *__restrict__ S, const float *__restrict__ z,
                                                            const float *__restrict__ phik, T *__restrict__ o) {
    __shared__ __align__(16) float qs[4][kMaxD];
    __shared__ __align__(16) float ps[4][kMaxDf];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y, b = bh / s.H, h = bh % s.H, G = s.G(), g = h / G;
    const int bg = b * s.Hkv + g;
    const int i = blockIdx.x * 4 + warp;
    if (i >= s.N) return;
    const int d = s.d, D = s.D, T_ = s.T(), m = s.m(), t = i / s.C;
    const T *qrow = q + ((size_t)bh * s.N + i) * d;
    for (int x = lane; x < d; x += 32) qs[warp][x] = to_f(qrow[x]);
    __syncwarp();
    npmap_row_warp<T>(qs[warp], Wq + (size_t)h * d * D, d, D, ps[warp], lane);
    __syncwarp();

    float acc[kMaxD / 32];
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) acc[u] = 0.f;
    float M = -INFINITY, L = 0.f;
    if (s.w > 0) {
        const int nk = s.k * max(0, t - m);
        const size_t hb = (size_t)bg * T_ * s.k * d;
        soft_keys<T>(qs[warp], khat + hb, vhat + hb, nk, s.scale, d, lane, M, L, acc);
        const int lo = max(0, (t - m) * s.C);
        const size_t kb = ((size_t)bg * s.N + lo) * d;
        soft_keys<T>(qs[warp], k + kb, v + kb, i - lo + 1, s.scale, d, lane, M, L, acc);
    }
    // linear branch: state seen by query chunk t (slot t of [T+1])
    const float *St = S + ((size_t)bg * (T_ + 1) + t) * D * d;
    const float *zt = z + ((size_t)bg * (T_ + 1) + t) * D;
    float lin[kMaxD / 32];
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) lin[u] = 0.f;
    float lden = 0.f;
    for (int a = 0; a < D; ++a) {
        const float pa = ps[warp][a];
        lden = fmaf(pa, zt[a], lden);
#pragma unroll
        for (int u = 0; u < kMaxD / 32; ++u) {
            int x = lane + 32 * u;
            if (x < d) lin[u] = fmaf(pa, St[(size_t)a * d + x], lin[u]);
        }
    }
    if (s.w == 0) {
        // chunk-local causal linear keys [tC, i]
        const int lo = t * s.C;
        for (int base = lo; base <= i; base += 32) {
            const int j = base + lane;
            float wgt = 0.f;
            if (j <= i) {
                const float *pk = phik + ((size_t)bg * s.N + j) * D;
                for (int a = 0; a < D; ++a) wgt = fmaf(ps[warp][a], pk[a], wgt);
            }
            lden += warp_sum(wgt);
            const int cnt = min(32, i - base + 1);
            for (int jj = 0; jj < cnt; ++jj) {
                float wj = __shfl_sync(0xffffffffu, wgt, jj);
                const T *vr = v + ((size_t)bg * s.N + base + jj) * d;
#pragma unroll
                for (int u = 0; u < kMaxD / 32; ++u) {
                    int x = lane + 32 * u;
                    if (x < d) lin[u] = fmaf(wj, to_f(vr[x]), lin[u]);
                }
            }
        }
    }
    float Ms = M;
    if (lden > 0.f) Ms = fmaxf(M, logf(lden));
    const float a_soft = (M == -INFINITY) ? 0.f : expf(M - Ms);
    const float a_lin = (Ms == -INFINITY) ? 0.f : expf(-Ms);
    const float den = L * a_soft + lden * a_lin;
    const float inv = den > 0.f ? 1.f / den : 0.f;
    T *orow = o + ((size_t)bh * s.N + i) * d;
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) {
        int x = lane + 32 * u;
        if (x < d) orow[x] = from_f<T>((acc[u] * a_soft + lin[u] * a_lin) * inv);
    }
}

}  // namespace

// ------------------------------------------------------------------ launchers
// Diagonal-only router ([p4] "Surprising findings": routing on the diagonal term by itself):
// r_{g,i} = mean over the G heads of g of tau <q_hi, k_gi>.  HBM-bound (reads Q and K once): a warp
// per (b, g, row); each lane holds its d/32 slice of k_gi and dots it with each head's q_hi.
template <typename T>
__global__ void __launch_bounds__(256) diagonal_score_kernel(Dims s, const T *__restrict__ q,
                                                             const T *__restrict__ k, float *__restrict__ r) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, G = s.G();
    const long long row = (long long)blockIdx.x * 8 + warp;  // over B * Hkv * N
    if (row >= (long long)s.B * s.Hkv * s.N) return;
    const long long bg = row / s.N;
    const int i = (int)(row % s.N), b = (int)(bg / s.Hkv), g = (int)(bg % s.Hkv);
    const T *ki = k + (size_t)row * s.d;
    float kv[kMaxD / 32];
#pragma unroll
    for (int u = 0; u < kMaxD / 32; ++u) {
        const int x = lane + 32 * u;
        kv[u] = x < s.d ? to_f(ki[x]) : 0.f;
    }
    float acc = 0.f;
    for (int hh = 0; hh < G; ++hh) {
        const T *qi = q + (((size_t)b * s.H + (size_t)g * G + hh) * s.N + i) * s.d;
        float dot = 0.f;
#pragma unroll
        for (int u = 0; u < kMaxD / 32; ++u) {
            const int x = lane + 32 * u;
            if (x < s.d) dot = fmaf(to_f(qi[x]), kv[u], dot);
        }
        acc += warp_sum(dot);
    }
    if (lane == 0) r[row] = s.scale * acc / (float)G;
}

cudaError_t launch_diagonal_score(const Dims &s, const void *q, const void *k, float *r_kv, cudaStream_t st) {
    const long long rows = (long long)s.B * s.Hkv * s.N;
    if (rows == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + 7) / 8);
    if (s.bf16)
        diagonal_score_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(s, (const __nv_bfloat16 *)q,
                                                                   (const __nv_bfloat16 *)k, r_kv);
    else
        diagonal_score_kernel<float><<<grid, 256, 0, st>>>(s, (const float *)q, (const float *)k, r_kv);
    return cudaGetLastError();
}

cudaError_t launch_saliency_generic(const Dims &s, const void *q, const void *k, float *r_kv, float *r_q,
                                    cudaStream_t st) {
    dim3 grid((s.N + kSalRows - 1) / kSalRows, s.B * s.Hkv);
    if (s.bf16)
        saliency_generic_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(
            s, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, r_kv, r_q);
    else
        saliency_generic_kernel<float><<<grid, 128, 0, st>>>(s, (const float *)q, (const float *)k, r_kv, r_q);
    return cudaGetLastError();
}

cudaError_t launch_topk_gather(const Dims &s, const float *r, int32_t *idx, const void *k, const void *v, void *khat,
                               void *vhat, cudaStream_t st) {
    const int T_ = s.T();
    if (T_ == 0 || s.k == 0 || s.B * s.Hkv == 0) return cudaSuccess;
    const int P = pow2_ceil(s.C), Pk = pow2_ceil(s.k);
    const size_t smem = (size_t)P * 8 + (size_t)Pk * 4;
    const int threads = P / 2 < 64 ? 64 : P / 2 > 1024 ? 1024 : P / 2;  // one compare-exchange per thread and stage
    dim3 grid(s.B * s.Hkv * T_);
    cudaError_t e;
    if (s.bf16) {
        e = cudaFuncSetAttribute(topk_gather_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        topk_gather_kernel<__nv_bfloat16><<<grid, threads, smem, st>>>(
            s, r, idx, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, (__nv_bfloat16 *)khat,
            (__nv_bfloat16 *)vhat, P, Pk);
    } else {
        e = cudaFuncSetAttribute(topk_gather_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        topk_gather_kernel<float><<<grid, threads, smem, st>>>(s, r, idx, (const float *)k, (const float *)v,
                                                               (float *)khat, (float *)vhat, P, Pk);
    }
    return cudaGetLastError();
}

cudaError_t launch_gather(const Dims &s, const int32_t *idx, const void *k, const void *v, void *khat, void *vhat,
                          unsigned *err, cudaStream_t st) {
    const int T_ = s.T();
    if (T_ == 0 || s.k == 0 || s.B * s.Hkv == 0) return cudaSuccess;
    dim3 grid(s.B * s.Hkv * T_);
    if (s.bf16)
        gather_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(s, idx, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v,
                                                           (__nv_bfloat16 *)khat, (__nv_bfloat16 *)vhat, err);
    else
        gather_kernel<float><<<grid, 256, 0, st>>>(s, idx, (const float *)k, (const float *)v, (float *)khat,
                                                   (float *)vhat, err);
    return cudaGetLastError();
}

cudaError_t launch_npmap(int rows, int Hx, int N, int d, int D, int bf16, const void *x, const void *W, float *phi,
                         cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    dim3 grid((rows + 3) / 4);
    if (bf16)
        npmap_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(rows, Hx, N, d, D, (const __nv_bfloat16 *)x,
                                                          (const __nv_bfloat16 *)W, phi);
    else
        npmap_kernel<float><<<grid, 128, 0, st>>>(rows, Hx, N, d, D, (const float *)x, (const float *)W, phi);
    return cudaGetLastError();
}

cudaError_t launch_linear_state(const Dims &s, const float *phik, const void *v, const int32_t *idx, float *S,
                                float *z, void *st_t, unsigned *err, cudaStream_t st) {
    const int T_ = s.T(), m = s.m();
    const int nc = T_ - m;  // chunks c <= T-m-1 are seen by some query chunk
    if (s.B * s.Hkv == 0) return cudaSuccess;
    cudaError_t e;
    if (nc > 0) {
        const int ent_per_block = 256 * kLinEnt;
        dim3 grid(nc, s.B * s.Hkv, (s.D * s.d + ent_per_block - 1) / ent_per_block);
        size_t smem = (size_t)kLinTok * (s.D + s.d) * 4 + (size_t)s.C;
        if (s.bf16) {
            e = cudaFuncSetAttribute(linear_delta_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem);
            if (e != cudaSuccess) return e;
            linear_delta_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(s, phik, (const __nv_bfloat16 *)v, idx, S, z,
                                                                        err);
        } else {
            e = cudaFuncSetAttribute(linear_delta_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem);
            if (e != cudaSuccess) return e;
            linear_delta_kernel<float><<<grid, 256, smem, st>>>(s, phik, (const float *)v, idx, S, z, err);
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return launch_linear_prefix(s, S, z, st_t, st);
}

cudaError_t launch_linear_prefix(const Dims &s, float *S, float *z, void *st_t, cudaStream_t st) {
    if ((size_t)s.B * s.Hkv * s.D * s.d == 0) return cudaSuccess;
    const dim3 grid((unsigned)((s.d + 31) / 32), (unsigned)((s.D + kPfxRows - 1) / kPfxRows), (unsigned)(s.B * s.Hkv));
    linear_prefix_kernel<<<grid, kPfxThreads, 0, st>>>(s, S, z, static_cast<__nv_bfloat16 *>(st_t));
    return cudaGetLastError();
}

cudaError_t launch_merge_generic(const Dims &s, const void *q, const void *k, const void *v, const void *Wq,
                                 const void *khat, const void *vhat, const float *S, const float *z,
                                 const float *phik, void *o, cudaStream_t st) {
    if (s.N == 0 || s.B == 0) return cudaSuccess;
    dim3 grid((s.N + 3) / 4, s.B * s.H);
    typedef __nv_bfloat16 bf;
    if (s.bf16)
        merge_generic_kernel<bf><<<grid, 128, 0, st>>>(s, (const bf *)q, (const bf *)k, (const bf *)v,
                                                       (const bf *)Wq, (const bf *)khat, (const bf *)vhat, S, z,
                                                       phik, (bf *)o);
    else
        merge_generic_kernel<float><<<grid, 128, 0, st>>>(s, (const float *)q, (const float *)k, (const float *)v,
                                                          (const float *)Wq, (const float *)khat,
                                                          (const float *)vhat, S, z, phik, (float *)o);
    return cudaGetLastError();
}

}  // namespace still
