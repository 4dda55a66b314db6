// kernels_decode.cu -- chunk-granular delayed decode ([p1] jsqmd.com "Chunk-Wise": during
// decoding the token selection is delayed at chunk granularity) and the prefill -> decode
// state hand-off, for "STILL: Selecting Tokens for Intra-Layer Hybrid Attention to Linearize LLMs".
//
// State per (b, g): kept K/V cache (chunk order), linear state S [D,d] / z [D], and a ring of
// m+1 chunk slots holding K/V rows and scores of the chunks t-m..t still inside the window.
// One step at position p (chunk t = p / C):
//   append  -> ring row of p;
//   attn    -> split-K online softmax over [kept rows 0..k(t-m)) ++ window [max(0,(t-m)C), p],
//              plus the band statistics of the new token's Self-Saliency Score;
//   combine -> merges the splits, adds phi(q)^T S and phi(q)^T z under one normaliser, writes o,
//              and stores the group score of p in the ring;
//   close   -> only when p ends chunk t and c = t-m >= 0: top-k of chunk c on the stored scores,
//              append its kept rows, fold the others into S and z.
#include "common.cuh"
#include "rowops.cuh"
#include "still_internal.h"
#include "tc_ptx.cuh"
#include "topk.cuh"

namespace still {

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

DecodeLayout decode_layout(const Dims &s, int capacity) {
    DecodeLayout L{};
    const size_t es = s.bf16 ? 2 : 4, BK = (size_t)s.B * s.Hkv;
    L.cap_chunks = capacity / s.C;
    L.ring_rows = (s.w > 0 ? s.m() + 1 : 1) * s.C;
    L.nsplit_max = kDecodeMaxSplits;
    size_t off = 0;
    L.header = off;
    off += 256;
    L.khat = off;
    off = align256(off + BK * L.cap_chunks * s.k * s.d * es);
    L.vhat = off;
    off = align256(off + BK * L.cap_chunks * s.k * s.d * es);
    L.S = off;
    off = align256(off + BK * s.D * s.d * 4);
    L.z = off;
    off = align256(off + BK * s.D * 4);
    L.ring_k = off;
    off = align256(off + BK * L.ring_rows * s.d * es);
    L.ring_v = off;
    off = align256(off + BK * L.ring_rows * s.d * es);
    L.ring_r = off;
    off = align256(off + BK * L.ring_rows * 4);
    L.part = off;
    off = align256(off + (size_t)s.B * s.H * kDecodeMaxSplits * (s.d + 2) * 4);
    L.band = off;
    off = align256(off + (size_t)s.B * s.H * kDecodeMaxSplits * 3 * 4);
    L.total = off;
    return L;
}

namespace {

struct StepGeom {
    int pos, t, lo, nk, n, nsplit, per;
};

__device__ __forceinline__ int ring_row(const Dims &s, int j) {
    const int slot = s.w > 0 ? (j / s.C) % (s.m() + 1) : 0;
    return slot * s.C + j % s.C;
}

template <typename T>
__global__ void decode_append_kernel(Dims s, DecodeLayout L, unsigned char *state, int pos, const T *__restrict__ k_t,
                                     const T *__restrict__ v_t, unsigned *err) {
    const int bg = blockIdx.x;
    if (bg == 0 && threadIdx.x == 0) {
        const DecodeHeader *hd = reinterpret_cast<const DecodeHeader *>(state + L.header);
        if (hd->pos != pos) report(err, DEV_ERR_POSITION);
    }
    T *rk = reinterpret_cast<T *>(state + L.ring_k) + ((size_t)bg * L.ring_rows + ring_row(s, pos)) * s.d;
    T *rv = reinterpret_cast<T *>(state + L.ring_v) + ((size_t)bg * L.ring_rows + ring_row(s, pos)) * s.d;
    for (int x = threadIdx.x; x < s.d; x += blockDim.x) {
        rk[x] = k_t[(size_t)bg * s.d + x];
        rv[x] = v_t[(size_t)bg * s.d + x];
    }
}

// Row of key number li of the softmax list [kept 0..nk) ++ window [lo, pos].
template <typename T>
__device__ __forceinline__ const T *list_row(const Dims &s, const DecodeLayout &L, const unsigned char *state, int bg,
                                             const StepGeom &gm, int li, bool value) {
    if (li < gm.nk) {
        const T *base = reinterpret_cast<const T *>(state + (value ? L.vhat : L.khat));
        return base + ((size_t)bg * L.cap_chunks * s.k + li) * s.d;
    }
    const int j = gm.lo + (li - gm.nk);
    const T *base = reinterpret_cast<const T *>(state + (value ? L.ring_v : L.ring_k));
    return base + ((size_t)bg * L.ring_rows + ring_row(s, j)) * s.d;
}

template <typename T>
__global__ void __launch_bounds__(128) decode_attn_kernel(Dims s, DecodeLayout L, unsigned char *state, StepGeom gm,
                                                          const T *__restrict__ q_t) {
    __shared__ __align__(16) float qs[4][kMaxD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bg = blockIdx.x, split = blockIdx.y, b = bg / s.Hkv, g = bg % s.Hkv, G = s.G();
    const int l0 = split * gm.per, l1 = min(gm.n, l0 + gm.per);
    const int band_lo = max(0, gm.pos - s.w + 1);  // band keys [band_lo, pos-1], diagonal pos
    float *part = reinterpret_cast<float *>(state + L.part);
    float *band = reinterpret_cast<float *>(state + L.band);
    for (int hh = warp; hh < G; hh += 4) {
        const int h = g * G + hh;
        for (int x = lane; x < s.d; x += 32) qs[warp][x] = to_f(q_t[((size_t)b * s.H + h) * s.d + x]);
        __syncwarp();
        float acc[kMaxD / 32];
#pragma unroll
        for (int u = 0; u < kMaxD / 32; ++u) acc[u] = 0.f;
        float M = -INFINITY, Ls = 0.f, bm = -INFINITY, bl = 0.f, sdiag = -INFINITY;
        for (int base = l0; base < l1; base += 32) {
            const int li = base + lane;
            float l = -INFINITY;
            if (li < l1) {
                l = s.scale * dot_row(qs[warp], list_row<T>(s, L, state, bg, gm, li, false), s.d);
                if (li >= gm.nk) {
                    const int j = gm.lo + (li - gm.nk);
                    if (j == gm.pos) sdiag = l;
                    else if (j >= band_lo) {
                        if (l > bm) {
                            bl = bl * expf(bm - l) + 1.f;
                            bm = l;
                        } else {
                            bl += expf(l - bm);
                        }
                    }
                }
            }
            float gmx = warp_max(l);
            float nm = fmaxf(M, gmx);
            float so = (M == -INFINITY) ? 0.f : expf(M - nm);
            float p = li < l1 ? expf(l - nm) : 0.f;
            Ls = Ls * so + warp_sum(p);
#pragma unroll
            for (int u = 0; u < kMaxD / 32; ++u) acc[u] *= so;
            const int cnt = min(32, l1 - base);
            for (int jj = 0; jj < cnt; ++jj) {
                float pj = __shfl_sync(0xffffffffu, p, jj);
                const T *vr = list_row<T>(s, L, state, bg, gm, base + jj, true);
#pragma unroll
                for (int u = 0; u < kMaxD / 32; ++u) {
                    int x = lane + 32 * u;
                    if (x < s.d) acc[u] = fmaf(pj, to_f(vr[x]), acc[u]);
                }
            }
            M = nm;
        }
        // combine the lanes' band statistics
        float BM = warp_max(bm);
        float BL = warp_sum(bm == -INFINITY ? 0.f : bl * expf(bm - BM));
        float SD = warp_max(sdiag);
        const size_t pi = ((size_t)b * s.H + h) * kDecodeMaxSplits + split;
        float *pp = part + pi * (s.d + 2);
        if (lane == 0) {
            pp[0] = M;
            pp[1] = Ls;
            band[pi * 3 + 0] = BM;
            band[pi * 3 + 1] = BL;
            band[pi * 3 + 2] = SD;
        }
#pragma unroll
        for (int u = 0; u < kMaxD / 32; ++u) {
            int x = lane + 32 * u;
            if (x < s.d) pp[2 + x] = acc[u];
        }
        __syncwarp();
    }
}

// One lane's DPL consecutive elements of a K or V row, held in the storage type until used.
template <typename T, int DPL>
struct RowSlice;
template <>
struct RowSlice<__nv_bfloat16, 4> {
    uint2 u;
    __device__ __forceinline__ void load(const __nv_bfloat16 *row, int lane) {
        u = __ldg(reinterpret_cast<const uint2 *>(row) + lane);
    }
    __device__ __forceinline__ void get(float (&f)[4]) const {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
        const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
        f[0] = a.x; f[1] = a.y; f[2] = c.x; f[3] = c.y;
    }
};
template <>
struct RowSlice<__nv_bfloat16, 2> {
    unsigned u;
    __device__ __forceinline__ void load(const __nv_bfloat16 *row, int lane) {
        u = __ldg(reinterpret_cast<const unsigned *>(row) + lane);
    }
    __device__ __forceinline__ void get(float (&f)[2]) const {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u));
        f[0] = a.x; f[1] = a.y;
    }
};
template <int DPL>
struct RowSlice<float, DPL> {
    float v[DPL];
    __device__ __forceinline__ void load(const float *row, int lane) {
#pragma unroll
        for (int e = 0; e < DPL; ++e) v[e] = __ldg(row + lane * DPL + e);
    }
    __device__ __forceinline__ void get(float (&f)[DPL]) const {
#pragma unroll
        for (int e = 0; e < DPL; ++e) f[e] = v[e];
    }
};

// Split-K decode attention with the G query heads of a KV group packed into each warp: a warp step
// takes KG = 32/G keys; every lane loads its DPL-element slice of those K and V rows (coalesced), forms
// the 32 partial dot products (key, head), and a reduce-scatter across the warp leaves the full score
// of pair (lane / G, lane % G) in each lane.  Online softmax per head (max and sum over the lanes of a
// head), P V accumulated per head in each lane's slice, and the band statistics of the new token's
// Self-Saliency Score ([i-w+1, i-1] plus the diagonal) from the same scores.  Scores are kept in log2
// units; the partials are written in natural units (same format as decode_attn_kernel).
template <int G>
__device__ __forceinline__ float reduce_scatter32(float (&v)[32], int lane) {
    // after the step with offset o the lane keeps the half of its values selected by bit o of its id
#pragma unroll
    for (int o = 16, n = 32; o >= 1; o >>= 1, n >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = upper ? v[i] : v[i + n / 2];
            const float keep = upper ? v[i + n / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return v[0];
}

template <typename T, int DPL, int G>
__global__ void __launch_bounds__(256) decode_attn_packed_kernel(Dims s, DecodeLayout L, unsigned char *state,
                                                                 StepGeom gm, const T *__restrict__ q_t) {
    constexpr int KG = 32 / G, NW = 8, DD = 32 * DPL;
    constexpr float kL2e = 1.4426950408889634f, kLn2f = 0.6931471805599453f;
    __shared__ float sm_ml[NW][G][5];          // m, l, bm, bl, sdiag (log2 units)
    __shared__ float sm_acc[NW][G][DD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bg = blockIdx.x, split = blockIdx.y, b = bg / s.Hkv, g = bg % s.Hkv;
    const int l0 = split * gm.per, l1 = min(gm.n, l0 + gm.per);
    const int band_lo = max(0, gm.pos - s.w + 1);
    const float sl2 = s.scale * kL2e;
    float qv[G][DPL];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        RowSlice<T, DPL> r;
        r.load(q_t + ((size_t)b * s.H + g * G + h) * s.d, lane);
        r.get(qv[h]);
#pragma unroll
        for (int e = 0; e < DPL; ++e) qv[h][e] *= sl2;
    }
    float m = -INFINITY, l = 0.f, bm = -INFINITY, bl = 0.f, sd = -INFINITY;
    float acc[G][DPL];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[h][e] = 0.f;
    const int my_kk = lane / G;
    const size_t dv_kept = L.vhat - L.khat, dv_ring = L.ring_v - L.ring_k;
    for (int base = l0 + warp * KG; base < l1; base += NW * KG) {
        // lane kk < KG works out where key base+kk lives (byte offset of its K row in the state; bit 0
        // set for a window-ring row) and the warp shares it; keys past the end re-read the last key of
        // the range, with probability zero
        unsigned long long my_off = 0;
        if (lane < KG) {
            const int li = min(base + lane, l1 - 1);
            if (li < gm.nk) {
                my_off = L.khat + ((size_t)bg * L.cap_chunks * s.k + li) * s.d * sizeof(T);
            } else {
                const int j = gm.lo + (li - gm.nk);
                my_off = (L.ring_k + ((size_t)bg * L.ring_rows + ring_row(s, j)) * s.d * sizeof(T)) | 1ull;
            }
        }
        RowSlice<T, DPL> kr[KG], vr[KG];
#pragma unroll
        for (int kk = 0; kk < KG; ++kk) {
            const unsigned long long off = __shfl_sync(0xffffffffu, my_off, kk);
            const size_t ko = off & ~1ull, vo = ko + ((off & 1ull) ? dv_ring : dv_kept);
            kr[kk].load(reinterpret_cast<const T *>(state + ko), lane);
            vr[kk].load(reinterpret_cast<const T *>(state + vo), lane);
        }
        float part[32];
#pragma unroll
        for (int kk = 0; kk < KG; ++kk) {
            float kf[DPL];
            kr[kk].get(kf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < DPL; ++e) a = fmaf(qv[h][e], kf[e], a);
                part[kk * G + h] = a;
            }
        }
        float sc = reduce_scatter32<G>(part, lane);
        const int li = base + my_kk;
        const bool valid = li < l1;
        if (!valid) sc = -INFINITY;
        if (valid && li >= gm.nk) {
            const int j = gm.lo + (li - gm.nk);
            if (j == gm.pos) {
                sd = sc;
            } else if (j >= band_lo) {
                if (sc > bm) {
                    bl = bl * exp2f(bm - sc) + 1.f;
                    bm = sc;
                } else {
                    bl += exp2f(sc - bm);
                }
            }
        }
        float gmx = sc;
#pragma unroll
        for (int o = G; o < 32; o <<= 1) gmx = fmaxf(gmx, __shfl_xor_sync(0xffffffffu, gmx, o));
        const float mn = fmaxf(m, gmx);
        const float so = (m == -INFINITY) ? 0.f : exp2f(m - mn);
        const float pr = valid ? exp2f(sc - mn) : 0.f;
        float gs = pr;
#pragma unroll
        for (int o = G; o < 32; o <<= 1) gs += __shfl_xor_sync(0xffffffffu, gs, o);
        l = l * so + gs;
        m = mn;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float a = __shfl_sync(0xffffffffu, so, h);
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[h][e] *= a;
        }
#pragma unroll
        for (int kk = 0; kk < KG; ++kk) {
            float vf[DPL];
            vr[kk].get(vf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float pk = __shfl_sync(0xffffffffu, pr, kk * G + h);
#pragma unroll
                for (int e = 0; e < DPL; ++e) acc[h][e] = fmaf(pk, vf[e], acc[h][e]);
            }
        }
    }
    // band statistics: combine the lanes of each head
#pragma unroll
    for (int o = G; o < 32; o <<= 1) {
        const float obm = __shfl_xor_sync(0xffffffffu, bm, o);
        const float obl = __shfl_xor_sync(0xffffffffu, bl, o);
        const float nbm = fmaxf(bm, obm);
        bl = (bm == -INFINITY ? 0.f : bl * exp2f(bm - nbm)) + (obm == -INFINITY ? 0.f : obl * exp2f(obm - nbm));
        bm = nbm;
        sd = fmaxf(sd, __shfl_xor_sync(0xffffffffu, sd, o));
    }
    if (lane < G) {
        sm_ml[warp][lane][0] = m;
        sm_ml[warp][lane][1] = l;
        sm_ml[warp][lane][2] = bm;
        sm_ml[warp][lane][3] = bl;
        sm_ml[warp][lane][4] = sd;
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < DPL; ++e) sm_acc[warp][h][lane * DPL + e] = acc[h][e];
    __syncthreads();
    // combine the warps: per head and element
    float *part_out = reinterpret_cast<float *>(state + L.part);
    float *band_out = reinterpret_cast<float *>(state + L.band);
    for (int t = threadIdx.x; t < G * DD; t += blockDim.x) {
        const int h = t / DD, x = t % DD;
        float M = -INFINITY;
#pragma unroll
        for (int w_ = 0; w_ < NW; ++w_) M = fmaxf(M, sm_ml[w_][h][0]);
        float A = 0.f, Ls = 0.f;
#pragma unroll
        for (int w_ = 0; w_ < NW; ++w_) {
            const float mw = sm_ml[w_][h][0];
            const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
            A = fmaf(sm_acc[w_][h][x], f, A);
            Ls = fmaf(sm_ml[w_][h][1], f, Ls);
        }
        const size_t pi = ((size_t)b * s.H + g * G + h) * kDecodeMaxSplits + split;
        float *pp = part_out + pi * (s.d + 2);
        pp[2 + x] = A;
        if (x == 0) {
            pp[0] = M == -INFINITY ? M : M * kLn2f;
            pp[1] = Ls;
            float BM = -INFINITY, SD = -INFINITY;
#pragma unroll
            for (int w_ = 0; w_ < NW; ++w_) {
                BM = fmaxf(BM, sm_ml[w_][h][2]);
                SD = fmaxf(SD, sm_ml[w_][h][4]);
            }
            float BL = 0.f;
#pragma unroll
            for (int w_ = 0; w_ < NW; ++w_) {
                const float b_ = sm_ml[w_][h][2];
                if (b_ != -INFINITY) BL = fmaf(sm_ml[w_][h][3], exp2f(b_ - BM), BL);
            }
            band_out[pi * 3 + 0] = BM == -INFINITY ? BM : BM * kLn2f;
            band_out[pi * 3 + 1] = BL;
            band_out[pi * 3 + 2] = SD == -INFINITY ? SD : SD * kLn2f;
        }
    }
}

// bf16 decode attention on the warp-level tensor-core instruction (mma.sync m16n8k16, fp32
// accumulate).  The step is bound by HBM (every kept and window row is read once); the SIMT form of
// the same contraction spends more issue slots on shuffles and conversions than the memory time
// allows, while one MMA covers a 16 x 8 x 16 block.  Per warp step of 16 keys:
//   S = Q K^T   (M = 16 rows: the G <= 8 query heads of the group, the rest zero; N = 8 keys; K = 16
//               dims): a lane loads one 16-byte slice of a K row and uses it as the B fragments of two
//               k-steps; Q's fragments follow the same permutation of the head dimension (a dot
//               product does not depend on the order of its terms);
//   O^T += V^T P^T  (M = 16 head dims, N = 8 heads, K = 16 keys): P^T is the score fragment as it
//               stands (bf16), V^T pairs two V rows per register with a byte permute; a lane loads a
//               contiguous DH/8-dim slice of four V rows, and row r of m-tile mt is head dim
//               (DH/8) * (r % 8) + (DH/16) * (r / 8) + mt.
// The next step's K/V rows are loaded before the current step is computed (two register buffers), so
// every warp keeps two steps of loads in flight.  Scores in log2 units; partials are written in
// natural units (same format as decode_attn_kernel).
__device__ __forceinline__ void mma16816(float (&c)[4], unsigned a0, unsigned a1, unsigned a2, unsigned a3,
                                         unsigned b0, unsigned b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int DH>
struct DecodeKV {
    uint4 k[2][DH / 32];  // K rows gq and gq+8: dims 32i + 8c .. +8
    uint4 v[4][DH / 64];  // V rows 2c, 2c+1, 2c+8, 2c+9: dims (DH/8) gq .. +DH/8
};

template <int DH, int G>
__global__ void __launch_bounds__(128, 2) decode_attn_mma_kernel(Dims s, DecodeLayout L, unsigned char *state,
                                                                 StepGeom gm, const __nv_bfloat16 *__restrict__ q_t) {
    constexpr int NW = 4, NQ = DH / 32, NM = DH / 16, VW = DH / 64;
    constexpr float kL2e = 1.4426950408889634f, kLn2f = 0.6931471805599453f;
    static_assert(G >= 1 && G <= 8 && (DH == 64 || DH == 128), "decode mma shape");
    __shared__ float sm_ml[NW][G][5];  // m, l, bm, bl, sdiag (log2 units)
    __shared__ float sm_acc[NW][G][DH];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, c = lane & 3;
    const int bg = blockIdx.x, split = blockIdx.y, b = bg / s.Hkv, g = bg % s.Hkv;
    const int l0 = split * gm.per, l1 = min(gm.n, l0 + gm.per);
    const int band_lo = max(0, gm.pos - s.w + 1);
    const float sl2 = s.scale * kL2e;
    const size_t dv_kept = L.vhat - L.khat, dv_ring = L.ring_v - L.ring_k;
    constexpr size_t kRow = DH * sizeof(__nv_bfloat16);

    unsigned qa0[2 * NQ], qa2[2 * NQ];
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        uint4 u = make_uint4(0u, 0u, 0u, 0u);
        if (gq < G) u = __ldg(reinterpret_cast<const uint4 *>(q_t + ((size_t)b * s.H + g * G + gq) * DH) + 4 * i + c);
        qa0[2 * i] = u.x;
        qa2[2 * i] = u.y;
        qa0[2 * i + 1] = u.z;
        qa2[2 * i + 1] = u.w;
    }
    float ot[NM][4];
#pragma unroll
    for (int mt = 0; mt < NM; ++mt) ot[mt][0] = ot[mt][1] = ot[mt][2] = ot[mt][3] = 0.f;
    float m = -INFINITY, l = 0.f, bm = -INFINITY, bl = 0.f, sd = -INFINITY;

    // lane kk < 16 locates key base+kk (byte offset of its K row in the state, bit 0 set for a
    // window-ring row) and the warp shares it; keys past the end re-read the last key of the range
    // with probability zero
    auto load = [&](DecodeKV<DH> &t, int base) {
        unsigned long long my_off = 0;
        if (lane < 16) {
            const int li = min(base + lane, l1 - 1);
            if (li < gm.nk) {
                my_off = L.khat + ((size_t)bg * L.cap_chunks * s.k + li) * kRow;
            } else {
                const int j = gm.lo + (li - gm.nk);
                my_off = (L.ring_k + ((size_t)bg * L.ring_rows + ring_row(s, j)) * kRow) | 1ull;
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const unsigned long long off = __shfl_sync(0xffffffffu, my_off, gq + 8 * h) & ~1ull;
            const uint4 *row = reinterpret_cast<const uint4 *>(state + off);
#pragma unroll
            for (int i = 0; i < NQ; ++i) t.k[h][i] = __ldg(row + 4 * i + c);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const unsigned long long off = __shfl_sync(0xffffffffu, my_off, 2 * c + (r & 1) + 8 * (r >> 1));
            const size_t vo = (off & ~1ull) + ((off & 1ull) ? dv_ring : dv_kept);
            const uint4 *row = reinterpret_cast<const uint4 *>(state + vo);
#pragma unroll
            for (int i = 0; i < VW; ++i) t.v[r][i] = __ldg(row + gq * VW + i);
        }
    };
    auto process = [&](const DecodeKV<DH> &t, int base) {
        // S for keys base+[0,8) and base+[8,16)
        float st[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            st[h][0] = st[h][1] = st[h][2] = st[h][3] = 0.f;
#pragma unroll
            for (int i = 0; i < NQ; ++i) {
                mma16816(st[h], qa0[2 * i], 0u, qa2[2 * i], 0u, t.k[h][i].x, t.k[h][i].y);
                mma16816(st[h], qa0[2 * i + 1], 0u, qa2[2 * i + 1], 0u, t.k[h][i].z, t.k[h][i].w);
            }
        }
        // this lane's scores: head gq, keys 2c, 2c+1, 8+2c, 9+2c
        float sc[4];
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int li = base + 2 * c + (e & 1) + 8 * (e >> 1);
            float x = st[e >> 1][e & 1] * sl2;
            if (li >= l1) x = -INFINITY;
            if (li < l1 && li >= gm.nk) {
                const int j = gm.lo + (li - gm.nk);
                if (j == gm.pos) {
                    sd = x;
                } else if (j >= band_lo) {
                    if (x > bm) {
                        bl = bl * tc::ex2(bm - x) + 1.f;
                        bm = x;
                    } else {
                        bl += tc::ex2(x - bm);
                    }
                }
            }
            sc[e] = x;
            mx = fmaxf(mx, x);
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float mn = fmaxf(m, mx);      // finite: key base+0 is always in range
        const float so = tc::ex2(m - mn);  // m = -inf gives 0
        float p[4], ps = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            p[e] = tc::ex2(sc[e] - mn);
            ps += p[e];
        }
        ps += __shfl_xor_sync(0xffffffffu, ps, 1);
        ps += __shfl_xor_sync(0xffffffffu, ps, 2);
        l = l * so + ps;
        m = mn;
        // O^T columns are heads 2c and 2c+1: their factors live in the lanes of rows 2c, 2c+1
        const float so0 = __shfl_sync(0xffffffffu, so, 8 * c), so1 = __shfl_sync(0xffffffffu, so, 8 * c + 4);
#pragma unroll
        for (int mt = 0; mt < NM; ++mt) {
            ot[mt][0] *= so0;
            ot[mt][1] *= so1;
            ot[mt][2] *= so0;
            ot[mt][3] *= so1;
        }
        const unsigned pb0 = tc::pack_bf16x2(p[0], p[1]), pb1 = tc::pack_bf16x2(p[2], p[3]);
        const unsigned *w0 = reinterpret_cast<const unsigned *>(&t.v[0][0]);
        const unsigned *w1 = reinterpret_cast<const unsigned *>(&t.v[1][0]);
        const unsigned *w2 = reinterpret_cast<const unsigned *>(&t.v[2][0]);
        const unsigned *w3 = reinterpret_cast<const unsigned *>(&t.v[3][0]);
#pragma unroll
        for (int mt = 0; mt < NM; ++mt) {
            const unsigned sel = (mt & 1) ? 0x7632u : 0x5410u;
            const int lo_w = mt >> 1, hi_w = (NM + mt) >> 1;
            const unsigned a0 = __byte_perm(w0[lo_w], w1[lo_w], sel);
            const unsigned a1 = __byte_perm(w0[hi_w], w1[hi_w], sel);
            const unsigned a2 = __byte_perm(w2[lo_w], w3[lo_w], sel);
            const unsigned a3 = __byte_perm(w2[hi_w], w3[hi_w], sel);
            mma16816(ot[mt], a0, a1, a2, a3, pb0, pb1);
        }
    };

    {
        DecodeKV<DH> ta, tb;
        constexpr int kStep = NW * 16;
        int base = l0 + warp * 16;
        if (base < l1) load(ta, base);
        while (base < l1) {
            if (base + kStep < l1) load(tb, base + kStep);
            process(ta, base);
            base += kStep;
            if (base >= l1) break;
            if (base + kStep < l1) load(ta, base + kStep);
            process(tb, base);
            base += kStep;
        }
    }
    // band statistics of head gq: combine the four lanes of the row
#pragma unroll
    for (int x = 1; x <= 2; x <<= 1) {
        const float obm = __shfl_xor_sync(0xffffffffu, bm, x);
        const float obl = __shfl_xor_sync(0xffffffffu, bl, x);
        const float nbm = fmaxf(bm, obm);
        bl = (bm == -INFINITY ? 0.f : bl * tc::ex2(bm - nbm)) + (obm == -INFINITY ? 0.f : obl * tc::ex2(obm - nbm));
        bm = nbm;
        sd = fmaxf(sd, __shfl_xor_sync(0xffffffffu, sd, x));
    }
    if (gq < G) {
        if (c == 0) {
            sm_ml[warp][gq][0] = m;
            sm_ml[warp][gq][1] = l;
            sm_ml[warp][gq][2] = bm;
            sm_ml[warp][gq][3] = bl;
            sm_ml[warp][gq][4] = sd;
        }
    }
    // O^T: columns heads 2c, 2c+1; rows gq (dims (DH/8) gq + mt) and gq+8 (dims (DH/8) gq + DH/16 + mt)
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
        const int hh = 2 * c + hc;
        if (hh < G) {
#pragma unroll
            for (int mt = 0; mt < NM; ++mt) {
                sm_acc[warp][hh][2 * NM * gq + mt] = ot[mt][hc];
                sm_acc[warp][hh][2 * NM * gq + NM + mt] = ot[mt][2 + hc];
            }
        }
    }
    __syncthreads();
    float *part_out = reinterpret_cast<float *>(state + L.part);
    float *band_out = reinterpret_cast<float *>(state + L.band);
    for (int t = threadIdx.x; t < G * DH; t += blockDim.x) {
        const int h = t / DH, x = t % DH;
        float M = -INFINITY;
#pragma unroll
        for (int w_ = 0; w_ < NW; ++w_) M = fmaxf(M, sm_ml[w_][h][0]);
        float A = 0.f, Ls = 0.f;
#pragma unroll
        for (int w_ = 0; w_ < NW; ++w_) {
            const float mw = sm_ml[w_][h][0];
            const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
            A = fmaf(sm_acc[w_][h][x], f, A);
            Ls = fmaf(sm_ml[w_][h][1], f, Ls);
        }
        const size_t pi = ((size_t)b * s.H + g * G + h) * kDecodeMaxSplits + split;
        float *pp = part_out + pi * (DH + 2);
        pp[2 + x] = A;
        if (x == 0) {
            pp[0] = M == -INFINITY ? M : M * kLn2f;
            pp[1] = Ls;
            float BM = -INFINITY, SD = -INFINITY;
#pragma unroll
            for (int w_ = 0; w_ < NW; ++w_) {
                BM = fmaxf(BM, sm_ml[w_][h][2]);
                SD = fmaxf(SD, sm_ml[w_][h][4]);
            }
            float BL = 0.f;
#pragma unroll
            for (int w_ = 0; w_ < NW; ++w_) {
                const float b_ = sm_ml[w_][h][2];
                if (b_ != -INFINITY) BL = fmaf(sm_ml[w_][h][3], exp2f(b_ - BM), BL);
            }
            band_out[pi * 3 + 0] = BM == -INFINITY ? BM : BM * kLn2f;
            band_out[pi * 3 + 1] = BL;
            band_out[pi * 3 + 2] = SD == -INFINITY ? SD : SD * kLn2f;
        }
    }
}

// The tensor-core decode attention with the K/V rows staged in shared memory by 1-D bulk
// copies (cp.async.bulk, no multicast): every warp owns a ring of NST stages of 16 keys (K and V
// tiles, 16 rows each) and keeps NST tiles in flight without holding them in registers; lane 0
// issues one copy per contiguous run of rows (kept cache rows of the group are contiguous, window
// rows are contiguous within a chunk's ring slot).  Fragments are read from the stage with 16-byte
// shared loads in the layout the register version used.
// 1-D bulk copy from global memory into this CTA's shared memory (no multicast), completing on an
// mbarrier.  Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before later async-proxy ones
// (a bulk copy into a buffer the thread has just read).
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

template <int DH>
struct DecodeBulkCfg {
    static constexpr int NW = 4, NST = 3, ROWS = 16;
    static constexpr int TILE = ROWS * DH * 2;  // bytes of the K (or V) rows of one stage
    static constexpr int STAGE = 2 * TILE;
    static constexpr int RING = NST * STAGE;    // per warp
    static constexpr int SMEM = NW * RING + NW * NST * 8;
};

__device__ __forceinline__ bool bar_wait_bounded(uint32_t bar, uint32_t parity) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = tc::globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0 && tc::globaltimer_ns() - t0 > tc::kWaitLimitNs) return false;
    }
}

// k_t, v_t (optional): the step's new key and value, appended here instead of by a kernel of their
// own: the CTA whose key range ends the list (it holds the diagonal, position pos) writes them into
// the window ring before any of its copies start.
template <int DH, int G>
__global__ void __launch_bounds__(128, 2) decode_attn_bulk_kernel(Dims s, DecodeLayout L, unsigned char *state,
                                                                  StepGeom gm, const __nv_bfloat16 *__restrict__ q_t,
                                                                  const __nv_bfloat16 *__restrict__ k_t,
                                                                  const __nv_bfloat16 *__restrict__ v_t,
                                                                  unsigned *err) {
    using Cfg = DecodeBulkCfg<DH>;
    constexpr int NW = Cfg::NW, NST = Cfg::NST, NQ = DH / 32, NM = DH / 16, VW = DH / 64;
    constexpr float kL2e = 1.4426950408889634f, kLn2f = 0.6931471805599453f;
    static_assert(G >= 1 && G <= 8 && (DH == 64 || DH == 128), "decode mma shape");
    static_assert(NW * G * (5 + DH) * 4 <= NW * Cfg::RING, "combine area fits in the rings");
    extern __shared__ __align__(128) unsigned char dsm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gq = lane >> 2, c = lane & 3;
    const int bg = blockIdx.x, split = blockIdx.y, b = bg / s.Hkv, g = bg % s.Hkv;
    const int l0 = split * gm.per, l1 = min(gm.n, l0 + gm.per);
    const int band_lo = max(0, gm.pos - s.w + 1);
    const float sl2 = s.scale * kL2e;
    unsigned char *ring = dsm + warp * Cfg::RING;
    const uint32_t bar0 = tc::smem_u32(dsm + NW * Cfg::RING) + warp * NST * 8;
    const __nv_bfloat16 *khat = reinterpret_cast<const __nv_bfloat16 *>(state + L.khat);
    const __nv_bfloat16 *vhat = reinterpret_cast<const __nv_bfloat16 *>(state + L.vhat);
    const __nv_bfloat16 *rk = reinterpret_cast<const __nv_bfloat16 *>(state + L.ring_k);
    const __nv_bfloat16 *rv = reinterpret_cast<const __nv_bfloat16 *>(state + L.ring_v);

    if (lane == 0) {
        for (int st = 0; st < NST; ++st) tc::mbar_init(bar0 + st * 8, 1);
        tc::mbar_fence_init();
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (k_t) {
        if (bg == 0 && split == 0 && threadIdx.x == 0 &&
            reinterpret_cast<const DecodeHeader *>(state + L.header)->pos != gm.pos)
            report(err, DEV_ERR_POSITION);
        if (l1 == gm.n) {
            const size_t row = (size_t)bg * L.ring_rows + ring_row(s, gm.pos);
            for (int x = threadIdx.x; x < DH / 8; x += blockDim.x) {
                reinterpret_cast<uint4 *>(const_cast<__nv_bfloat16 *>(rk) + row * DH)[x] =
                    __ldg(reinterpret_cast<const uint4 *>(k_t + (size_t)bg * DH) + x);
                reinterpret_cast<uint4 *>(const_cast<__nv_bfloat16 *>(rv) + row * DH)[x] =
                    __ldg(reinterpret_cast<const uint4 *>(v_t + (size_t)bg * DH) + x);
            }
            asm volatile("fence.proxy.async.global;" ::: "memory");  // the row, before the bulk copies read it
        }
        __syncthreads();
    }

    const int ntiles = (l1 - l0 + 15) / 16;
    const int my_tiles = ntiles > warp ? (ntiles - warp + NW - 1) / NW : 0;
    // lane 0: copies of this warp's tile number `it` into stage it % NST
    auto issue = [&](int it) {
        const int st = it % NST;
        const int k0 = l0 + 16 * (warp + NW * it), k1 = min(l1, k0 + 16);
        const uint32_t sK = tc::smem_u32(ring + st * Cfg::STAGE), sV = sK + Cfg::TILE, bar = bar0 + st * 8;
        tc::mbar_arrive_expect_tx(bar, (uint32_t)(k1 - k0) * DH * 2 * 2);
        for (int li = k0; li < k1;) {
            int end;
            size_t row;
            const __nv_bfloat16 *kb, *vb;
            if (li < gm.nk) {
                end = min(k1, gm.nk);
                row = (size_t)bg * L.cap_chunks * s.k + li;
                kb = khat;
                vb = vhat;
            } else {
                const int j = gm.lo + (li - gm.nk);
                end = min(k1, li + (s.C - j % s.C));  // to the end of j's chunk slot
                row = (size_t)bg * L.ring_rows + ring_row(s, j);
                kb = rk;
                vb = rv;
            }
            const uint32_t bytes = (uint32_t)(end - li) * DH * 2, off = (uint32_t)(li - k0) * DH * 2;
            bulk_load(sK + off, kb + row * DH, bytes, bar);
            bulk_load(sV + off, vb + row * DH, bytes, bar);
            li = end;
        }
    };
    if (lane == 0)
        for (int it = 0; it < min(NST, my_tiles); ++it) issue(it);

    unsigned qa0[2 * NQ], qa2[2 * NQ];
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        uint4 u = make_uint4(0u, 0u, 0u, 0u);
        if (gq < G) u = __ldg(reinterpret_cast<const uint4 *>(q_t + ((size_t)b * s.H + g * G + gq) * DH) + 4 * i + c);
        qa0[2 * i] = u.x;
        qa2[2 * i] = u.y;
        qa0[2 * i + 1] = u.z;
        qa2[2 * i + 1] = u.w;
    }
    float ot[NM][4];
#pragma unroll
    for (int mt = 0; mt < NM; ++mt) ot[mt][0] = ot[mt][1] = ot[mt][2] = ot[mt][3] = 0.f;
    float m = -INFINITY, l = 0.f, bm = -INFINITY, bl = 0.f, sd = -INFINITY;

    bool ok = true;
    int it = 0;
    for (; it < my_tiles; ++it) {
        const int st = it % NST;
        ok = bar_wait_bounded(bar0 + st * 8, (it / NST) & 1);
        if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
        }
        const int base = l0 + 16 * (warp + NW * it);
        const uint4 *K4 = reinterpret_cast<const uint4 *>(ring + st * Cfg::STAGE);
        const uint4 *V4 = reinterpret_cast<const uint4 *>(ring + st * Cfg::STAGE + Cfg::TILE);
        // rows past the end of a partial tile were not copied (stale or never written): read as zeros
        DecodeKV<DH> t;
        const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const bool in = base + gq + 8 * h < l1;
#pragma unroll
            for (int i = 0; i < NQ; ++i) t.k[h][i] = in ? K4[(gq + 8 * h) * (DH / 8) + 4 * i + c] : z4;
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int key = 2 * c + (r & 1) + 8 * (r >> 1);
            const bool in = base + key < l1;
#pragma unroll
            for (int i = 0; i < VW; ++i) t.v[r][i] = in ? V4[key * (DH / 8) + gq * VW + i] : z4;
        }
        // ---- S = Q K^T, online softmax, band statistics, O^T += V^T P^T (as decode_attn_mma_kernel)
        float stt[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            stt[h][0] = stt[h][1] = stt[h][2] = stt[h][3] = 0.f;
#pragma unroll
            for (int i = 0; i < NQ; ++i) {
                mma16816(stt[h], qa0[2 * i], 0u, qa2[2 * i], 0u, t.k[h][i].x, t.k[h][i].y);
                mma16816(stt[h], qa0[2 * i + 1], 0u, qa2[2 * i + 1], 0u, t.k[h][i].z, t.k[h][i].w);
            }
        }
        float sc[4];
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int li = base + 2 * c + (e & 1) + 8 * (e >> 1);
            float x = stt[e >> 1][e & 1] * sl2;
            if (li >= l1) x = -INFINITY;
            if (li < l1 && li >= gm.nk) {
                const int j = gm.lo + (li - gm.nk);
                if (j == gm.pos) {
                    sd = x;
                } else if (j >= band_lo) {
                    if (x > bm) {
                        bl = bl * tc::ex2(bm - x) + 1.f;
                        bm = x;
                    } else {
                        bl += tc::ex2(x - bm);
                    }
                }
            }
            sc[e] = x;
            mx = fmaxf(mx, x);
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float mn = fmaxf(m, mx);      // finite: key base+0 is always in range
        const float so = tc::ex2(m - mn);  // m = -inf gives 0
        float pp[4], ps = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            pp[e] = tc::ex2(sc[e] - mn);
            ps += pp[e];
        }
        ps += __shfl_xor_sync(0xffffffffu, ps, 1);
        ps += __shfl_xor_sync(0xffffffffu, ps, 2);
        l = l * so + ps;
        m = mn;
        const float so0 = __shfl_sync(0xffffffffu, so, 8 * c), so1 = __shfl_sync(0xffffffffu, so, 8 * c + 4);
#pragma unroll
        for (int mt = 0; mt < NM; ++mt) {
            ot[mt][0] *= so0;
            ot[mt][1] *= so1;
            ot[mt][2] *= so0;
            ot[mt][3] *= so1;
        }
        const unsigned pb0 = tc::pack_bf16x2(pp[0], pp[1]), pb1 = tc::pack_bf16x2(pp[2], pp[3]);
        const unsigned *w0 = reinterpret_cast<const unsigned *>(&t.v[0][0]);
        const unsigned *w1 = reinterpret_cast<const unsigned *>(&t.v[1][0]);
        const unsigned *w2 = reinterpret_cast<const unsigned *>(&t.v[2][0]);
        const unsigned *w3 = reinterpret_cast<const unsigned *>(&t.v[3][0]);
#pragma unroll
        for (int mt = 0; mt < NM; ++mt) {
            const unsigned sel = (mt & 1) ? 0x7632u : 0x5410u;
            const int lo_w = mt >> 1, hi_w = (NM + mt) >> 1;
            mma16816(ot[mt], __byte_perm(w0[lo_w], w1[lo_w], sel), __byte_perm(w0[hi_w], w1[hi_w], sel),
                     __byte_perm(w2[lo_w], w3[lo_w], sel), __byte_perm(w2[hi_w], w3[hi_w], sel), pb0, pb1);
        }
        // the stage's rows are in registers and used: hand it to the next copy
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && it + NST < my_tiles) issue(it + NST);
    }
    if (!ok) {
        if (lane == 0) {
            report(err, DEV_ERR_TIMEOUT);
            // copies this warp issued and did not consume: wait for them (bounded) before exiting
            for (int k = it; k < min(my_tiles, it + NST); ++k)
                tc::mbar_wait_drain(bar0 + (k % NST) * 8, (k / NST) & 1, 100000000ull);
        }
        __syncwarp();
    }
    // band statistics of head gq: combine the four lanes of the row
#pragma unroll
    for (int x = 1; x <= 2; x <<= 1) {
        const float obm = __shfl_xor_sync(0xffffffffu, bm, x);
        const float obl = __shfl_xor_sync(0xffffffffu, bl, x);
        const float nbm = fmaxf(bm, obm);
        bl = (bm == -INFINITY ? 0.f : bl * tc::ex2(bm - nbm)) + (obm == -INFINITY ? 0.f : obl * tc::ex2(obm - nbm));
        bm = nbm;
        sd = fmaxf(sd, __shfl_xor_sync(0xffffffffu, sd, x));
    }
    __syncthreads();  // every warp is done with its ring: reuse it for the combine
    auto sm_ml = reinterpret_cast<float (*)[G][5]>(dsm);
    auto sm_acc = reinterpret_cast<float (*)[G][DH]>(dsm + NW * G * 5 * 4);
    if (gq < G && c == 0) {
        sm_ml[warp][gq][0] = m;
        sm_ml[warp][gq][1] = l;
        sm_ml[warp][gq][2] = bm;
        sm_ml[warp][gq][3] = bl;
        sm_ml[warp][gq][4] = sd;
    }
#pragma unroll
    for (int hc = 0; hc < 2; ++hc) {
        const int hh = 2 * c + hc;
        if (hh < G) {
#pragma unroll
            for (int mt = 0; mt < NM; ++mt) {
                sm_acc[warp][hh][2 * NM * gq + mt] = ot[mt][hc];
                sm_acc[warp][hh][2 * NM * gq + NM + mt] = ot[mt][2 + hc];
            }
        }
    }
    __syncthreads();
    float *part_out = reinterpret_cast<float *>(state + L.part);
    float *band_out = reinterpret_cast<float *>(state + L.band);
    for (int t2 = threadIdx.x; t2 < G * DH; t2 += blockDim.x) {
        const int h = t2 / DH, x = t2 % DH;
        float M = -INFINITY;
#pragma unroll
        for (int w_ = 0; w_ < NW; ++w_) M = fmaxf(M, sm_ml[w_][h][0]);
        float A = 0.f, Ls = 0.f;
#pragma unroll
        for (int w_ = 0; w_ < NW; ++w_) {
            const float mw = sm_ml[w_][h][0];
            const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
            A = fmaf(sm_acc[w_][h][x], f, A);
            Ls = fmaf(sm_ml[w_][h][1], f, Ls);
        }
        const size_t pi = ((size_t)b * s.H + g * G + h) * kDecodeMaxSplits + split;
        float *pp2 = part_out + pi * (DH + 2);
        pp2[2 + x] = A;
        if (x == 0) {
            pp2[0] = M == -INFINITY ? M : M * kLn2f;
            pp2[1] = Ls;
            float BM = -INFINITY, SD = -INFINITY;
#pragma unroll
            for (int w_ = 0; w_ < NW; ++w_) {
                BM = fmaxf(BM, sm_ml[w_][h][2]);
                SD = fmaxf(SD, sm_ml[w_][h][4]);
            }
            float BL = 0.f;
#pragma unroll
            for (int w_ = 0; w_ < NW; ++w_) {
                const float b_ = sm_ml[w_][h][2];
                if (b_ != -INFINITY) BL = fmaf(sm_ml[w_][h][3], exp2f(b_ - BM), BL);
            }
            band_out[pi * 3 + 0] = BM == -INFINITY ? BM : BM * kLn2f;
            band_out[pi * 3 + 1] = BL;
            band_out[pi * 3 + 2] = SD == -INFINITY ? SD : SD * kLn2f;
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(128) decode_combine_kernel(Dims s, DecodeLayout L, unsigned char *state, StepGeom gm,
                                                             const T *__restrict__ q_t, const T *__restrict__ Wq,
                                                             const T *__restrict__ Wk, T *__restrict__ o_t) {
    __shared__ __align__(16) float qs[4][kMaxD];
    __shared__ __align__(16) float ps[4][kMaxDf];
    __shared__ __align__(16) float ks[4][kMaxD];
    __shared__ __align__(16) float pk[4][kMaxDf];
    __shared__ float sig[32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bg = blockIdx.x, b = bg / s.Hkv, g = bg % s.Hkv, G = s.G(), d = s.d, D = s.D;
    const float *part = reinterpret_cast<const float *>(state + L.part);
    const float *band = reinterpret_cast<const float *>(state + L.band);
    const float *S = reinterpret_cast<const float *>(state + L.S) + (size_t)bg * D * d;
    const float *z = reinterpret_cast<const float *>(state + L.z) + (size_t)bg * D;
    for (int hh = warp; hh < G; hh += 4) {
        const int h = g * G + hh;
        float M = -INFINITY, Ls = 0.f, BM = -INFINITY, BL = 0.f, SD = -INFINITY;
        for (int sp = 0; sp < gm.nsplit; ++sp) {
            const size_t pi = ((size_t)b * s.H + h) * kDecodeMaxSplits + sp;
            M = fmaxf(M, part[pi * (d + 2)]);
            BM = fmaxf(BM, band[pi * 3]);
            SD = fmaxf(SD, band[pi * 3 + 2]);
        }
        float acc[kMaxD / 32];
#pragma unroll
        for (int u = 0; u < kMaxD / 32; ++u) acc[u] = 0.f;
        for (int sp = 0; sp < gm.nsplit; ++sp) {
            const size_t pi = ((size_t)b * s.H + h) * kDecodeMaxSplits + sp;
            const float *pp = part + pi * (d + 2);
            const float ms = pp[0];
            const float f = ms == -INFINITY ? 0.f : expf(ms - M);
            Ls += pp[1] * f;
#pragma unroll
            for (int u = 0; u < kMaxD / 32; ++u) {
                int x = lane + 32 * u;
                if (x < d) acc[u] = fmaf(pp[2 + x], f, acc[u]);
            }
            const float bms = band[pi * 3];
            if (bms != -INFINITY) BL += band[pi * 3 + 1] * expf(bms - BM);
        }
        // saliency of the new token for this head
        float sigma = 0.f;
        if (s.w > 0) {
            const int band_lo = max(0, gm.pos - s.w + 1);
            sigma = (band_lo == gm.pos) ? INFINITY : softplus_f(SD - (BM + logf(BL)));
        }
        if (lane == 0) sig[hh] = sigma;
        // linear branch
        for (int x = lane; x < d; x += 32) qs[warp][x] = to_f(q_t[((size_t)b * s.H + h) * d + x]);
        __syncwarp();
        npmap_row_warp<T>(qs[warp], Wq + (size_t)h * d * D, d, D, ps[warp], lane);
        __syncwarp();
        float lin[kMaxD / 32];
#pragma unroll
        for (int u = 0; u < kMaxD / 32; ++u) lin[u] = 0.f;
        float lden = 0.f;
        for (int a = 0; a < D; ++a) {
            const float pa = ps[warp][a];
            lden = fmaf(pa, z[a], lden);
#pragma unroll
            for (int u = 0; u < kMaxD / 32; ++u) {
                int x = lane + 32 * u;
                if (x < d) lin[u] = fmaf(pa, S[(size_t)a * d + x], lin[u]);
            }
        }
        if (s.w == 0) {
            // open chunk [tC, pos] is linear too; features computed on the fly
            const T *rk = reinterpret_cast<const T *>(state + L.ring_k) + (size_t)bg * L.ring_rows * d;
            const T *rv = reinterpret_cast<const T *>(state + L.ring_v) + (size_t)bg * L.ring_rows * d;
            for (int j = gm.t * s.C; j <= gm.pos; ++j) {
                const int rr = j % s.C;
                for (int x = lane; x < d; x += 32) ks[warp][x] = to_f(rk[(size_t)rr * d + x]);
                __syncwarp();
                npmap_row_warp<T>(ks[warp], Wk + (size_t)g * d * D, d, D, pk[warp], lane);
                __syncwarp();
                float wpart = 0.f;
                for (int a = lane; a < D; a += 32) wpart = fmaf(ps[warp][a], pk[warp][a], wpart);
                const float wj = warp_sum(wpart);
                lden += wj;
#pragma unroll
                for (int u = 0; u < kMaxD / 32; ++u) {
                    int x = lane + 32 * u;
                    if (x < d) lin[u] = fmaf(wj, to_f(rv[(size_t)rr * d + x]), lin[u]);
                }
                __syncwarp();
            }
        }
        float Ms = M;
        if (lden > 0.f) Ms = fmaxf(M, logf(lden));
        const float a_soft = (M == -INFINITY) ? 0.f : expf(M - Ms);
        const float a_lin = (Ms == -INFINITY) ? 0.f : expf(-Ms);
        const float den = Ls * a_soft + lden * a_lin;
        const float inv = den > 0.f ? 1.f / den : 0.f;
        T *orow = o_t + ((size_t)b * s.H + h) * d;
#pragma unroll
        for (int u = 0; u < kMaxD / 32; ++u) {
            int x = lane + 32 * u;
            if (x < d) orow[x] = from_f<T>((acc[u] * a_soft + lin[u] * a_lin) * inv);
        }
        __syncwarp();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float acc = 0.f;
        for (int hh = 0; hh < G; ++hh) acc += sig[hh];
        float *rr = reinterpret_cast<float *>(state + L.ring_r);
        rr[(size_t)bg * L.ring_rows + ring_row(s, gm.pos)] = s.w > 0 ? acc / (float)G : 0.f;
        if (bg == 0) reinterpret_cast<DecodeHeader *>(state + L.header)->pos = gm.pos + 1;
    }
}

// Combine for a window (w > 0) and G <= 8: one CTA of 256 threads per (b, g) does every head of the
// group at once.  The kernel is latency bound (a few hundred KB per CTA, mostly from L2), so every
// phase gives each thread many independent 8- or 16-byte loads:
//   split weights per head (a warp per head);
//   softmax numerator: thread per (head, element pair), the splits' partials as float2;
//   Y = q Wq: thread per (head, 16-byte group of features, slice of the head dim), reduced in smem;
//   NP-Map per head ([p1] "Norm-Preserved Feature Map") and phi(q) . z (a warp per head);
//   phi(q)^T S: thread per (4 head-dim elements, slice of the features), S read once for the group
//   as float4, reduced in smem;
//   merge under the shared normaliser, group score of the new token into the ring.
constexpr int kCombineThreads = 256;

template <typename T>
struct CombineGeom {
    int G, d, D;
    int nfv, xq, xlen;  // Y: feature vectors per head (16 bytes of Wq each), head-dim slices, slice length
    int ar, alen;       // phi^T S: feature slices, slice length
    __host__ __device__ explicit CombineGeom(const Dims &s) : G(s.G()), d(s.d), D(s.D) {
        constexpr int V = 16 / (int)sizeof(T);
        nfv = D / V;
        const int combos = G * nfv;
        xq = combos >= kCombineThreads ? 1 : kCombineThreads / combos;
        xlen = (d + xq - 1) / xq;
        ar = kCombineThreads / (d / 4) > 0 ? kCombineThreads / (d / 4) : 1;
        alen = (D + ar - 1) / ar;
    }
    // floats of shared memory: weights, stats, numerator, q, phi, then one scratch area shared by the
    // Y partials [xq][G][D] and the phi^T S partials [ar][G][d]
    __host__ __device__ int smem_floats() const {
        const int scratch = max(xq * G * D, ar * G * d);
        return G * 64 + G * 8 + 2 * G * d + G * D + scratch;
    }
};

size_t combine_wide_smem(const Dims &s) {
    if (s.bf16) return (size_t)CombineGeom<__nv_bfloat16>(s).smem_floats() * sizeof(float);
    return (size_t)CombineGeom<float>(s).smem_floats() * sizeof(float);
}

__device__ __forceinline__ void unpack16(const uint4 &u, const __nv_bfloat16 *, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
        f[2 * e] = t.x;
        f[2 * e + 1] = t.y;
    }
}
__device__ __forceinline__ void unpack16(const uint4 &u, const float *, float (&f)[4]) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
}

template <typename T>
__global__ void __launch_bounds__(kCombineThreads) decode_combine_wide_kernel(Dims s, DecodeLayout L,
                                                                              unsigned char *state, StepGeom gm,
                                                                              const T *__restrict__ q_t,
                                                                              const T *__restrict__ Wq,
                                                                              T *__restrict__ o_t) {
    constexpr int V = 16 / (int)sizeof(T);
    extern __shared__ float cs[];
    const CombineGeom<T> cg(s);
    const int G = cg.G, d = cg.d, D = cg.D, ns = gm.nsplit;
    float *sf = cs;           // [G][64] weight of each split
    float *st = sf + G * 64;  // [G][8]: M, Ls, -, -, -, lden, sigma
    float *os = st + G * 8;   // [G][d] softmax numerator
    float *qs = os + G * d;   // [G][d]
    float *ph = qs + G * d;   // [G][D] Y, then phi(q)
    float *scr = ph + G * D;  // Y partials [xq][G][D], then phi^T S partials [ar][G][d]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bg = blockIdx.x, b = bg / s.Hkv, g = bg % s.Hkv;
    const float *part = reinterpret_cast<const float *>(state + L.part);
    const float *band = reinterpret_cast<const float *>(state + L.band);
    const float *S = reinterpret_cast<const float *>(state + L.S) + (size_t)bg * D * d;
    const float *z = reinterpret_cast<const float *>(state + L.z) + (size_t)bg * D;
    const size_t pb0 = ((size_t)b * s.H + g * G) * kDecodeMaxSplits;
    // the group's linear state is read late (phi^T S): start bringing it into L2 now
    for (size_t off = (size_t)tid * 128; off < (size_t)D * d * 4; off += (size_t)kCombineThreads * 128)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char *>(S) + off));

    for (int hh = warp; hh < G; hh += kCombineThreads / 32) {
        const size_t pb = pb0 + (size_t)hh * kDecodeMaxSplits;
        float M = -INFINITY, BM = -INFINITY, SD = -INFINITY;
        for (int sp = lane; sp < ns; sp += 32) {
            M = fmaxf(M, part[(pb + sp) * (d + 2)]);
            BM = fmaxf(BM, band[(pb + sp) * 3]);
            SD = fmaxf(SD, band[(pb + sp) * 3 + 2]);
        }
        M = warp_max(M);
        BM = warp_max(BM);
        SD = warp_max(SD);
        float Ls = 0.f, BL = 0.f;
        for (int sp = lane; sp < ns; sp += 32) {
            const float ms = part[(pb + sp) * (d + 2)];
            const float f = ms == -INFINITY ? 0.f : expf(ms - M);
            sf[hh * 64 + sp] = f;
            Ls = fmaf(part[(pb + sp) * (d + 2) + 1], f, Ls);
            const float bms = band[(pb + sp) * 3];
            if (bms != -INFINITY) BL = fmaf(band[(pb + sp) * 3 + 1], expf(bms - BM), BL);
        }
        Ls = warp_sum(Ls);
        BL = warp_sum(BL);
        if (lane == 0) {
            st[hh * 8 + 0] = M;
            st[hh * 8 + 1] = Ls;
            const int band_lo = max(0, gm.pos - s.w + 1);
            st[hh * 8 + 6] = (band_lo == gm.pos) ? INFINITY : softplus_f(SD - (BM + logf(BL)));
        }
    }
    for (int t = tid; t < G * d; t += kCombineThreads) qs[t] = to_f(q_t[((size_t)b * s.H + g * G) * d + t]);
    __syncthreads();
    // softmax numerator: (head, element pair); partial rows are (d + 2) floats, so 8-byte aligned
    for (int t = tid; t < G * d / 2; t += kCombineThreads) {
        const int hh = t / (d / 2), x2 = t % (d / 2);
        const float2 *pp = reinterpret_cast<const float2 *>(part + (pb0 + (size_t)hh * kDecodeMaxSplits) * (d + 2) + 2) + x2;
        const size_t stride2 = (size_t)(d + 2) / 2;
        float2 a = make_float2(0.f, 0.f);
        int sp = 0;
        for (; sp + 4 <= ns; sp += 4) {
            float2 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = pp[(size_t)(sp + u) * stride2];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float f = sf[hh * 64 + sp + u];
                a.x = fmaf(v[u].x, f, a.x);
                a.y = fmaf(v[u].y, f, a.y);
            }
        }
        for (; sp < ns; ++sp) {
            const float2 v = pp[(size_t)sp * stride2];
            const float f = sf[hh * 64 + sp];
            a.x = fmaf(v.x, f, a.x);
            a.y = fmaf(v.y, f, a.y);
        }
        os[hh * d + 2 * x2] = a.x;
        os[hh * d + 2 * x2 + 1] = a.y;
    }
    // Y = q Wq: (head, feature vector, head-dim slice)
    for (int t = tid; t < G * cg.nfv * cg.xq; t += kCombineThreads) {
        const int xs = t % cg.xq, cv = t / cg.xq, hh = cv / cg.nfv, fv = cv % cg.nfv;
        const int x0 = xs * cg.xlen, x1 = min(d, x0 + cg.xlen);
        const uint4 *w = reinterpret_cast<const uint4 *>(Wq + (size_t)(g * G + hh) * d * D) + fv;
        const int wstride = D / V;
        float y[V];
#pragma unroll
        for (int e = 0; e < V; ++e) y[e] = 0.f;
        int x = x0;
        for (; x + 8 <= x1; x += 8) {
            uint4 u[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) u[r] = __ldg(w + (size_t)(x + r) * wstride);
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                float f[V];
                unpack16(u[r], Wq, f);
                const float qv = qs[hh * d + x + r];
#pragma unroll
                for (int e = 0; e < V; ++e) y[e] = fmaf(qv, f[e], y[e]);
            }
        }
        for (; x < x1; ++x) {
            float f[V];
            unpack16(__ldg(w + (size_t)x * wstride), Wq, f);
            const float qv = qs[hh * d + x];
#pragma unroll
            for (int e = 0; e < V; ++e) y[e] = fmaf(qv, f[e], y[e]);
        }
#pragma unroll
        for (int e = 0; e < V; ++e) scr[(xs * G + hh) * D + fv * V + e] = y[e];
    }
    __syncthreads();
    for (int t = tid; t < G * D; t += kCombineThreads) {
        float y = 0.f;
        for (int xs = 0; xs < cg.xq; ++xs) y += scr[xs * G * D + t];
        ph[t] = y;
    }
    __syncthreads();
    for (int hh = warp; hh < G; hh += kCombineThreads / 32) {
        float *yh = ph + hh * D;
        float mx = -INFINITY;
        for (int a = lane; a < D; a += 32) mx = fmaxf(mx, yh[a]);
        mx = warp_max(mx);
        float ee = 0.f;
        for (int a = lane; a < D; a += 32) {
            const float e = expf(yh[a] - mx);
            yh[a] = e;
            ee = fmaf(e, e, ee);
        }
        ee = warp_sum(ee);
        float nq = 0.f;
        for (int x = lane; x < d; x += 32) nq = fmaf(qs[hh * d + x], qs[hh * d + x], nq);
        nq = warp_sum(nq);
        const float f = sqrtf(nq) / sqrtf(ee);
        float ld = 0.f;
        for (int a = lane; a < D; a += 32) {
            const float v = yh[a] * f;
            yh[a] = v;
            ld = fmaf(v, z[a], ld);
        }
        ld = warp_sum(ld);
        if (lane == 0) st[hh * 8 + 5] = ld;
    }
    __syncthreads();
    // phi(q)^T S: (4 head-dim elements, feature slice); S rows are d floats, 16-byte aligned
    if (tid < (d / 4) * cg.ar) {
        const int x4 = tid % (d / 4), as = tid / (d / 4);
        const int a0 = as * cg.alen, a1 = min(D, a0 + cg.alen);
        float4 acc[8];
#pragma unroll
        for (int hh = 0; hh < 8; ++hh) acc[hh] = make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 *S4 = reinterpret_cast<const float4 *>(S) + x4;
        int a = a0;
        for (; a + 8 <= a1; a += 8) {
            float4 sv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) sv[u] = S4[(size_t)(a + u) * (d / 4)];
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int hh = 0; hh < 8; ++hh)
                    if (hh < G) {
                        const float pv = ph[hh * D + a + u];
                        acc[hh].x = fmaf(pv, sv[u].x, acc[hh].x);
                        acc[hh].y = fmaf(pv, sv[u].y, acc[hh].y);
                        acc[hh].z = fmaf(pv, sv[u].z, acc[hh].z);
                        acc[hh].w = fmaf(pv, sv[u].w, acc[hh].w);
                    }
        }
        for (; a < a1; ++a) {
            const float4 sv = S4[(size_t)a * (d / 4)];
#pragma unroll
            for (int hh = 0; hh < 8; ++hh)
                if (hh < G) {
                    const float pv = ph[hh * D + a];
                    acc[hh].x = fmaf(pv, sv.x, acc[hh].x);
                    acc[hh].y = fmaf(pv, sv.y, acc[hh].y);
                    acc[hh].z = fmaf(pv, sv.z, acc[hh].z);
                    acc[hh].w = fmaf(pv, sv.w, acc[hh].w);
                }
        }
#pragma unroll
        for (int hh = 0; hh < 8; ++hh)
            if (hh < G) reinterpret_cast<float4 *>(scr + (as * G + hh) * d)[x4] = acc[hh];
    }
    __syncthreads();
    for (int t = tid; t < G * d; t += kCombineThreads) {
        const int hh = t / d, x = t % d;
        float lin = 0.f;
        for (int as = 0; as < cg.ar; ++as) lin += scr[(as * G + hh) * d + x];
        const float M = st[hh * 8 + 0], Ls = st[hh * 8 + 1], ld = st[hh * 8 + 5];
        const float Ms = ld > 0.f ? fmaxf(M, logf(ld)) : M;
        const float a_soft = (M == -INFINITY) ? 0.f : expf(M - Ms);
        const float a_lin = (Ms == -INFINITY) ? 0.f : expf(-Ms);
        const float den = Ls * a_soft + ld * a_lin;
        const float inv = den > 0.f ? 1.f / den : 0.f;
        o_t[((size_t)b * s.H + g * G + hh) * d + x] = from_f<T>((os[t] * a_soft + lin * a_lin) * inv);
    }
    if (tid == 0) {
        float acc = 0.f;
        for (int hh = 0; hh < G; ++hh) acc += st[hh * 8 + 6];
        float *rr = reinterpret_cast<float *>(state + L.ring_r);
        rr[(size_t)bg * L.ring_rows + ring_row(s, gm.pos)] = acc / (float)G;
        if (bg == 0) reinterpret_cast<DecodeHeader *>(state + L.header)->pos = gm.pos + 1;
    }
}

// Decide chunk c = t-m of (b, g): top-k on its stored scores, append kept rows, fold the rest.
// grid (B*Hkv, passes): each pass owns kFoldEnt*512 entries of S; pass 0 also appends the kept rows.
constexpr int kFoldTok = 16;   // rows featurised per step (one per warp)
constexpr int kFoldEnt = 32;   // S entries per thread per pass
constexpr int kFoldThreads = 512;

template <typename T>
__global__ void __launch_bounds__(kFoldThreads) decode_close_kernel(Dims s, DecodeLayout L, unsigned char *state,
                                                                    int c, const T *__restrict__ Wk, int P, int Pk) {
    extern __shared__ unsigned long long csm[];
    unsigned long long *keys = csm;                                     // P
    uint32_t *pos = reinterpret_cast<uint32_t *>(keys + P);             // Pk
    unsigned char *kept = reinterpret_cast<unsigned char *>(pos + Pk);  // C (rounded to 16)
    float *xs = reinterpret_cast<float *>(kept + ((s.C + 15) & ~15));   // [kFoldTok][d]
    float *ph = xs + kFoldTok * s.d;                                    // [kFoldTok][D]
    float *vs = ph + kFoldTok * s.D;                                    // [kFoldTok][d]
    const int bg = blockIdx.x, g = bg % s.Hkv, d = s.d, D = s.D;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = s.w > 0 ? c % (s.m() + 1) : 0;
    const float *rc = reinterpret_cast<const float *>(state + L.ring_r) + (size_t)bg * L.ring_rows + slot * s.C;
    const T *rk = reinterpret_cast<const T *>(state + L.ring_k) + ((size_t)bg * L.ring_rows + slot * s.C) * d;
    const T *rv = reinterpret_cast<const T *>(state + L.ring_v) + ((size_t)bg * L.ring_rows + slot * s.C) * d;
    for (int j = threadIdx.x; j < s.C; j += blockDim.x) kept[j] = 0;
    __syncthreads();
    if (s.k > 0) {
        block_topk(rc, s.C, s.k, keys, pos, P, Pk);  // syncs internally
        if (blockIdx.y == 0) {
            T *kh = reinterpret_cast<T *>(state + L.khat) + ((size_t)bg * L.cap_chunks * s.k + (size_t)c * s.k) * d;
            T *vh = reinterpret_cast<T *>(state + L.vhat) + ((size_t)bg * L.cap_chunks * s.k + (size_t)c * s.k) * d;
            for (int t = threadIdx.x; t < s.k * d; t += blockDim.x) {
                const int rr = t / d, x = t % d;
                kh[(size_t)rr * d + x] = rk[(size_t)pos[rr] * d + x];
                vh[(size_t)rr * d + x] = rv[(size_t)pos[rr] * d + x];
            }
        }
        for (int t = threadIdx.x; t < s.k; t += blockDim.x) kept[pos[t]] = 1;
    }
    __syncthreads();
    // fold: S += sum_{unkept j} phi(k_j) v_j^T, z += sum phi(k_j)
    const int Dd = D * d;
    const int ebase = blockIdx.y * kFoldThreads * kFoldEnt;
    float acc[kFoldEnt];
#pragma unroll
    for (int u = 0; u < kFoldEnt; ++u) acc[u] = 0.f;
    float zacc = 0.f;
    for (int jb = 0; jb < s.C; jb += kFoldTok) {
        const int j = jb + warp;
        if (warp < kFoldTok) {
            float *xr = xs + warp * d;
            for (int x = lane; x < d; x += 32) xr[x] = j < s.C ? to_f(rk[(size_t)j * d + x]) : 0.f;
            for (int x = lane; x < d; x += 32) vs[warp * d + x] = j < s.C ? to_f(rv[(size_t)j * d + x]) : 0.f;
            __syncwarp();
            if (j < s.C && !kept[j]) {
                npmap_row_warp<T>(xr, Wk + (size_t)g * d * D, d, D, ph + warp * D, lane);
            } else {
                for (int a = lane; a < D; a += 32) ph[warp * D + a] = 0.f;
            }
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kFoldEnt; ++u) {
            const int e = ebase + threadIdx.x + u * kFoldThreads;
            if (e < Dd) {
                const int a = e / d, x = e % d;
                float sa = acc[u];
                for (int rr = 0; rr < kFoldTok; ++rr) sa = fmaf(ph[rr * D + a], vs[rr * d + x], sa);
                acc[u] = sa;
            }
        }
        if (blockIdx.y == 0 && threadIdx.x < D)
            for (int rr = 0; rr < kFoldTok; ++rr) zacc += ph[rr * D + threadIdx.x];
        __syncthreads();
    }
    float *S = reinterpret_cast<float *>(state + L.S) + (size_t)bg * Dd;
    float *z = reinterpret_cast<float *>(state + L.z) + (size_t)bg * D;
#pragma unroll
    for (int u = 0; u < kFoldEnt; ++u) {
        const int e = ebase + threadIdx.x + u * kFoldThreads;
        if (e < Dd) S[e] += acc[u];
    }
    if (blockIdx.y == 0 && threadIdx.x < D) z[threadIdx.x] += zacc;
}

// Prefill -> decode hand-off: after N tokens the state holds chunks c <= T-m-1 decided (kept rows
// and S_T, z_T), and the ring holds positions [max(0,(T-m)C), N) (w = 0: [TC, N)).
template <typename T>
__global__ void state_export_kernel(Dims s, DecodeLayout L, unsigned char *state, const T *__restrict__ k,
                                    const T *__restrict__ v, const float *__restrict__ r, const T *__restrict__ khat,
                                    const T *__restrict__ vhat, const float *__restrict__ Sw,
                                    const float *__restrict__ zw) {
    const int bg = blockIdx.x, d = s.d, D = s.D, T_ = s.T(), m = s.m();
    const int lo = s.w > 0 ? max(0, (T_ - m) * s.C) : T_ * s.C;
    for (int t = threadIdx.x; t < (s.N - lo) * d; t += blockDim.x) {
        const int j = lo + t / d, x = t % d;
        const size_t dst = ((size_t)bg * L.ring_rows + ring_row(s, j)) * d + x;
        reinterpret_cast<T *>(state + L.ring_k)[dst] = k[((size_t)bg * s.N + j) * d + x];
        reinterpret_cast<T *>(state + L.ring_v)[dst] = v[((size_t)bg * s.N + j) * d + x];
    }
    for (int j = lo + threadIdx.x; j < s.N; j += blockDim.x)
        reinterpret_cast<float *>(state + L.ring_r)[(size_t)bg * L.ring_rows + ring_row(s, j)] =
            r ? r[(size_t)bg * s.N + j] : 0.f;
    const int nkept = s.w > 0 ? s.k * max(0, T_ - m) : 0;
    for (int t = threadIdx.x; t < nkept * d; t += blockDim.x) {
        const size_t src = (size_t)bg * T_ * s.k * d + t;
        const size_t dst = (size_t)bg * L.cap_chunks * s.k * d + t;
        reinterpret_cast<T *>(state + L.khat)[dst] = khat[src];
        reinterpret_cast<T *>(state + L.vhat)[dst] = vhat[src];
    }
    const float *Ss = Sw + ((size_t)bg * (T_ + 1) + T_) * D * d;
    const float *zs = zw + ((size_t)bg * (T_ + 1) + T_) * D;
    for (int t = threadIdx.x; t < D * d; t += blockDim.x)
        reinterpret_cast<float *>(state + L.S)[(size_t)bg * D * d + t] = Ss[t];
    for (int t = threadIdx.x; t < D; t += blockDim.x)
        reinterpret_cast<float *>(state + L.z)[(size_t)bg * D + t] = zs[t];
    if (bg == 0 && threadIdx.x == 0) {
        DecodeHeader *hd = reinterpret_cast<DecodeHeader *>(state + L.header);
        hd->pos = s.N;
    }
}

__global__ void decode_header_kernel(unsigned char *state, DecodeLayout L, int capacity) {
    DecodeHeader *hd = reinterpret_cast<DecodeHeader *>(state + L.header);
    hd->pos = 0;
    hd->capacity = capacity;
    hd->magic = kDecodeMagic;
}

}  // namespace

cudaError_t launch_decode_init(const Dims &s, unsigned char *state, const DecodeLayout &L, int capacity,
                               cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(state + L.S, 0, L.ring_k - L.S, st);  // S and z
    if (e != cudaSuccess) return e;
    decode_header_kernel<<<1, 1, 0, st>>>(state, L, capacity);
    return cudaGetLastError();
}

// K/V rows of the tensor-core decode attention: staged in shared memory by bulk copies (true) or
// loaded into registers (false).
constexpr bool kDecodeBulk = true;

// SMs of the current device (looked up once per device).
int decode_sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

template <typename T>
static cudaError_t decode_step_t(const Dims &s, unsigned char *state, const DecodeLayout &L, int pos, const void *Wq,
                                 const void *Wk, const void *q_t, const void *k_t, const void *v_t, void *o_t,
                                 unsigned *err, cudaStream_t st, int *launches) {
    StepGeom gm{};
    gm.pos = pos;
    gm.t = pos / s.C;
    const int m = s.m();
    if (s.w > 0) {
        gm.lo = max(0, (gm.t - m) * s.C);
        gm.nk = s.k * max(0, gm.t - m);
        gm.n = gm.nk + (pos - gm.lo + 1);
    } else {
        gm.lo = pos + 1;
        gm.nk = 0;
        gm.n = 0;
    }
    const int BK = s.B * s.Hkv;
    gm.nsplit = gm.n == 0 ? 0 : min(kDecodeMaxSplits, (gm.n + 511) / 512);
    const bool tc_path = sizeof(T) == 2 && (s.d == 64 || s.d == 128) && s.G() <= 8 && (8 % s.G()) == 0;
    if (tc_path && kDecodeBulk && gm.n > 0) {
        // splits of 512..2048 keys, as few as keep the last wave of CTAs nearly full (the
        // bulk-copy kernel keeps 2 CTAs per SM at d = 128, 4 at d = 64)
        const int slots = decode_sm_count() * (s.d == 128 ? 2 : 4);
        const int lo_ns = max(1, (gm.n + 2047) / 2048), hi_ns = min(kDecodeMaxSplits, max(lo_ns, (gm.n + 511) / 512));
        int best = hi_ns;
        double best_eff = -1.0;
        for (int ns = lo_ns; ns <= hi_ns; ++ns) {
            const long long ctas = (long long)BK * ns, waves = (ctas + slots - 1) / slots;
            const double eff = (double)ctas / (double)(waves * slots);
            if (eff >= 0.95) {
                best = ns;
                break;
            }
            if (eff > best_eff) {
                best_eff = eff;
                best = ns;
            }
        }
        gm.nsplit = best;
    }
    gm.per = gm.nsplit ? (gm.n + gm.nsplit - 1) / gm.nsplit : 0;
    // the bulk-copy attention kernel appends the step's key and value itself
    const int Gs = s.G();
    const bool fold_append = kDecodeBulk && gm.nsplit > 0 && sizeof(T) == 2 && (s.d == 64 || s.d == 128) &&
                             (Gs == 1 || Gs == 2 || Gs == 4 || Gs == 8);
    int ts = -1;
    if (!fold_append) {
        ts = timing_begin(kTimeDecodeAppend, st);
        decode_append_kernel<T><<<BK, 128, 0, st>>>(s, L, state, pos, (const T *)k_t, (const T *)v_t, err);
        timing_end(ts, st);
        ++*launches;
    }
    if (gm.nsplit) {
        ts = timing_begin(kTimeDecodeAttn, st);
        const dim3 grid(BK, gm.nsplit);
        const int G = s.G();
#define STILL_DECODE_PACKED(DPL, GG) \
    decode_attn_packed_kernel<T, DPL, GG><<<grid, 256, 0, st>>>(s, L, state, gm, (const T *)q_t)
#define STILL_DECODE_MMA(DH, GG)                                                                          \
    do {                                                                                                    \
        if (kDecodeBulk) {                                                                                  \
            const int smem_ = DecodeBulkCfg<DH>::SMEM;                                                      \
            cudaError_t e_ = cudaFuncSetAttribute(decode_attn_bulk_kernel<DH, GG>,                          \
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, smem_);      \
            if (e_ != cudaSuccess) return e_;                                                               \
            decode_attn_bulk_kernel<DH, GG><<<grid, 128, smem_, st>>>(                                      \
                s, L, state, gm, (const __nv_bfloat16 *)q_t, (const __nv_bfloat16 *)k_t,                    \
                (const __nv_bfloat16 *)v_t, err);                                                           \
        } else {                                                                                            \
            decode_attn_mma_kernel<DH, GG><<<grid, 128, 0, st>>>(s, L, state, gm, (const __nv_bfloat16 *)q_t); \
        }                                                                                                   \
    } while (0)
        const bool mma = sizeof(T) == 2 && (s.d == 64 || s.d == 128) && (G == 1 || G == 2 || G == 4 || G == 8);
        if (mma) {
            if (s.d == 128) {
                if (G == 1) STILL_DECODE_MMA(128, 1);
                else if (G == 2) STILL_DECODE_MMA(128, 2);
                else if (G == 4) STILL_DECODE_MMA(128, 4);
                else STILL_DECODE_MMA(128, 8);
            } else {
                if (G == 1) STILL_DECODE_MMA(64, 1);
                else if (G == 2) STILL_DECODE_MMA(64, 2);
                else if (G == 4) STILL_DECODE_MMA(64, 4);
                else STILL_DECODE_MMA(64, 8);
            }
        }
        else if (s.d == 128 && G == 4) STILL_DECODE_PACKED(4, 4);
        else if (s.d == 128 && G == 8) STILL_DECODE_PACKED(4, 8);
        else if (s.d == 128 && G == 2) STILL_DECODE_PACKED(4, 2);
        else if (s.d == 128 && G == 1 && sizeof(T) == 2) STILL_DECODE_PACKED(4, 1);
        else if (s.d == 64 && G == 4) STILL_DECODE_PACKED(2, 4);
        else if (s.d == 64 && G == 8) STILL_DECODE_PACKED(2, 8);
        else if (s.d == 64 && G == 2) STILL_DECODE_PACKED(2, 2);
        else if (s.d == 64 && G == 1) STILL_DECODE_PACKED(2, 1);
        else decode_attn_kernel<T><<<grid, 128, 0, st>>>(s, L, state, gm, (const T *)q_t);
#undef STILL_DECODE_PACKED
#undef STILL_DECODE_MMA
        timing_end(ts, st);
        ++*launches;
    }
    ts = timing_begin(kTimeDecodeCombine, st);
    if (s.w > 0 && s.G() <= 8) {
        const size_t smem = combine_wide_smem(s);
        if (smem > 48 * 1024) {  // at most ~66 KB (G = 8, d = D = 256)
            cudaError_t e = cudaFuncSetAttribute(decode_combine_wide_kernel<T>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
        decode_combine_wide_kernel<T><<<BK, kCombineThreads, smem, st>>>(s, L, state, gm, (const T *)q_t,
                                                                        (const T *)Wq, (T *)o_t);
    } else {
        decode_combine_kernel<T><<<BK, 128, 0, st>>>(s, L, state, gm, (const T *)q_t, (const T *)Wq, (const T *)Wk,
                                                     (T *)o_t);
    }
    timing_end(ts, st);
    ++*launches;
    if (pos % s.C == s.C - 1 && gm.t - m >= 0) {
        const int P = pow2_ceil(s.C), Pk = pow2_ceil(s.k > 0 ? s.k : 1);
        size_t smem = (size_t)P * 8 + (size_t)Pk * 4 + ((s.C + 15) & ~15) + (size_t)kFoldTok * (2 * s.d + s.D) * 4;
        cudaError_t e =
            cudaFuncSetAttribute(decode_close_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const int passes = (s.D * s.d + kFoldThreads * kFoldEnt - 1) / (kFoldThreads * kFoldEnt);
        ts = timing_begin(kTimeDecodeClose, st);
        decode_close_kernel<T><<<dim3(BK, passes), kFoldThreads, smem, st>>>(s, L, state, gm.t - m, (const T *)Wk, P,
                                                                             Pk);
        timing_end(ts, st);
        ++*launches;
    }
    return cudaGetLastError();
}

cudaError_t launch_decode_step(const Dims &s, unsigned char *state, const DecodeLayout &L, int pos, const void *Wq,
                               const void *Wk, const void *q_t, const void *k_t, const void *v_t, void *o_t,
                               unsigned *err, cudaStream_t st, int *launches) {
    if (s.bf16)
        return decode_step_t<__nv_bfloat16>(s, state, L, pos, Wq, Wk, q_t, k_t, v_t, o_t, err, st, launches);
    return decode_step_t<float>(s, state, L, pos, Wq, Wk, q_t, k_t, v_t, o_t, err, st, launches);
}

cudaError_t launch_state_export(const Dims &s, unsigned char *state, const DecodeLayout &L, const void *k,
                                const void *v, const float *r, const void *khat, const void *vhat, const float *S,
                                const float *z, cudaStream_t st) {
    const int BK = s.B * s.Hkv;
    if (BK == 0) return cudaSuccess;
    typedef __nv_bfloat16 bf;
    if (s.bf16)
        state_export_kernel<bf><<<BK, 256, 0, st>>>(s, L, state, (const bf *)k, (const bf *)v, r, (const bf *)khat,
                                                    (const bf *)vhat, S, z);
    else
        state_export_kernel<float><<<BK, 256, 0, st>>>(s, L, state, (const float *)k, (const float *)v, r,
                                                       (const float *)khat, (const float *)vhat, S, z);
    return cudaGetLastError();
}

}  // namespace still
