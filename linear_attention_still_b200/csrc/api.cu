// api.cu -- the C ABI of libstill.so (declared in include/still.h): argument validation on the
// host, workspace and state layout, and the launch sequence of each entry point.
#include <atomic>
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "still.h"
#include "still_internal.h"

namespace still {
cudaError_t launch_gather(const Dims &s, const int32_t *idx, const void *k, const void *v, void *khat, void *vhat,
                          unsigned *err, cudaStream_t st);
bool tc_merge_supported(const Dims &s);
cudaError_t launch_w_transpose(int Hx, int d, int D, const void *w, void *wt, cudaStream_t st);
bool tc_linear_supported(const Dims &s);
cudaError_t launch_linear_tc(const Dims &s, const void *k, const void *v, const void *wkt, const int32_t *idx,
                             float *S, float *z, unsigned *err, cudaStream_t st);
cudaError_t launch_merge_tc(int mode, const Dims &s, const MergeOperands &a, unsigned *err, cudaStream_t st);
cudaError_t launch_mean_heads(const Dims &s, const float *sigma, float *r, cudaStream_t st);
cudaError_t launch_saliency_fixup(const Dims &s, const void *q, const void *k, const int *list, const unsigned *count,
                                  float *sigma, cudaStream_t st);
bool tc_saliency_supported(const Dims &s);
bool tc_nowin_supported(const Dims &s);
cudaError_t launch_nowin_phik(const Dims &s, const void *k, const void *wkt, void *phik, unsigned *err,
                              cudaStream_t st);
cudaError_t launch_nowin_tc(const Dims &s, const void *q, const void *v, const void *wqt, const void *st_t,
                            const float *z, const void *phik, void *o, unsigned *err, cudaStream_t st);
void set_merge_debug(int stall, int max_ctas);
cudaError_t launch_saliency_tc(const Dims &s, const void *q, const void *k, float *r_kv, float *r_q, unsigned *err,
                               cudaStream_t st);
}  // namespace still

using namespace still;

__device__ unsigned g_still_device_error;  // one per device (module globals are per context)

namespace {

std::atomic<uint64_t> g_launches{0};
std::mutex g_err_mu;
unsigned *g_err_ptr[128] = {nullptr};

unsigned *device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
    std::lock_guard<std::mutex> lk(g_err_mu);
    if (!g_err_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_still_device_error) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<unsigned *>(p);
    }
    return g_err_ptr[dev];
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

still_status check_dims(const still_dims *in, Dims *out, bool need_N = true) {
    if (!in) return STILL_ERR_INVALID_ARG;
    const still_dims &d = *in;
    if (d.B < 0 || d.H < 1 || d.Hkv < 1 || (need_N && d.N < 0) || d.C < 1 || d.k < 0 || d.w < 0)
        return STILL_ERR_INVALID_ARG;
    if (d.H % d.Hkv != 0 || d.k > d.C || d.w % d.C != 0) return STILL_ERR_INVALID_ARG;
    if (d.w == 0 && d.k != 0) return STILL_ERR_INVALID_ARG;
    if (d.dtype != STILL_F32 && d.dtype != STILL_BF16) return STILL_ERR_INVALID_ARG;
    if (d.d < 8 || d.d % 8 != 0 || d.D < 8 || d.D % 8 != 0) return STILL_ERR_INVALID_ARG;
    if (!std::isfinite(d.scale) || d.scale < 0.f) return STILL_ERR_INVALID_ARG;
    if (d.d > 256 || d.D > 256 || d.H / d.Hkv > 32 || d.C > 16384) return STILL_ERR_UNSUPPORTED;
    if ((long long)d.B * d.H > 65535 || (need_N && d.N > (1 << 26))) return STILL_ERR_UNSUPPORTED;
    Dims s{};
    s.B = d.B;
    s.H = d.H;
    s.Hkv = d.Hkv;
    s.N = need_N ? d.N : 0;
    s.d = d.d;
    s.D = d.D;
    s.w = d.w;
    s.C = d.C;
    s.k = d.k;
    s.scale = d.scale == 0.f ? 1.0f / std::sqrt((float)d.d) : d.scale;
    s.bf16 = d.dtype == STILL_BF16;
    *out = s;
    return STILL_OK;
}

still_ws_layout ws_layout(const Dims &s) {
    still_ws_layout L{};
    const size_t es = s.bf16 ? 2 : 4, BK = (size_t)s.B * s.Hkv, T = (size_t)s.T();
    size_t off = 0;
    L.r = off;
    off = al256(off + BK * s.N * 4);
    L.idx = off;
    off = al256(off + BK * T * s.k * 4);
    L.khat = off;
    off = al256(off + BK * T * s.k * s.d * es);
    L.vhat = off;
    off = al256(off + BK * T * s.k * s.d * es);
    L.S = off;
    off = al256(off + BK * (T + 1) * s.D * s.d * 4);
    L.z = off;
    off = al256(off + BK * (T + 1) * s.D * 4);
    // phi(K): fp32 on the SIMT path; bf16 for the intra-chunk tiles of the tensor-core w = 0 path; none
    // on the tensor-core hybrid path (its linear state featurises the keys in place)
    L.phik = off;
    const bool nowin = tc_nowin_supported(s);
    const bool fused_lin = s.bf16 && tc_merge_supported(s) && tc_linear_supported(s);
    off = al256(off + (nowin ? BK * s.N * s.D * 2 : fused_lin ? 0 : BK * s.N * s.D * 4));
    const bool tc = s.bf16 != 0;  // per-head scores and transposed bf16 operands of the tensor-core path
    L.sig = off;
    off = al256(off + (tc ? (size_t)s.B * s.H * s.N * 4 : 0));
    L.lse = off;
    off = al256(off + (tc ? (size_t)s.B * s.H * s.N * 4 : 0));
    L.fix = off;  // u32 count, then up to B*H*N row indices
    off = al256(off + (tc ? 256 + (size_t)s.B * s.H * s.N * 4 : 0));
    L.wqt = off;
    off = al256(off + (tc ? (size_t)s.H * s.D * s.d * 2 : 0));
    L.wkt = off;
    off = al256(off + (tc ? (size_t)s.Hkv * s.D * s.d * 2 : 0));
    L.st = off;
    off = al256(off + (tc ? BK * (T + 1) * s.D * s.d * 2 : 0));
    L.total = off;
    return L;
}

inline still_status cuda_status(cudaError_t e) { return e == cudaSuccess ? STILL_OK : STILL_ERR_CUDA; }

#define STILL_LAUNCH(expr)                                   \
    do {                                                     \
        cudaError_t e_ = (expr);                             \
        if (e_ != cudaSuccess) return STILL_ERR_CUDA;        \
        g_launches.fetch_add(1, std::memory_order_relaxed);  \
    } while (0)

// ---- optional per-kernel event timing (still_timing_enable / still_timing_read)
struct TimedLaunch {
    cudaEvent_t a, b;
    int cls;
};
bool g_timing = false;
TimedLaunch g_timed[STILL_TIMING_MAX_LAUNCHES];
int g_ntimed = 0;
cudaEvent_t g_ev_pool[2 * STILL_TIMING_MAX_LAUNCHES];
int g_ev_made = 0;

struct TimingScope {
    int slot;
    cudaStream_t st;
    TimingScope(int cls, cudaStream_t s) : slot(still::timing_begin(cls, s)), st(s) {}
    ~TimingScope() { still::timing_end(slot, st); }
};

}  // namespace

namespace still {

int timing_begin(int cls, cudaStream_t st) {
    if (!g_timing || g_ntimed >= STILL_TIMING_MAX_LAUNCHES) return -1;
    const int i = g_ntimed;
    for (int e = 0; e < 2; ++e)
        if (g_ev_made <= 2 * i + e) {
            if (cudaEventCreate(&g_ev_pool[2 * i + e]) != cudaSuccess) return -1;
            ++g_ev_made;
        }
    g_timed[i] = {g_ev_pool[2 * i], g_ev_pool[2 * i + 1], cls};
    if (cudaEventRecord(g_timed[i].a, st) != cudaSuccess) return -1;
    ++g_ntimed;
    return i;
}

void timing_end(int slot, cudaStream_t st) {
    if (slot >= 0) cudaEventRecord(g_timed[slot].b, st);
}

}  // namespace still

extern "C" {

const char *still_status_string(int status) {
    switch (status) {
        case STILL_OK: return "ok";
        case STILL_ERR_INVALID_ARG: return "invalid argument";
        case STILL_ERR_UNSUPPORTED: return "unsupported shape or type";
        case STILL_ERR_WORKSPACE: return "workspace or state buffer too small";
        case STILL_ERR_CUDA: return "CUDA error";
        case STILL_ERR_DEVICE_CHECK: return "device-side check failed";
        case STILL_ERR_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

uint64_t still_launch_count(void) { return g_launches.load(); }

still_status still_saliency(const still_dims *dims, const void *q, const void *k, float *r_kv, float *r_q,
                            void *stream) {
    Dims s;
    still_status st = check_dims(dims, &s);
    if (st) return st;
    if (s.w < 1) return STILL_ERR_INVALID_ARG;
    if ((long long)s.B * s.N == 0) return STILL_OK;
    if (!q || !k || !r_kv || !aligned16(q) || !aligned16(k) || !aligned16(r_kv)) return STILL_ERR_INVALID_ARG;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (tc_saliency_supported(s) && (r_q || s.G() <= 2)) {
        unsigned *err = device_error_word();
        STILL_LAUNCH(launch_saliency_tc(s, q, k, r_kv, r_q, err, cs));
    } else {
        STILL_LAUNCH(launch_saliency_generic(s, q, k, r_kv, r_q, cs));
    }
    return STILL_OK;
}

still_status still_diagonal_score(const still_dims *dims, const void *q, const void *k, float *r_kv, void *stream) {
    Dims s;
    still_status st = check_dims(dims, &s);
    if (st) return st;
    if ((long long)s.B * s.N == 0) return STILL_OK;
    if (!q || !k || !r_kv || !aligned16(q) || !aligned16(k) || !aligned16(r_kv)) return STILL_ERR_INVALID_ARG;
    STILL_LAUNCH(launch_diagonal_score(s, q, k, r_kv, static_cast<cudaStream_t>(stream)));
    return STILL_OK;
}

namespace {
// Backward scratch layout (256-byte aligned fp32 segments).
constexpr int kBwdSegments = 17;
size_t backward_layout(const Dims &s, size_t *off) {
    const size_t BH = (size_t)s.B * s.H, BK = (size_t)s.B * s.Hkv, T1 = (size_t)s.T() + 1;
    // tensor-core path: the rows' log2 normalisers and the gathered kept rows (bf16, in fp32 units)
    const bool tc = tc_backward_supported(s);
    const size_t kept = tc ? (BK * s.T() * s.k * s.d * 2 + 3) / 4 : 0;
    const size_t sizes[kBwdSegments] = {BK * s.N * s.D, BK * T1 * s.D * s.d, BK * T1 * s.D, BH * s.N * s.D, BH * s.N,
                                        BH * s.N * s.D, BK * T1 * s.D * s.d, BK * T1 * s.D, BK * s.N * s.D, BH * s.N,
                                        BH * s.N, tc ? BH * s.N : 0, kept, kept,
                                        tc ? ((size_t)s.Hkv * s.d * s.D * 2 + 3) / 4 : 0,
                                        tc ? ((size_t)s.H * s.d * s.D * 2 + 3) / 4 : 0,
                                        tc ? (BK * T1 * s.d * s.D * 2 + 3) / 4 : 0};
    size_t o = 0;
    for (int i = 0; i < kBwdSegments; ++i) {
        off[i] = o;
        o += (sizes[i] * 4 + 255) & ~(size_t)255;
    }
    return o;
}
}  // namespace

size_t still_backward_workspace_bytes(const still_dims *dims) {
    Dims s;
    if (check_dims(dims, &s)) return 0;
    size_t off[kBwdSegments];
    return backward_layout(s, off);
}

still_status still_hybrid_backward(const still_dims *dims, const void *q, const void *k, const void *v,
                                   const void *Wq, const void *Wk, const int32_t *idx, const void *dO, float *dq,
                                   float *dk, float *dv, float *dWq, float *dWk, void *workspace,
                                   size_t workspace_bytes, void *stream) {
    Dims s;
    still_status st = check_dims(dims, &s);
    if (st) return st;
    if ((long long)s.B * s.N == 0) return STILL_OK;
    const void *ptrs[] = {q, k, v, Wq, Wk, dO, dq, dk, dv, dWq, dWk, workspace};
    for (const void *p : ptrs)
        if (!p || !aligned16(p)) return STILL_ERR_INVALID_ARG;
    const bool select = s.k > 0 && s.T() > 0;
    if (select && (!idx || !aligned16(idx))) return STILL_ERR_INVALID_ARG;
    size_t off[kBwdSegments];
    if (workspace_bytes < backward_layout(s, off)) return STILL_ERR_WORKSPACE;
    if (((uintptr_t)workspace & 255u) != 0) return STILL_ERR_INVALID_ARG;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    auto F = [&](int i) { return reinterpret_cast<float *>(ws + off[i]); };
    BackwardScratch w{F(0), F(1), F(2), F(3), F(4), F(9), F(10), F(5), F(6), F(7), F(8), F(11), F(12), F(13), F(14), F(15), F(16)};
    int launches = 0;
    cudaError_t e = launch_backward(s, q, k, v, Wq, Wk, select ? idx : nullptr, dO, dq, dk, dv, dWq, dWk, w,
                                    device_error_word(), static_cast<cudaStream_t>(stream), &launches);
    g_launches.fetch_add((uint64_t)launches, std::memory_order_relaxed);
    return e == cudaSuccess ? STILL_OK : STILL_ERR_CUDA;
}

still_status still_hybrid_backward_saved(const still_dims *dims, const void *q, const void *k, const void *v,
                                         const void *Wq, const void *Wk, const int32_t *idx, const void *dO,
                                         const void *o, const float *lse, float *dq, float *dk, float *dv,
                                         float *dWq, float *dWk, void *workspace, size_t workspace_bytes,
                                         void *stream) {
    Dims s;
    still_status st = check_dims(dims, &s);
    if (st) return st;
    if ((long long)s.B * s.N == 0) return STILL_OK;
    const void *ptrs[] = {q, k, v, Wq, Wk, dO, o, lse, dq, dk, dv, dWq, dWk, workspace};
    for (const void *p : ptrs)
        if (!p || !aligned16(p)) return STILL_ERR_INVALID_ARG;
    const bool select = s.k > 0 && s.T() > 0;
    if (select && (!idx || !aligned16(idx))) return STILL_ERR_INVALID_ARG;
    size_t off[kBwdSegments];
    if (workspace_bytes < backward_layout(s, off)) return STILL_ERR_WORKSPACE;
    if (((uintptr_t)workspace & 255u) != 0) return STILL_ERR_INVALID_ARG;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    auto F = [&](int i) { return reinterpret_cast<float *>(ws + off[i]); };
    BackwardScratch w{F(0), F(1), F(2), F(3), F(4), F(9), F(10), F(5), F(6), F(7), F(8), F(11), F(12), F(13), F(14), F(15), F(16)};
    // the forward leaves every row's whole normaliser in its workspace on the tensor-core merge path only;
    // elsewhere the statistics are formed again as in still_hybrid_backward
    const bool saved = tc_merge_supported(s);
    int launches = 0;
    cudaError_t e = launch_backward(s, q, k, v, Wq, Wk, select ? idx : nullptr, dO, dq, dk, dv, dWq, dWk, w,
                                    device_error_word(), static_cast<cudaStream_t>(stream), &launches,
                                    saved ? o : nullptr, saved ? lse : nullptr);
    g_launches.fetch_add((uint64_t)launches, std::memory_order_relaxed);
    return e == cudaSuccess ? STILL_OK : STILL_ERR_CUDA;
}

still_status still_select_topk(const still_dims *dims, const float *r_kv, int32_t *idx, void *stream) {
    Dims s;
    still_status st = check_dims(dims, &s);
    if (st) return st;
    if ((long long)s.B * s.T() * s.k == 0) return STILL_OK;
    if (!r_kv || !idx || !aligned16(r_kv) || !aligned16(idx)) return STILL_ERR_INVALID_ARG;
    STILL_LAUNCH(launch_topk_gather(s, r_kv, idx, nullptr, nullptr, nullptr, nullptr, static_cast<cudaStream_t>(stream)));
    return STILL_OK;
}

still_status still_npmap(int B, int Hx, int N, int d, int D, still_dtype dtype, const void *x, const void *W,
                         float *phi, void *stream) {
    if (B < 0 || Hx < 1 || N < 0 || d < 8 || d % 8 || D < 8 || D % 8) return STILL_ERR_INVALID_ARG;
    if (dtype != STILL_F32 && dtype != STILL_BF16) return STILL_ERR_INVALID_ARG;
    if (d > 256 || D > 256) return STILL_ERR_UNSUPPORTED;
    const long long rows = (long long)B * Hx * N;
    if (rows == 0) return STILL_OK;
    if (rows > (1ll << 31) - 4) return STILL_ERR_UNSUPPORTED;
    if (!x || !W || !phi || !aligned16(x) || !aligned16(W) || !aligned16(phi)) return STILL_ERR_INVALID_ARG;
    STILL_LAUNCH(launch_npmap((int)rows, Hx, N, d, D, dtype == STILL_BF16, x, W, phi, static_cast<cudaStream_t>(stream)));
    return STILL_OK;
}

size_t still_prefill_workspace_bytes(const still_dims *dims) {
    Dims s;
    if (check_dims(dims, &s)) return 0;
    return ws_layout(s).total;
}

still_status still_prefill_workspace_layout(const still_dims *dims, still_ws_layout *out) {
    Dims s;
    still_status st = check_dims(dims, &s);
    if (st) return st;
    if (!out) return STILL_ERR_INVALID_ARG;
    *out = ws_layout(s);
    return STILL_OK;
}

size_t still_decode_state_bytes(const still_dims *dims, int capacity) {
    Dims s;
    if (check_dims(dims, &s, false) || capacity < 0) return 0;
    return decode_layout(s, capacity).total;
}

still_status still_decode_state_layout(const still_dims *dims, int capacity, still_state_layout *out) {
    Dims s;
    still_status st = check_dims(dims, &s, false);
    if (st) return st;
    if (capacity < 0 || capacity > (1 << 26) || !out) return STILL_ERR_INVALID_ARG;
    const DecodeLayout L = decode_layout(s, capacity);
    out->header = L.header;
    out->khat = L.khat;
    out->vhat = L.vhat;
    out->S = L.S;
    out->z = L.z;
    out->ring_k = L.ring_k;
    out->ring_v = L.ring_v;
    out->ring_r = L.ring_r;
    out->total = L.total;
    out->ring_rows = L.ring_rows;
    out->cap_chunks = L.cap_chunks;
    return STILL_OK;
}

still_status still_decode_init(const still_dims *dims, int capacity, void *state, void *stream) {
    Dims s;
    still_status st = check_dims(dims, &s, false);
    if (st) return st;
    if (capacity < 0 || capacity > (1 << 26)) return STILL_ERR_INVALID_ARG;
    if (!state || !aligned16(state)) return STILL_ERR_INVALID_ARG;
    DecodeLayout L = decode_layout(s, capacity);
    STILL_LAUNCH(launch_decode_init(s, static_cast<unsigned char *>(state), L, capacity,
                                    static_cast<cudaStream_t>(stream)));
    return STILL_OK;
}

}  // extern "C"

namespace still {
// Every check of still_hybrid_prefill except those of the workspace, in the order that call makes
// them (dims, decode state, then the tensors); STILL_OK with *empty set when B * N == 0.
still_status check_prefill_args(const still_dims *dims, const void *q, const void *k, const void *v, const void *Wq,
                                const void *Wk, const void *o, const int32_t *idx_in, const void *state,
                                int state_capacity, bool *empty) {
    Dims s;
    still_status st = check_dims(dims, &s);
    if (st) return st;
    if (state && (state_capacity < s.N || !aligned16(state))) return STILL_ERR_INVALID_ARG;
    *empty = (long long)s.B * s.N == 0;
    if (*empty) return STILL_OK;
    const void *ptrs[] = {q, k, v, Wq, Wk, o};
    for (const void *p : ptrs)
        if (!p || !aligned16(p)) return STILL_ERR_INVALID_ARG;
    if (idx_in && !aligned16(idx_in)) return STILL_ERR_INVALID_ARG;
    return STILL_OK;
}
}  // namespace still

extern "C" {

still_status still_hybrid_prefill(const still_dims *dims, const void *q, const void *k, const void *v, const void *Wq,
                                  const void *Wk, void *o, const int32_t *idx_in, void *workspace,
                                  size_t workspace_bytes, void *state, int state_capacity, void *stream) {
    bool empty = false;
    still_status st = check_prefill_args(dims, q, k, v, Wq, Wk, o, idx_in, state, state_capacity, &empty);
    if (st || empty) return st;
    if (!workspace || !aligned16(workspace)) return STILL_ERR_INVALID_ARG;
    Dims s;
    check_dims(dims, &s);
    const still_ws_layout W = ws_layout(s);
    if (workspace_bytes < W.total) return STILL_ERR_WORKSPACE;
    if (((uintptr_t)workspace & 255u) != 0) return STILL_ERR_INVALID_ARG;

    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    unsigned *err = device_error_word();
    float *r = reinterpret_cast<float *>(ws + W.r);
    int32_t *idx = reinterpret_cast<int32_t *>(ws + W.idx);
    void *khat = ws + W.khat, *vhat = ws + W.vhat;
    float *S = reinterpret_cast<float *>(ws + W.S), *z = reinterpret_cast<float *>(ws + W.z);
    float *phik = reinterpret_cast<float *>(ws + W.phik);
    void *wqt = ws + W.wqt, *st_t = ws + W.st, *wkt = ws + W.wkt;
    const bool use_tc = tc_merge_supported(s);
    const bool use_tc_lin = use_tc && tc_linear_supported(s);
    const bool select = s.w > 0 && s.k > 0 && s.T() > 0;
    const bool need_r = s.w > 0 && s.k > 0 && (!idx_in || state);

    float *sig = reinterpret_cast<float *>(ws + W.sig), *lse = reinterpret_cast<float *>(ws + W.lse);
    unsigned *fix_count = reinterpret_cast<unsigned *>(ws + W.fix);
    int *fix_list = reinterpret_cast<int *>(ws + W.fix + 256);
    MergeOperands mo{q, k, v, wqt, khat, vhat, st_t, z, o, lse, sig, fix_list, fix_count};
    if (tc_nowin_supported(s)) {
        // w = 0 (no softmax branch): the inter-chunk linear state on tensor cores (NP-Map of the keys
        // fused), then phi(k) of every key once (bf16, for the intra-chunk tiles) and every row's
        // intra-chunk causal tile plus phi(q)^T S_t on tensor cores
        {
            TimingScope ts(3, cs);
            STILL_LAUNCH(launch_w_transpose(s.Hkv, s.d, s.D, Wk, wkt, cs));
            STILL_LAUNCH(launch_linear_tc(s, k, v, wkt, nullptr, S, z, err, cs));
            STILL_LAUNCH(launch_linear_prefix(s, S, z, st_t, cs));
        }
        {
            TimingScope ts(4, cs);
            STILL_LAUNCH(launch_w_transpose(s.H, s.d, s.D, Wq, wqt, cs));
            STILL_LAUNCH(launch_nowin_phik(s, k, wkt, ws + W.phik, err, cs));
            STILL_LAUNCH(launch_nowin_tc(s, q, v, wqt, st_t, z, ws + W.phik, o, err, cs));
        }
        if (state) {
            DecodeLayout L = decode_layout(s, state_capacity);
            TimingScope ts(5, cs);
            STILL_LAUNCH(launch_state_export(s, static_cast<unsigned char *>(state), L, k, v, nullptr, khat, vhat, S,
                                             z, cs));
        }
        return STILL_OK;
    }
    if (use_tc) {
        // 1a. window part of the softmax branch and, from the same exponentials, the Self-Saliency
        //     Score of every query head (tensor cores)
        TimingScope ts(4, cs);
        if (cudaMemsetAsync(fix_count, 0, sizeof(unsigned), cs) != cudaSuccess) return STILL_ERR_CUDA;
        STILL_LAUNCH(launch_w_transpose(s.H, s.d, s.D, Wq, wqt, cs));
        STILL_LAUNCH(launch_merge_tc(0, s, mo, err, cs));
    }
    // 1b. Self-Saliency Score per KV group
    if (need_r) {
        TimingScope ts(0, cs);
        if (use_tc) {
            STILL_LAUNCH(launch_saliency_fixup(s, q, k, fix_list, fix_count, sig, cs));
            STILL_LAUNCH(launch_mean_heads(s, sig, r, cs));
        } else {
            STILL_LAUNCH(launch_saliency_generic(s, q, k, r, nullptr, cs));
        }
    }
    // 2. per-chunk top-k and gather of the kept rows
    const int32_t *idx_used = idx;
    if (select) {
        TimingScope ts(1, cs);
        if (idx_in) {
            idx_used = idx_in;
            STILL_LAUNCH(launch_gather(s, idx_in, k, v, khat, vhat, err, cs));
        } else {
            STILL_LAUNCH(launch_topk_gather(s, r, idx, k, v, khat, vhat, cs));
        }
    }
    // 3./4. NP-Map of the keys and the linear state seen by every query chunk
    if (use_tc_lin) {
        // NP-Map of the keys fused into the tensor-core linear-state kernel
        TimingScope ts(3, cs);
        STILL_LAUNCH(launch_w_transpose(s.Hkv, s.d, s.D, Wk, wkt, cs));
        STILL_LAUNCH(launch_linear_tc(s, k, v, wkt, idx_used, S, z, err, cs));
        STILL_LAUNCH(launch_linear_prefix(s, S, z, use_tc ? st_t : nullptr, cs));
    } else {
        {
            TimingScope ts(2, cs);
            STILL_LAUNCH(launch_npmap(s.B * s.Hkv * s.N, s.Hkv, s.N, s.d, s.D, s.bf16, k, Wk, phik, cs));
        }
        TimingScope ts(3, cs);
        STILL_LAUNCH(launch_linear_state(s, phik, v, idx_used, S, z, use_tc ? st_t : nullptr, err, cs));
        g_launches.fetch_add(s.T() - s.m() > 0 ? 1 : 0);  // the delta kernel (the prefix was counted)
    }
    // 5. kept-prefix part of the softmax branch + linear branch, merged with the window part
    if (use_tc) {
        TimingScope ts(6, cs);
        STILL_LAUNCH(launch_merge_tc(1, s, mo, err, cs));
    } else {
        TimingScope ts(4, cs);
        STILL_LAUNCH(launch_merge_generic(s, q, k, v, Wq, khat, vhat, S, z, phik, o, cs));
    }
    // hand-off to decode
    if (state) {
        DecodeLayout L = decode_layout(s, state_capacity);
        TimingScope ts(5, cs);
        STILL_LAUNCH(launch_state_export(s, static_cast<unsigned char *>(state), L, k, v, need_r ? r : nullptr, khat,
                                         vhat, S, z, cs));
    }
    return STILL_OK;
}

still_status still_decode_step(const still_dims *dims, void *state, int capacity, int pos, const void *Wq,
                               const void *Wk, const void *q_t, const void *k_t, const void *v_t, void *o_t,
                               void *stream) {
    Dims s;
    still_status st = check_dims(dims, &s, false);
    if (st) return st;
    if (capacity < 1 || pos < 0 || pos >= capacity) return STILL_ERR_INVALID_ARG;
    if (s.B == 0) return STILL_OK;
    const void *ptrs[] = {state, Wq, Wk, q_t, k_t, v_t, o_t};
    for (const void *p : ptrs)
        if (!p || !aligned16(p)) return STILL_ERR_INVALID_ARG;
    s.N = capacity;
    DecodeLayout L = decode_layout(s, capacity);
    int launches = 0;
    cudaError_t e = launch_decode_step(s, static_cast<unsigned char *>(state), L, pos, Wq, Wk, q_t, k_t, v_t, o_t,
                                       device_error_word(), static_cast<cudaStream_t>(stream), &launches);
    g_launches.fetch_add(launches);
    return cuda_status(e);
}

void still_debug_merge(int stall, int max_ctas) { set_merge_debug(stall, max_ctas); }

still_status still_timing_enable(int on) {
    g_timing = on != 0;
    return STILL_OK;
}

still_status still_timing_read(double *ms, int *launches, int n) {
    if (n < 0 || (n > 0 && (!ms || !launches))) return STILL_ERR_INVALID_ARG;
    for (int c = 0; c < n; ++c) {
        ms[c] = 0.0;
        launches[c] = 0;
    }
    still_status st = STILL_OK;
    for (int i = 0; i < g_ntimed; ++i) {
        float t = 0.f;
        if (cudaEventSynchronize(g_timed[i].b) != cudaSuccess ||
            cudaEventElapsedTime(&t, g_timed[i].a, g_timed[i].b) != cudaSuccess) {
            st = STILL_ERR_CUDA;
            continue;
        }
        const int c = g_timed[i].cls;
        if (c < n) {
            ms[c] += t;
            launches[c] += 1;
        }
    }
    g_ntimed = 0;
    return st;
}

still_status still_get_device_status(void *stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return STILL_ERR_CUDA;
    unsigned *p = device_error_word();
    if (!p) return STILL_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return STILL_ERR_CUDA;
    if (v) {
        unsigned zero = 0;
        if (cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return STILL_ERR_CUDA;
    }
    if (v & DEV_ERR_TIMEOUT) return STILL_ERR_TIMEOUT;
    if (v) return STILL_ERR_DEVICE_CHECK;
    return STILL_OK;
}

}  // extern "C"
