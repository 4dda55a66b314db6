// still_internal.h -- launcher interface between the C-ABI layer (api.cu) and
// the kernel translation units.  Not installed; C++ only.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "still.h"

namespace still {

struct Dims {
    int B, H, Hkv, N, d, D, w, C, k;
    float scale;  // resolved (never 0)
    int bf16;     // 1: q/k/v/o/W are bf16, 0: fp32
    __host__ __device__ int G() const { return H / Hkv; }
    __host__ __device__ int T() const { return N / C; }
    __host__ __device__ int m() const { return w / C; }
};

// Decode state buffer layout (byte offsets from the state base pointer).
struct DecodeLayout {
    size_t header, khat, vhat, S, z, ring_k, ring_v, ring_r, part, band, total;
    int cap_chunks;  // capacity / C
    int ring_rows;   // (m+1)*C, or C when w == 0
    int nsplit_max;
};

struct DecodeHeader {
    long long pos;
    int capacity;
    int magic;
};
constexpr int kDecodeMagic = 0x5711D ^ 0x1234;
constexpr int kDecodeMaxSplits = 64;

DecodeLayout decode_layout(const Dims &s, int capacity);

// Operands of the tensor-core merge phases (device pointers).
struct MergeOperands {
    const void *q, *k, *v, *wqt, *khat, *vhat, *st_t;
    const float *z;
    void *o;
    float *lse, *sigma;
    int *fix_list;
    unsigned *fix_count;
};

// ---- generic kernels (fp32 or bf16 storage, fp32 arithmetic) ----
cudaError_t launch_diagonal_score(const Dims &s, const void *q, const void *k, float *r_kv, cudaStream_t st);
cudaError_t launch_saliency_generic(const Dims &s, const void *q, const void *k, float *r_kv, float *r_q,
                                    cudaStream_t st);
cudaError_t launch_topk_gather(const Dims &s, const float *r, int32_t *idx, const void *k, const void *v, void *khat,
                               void *vhat, cudaStream_t st);
cudaError_t launch_npmap(int rows, int Hx, int N, int d, int D, int bf16, const void *x, const void *W, float *phi,
                         cudaStream_t st);
cudaError_t launch_linear_state(const Dims &s, const float *phik, const void *v, const int32_t *idx, float *S,
                                float *z, void *st_t, unsigned *err, cudaStream_t st);
cudaError_t launch_linear_prefix(const Dims &s, float *S, float *z, void *st_t, cudaStream_t st);
cudaError_t launch_merge_generic(const Dims &s, const void *q, const void *k, const void *v, const void *Wq,
                                 const void *khat, const void *vhat, const float *S, const float *z,
                                 const float *phik, void *o, cudaStream_t st);

// ---- decode ----
// Scratch of the backward pass (fp32, inside the caller's workspace).
struct BackwardScratch {
    float *phik;   // [B,Hkv,N,D]   NP-Map features of the keys
    float *S, *z;  // [B,Hkv,T+1,D,d], [B,Hkv,T+1,D]  forward linear state per query chunk
    float *A;      // [B,H,N,D]     a_i = exp(-Ms) / Z * phi(q_i)
    float *Dv;     // [B,H,N]       D_i = <dO_i, o_i>
    float *Ms, *iZ;  // [B,H,N]     each row's joint shift and 1 / shifted normaliser
    float *dYq;    // [B,H,N,D]     dL/d(q Wq)
    float *R, *r;  // [B,Hkv,T+1,D,d], [B,Hkv,T+1,D]  suffix sums over query chunks
    float *dYk;    // [B,Hkv,N,D]   dL/d(k Wk)
    float *L;      // [B,H,N]       tensor-core path: each row's log2 normaliser Ms log2(e) + log2 Z
    void *khat, *vhat;  // [B,Hkv,T*k,d] tensor-core path: the kept rows, gathered (bf16)
    void *wkt;     // [Hkv,D,d] tensor-core path: Wk^T (bf16), operand of the linear-state kernel
    void *wqt;     // [H,D,d] tensor-core path: Wq^T (bf16), operand of the dq kernel's prologue
    void *st_t;    // [B,Hkv,T+1,d,D] tensor-core path: S_t^T (bf16), operand of the dq kernel's prologue
};
bool tc_linear_supported(const Dims &s);
cudaError_t launch_w_transpose(int Hx, int d, int D, const void *w, void *wt, cudaStream_t st);
cudaError_t launch_linear_tc(const Dims &s, const void *k, const void *v, const void *wkt, const int32_t *idx,
                             float *S, float *z, unsigned *err, cudaStream_t st);
bool tc_backward_supported(const Dims &s);
bool tiled_linear_backward_supported(const Dims &s);
cudaError_t launch_linear_backward_tiled(int which, const Dims &s, const void *q, const void *k, const void *v,
                                         const void *Wq, const void *Wk, const void *dO, const int32_t *idx,
                                         const BackwardScratch &w, float *dq, float *dk, float *dv, float *dWq,
                                         float *dWk, cudaStream_t st);
cudaError_t launch_bwd_suffix(const Dims &s, float *R, float *r, cudaStream_t st);
cudaError_t launch_gather(const Dims &s, const int32_t *idx, const void *k, const void *v, void *khat, void *vhat,
                          unsigned *err, cudaStream_t st);
// Inputs of the dq kernel's own linear prologue (wqt = nullptr: none; lden, dl are read instead).
struct BwdPrologue {
    const void *wqt;    // [H,D,d] Wq^T (bf16)
    const void *Wq;     // [H,d,D] Wq (bf16): its epilogue adds dY Wq^T to dq
    const void *st_t;   // [B,Hkv,T+1,d,D] S_t^T (bf16)
    const float *z;     // [B,Hkv,T+1,D]
    float *Phi, *SG;    // [B,H,N,D] out: a = 2^-L phi(q) and dY = dL/d(q Wq) (phi(q), S_t dO on the way)
    // the forward's output [B,H,N,d] and per-row log2 normaliser [B,H,N], or null: with them the dq
    // kernel takes L_i and D_i = <dO_i, o_i> as given and skips its statistics sweep
    const void *o_fwd = nullptr;
    const float *lse_fwd = nullptr;
};
cudaError_t launch_backward_tc(const Dims &s, const void *q, const void *k, const void *v, const void *khat,
                               const void *vhat, const int32_t *idx, const void *dO, const float *lden,
                               const float *dl, const BwdPrologue &pro, float *L, float *Dv, float *dq, float *dk,
                               float *dv, unsigned *err, cudaStream_t st, int *launches);
cudaError_t launch_backward(const Dims &s, const void *q, const void *k, const void *v, const void *Wq,
                            const void *Wk, const int32_t *idx, const void *dO, float *dq, float *dk, float *dv,
                            float *dWq, float *dWk, const BackwardScratch &w, unsigned *err, cudaStream_t st,
                            int *launches, const void *o_fwd = nullptr, const float *lse_fwd = nullptr);

// Every argument check of still_hybrid_prefill except the workspace's (api.cu).
still_status check_prefill_args(const still_dims *dims, const void *q, const void *k, const void *v, const void *Wq,
                                const void *Wk, const void *o, const int32_t *idx_in, const void *state,
                                int state_capacity, bool *empty);

// Per-kernel event timing (still_timing_enable): returns a slot for timing_end, or -1 when off.
int timing_begin(int cls, cudaStream_t st);
void timing_end(int slot, cudaStream_t st);
enum TimingClass {
    kTimeDecodeAppend = 7,
    kTimeDecodeAttn = 8,
    kTimeDecodeCombine = 9,
    kTimeDecodeClose = 10,
    kTimeBwdDq = 11,
    kTimeBwdDkv = 12,
    kTimeBwdLinear = 13
};

cudaError_t launch_decode_step(const Dims &s, unsigned char *state, const DecodeLayout &L, int pos, const void *Wq,
                               const void *Wk, const void *q_t, const void *k_t, const void *v_t, void *o_t,
                               unsigned *err, cudaStream_t st, int *launches);
cudaError_t launch_state_export(const Dims &s, unsigned char *state, const DecodeLayout &L, const void *k,
                                const void *v, const float *r, const void *khat, const void *vhat, const float *S,
                                const float *z, cudaStream_t st);
cudaError_t launch_decode_init(const Dims &s, unsigned char *state, const DecodeLayout &L, int capacity,
                               cudaStream_t st);

}  // namespace still
