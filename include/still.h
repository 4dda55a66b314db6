/*
 * still.h -- C ABI of libstill.so, the B200 (sm_100a) implementation of the
 * STILL intra-layer hybrid attention layer.
 *
 * Method: "STILL: Selecting Tokens for Intra-Layer Hybrid Attention to
 * Linearize LLMs".  Passages cited below:
 *   [p1] jsqmd.com news article -- introduction (two branches in one layer:
 *        selected tokens go to softmax attention, the rest to linear
 *        attention), "Self-Saliency Score", "Norm-Preserved Feature Map
 *        (NP-Map)", "Chunk-Wise parallel + delayed selection";
 *   [p4] atlas.scime.ai summary -- "Approach".
 *
 * Conventions (all entry points):
 *  - Every tensor argument is a caller-owned DEVICE pointer in the row-major
 *    layout stated at the call, 16-byte aligned.  No call allocates memory;
 *    scratch space is passed in by the caller (still_hybrid_prefill_static
 *    uses a fixed array of the library instead).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Every call is asynchronous on that stream.
 *  - Argument errors are detected on the host before anything is launched and
 *    returned as a still_status; nothing is launched then.  Errors found by a
 *    kernel (an injected index outside its chunk, a decode position that does
 *    not match the state, a bounded wait that ran out) are recorded in a
 *    per-device error word and reported by still_get_device_status().
 *  - Shapes: B batch, H query heads, Hkv key/value heads (H % Hkv == 0, query
 *    head h reads KV head h / (H/Hkv)), N tokens, head dim d, NP-Map feature
 *    width D, window w, chunk C, k tokens kept per full chunk.  The window is
 *    a whole number of chunks, w = m*C with m >= 1, or w = 0 (no window: pure
 *    linear attention, then k must be 0).  0 <= k <= C.  N is arbitrary; a
 *    trailing partial chunk is never selected from.  d and D are multiples
 *    of 8 (at least 8); scale is finite and >= 0; B, N >= 0; H, Hkv, C >= 1
 *    (STILL_ERR_INVALID_ARG otherwise).  Limits of this implementation
 *    (STILL_ERR_UNSUPPORTED beyond them): d, D <= 256; H/Hkv <= 32;
 *    C <= 16384; B*H <= 65535; N <= 2^26.  The size queries return 0 for
 *    dims that either check rejects.
 *  - dtype applies to q, k, v, o, Wq, Wk; scores, features and linear states
 *    are always fp32.
 */
#ifndef STILL_H
#define STILL_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define STILL_API __attribute__((visibility("default")))
#else
#define STILL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    STILL_OK = 0,
    STILL_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad shape, constraint violated */
    STILL_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. d > 256) */
    STILL_ERR_WORKSPACE = 3,    /* workspace or state buffer too small */
    STILL_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    STILL_ERR_DEVICE_CHECK = 5, /* a kernel found bad data (see still_get_device_status) */
    STILL_ERR_TIMEOUT = 6       /* a kernel's bounded wait ran out */
} still_status;

typedef enum { STILL_F32 = 0, STILL_BF16 = 1 } still_dtype;

typedef struct {
    int B, H, Hkv, N, d, D, w, C, k;
    float scale;       /* logit scale tau; 0 selects 1/sqrt(d) */
    still_dtype dtype;
} still_dims;

/* Text of a status code (static storage). */
STILL_API const char *still_status_string(int status);

/*
 * Self-Saliency Score ([p1] "Self-Saliency Score"; [p4] "Approach").
 * For query head h and token i, with band B(i) = [max(0, i-w+1), i] and
 * logits s_ij = tau <q_hi, k_gj>:
 *     sigma_hi = KL(p' || p) = -ln(1 - p_ii) = softplus(s_ii - LSE_{j in B(i), j != i} s_ij)
 * (p: band softmax with the diagonal, p': without it); +inf when the band
 * holds only i.  Group score r_gi = mean of sigma over the G query heads of g.
 *   q    [B,H,N,d]   dtype
 *   k    [B,Hkv,N,d] dtype
 *   r_kv [B,Hkv,N]   fp32 out
 *   r_q  [B,H,N]     fp32 out, may be NULL (per-query-head sigma)
 * Requires w >= 1.  bf16 with d in {64, 128} and w a multiple of 128 runs on
 * the tensor cores when r_q is given or G <= 2 (r_q doubles as the per-head
 * buffer); otherwise the SIMT kernel computes the same scores.
 */
STILL_API still_status still_saliency(const still_dims *dims, const void *q, const void *k, float *r_kv, float *r_q,
                            void *stream);

/*
 * Diagonal-only router score ([p4] "Surprising findings": an ablation routes on
 * the diagonal term by itself): r_gi = mean over the G query heads of g of the
 * raw diagonal logit tau <q_hi, k_gi> (read as the logit, not its band
 * probability).  An alternative to still_saliency's r_kv: its per-chunk top-k
 * (still_select_topk) passed as idx_in to still_hybrid_prefill runs the layer
 * with this router.  w may be 0.
 *   q [B,H,N,d], k [B,Hkv,N,d] dtype;  r_kv [B,Hkv,N] fp32 out
 */
STILL_API still_status still_diagonal_score(const still_dims *dims, const void *q, const void *k, float *r_kv,
                                            void *stream);

/*
 * Per-chunk top-k ([p1] "Chunk-Wise": scores per chunk, kept tokens chosen in
 * one batch; [p4] "Approach": top-scoring tokens go to softmax attention).
 * For every full chunk c < T = floor(N/C) of every (b, g): the k positions
 * with the largest r, ties broken by the lower position, written in
 * ascending order.  Bit-exact given r.
 *   r_kv [B,Hkv,N]    fp32 in
 *   idx  [B,Hkv,T,k]  int32 out (absolute token positions)
 */
STILL_API still_status still_select_topk(const still_dims *dims, const float *r_kv, int32_t *idx, void *stream);

/*
 * NP-Map feature map ([p1] "Norm-Preserved Feature Map"; [p4] "Approach"):
 *     phi(x) = ||x||_2 * f(x W) / ||f(x W)||_2,   f = softmax over the D features
 * with one bias-free d->D map per head.
 *   x   [B,Hx,N,d] dtype
 *   W   [Hx,d,D]   dtype
 *   phi [B,Hx,N,D] fp32 out
 */
STILL_API still_status still_npmap(int B, int Hx, int N, int d, int D, still_dtype dtype, const void *x, const void *W,
                         float *phi, void *stream);

/* Bytes of scratch still_hybrid_prefill needs for `dims` (256-byte aligned pointer). */
STILL_API size_t still_prefill_workspace_bytes(const still_dims *dims);

/* Byte offsets of the intermediate results inside the prefill workspace, for inspection. */
typedef struct {
    size_t r;      /* fp32  [B,Hkv,N]          group saliency scores          */
    size_t idx;    /* int32 [B,Hkv,T,k]        kept positions per chunk        */
    size_t khat;   /* dtype [B,Hkv,T*k,d]      kept keys, chunk order          */
    size_t vhat;   /* dtype [B,Hkv,T*k,d]      kept values                     */
    size_t S;      /* fp32  [B,Hkv,T+1,D,d]    linear state seen by chunk t    */
    size_t z;      /* fp32  [B,Hkv,T+1,D]      linear normaliser seen by chunk t */
    size_t phik;   /* fp32  [B,Hkv,N,D]        NP-Map features of the keys (SIMT path; bf16 on the
                      tensor-core w = 0 path; empty on the tensor-core hybrid path) */
    size_t sig;    /* fp32  [B,H,N]            per-query-head saliency (bf16 tensor-core path) */
    size_t lse;    /* fp32  [B,H,N]            log2-sum-exp of each row's window part (same path) */
    size_t fix;    /* u32 count + int32 [B*H*N] rows whose band score is recomputed (same path) */
    size_t wqt;    /* bf16  [H,D,d]            Wq transposed (bf16 tensor-core path) */
    size_t wkt;    /* bf16  [Hkv,D,d]          Wk transposed (bf16 tensor-core path) */
    size_t st;     /* bf16  [B,Hkv,T+1,d,D]    S_t transposed (bf16 tensor-core path) */
    size_t total;
} still_ws_layout;

STILL_API still_status still_prefill_workspace_layout(const still_dims *dims, still_ws_layout *out);

/*
 * Hybrid-attention forward of one layer (prefill), all five steps ([p1]
 * introduction and "Chunk-Wise"; [p4] "Approach"):
 *   1. group saliency r (skipped if idx_in is given or k == 0);
 *   2. per-chunk top-k -> idx, and the kept K/V rows gathered into a compact
 *      chunk-ordered cache;
 *   3. softmax branch of query i in chunk t = floor(i/C), m = w/C:
 *      Soft(i) = [max(0,(t-m)C), i]  U  kept rows of chunks c <= t-m-1;
 *   4. linear branch over the other tokens of the chunks c <= t-m-1, with NP-Map
 *      features: S_t = sum phi(k_j) v_j^T, z_t = sum phi(k_j);
 *   5. one shared normaliser:
 *      o_i = (sum_Soft e^{s_ij} v_j + phi(q_i)^T S_t) / (sum_Soft e^{s_ij} + phi(q_i)^T z_t).
 *   w = 0: no softmax branch; every j <= i is linear.
 *   q [B,H,N,d], k/v [B,Hkv,N,d], Wq [H,d,D], Wk [Hkv,d,D], o [B,H,N,d]  (dtype)
 *   idx_in     [B,Hkv,T,k] int32 or NULL: use this selection instead of computing it
 *              (each index must lie in its chunk; violations set the device error word
 *              and the row is ignored)
 *   workspace  device scratch of workspace_bytes >= still_prefill_workspace_bytes(dims)
 *   state      NULL, or a decode state made by still_decode_init with capacity
 *              state_capacity >= N: it is left holding the layer's cache after N tokens
 *              (positioned at N), ready for still_decode_step.
 */
STILL_API still_status still_hybrid_prefill(const still_dims *dims, const void *q, const void *k, const void *v, const void *Wq,
                                  const void *Wk, void *o, const int32_t *idx_in, void *workspace,
                                  size_t workspace_bytes, void *state, int state_capacity, void *stream);

/*
 * still_hybrid_prefill with its scratch in a fixed device array inside this
 * library instead of a caller workspace (no counterpart in the method: the
 * pages describe no memory management).  It is for callers that cannot
 * allocate device memory around the call: a serving loop that must keep its
 * footprint fixed once it has started, code running under a memory budget that
 * another owner enforces, or a host thread that must not call cudaMalloc (which
 * can synchronise the device) while other work is in flight.  Same arguments, results and errors as
 * still_hybrid_prefill, minus workspace and workspace_bytes: the same argument
 * checks run first, in the same order, then the size limit below.  A call
 * allocates nothing: no device, host or pinned memory, directly or through a
 * library.
 *   - Limit: shapes with still_prefill_workspace_bytes(dims) greater than
 *     STILL_STATIC_WORKSPACE_BYTES (64 MiB) are rejected with
 *     STILL_ERR_WORKSPACE before any work; use still_hybrid_prefill for them.
 *   - The 64 MiB array is reserved on a device when the library's module
 *     holding it is loaded there: by default (lazy module loading) on the
 *     first call of this entry point on that device, with
 *     CUDA_MODULE_LOADING=EAGER when the process's context is created on it.
 *     That reservation can fail for lack of device memory, which returns
 *     STILL_ERR_CUDA; callers that must not allocate later should make one
 *     warm-up call before entering their allocation-free loop.
 *   - Nothing in the array has to start at zero: each call writes every part of
 *     the scratch it reads (its counter of recomputed rows is reset by the call
 *     itself), so leftovers of earlier calls, of any shape, do no harm.
 *   - One array per device: calls that overlap in time on one device (other
 *     streams, other host threads) share it and race; serialise them.
 *   - The array's address is looked up once per device, with that device
 *     current, on the first call there (which may load the library's module for
 *     it); make that first call before any stream capture.
 * STILL_ERR_CUDA if the current device or the array's address cannot be had
 * (device ordinals 128 and above are not supported).
 */
#define STILL_STATIC_WORKSPACE_BYTES (64u << 20)
STILL_API still_status still_hybrid_prefill_static(const still_dims *dims, const void *q, const void *k,
                                                   const void *v, const void *Wq, const void *Wk, void *o,
                                                   const int32_t *idx_in, void *state, int state_capacity,
                                                   void *stream);

/*
 * Backward pass of still_hybrid_prefill ([p1] introduction and "Chunk-Wise":
 * one chunk-parallel implementation for training and inference): gradients of
 * L = sum(dO * o) with respect to q, k, v, Wq and Wk, with the per-chunk
 * selection idx held fixed (top-k is a discrete choice with no gradient).
 * w = 0 (no window, k = 0: every earlier token in the linear set) is covered.
 *   q, k, v, Wq, Wk  as for still_hybrid_prefill (dtype)
 *   idx   [B,Hkv,T,k] int32, the selection the forward used (NULL when k = 0 or T = 0)
 *   dO    [B,H,N,d] dtype, the gradient of the layer output
 *   dq    [B,H,N,d], dk/dv [B,Hkv,N,d], dWq [H,d,D], dWk [Hkv,d,D]: fp32 out (overwritten)
 *   workspace  device scratch of still_backward_workspace_bytes(dims) bytes, 256-byte aligned
 * bf16 with d in {64, 128}, C a multiple of 128 and w >= 1: the softmax branch
 * runs on tensor cores (P and dS enter the MMAs in bf16) and, for D in {64, 128},
 * the linear branch in tiled fp32 kernels whose weight and chunk sums add with
 * atomics; otherwise SIMT kernels with fp32 arithmetic (w = 0 among them).
 * Sums that use atomics round in schedule order.
 */
STILL_API size_t still_backward_workspace_bytes(const still_dims *dims);
STILL_API still_status still_hybrid_backward(const still_dims *dims, const void *q, const void *k, const void *v,
                                             const void *Wq, const void *Wk, const int32_t *idx, const void *dO,
                                             float *dq, float *dk, float *dv, float *dWq, float *dWk,
                                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * The same backward pass given what the forward left behind ([p1] "Chunk-Wise":
 * one implementation for training and inference, where a training step runs
 * the forward first).  Every row's gradient needs its normaliser L_i (both
 * branches) and D_i = <dO_i, o_i>; still_hybrid_backward forms them with a
 * first sweep over the row's keys, this call takes them from the forward:
 *   o     [B,H,N,d] dtype, the output of still_hybrid_prefill on the same inputs
 *         (and the same selection idx)
 *   lse   [B,H,N] fp32, the forward's per-row log2 normaliser: the region "lse" of
 *         the workspace of that still_hybrid_prefill call (offset in
 *         still_prefill_workspace_layout), read after the call completed and
 *         before the workspace is used again
 * Other arguments, errors and workspace as for still_hybrid_backward; o and lse
 * must be non-NULL and 16-byte aligned.  They are used where the forward ran its
 * tensor-core merge and the backward its tensor-core softmax branch (bf16,
 * d and D in {64, 128}, C a multiple of 128, w >= 1); elsewhere the call forms the
 * statistics itself, as still_hybrid_backward does.  D_i comes from the rounded
 * o (dtype), so the gradients differ from still_hybrid_backward's by rounding.
 */
STILL_API still_status still_hybrid_backward_saved(const still_dims *dims, const void *q, const void *k,
                                                   const void *v, const void *Wq, const void *Wk,
                                                   const int32_t *idx, const void *dO, const void *o,
                                                   const float *lse, float *dq, float *dk, float *dv, float *dWq,
                                                   float *dWk, void *workspace, size_t workspace_bytes,
                                                   void *stream);

/*
 * Chunk-granular delayed decode ([p1] "Chunk-Wise": during decoding the
 * selection is delayed at chunk granularity).  The state is one caller-owned
 * device buffer holding, per (b, g): the kept K/V cache, the linear state
 * S [D,d] and z [D], the window ring (K/V and scores of chunks t-m..t) and
 * the position.  dims->N is ignored; `capacity` is the largest number of
 * tokens the state can hold.
 */
STILL_API size_t still_decode_state_bytes(const still_dims *dims, int capacity);

/*
 * Byte offsets of the decode state's segments, for inspection (the kernels own
 * the contents; a caller reads them only between calls on the stream).  Per
 * (b, g), G = B*Hkv groups, cap_chunks = capacity / C:
 *   khat, vhat  dtype [B,Hkv,cap_chunks*k,d]  kept rows of each closed chunk c at
 *               rows [c*k, c*k+k), ascending positions
 *   S, z        fp32 [B,Hkv,D,d], [B,Hkv,D]   linear state of the folded tokens
 *   ring_k/v    dtype [B,Hkv,ring_rows,d]     rows of the last m+1 chunks
 *   ring_r      fp32 [B,Hkv,ring_rows]        their group saliency scores
 * Position j of the ring sits at row ((j / C) % (m+1)) * C + j % C
 * (m = w / C; w = 0: row j % C); ring_rows = (m+1) * C (C when w = 0).
 */
typedef struct {
    size_t header, khat, vhat, S, z, ring_k, ring_v, ring_r, total;
    int ring_rows, cap_chunks;
} still_state_layout;
STILL_API still_status still_decode_state_layout(const still_dims *dims, int capacity, still_state_layout *out);

/* Empty state at position 0. */
STILL_API still_status still_decode_init(const still_dims *dims, int capacity, void *state, void *stream);

/*
 * One token per sequence at position `pos` (must equal the state's position;
 * 0 <= pos < capacity): scores it, attends over window + kept cache + linear
 * state exactly as the prefill does for row pos, and, if pos closes chunk t
 * (pos % C == C-1) and t-m >= 0, selects chunk t-m, appends its kept rows and
 * folds the others into S, z.
 *   q_t [B,H,d], k_t/v_t [B,Hkv,d], o_t [B,H,d] (dtype); Wq, Wk as for prefill.
 */
STILL_API still_status still_decode_step(const still_dims *dims, void *state, int capacity, int pos, const void *Wq,
                               const void *Wk, const void *q_t, const void *k_t, const void *v_t, void *o_t,
                               void *stream);

/*
 * Synchronises `stream`, then returns and clears the current device's error
 * word: STILL_OK, STILL_ERR_DEVICE_CHECK or STILL_ERR_TIMEOUT (or
 * STILL_ERR_CUDA if the synchronisation itself failed).
 */
STILL_API still_status still_get_device_status(void *stream);

/* Number of kernels this library has launched in this process (all devices). */
STILL_API uint64_t still_launch_count(void);

/*
 * Per-kernel timing for benchmarks (no counterpart in the method; host-side
 * instrumentation).  While enabled, every kernel launched by
 * still_hybrid_prefill, still_decode_step and still_hybrid_backward is bracketed by a pair of CUDA
 * events recorded on the caller's stream (created on first use; at most
 * STILL_TIMING_MAX_LAUNCHES launches are kept; later ones are not timed).  still_timing_read synchronises those events and, for
 * each kernel class c < n, writes the summed milliseconds to ms[c] and the
 * number of timed launches to launches[c], then forgets them.  Classes:
 * 0 saliency (group mean on the tensor-core path), 1 top-k + gather, 2 NP-Map,
 * 3 linear state, 4 softmax/linear merge (tensor-core path: window part with
 * the fused saliency), 5 decode-state export, 6 tensor-core merge of the kept
 * prefix and the linear branch, 7 decode append, 8 decode attention, 9 decode
 * combine, 10 decode chunk close, 11 backward dq (tensor cores), 12 backward dk/dv
 * (tensor cores, window and kept keys), 13 backward linear branch (linear state,
 * NP-Map backward, chunk sums, key side; the tiled path).  Single-threaded use only.
 */
/*
 * Test hooks of the head-dimension-64 tensor-core merge (no counterpart in the
 * method; host state of the library, read when a merge is launched;
 * single-threaded use only; (0, 0), the default, leaves the kernels alone).
 *   stall != 0: the first CTA of every later launch loads its query tiles but
 *     issues no key/value tile, so its MMA warp's bounded wait (2 s) runs out:
 *     the CTA records STILL_ERR_TIMEOUT in the device status word (read it
 *     with still_get_device_status), drains its own copies, frees its tensor
 *     memory and returns, and every other CTA finishes normally.  The output
 *     of that call is undefined; the context stays usable.
 *   max_ctas > 0: the persistent merge grid holds at most max_ctas CTAs (one
 *     per SM otherwise), so small problems also run many work items per CTA.
 *     Results do not depend on it.
 */
STILL_API void still_debug_merge(int stall, int max_ctas);

#define STILL_TIMING_MAX_LAUNCHES 4096
#define STILL_TIMING_CLASSES 14
STILL_API still_status still_timing_enable(int on);
STILL_API still_status still_timing_read(double *ms, int *launches, int n);

#ifdef __cplusplus
}
#endif

#endif /* STILL_H */
