/*
 * still_oracle.c -- plain fp64 CPU oracle for the STILL hybrid-attention layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product (the CUDA library and its
 * Python binding) links, loads or calls this file; only the tests, the
 * package's smoke check and the benchmark's CPU-baseline leg do.  It shares no
 * code, header, table or helper with the CUDA path.
 *
 * Source of every definition: "STILL: Selecting Tokens for Intra-Layer Hybrid
 * Attention to Linearize LLMs" as described on the pages
 *   [p1] jsqmd.com news article: sections "Self-Saliency Score",
 *        "Norm-Preserved Feature Map (NP-Map)", "Chunk-Wise parallel + delayed
 *        selection", and the introduction (two branches inside one layer);
 *   [p4] atlas.scime.ai summary: section "Approach".
 * The pages give prose only (no formulas, no code); every place where a
 * reading had to be chosen is marked READING below.
 *
 * Notation: B batch, H query heads, Hkv key/value heads, G = H/Hkv, head dim d,
 * NP-Map width D, window w = m*C, chunk C, k kept per chunk, T = floor(N/C)
 * full chunks, g(h) = h / G.  Tensors are row-major:
 *   q [B,H,N,d], k/v [B,Hkv,N,d], Wq [H,d,D], Wk [Hkv,d,D], o [B,H,N,d].
 *
 * Everything is computed in double precision directly from the definitions,
 * one query row at a time; no blocking, fusion or reordering.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, H, Hkv, N, d, D, w, C, k;
    double scale; /* softmax logit scale tau; READING: 1/sqrt(d) (pretrained default) */
} od_dims;

enum { OD_OK = 0, OD_EINVAL = -1, OD_ENOMEM = -2, OD_ENONFINITE = -3 };

static int od_check(const od_dims *s)
{
    if (!s || s->B < 0 || s->H <= 0 || s->Hkv <= 0 || s->N < 0 || s->d <= 0 || s->D <= 0 ||
        s->C <= 0 || s->k < 0 || s->k > s->C || s->w < 0)
        return OD_EINVAL;
    if (s->H % s->Hkv) return OD_EINVAL;
    if (s->w % s->C) return OD_EINVAL;          /* window is a whole number of chunks */
    if (s->w == 0 && s->k != 0) return OD_EINVAL; /* no window: nothing is ever selected */
    return OD_OK;
}

/* ------------------------------------------------------------------------ */
/* simple thread pool: run fn(arg, i) for i in [0, n) on nthreads threads    */

typedef void (*od_task_fn)(void *arg, long i);
typedef struct {
    od_task_fn fn;
    void *arg;
    long n;
    long next;
    pthread_mutex_t mu;
} od_pool;

static void *od_worker(void *p)
{
    od_pool *pool = (od_pool *)p;
    for (;;) {
        pthread_mutex_lock(&pool->mu);
        long i = pool->next++;
        pthread_mutex_unlock(&pool->mu);
        if (i >= pool->n) break;
        pool->fn(pool->arg, i);
    }
    return NULL;
}

static void od_parallel_for(long n, int nthreads, od_task_fn fn, void *arg)
{
    od_pool pool = {fn, arg, n, 0, PTHREAD_MUTEX_INITIALIZER};
    if (nthreads <= 1 || n <= 1) {
        for (long i = 0; i < n; ++i) fn(arg, i);
        return;
    }
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    int started = 0;
    for (int t = 0; t < nthreads; ++t)
        if (pthread_create(&th[t], NULL, od_worker, &pool) == 0) ++started;
    if (started == 0) od_worker(&pool);
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
}

/* ------------------------------------------------------------------------ */
/* scores                                                                    */

/* s_{h,i,j} = tau * <q_{h,i}, k_{g(h),j}>  */
static double od_logit(const od_dims *s, const double *qi, const double *kj)
{
    double acc = 0.0;
    for (int x = 0; x < s->d; ++x) acc += qi[x] * kj[x];
    return s->scale * acc;
}

/*
 * Self-Saliency Score of one query row ([p1] "Self-Saliency Score"; [p4]
 * "Approach": a divergence of the Kullback-Leibler kind that compares the
 * window attention of the token with the same attention once its own key is
 * left out).
 *
 * READINGS:
 *  - the band is B(i) = {j : max(0, i-w+1) <= j <= i}, i.e. w keys including
 *    the token itself;
 *  - p  = softmax of the logits over B(i)        (with the diagonal),
 *    p' = softmax of the logits over B(i)\{i}    (without it),
 *    sigma = KL(p' || p) = sum_{j != i} p'_j ln(p'_j / p_j)
 *    (the other direction is infinite since p'_i = 0);
 *  - if B(i)\{i} is empty (i = 0 or w = 1), sigma = +inf.
 * The sum is evaluated term by term.
 */
static double od_sigma_row(const od_dims *s, const double *qi, const double *kg, int i)
{
    int lo = i - s->w + 1;
    if (lo < 0) lo = 0;
    int n = i - lo + 1;
    if (n <= 1) return INFINITY;
    double *lg = (double *)malloc(sizeof(double) * (size_t)n);
    if (!lg) return NAN;
    for (int j = lo; j <= i; ++j) lg[j - lo] = od_logit(s, qi, kg + (size_t)j * s->d);
    /* with diagonal */
    double mx = -INFINITY;
    for (int t = 0; t < n; ++t) mx = lg[t] > mx ? lg[t] : mx;
    double z = 0.0;
    for (int t = 0; t < n; ++t) z += exp(lg[t] - mx);
    double logz = mx + log(z);
    /* without diagonal (last entry is j = i) */
    double mx2 = -INFINITY;
    for (int t = 0; t < n - 1; ++t) mx2 = lg[t] > mx2 ? lg[t] : mx2;
    double z2 = 0.0;
    for (int t = 0; t < n - 1; ++t) z2 += exp(lg[t] - mx2);
    double logz2 = mx2 + log(z2);
    double kl = 0.0;
    for (int t = 0; t < n - 1; ++t) {
        double lp2 = lg[t] - logz2; /* ln p'_j */
        double lp = lg[t] - logz;   /* ln p_j  */
        kl += exp(lp2) * (lp2 - lp);
    }
    free(lg);
    return kl;
}

typedef struct {
    const od_dims *s;
    const double *q, *k;
    double *sigma; /* [B,H,N] */
} od_sal_job;

#define OD_ROWS_PER_TASK 256

static void od_sal_task(void *p, long u)
{
    od_sal_job *J = (od_sal_job *)p;
    const od_dims *s = J->s;
    int G = s->H / s->Hkv;
    long nblk = (s->N + OD_ROWS_PER_TASK - 1) / OD_ROWS_PER_TASK;
    long bh = u / nblk, blk = u % nblk;
    long b = bh / s->H, h = bh % s->H;
    const double *kg = J->k + ((size_t)b * s->Hkv + h / G) * (size_t)s->N * s->d;
    const double *qh = J->q + ((size_t)b * s->H + h) * (size_t)s->N * s->d;
    int i1 = (int)((blk + 1) * OD_ROWS_PER_TASK);
    if (i1 > s->N) i1 = s->N;
    for (int i = (int)(blk * OD_ROWS_PER_TASK); i < i1; ++i)
        J->sigma[((size_t)b * s->H + h) * s->N + i] = od_sigma_row(s, qh + (size_t)i * s->d, kg, i);
}

/*
 * sigma [B,H,N] per query head, r [B,Hkv,N] per KV head.
 * READING (GQA): the routing decision is per KV head (the kept cache and the
 * linear state belong to a KV head), and r_{g,i} is the plain mean of the
 * sigma of the G query heads of group g.
 */
int od_saliency(const od_dims *s, const double *q, const double *k, double *sigma, double *r, int nthreads)
{
    int e = od_check(s);
    if (e) return e;
    if (s->w < 1) return OD_EINVAL;
    int G = s->H / s->Hkv;
    double *sg = sigma;
    if (!sg) {
        sg = (double *)malloc(sizeof(double) * (size_t)s->B * s->H * s->N + 1);
        if (!sg) return OD_ENOMEM;
    }
    od_sal_job J = {s, q, k, sg};
    od_parallel_for((long)s->B * s->H * ((s->N + OD_ROWS_PER_TASK - 1) / OD_ROWS_PER_TASK), nthreads, od_sal_task, &J);
    if (r) {
        for (int b = 0; b < s->B; ++b)
            for (int g = 0; g < s->Hkv; ++g)
                for (int i = 0; i < s->N; ++i) {
                    double acc = 0.0;
                    for (int hh = 0; hh < G; ++hh) acc += sg[((size_t)b * s->H + g * G + hh) * s->N + i];
                    r[((size_t)b * s->Hkv + g) * s->N + i] = acc / G;
                }
    }
    if (!sigma) free(sg);
    return OD_OK;
}

/*
 * Diagonal-only router ([p4] "Surprising findings": an ablation that routes on
 * the diagonal term by itself): r_{g,i} = mean over the G query heads of g of
 * the raw diagonal logit s_ii = tau <q_hi, k_gi>.
 * READING: "the diagonal term" is taken as the raw logit s_ii, not
 * its probability within the band (which would make it the saliency score's
 * own ingredient p_ii); the GQA mean follows the saliency score's reading.
 */
int od_diagonal_score(const od_dims *s, const double *q, const double *k, double *r)
{
    int e = od_check(s);
    if (e) return e;
    int G = s->H / s->Hkv;
    for (int b = 0; b < s->B; ++b)
        for (int g = 0; g < s->Hkv; ++g)
            for (int i = 0; i < s->N; ++i) {
                const double *ki = k + (((size_t)b * s->Hkv + g) * s->N + i) * s->d;
                double acc = 0.0;
                for (int hh = 0; hh < G; ++hh) {
                    const double *qi = q + (((size_t)b * s->H + g * G + hh) * s->N + i) * s->d;
                    double dot = 0.0;
                    for (int x = 0; x < s->d; ++x) dot += qi[x] * ki[x];
                    acc += s->scale * dot;
                }
                r[((size_t)b * s->Hkv + g) * s->N + i] = acc / G;
            }
    return OD_OK;
}

/* ------------------------------------------------------------------------ */
/* per-chunk top-k ([p1] "Chunk-Wise": scores are computed per chunk and the  */
/* kept tokens are chosen in one batch; [p4] "Approach": the top-scoring      */
/* tokens go to softmax attention).                                          */
/* READING: order = score descending, then index ascending; output ascending. */

static int od_better(double ra, int a, double rb, int b)
{
    if (ra > rb) return 1;
    if (ra < rb) return 0;
    return a < b;
}

/* Select k of the C scores r[0..C) into out[0..k) (local indices, ascending). */
static void od_topk_chunk(const double *r, int C, int k, int32_t *out)
{
    unsigned char *taken = (unsigned char *)calloc((size_t)C, 1);
    for (int n = 0; n < k; ++n) {
        int best = -1;
        for (int j = 0; j < C; ++j) {
            if (taken[j]) continue;
            if (best < 0 || od_better(r[j], j, r[best], best)) best = j;
        }
        taken[best] = 1;
    }
    int n = 0;
    for (int j = 0; j < C; ++j)
        if (taken[j]) out[n++] = j;
    free(taken);
}

/* r [B,Hkv,N] -> idx [B,Hkv,T,k] of absolute token positions, ascending per chunk. */
int od_topk(const od_dims *s, const double *r, int32_t *idx)
{
    int e = od_check(s);
    if (e) return e;
    int T = s->N / s->C;
    for (int b = 0; b < s->B; ++b)
        for (int g = 0; g < s->Hkv; ++g)
            for (int c = 0; c < T; ++c) {
                const double *rc = r + ((size_t)b * s->Hkv + g) * s->N + (size_t)c * s->C;
                int32_t *o = idx + (((size_t)b * s->Hkv + g) * T + c) * s->k;
                od_topk_chunk(rc, s->C, s->k, o);
                for (int n = 0; n < s->k; ++n) o[n] += c * s->C;
            }
    return OD_OK;
}

/* ------------------------------------------------------------------------ */
/* NP-Map ([p1] "Norm-Preserved Feature Map"; [p4] "Approach"): the direction */
/* comes from the normalised MLP output and the input's own norm is put back: */
/*   phi(x) = ||x||_2 * f(x W) / ||f(x W)||_2,  f = softmax over the D features */
/* READINGS: the MLP is one bias-free linear map d -> D (separate maps for q   */
/* and k, one per head); f is the Hedgehog-style softmax over features without */
/* the +/- doubling; phi is applied to q and k as given (no 1/sqrt(d)).        */

static void od_phi_row(int d, int D, const double *x, const double *W, double *phi)
{
    double nx = 0.0;
    for (int a = 0; a < d; ++a) nx += x[a] * x[a];
    nx = sqrt(nx);
    double mx = -INFINITY;
    for (int c = 0; c < D; ++c) {
        double y = 0.0;
        for (int a = 0; a < d; ++a) y += x[a] * W[(size_t)a * D + c];
        phi[c] = y;
        mx = y > mx ? y : mx;
    }
    double z = 0.0;
    for (int c = 0; c < D; ++c) {
        phi[c] = exp(phi[c] - mx);
        z += phi[c];
    }
    double nf = 0.0;
    for (int c = 0; c < D; ++c) {
        phi[c] /= z;
        nf += phi[c] * phi[c];
    }
    nf = sqrt(nf);
    for (int c = 0; c < D; ++c) phi[c] = nx * phi[c] / nf;
}

/* x [n,d], W [d,D] -> phi [n,D] */
int od_npmap(int n, int d, int D, const double *x, const double *W, double *phi)
{
    if (n < 0 || d <= 0 || D <= 0) return OD_EINVAL;
    for (int i = 0; i < n; ++i) od_phi_row(d, D, x + (size_t)i * d, W, phi + (size_t)i * D);
    return OD_OK;
}

/* ------------------------------------------------------------------------ */
/* routing sets ([p1] intro: selected tokens -> softmax branch, the others    */
/* -> linear branch, in the same layer; [p1] "Chunk-Wise": selection in       */
/* batches per chunk, delayed; [p4] "Approach": the routing decision waits    */
/* and is taken a chunk at a time).                                          */
/*
 * READING (chunk-granular delay): for query i in chunk t = floor(i/C) with
 * m = w/C,
 *   Local(i) = { j : max(0,(t-m)C) <= j <= i }
 *   chunk c is decided for i iff c <= t-m-1 (it has left the window of the
 *   whole query chunk), and then Sel(c) is its top-k set;
 *   Soft(i)  = Local(i)  U  Sel(c) over decided c,
 *   Lin(i)   = (c \ Sel(c)) over decided c.
 * w = 0 (no window, k = 0): Soft(i) is empty and Lin(i) = { j <= i }.
 * Output: 0 = not attended, 1 = softmax branch, 2 = linear branch, for j <= i.
 */
static void od_route_row(const od_dims *s, const unsigned char *selmask_g, int i, unsigned char *route)
{
    if (s->w == 0) {
        for (int j = 0; j <= i; ++j) route[j] = 2;
        return;
    }
    int m = s->w / s->C;
    int t = i / s->C;
    int lo = (t - m) * s->C;
    if (lo < 0) lo = 0;
    for (int j = 0; j <= i; ++j) {
        if (j >= lo) {
            route[j] = 1;
        } else {
            int c = j / s->C; /* c <= t-m-1: decided */
            (void)c;
            route[j] = selmask_g[j] ? 1 : 2;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* merge ([p1] intro and "NP-Map": both branches are fused inside one layer   */
/* and must agree in distribution).                                           */
/* READING: one shared normaliser, no learned mixing factor:                  */
/*   o_i = [ sum_{Soft} e^{s_ij} v_j + sum_{Lin} <phi(q_i),phi(k_j)> v_j ]   */
/*       / [ sum_{Soft} e^{s_ij}     + sum_{Lin} <phi(q_i),phi(k_j)>     ]   */
/* evaluated with the shift M = max_{Soft} s_ij applied to both branches      */
/* (multiplying numerator and denominator by e^{-M} changes nothing).         */

typedef struct {
    const od_dims *s;
    const double *q, *k, *v, *Wq;
    const double *phik;            /* [B,Hkv,N,D] */
    const unsigned char *selmask;  /* [B,Hkv,N] */
    double *o;                     /* [B,H,N,d] (only listed rows written) */
    const int32_t *rows;           /* nrows x (b,h,i) or NULL = all */
    long nrows;
    int bad;
} od_out_job;

static void od_out_task(void *p, long u)
{
    od_out_job *J = (od_out_job *)p;
    const od_dims *s = J->s;
    int b, h, i;
    if (J->rows) {
        b = J->rows[3 * u];
        h = J->rows[3 * u + 1];
        i = J->rows[3 * u + 2];
    } else {
        b = (int)(u / ((long)s->H * s->N));
        h = (int)((u / s->N) % s->H);
        i = (int)(u % s->N);
    }
    int G = s->H / s->Hkv, g = h / G, d = s->d, D = s->D;
    size_t kvo = ((size_t)b * s->Hkv + g) * (size_t)s->N;
    const double *qi = J->q + (((size_t)b * s->H + h) * s->N + i) * d;
    unsigned char *route = (unsigned char *)malloc((size_t)i + 1);
    double *phiq = (double *)malloc(sizeof(double) * D);
    double *num = (double *)calloc((size_t)d, sizeof(double));
    od_route_row(s, J->selmask + kvo, i, route);
    od_phi_row(d, D, qi, J->Wq + (size_t)h * d * D, phiq);
    double M = -INFINITY;
    for (int j = 0; j <= i; ++j)
        if (route[j] == 1) {
            double l = od_logit(s, qi, J->k + (kvo + j) * d);
            M = l > M ? l : M;
        }
    if (M == -INFINITY) M = 0.0; /* no softmax keys: no shift needed */
    double den = 0.0;
    for (int j = 0; j <= i; ++j) {
        double wgt;
        if (route[j] == 1) {
            wgt = exp(od_logit(s, qi, J->k + (kvo + j) * d) - M);
        } else if (route[j] == 2) {
            const double *pk = J->phik + (kvo + j) * D;
            double dot = 0.0;
            for (int c = 0; c < D; ++c) dot += phiq[c] * pk[c];
            wgt = dot * exp(-M);
        } else {
            continue;
        }
        const double *vj = J->v + (kvo + j) * d;
        for (int x = 0; x < d; ++x) num[x] += wgt * vj[x];
        den += wgt;
    }
    double *oi = J->o + (((size_t)b * s->H + h) * s->N + i) * d;
    for (int x = 0; x < d; ++x) {
        oi[x] = num[x] / den;
        if (!isfinite(oi[x])) J->bad = 1;
    }
    free(route);
    free(phiq);
    free(num);
}

typedef struct {
    const od_dims *s;
    const double *k, *Wk;
    double *phik;
} od_phik_job;

static void od_phik_task(void *p, long u)
{
    od_phik_job *J = (od_phik_job *)p;
    const od_dims *s = J->s;
    long g = u % s->Hkv;
    od_npmap(s->N, s->d, s->D, J->k + (size_t)u * s->N * s->d, J->Wk + (size_t)g * s->d * s->D,
             J->phik + (size_t)u * s->N * s->D);
}

static int od_selection(const od_dims *s, const double *q, const double *k, const int32_t *idx_in,
                        double *r_out, int32_t *idx_out, unsigned char *selmask, int nthreads)
{
    int T = s->N / s->C;
    size_t nidx = (size_t)s->B * s->Hkv * T * s->k;
    int32_t *idx = idx_out;
    int own_idx = 0;
    memset(selmask, 0, (size_t)s->B * s->Hkv * s->N);
    if (r_out && s->w > 0 && !idx_in && (s->k == 0 || T == 0))
        return od_saliency(s, q, k, NULL, r_out, nthreads); /* scores asked for, nothing to select */
    if (s->k == 0 || T == 0) return OD_OK;
    if (!idx) {
        idx = (int32_t *)malloc(sizeof(int32_t) * nidx + 1);
        if (!idx) return OD_ENOMEM;
        own_idx = 1;
    }
    if (idx_in) {
        memcpy(idx, idx_in, sizeof(int32_t) * nidx);
    } else {
        double *r = r_out;
        if (!r) r = (double *)malloc(sizeof(double) * (size_t)s->B * s->Hkv * s->N + 1);
        int e = od_saliency(s, q, k, NULL, r, nthreads);
        if (!e) e = od_topk(s, r, idx);
        if (!r_out) free(r);
        if (e) {
            if (own_idx) free(idx);
            return e;
        }
    }
    for (int b = 0; b < s->B; ++b)
        for (int g = 0; g < s->Hkv; ++g)
            for (int c = 0; c < T; ++c)
                for (int n = 0; n < s->k; ++n) {
                    int j = idx[(((size_t)b * s->Hkv + g) * T + c) * s->k + n];
                    if (j < c * s->C || j >= (c + 1) * s->C) {
                        if (own_idx) free(idx);
                        return OD_EINVAL; /* an injected index outside its chunk */
                    }
                    selmask[((size_t)b * s->Hkv + g) * s->N + j] = 1;
                }
    if (own_idx) free(idx);
    return OD_OK;
}

/*
 * Full layer forward.  idx_in (nullable) injects the per-chunk selection
 * instead of computing it; r_out / idx_out (nullable) return the scores and
 * the selection; rows (nullable) restricts the output to nrows (b,h,i)
 * triples.  phik_in (nullable) supplies phi(k) [B,Hkv,N,D] of every key, as
 * od_npmap computes it, instead of computing it from k and Wk here (callers
 * that evaluate rows of the same keys many times pass it once computed).
 */
static int od_prefill_core(const od_dims *s, const double *q, const double *k, const double *v, const double *Wq,
                           const double *Wk, const double *phik_in, const int32_t *idx_in, double *o,
                           double *r_out, int32_t *idx_out, const int32_t *rows, long nrows, int nthreads)
{
    int e = od_check(s);
    if (e) return e;
    size_t nkv = (size_t)s->B * s->Hkv * s->N;
    unsigned char *selmask = (unsigned char *)malloc(nkv + 1);
    double *phik = phik_in ? NULL : (double *)malloc(sizeof(double) * nkv * s->D + 1);
    if (!selmask || (!phik_in && !phik)) {
        free(selmask);
        free(phik);
        return OD_ENOMEM;
    }
    e = od_selection(s, q, k, idx_in, r_out, idx_out, selmask, nthreads);
    if (!e) {
        if (!phik_in) {
            od_phik_job PJ = {s, k, Wk, phik};
            od_parallel_for((long)s->B * s->Hkv, nthreads, od_phik_task, &PJ);
        }
        od_out_job J = {s, q, k, v, Wq, phik_in ? phik_in : phik, selmask, o, rows,
                        rows ? nrows : (long)s->B * s->H * s->N, 0};
        od_parallel_for(J.nrows, nthreads, od_out_task, &J);
        if (J.bad) e = OD_ENONFINITE;
    }
    free(selmask);
    free(phik);
    return e;
}

int od_prefill(const od_dims *s, const double *q, const double *k, const double *v, const double *Wq,
               const double *Wk, const int32_t *idx_in, double *o, double *r_out, int32_t *idx_out,
               const int32_t *rows, long nrows, int nthreads)
{
    return od_prefill_core(s, q, k, v, Wq, Wk, NULL, idx_in, o, r_out, idx_out, rows, nrows, nthreads);
}

int od_prefill_given_phik(const od_dims *s, const double *q, const double *k, const double *v, const double *Wq,
                          const double *phik, const int32_t *idx_in, double *o, double *r_out, int32_t *idx_out,
                          const int32_t *rows, long nrows, int nthreads)
{
    if (!phik) return OD_EINVAL;
    return od_prefill_core(s, q, k, v, Wq, NULL, phik, idx_in, o, r_out, idx_out, rows, nrows, nthreads);
}

/*
 * Linear-branch state seen by query chunk t of (b, g):
 *   S_t = sum over decided chunks c <= t-m-1 of sum_{j in c \ Sel(c)} phi(k_j) v_j^T   [D,d]
 *   z_t = the same sum of phi(k_j)                                                    [D]
 * (w = 0: every chunk c < t, all of its tokens).  idx [B,Hkv,T,k] is given.
 */
int od_linear_state(const od_dims *s, const double *k, const double *v, const double *Wk, const int32_t *idx,
                    int b, int g, int t, double *S, double *z)
{
    int e = od_check(s);
    if (e) return e;
    int T = s->N / s->C, m = s->w / s->C, d = s->d, D = s->D;
    int last = s->w == 0 ? t - 1 : t - m - 1;
    if (last > T - 1) last = T - 1;
    memset(S, 0, sizeof(double) * (size_t)D * d);
    memset(z, 0, sizeof(double) * (size_t)D);
    double *phi = (double *)malloc(sizeof(double) * D);
    size_t kvo = ((size_t)b * s->Hkv + g) * (size_t)s->N;
    for (int c = 0; c <= last; ++c) {
        for (int j = c * s->C; j < (c + 1) * s->C; ++j) {
            int sel = 0;
            for (int n = 0; n < s->k; ++n)
                if (idx[(((size_t)b * s->Hkv + g) * T + c) * s->k + n] == j) sel = 1;
            if (sel) continue;
            od_phi_row(d, D, k + (kvo + j) * d, Wk + (size_t)g * d * D, phi);
            for (int a = 0; a < D; ++a) {
                z[a] += phi[a];
                for (int x = 0; x < d; ++x) S[(size_t)a * d + x] += phi[a] * v[(kvo + j) * d + x];
            }
        }
    }
    free(phi);
    return OD_OK;
}

/* ------------------------------------------------------------------------ */
/* decode: chunk-granular delayed selection ([p1] "Chunk-Wise": during       */
/* decoding the selection is delayed at chunk granularity).                  */
/*
 * An incremental state machine, written independently of od_prefill's
 * per-row sets.  Per (b, g) it keeps: every K/V row seen, the saliency of
 * every token, a list of kept (softmax) positions, and the folded linear state
 * S [D,d], z [D].  At position p (chunk t = p/C):
 *   1. append k_p, v_p; score token p over its band (w >= 1);
 *   2. o_p = merge over  window positions [max(0,(t-m)C), p]  U  kept list
 *      (softmax) and phi(q_p)^T S, phi(q_p)^T z (linear); for w = 0 the
 *      current chunk's positions [tC, p] are linear too;
 *   3. if p closes chunk t (p % C == C-1) and c = t-m >= 0: select top-k of
 *      chunk c on the stored scores, append them to the kept list, fold the
 *      others into S, z.  The change is seen from position (t+1)C on.
 */
typedef struct {
    od_dims s;      /* N = capacity in tokens */
    double *Wq, *Wk;
    int pos;
    double *K, *V;  /* [B,Hkv,cap,d] */
    double *r;      /* [B,Hkv,cap] */
    int32_t *kept;  /* [B,Hkv,cap] */
    int *nkept;     /* [B,Hkv] */
    double *S, *z;  /* [B,Hkv,D,d], [B,Hkv,D] */
} od_decode;

void od_decode_free(od_decode *st)
{
    if (!st) return;
    free(st->Wq);
    free(st->Wk);
    free(st->K);
    free(st->V);
    free(st->r);
    free(st->kept);
    free(st->nkept);
    free(st->S);
    free(st->z);
    free(st);
}

od_decode *od_decode_new(const od_dims *s, const double *Wq, const double *Wk)
{
    if (od_check(s)) return NULL;
    od_decode *st = (od_decode *)calloc(1, sizeof(od_decode));
    if (!st) return NULL;
    st->s = *s;
    size_t cap = (size_t)s->N, BK = (size_t)s->B * s->Hkv;
    st->Wq = (double *)malloc(sizeof(double) * (size_t)s->H * s->d * s->D);
    st->Wk = (double *)malloc(sizeof(double) * (size_t)s->Hkv * s->d * s->D);
    st->K = (double *)malloc(sizeof(double) * BK * cap * s->d + 1);
    st->V = (double *)malloc(sizeof(double) * BK * cap * s->d + 1);
    st->r = (double *)malloc(sizeof(double) * BK * cap + 1);
    st->kept = (int32_t *)malloc(sizeof(int32_t) * BK * cap + 1);
    st->nkept = (int *)calloc(BK, sizeof(int));
    st->S = (double *)calloc(BK * s->D * s->d, sizeof(double));
    st->z = (double *)calloc(BK * s->D, sizeof(double));
    if (!st->Wq || !st->Wk || !st->K || !st->V || !st->r || !st->kept || !st->nkept || !st->S ||
        !st->z) {
        od_decode_free(st);
        return NULL;
    }
    memcpy(st->Wq, Wq, sizeof(double) * (size_t)s->H * s->d * s->D);
    memcpy(st->Wk, Wk, sizeof(double) * (size_t)s->Hkv * s->d * s->D);
    return st;
}

int od_decode_pos(const od_decode *st) { return st->pos; }

/* q_t [B,H,d], k_t/v_t [B,Hkv,d] -> o_t [B,H,d]; r_t [B,Hkv] (nullable) gets the new token's score. */
int od_decode_step(od_decode *st, const double *q_t, const double *k_t, const double *v_t, double *o_t,
                   double *r_t)
{
    const od_dims *s = &st->s;
    int p = st->pos, d = s->d, D = s->D, C = s->C, G = s->H / s->Hkv, cap = s->N;
    if (p >= cap) return OD_EINVAL;
    int m = s->w / C, t = p / C;
    double *phi = (double *)malloc(sizeof(double) * D);
    double *num = (double *)malloc(sizeof(double) * d);
    int bad = 0;
    for (int b = 0; b < s->B; ++b) {
        for (int g = 0; g < s->Hkv; ++g) {
            size_t u = (size_t)b * s->Hkv + g;
            double *Kg = st->K + u * cap * d, *Vg = st->V + u * cap * d;
            memcpy(Kg + (size_t)p * d, k_t + u * d, sizeof(double) * d);
            memcpy(Vg + (size_t)p * d, v_t + u * d, sizeof(double) * d);
            double rsum = 0.0;
            for (int hh = 0; hh < G; ++hh) {
                int h = g * G + hh;
                const double *qi = q_t + ((size_t)b * s->H + h) * d;
                if (s->w >= 1) rsum += od_sigma_row(s, qi, Kg, p);
                /* softmax set: window and kept list */
                int lo = s->w == 0 ? p + 1 : (t - m) * C;
                if (lo < 0) lo = 0;
                double M = -INFINITY;
                for (int j = lo; j <= p; ++j) {
                    double l = od_logit(s, qi, Kg + (size_t)j * d);
                    M = l > M ? l : M;
                }
                for (int n = 0; n < st->nkept[u]; ++n) {
                    double l = od_logit(s, qi, Kg + (size_t)st->kept[u * cap + n] * d);
                    M = l > M ? l : M;
                }
                if (M == -INFINITY) M = 0.0;
                double den = 0.0;
                for (int x = 0; x < d; ++x) num[x] = 0.0;
                for (int j = lo; j <= p; ++j) {
                    double e = exp(od_logit(s, qi, Kg + (size_t)j * d) - M);
                    for (int x = 0; x < d; ++x) num[x] += e * Vg[(size_t)j * d + x];
                    den += e;
                }
                for (int n = 0; n < st->nkept[u]; ++n) {
                    int j = st->kept[u * cap + n];
                    double e = exp(od_logit(s, qi, Kg + (size_t)j * d) - M);
                    for (int x = 0; x < d; ++x) num[x] += e * Vg[(size_t)j * d + x];
                    den += e;
                }
                /* linear: folded state, plus the open chunk when there is no window */
                od_phi_row(d, D, qi, st->Wq + (size_t)h * d * D, phi);
                double sh = exp(-M);
                const double *S = st->S + u * D * d, *z = st->z + u * D;
                for (int a = 0; a < D; ++a) {
                    den += sh * phi[a] * z[a];
                    for (int x = 0; x < d; ++x) num[x] += sh * phi[a] * S[(size_t)a * d + x];
                }
                if (s->w == 0) {
                    double *pk = (double *)malloc(sizeof(double) * D);
                    for (int j = t * C; j <= p; ++j) {
                        od_phi_row(d, D, Kg + (size_t)j * d, st->Wk + (size_t)g * d * D, pk);
                        double wgt = 0.0;
                        for (int a = 0; a < D; ++a) wgt += phi[a] * pk[a];
                        wgt *= sh;
                        for (int x = 0; x < d; ++x) num[x] += wgt * Vg[(size_t)j * d + x];
                        den += wgt;
                    }
                    free(pk);
                }
                double *oi = o_t + ((size_t)b * s->H + h) * d;
                for (int x = 0; x < d; ++x) {
                    oi[x] = num[x] / den;
                    if (!isfinite(oi[x])) bad = 1;
                }
            }
            st->r[u * cap + p] = s->w >= 1 ? rsum / G : 0.0;
            if (r_t) r_t[u] = st->r[u * cap + p];
            /* chunk close: decide chunk t-m */
            if (p % C == C - 1 && t - m >= 0) {
                int c = t - m;
                int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (s->k + 1));
                if (s->k > 0) od_topk_chunk(st->r + u * cap + (size_t)c * C, C, s->k, sel);
                for (int n = 0; n < s->k; ++n) st->kept[u * cap + st->nkept[u]++] = c * C + sel[n];
                double *S = st->S + u * D * d, *z = st->z + u * D;
                for (int j = c * C; j < (c + 1) * C; ++j) {
                    int is_sel = 0;
                    for (int n = 0; n < s->k; ++n)
                        if (c * C + sel[n] == j) is_sel = 1;
                    if (is_sel) continue;
                    od_phi_row(d, D, Kg + (size_t)j * d, st->Wk + (size_t)g * d * D, phi);
                    for (int a = 0; a < D; ++a) {
                        z[a] += phi[a];
                        for (int x = 0; x < d; ++x) S[(size_t)a * d + x] += phi[a] * Vg[(size_t)j * d + x];
                    }
                }
                free(sel);
            }
        }
    }
    free(phi);
    free(num);
    st->pos = p + 1;
    return bad ? OD_ENONFINITE : OD_OK;
}
