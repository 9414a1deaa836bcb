/*
 * Attention-KL oracle: a plain, slow, fp64 CPU implementation of the
 * attention-distillation KL divergence and its gradients.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this library.  It shares no code, header, table or
 * helper with the CUDA path, and nothing here is derived from that path.
 *
 * What it computes (sources, cited by page title and section):
 *  - "StreamKL: Fast and Memory-Efficient KL Divergence for Boosting Attention
 *    Distillation", abstract: one attention distribution is trained to match
 *    another by minimising their KL divergence; the existing approach
 *    materialises both distributions and then reduces.  This file IS that
 *    materialised approach, one query row at a time.
 *  - "Lecture 05 - Where It All Lands ...", section 1 (the identity as a
 *    toolkit) and section 3.1 (forward KL at temperature T): D_KL(p||q) =
 *    sum_v p(v) (log p(v) - log q(v)), teacher p in the first slot.
 *
 * For every (b, h, i):
 *   s_t[j] = scale_t * <Q_t[i], K_t[j]>,  s_s[j] = scale_s * <Q_s[i], K_s[j]>
 *   over the visible keys j (all keys, or j <= i + N_K - N_Q when causal);
 *   LSE = max + log(sum exp(s - max)); logP = s_t - LSE_t; logQ = s_s - LSE_s;
 *   KL_i = sum_j exp(logP_j) * (logP_j - logQ_j).
 * Backward with the per-row upstream gradient g_i (chain rule through the two
 * softmaxes; derivation in the design notes):
 *   dS_s[j] = g_i * (Q_j - P_j)
 *   dS_t[j] = g_i * P_j * (logP_j - logQ_j - KL_i)
 *   dQ_s[i] = scale_s * sum_j dS_s[j] K_s[j],  dK_s[j] += scale_s * dS_s[j] Q_s[i]
 *   and the same for the teacher with scale_t.
 *
 * Two variants of the visible set and of the key heads (readings of the
 * abstract's use cases, sparse-attention training and long-context
 * distillation, which need padded batches and grouped key heads; the pages
 * give no formula for either, so these are the plain readings):
 *  - padding: with per-batch key lengths kv_len[b] (NULL = all N_K keys), key
 *    j is visible to row i iff it is visible under the mask above AND
 *    j < kv_len[b] (lengths outside [0, N_K] are clamped to it).  A row with no
 *    visible key has KL = 0, LSE = -inf and no gradient (the empty sums).
 *  - grouped key heads: K_t has H_kt heads and K_s has H_ks heads, each
 *    dividing H; query head h of batch b reads key head h / (H / H_k) of the
 *    same batch, and a key head's gradient is the sum over its query heads.
 *
 * Layouts: row-major [B, H, N_Q, d] queries and [B, H_k, N_K, d] keys in
 * doubles; per-row outputs [B, H, N_Q].
 * Threads split the query rows; each thread keeps private dK accumulators that
 * are summed in thread order at the end (so a fixed thread count gives a fixed
 * result).  Return value 0 = ok, nonzero = bad arguments / out of memory.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    const double *q_t, *k_t, *q_s, *k_s;
    int B, H, N_Q, N_K, d_t, d_s, causal;
    int H_kt, H_ks;                   /* key heads of the teacher / student */
    const int *kv_len;                /* per-batch key lengths, or NULL */
    double scale_t, scale_s;
    /* forward outputs (may be NULL) */
    double *kl, *lse_t, *lse_s;
    /* backward: per-row upstream gradient (NULL = forward only) */
    const double *g;
    double *dq_s, *dq_t;              /* indexed like the inputs */
    double *dk_s_priv, *dk_t_priv;    /* this thread's private [B,H_k,N_K,d] */
    /* the rows this worker owns: flat ids r = (b*H + h)*N_Q + i */
    const int64_t *rows;              /* NULL = contiguous range */
    int64_t r_begin, r_end;
} work_t;

static int num_visible(int i, int N_Q, int N_K, int causal)
{
    if (!causal) return N_K;
    int last = i + (N_K - N_Q);          /* bottom-right aligned diagonal */
    int n = last + 1;
    if (n < 0) n = 0;
    if (n > N_K) n = N_K;
    return n;
}

/* Visible keys of row i of batch b: a prefix [0, n) of the keys. */
static int row_visible(const work_t *w, int b, int i)
{
    int n = num_visible(i, w->N_Q, w->N_K, w->causal);
    if (w->kv_len) {
        int len = w->kv_len[b];
        if (len < 0) len = 0;
        if (len > w->N_K) len = w->N_K;
        if (len < n) n = len;
    }
    return n;
}

static double dot(const double *a, const double *b, int d)
{
    double s = 0.0;
    for (int k = 0; k < d; ++k) s += a[k] * b[k];
    return s;
}

static double log_sum_exp(const double *s, int n)
{
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) if (s[j] > m) m = s[j];
    double acc = 0.0;
    for (int j = 0; j < n; ++j) acc += exp(s[j] - m);
    return m + log(acc);
}

/* One query row: materialise both logit rows, both log-softmaxes, the KL,
 * and (if asked) the row's dQ and its contribution to dK. */
static void one_row(const work_t *w, int64_t r, double *s_t, double *s_s)
{
    const int N_Q = w->N_Q, N_K = w->N_K, d_t = w->d_t, d_s = w->d_s;
    const int64_t bh = r / N_Q;
    const int i = (int)(r % N_Q);
    const int b = (int)(bh / w->H), h = (int)(bh % w->H);
    /* the key heads this query head reads */
    const int64_t kht = (int64_t)b * w->H_kt + h / (w->H / w->H_kt);
    const int64_t khs = (int64_t)b * w->H_ks + h / (w->H / w->H_ks);
    const double *qt = w->q_t + (bh * N_Q + i) * d_t;
    const double *qs = w->q_s + (bh * N_Q + i) * d_s;
    const double *kt = w->k_t + kht * (int64_t)N_K * d_t;
    const double *ks = w->k_s + khs * (int64_t)N_K * d_s;
    const int n = row_visible(w, b, i);

    for (int j = 0; j < n; ++j) {
        s_t[j] = w->scale_t * dot(qt, kt + (int64_t)j * d_t, d_t);
        s_s[j] = w->scale_s * dot(qs, ks + (int64_t)j * d_s, d_s);
    }
    const double lse_t = log_sum_exp(s_t, n);
    const double lse_s = log_sum_exp(s_s, n);
    double kl = 0.0;
    for (int j = 0; j < n; ++j) {
        const double logp = s_t[j] - lse_t, logq = s_s[j] - lse_s;
        kl += exp(logp) * (logp - logq);
    }
    if (w->kl) w->kl[r] = kl;
    if (w->lse_t) w->lse_t[r] = lse_t;
    if (w->lse_s) w->lse_s[r] = lse_s;
    if (!w->g) return;

    const double g = w->g[r];
    double *dqs = w->dq_s ? w->dq_s + (bh * N_Q + i) * d_s : NULL;
    double *dqt = w->dq_t ? w->dq_t + (bh * N_Q + i) * d_t : NULL;
    if (dqs) memset(dqs, 0, sizeof(double) * d_s);
    if (dqt) memset(dqt, 0, sizeof(double) * d_t);
    double *dks = w->dk_s_priv ? w->dk_s_priv + khs * (int64_t)N_K * d_s : NULL;
    double *dkt = w->dk_t_priv ? w->dk_t_priv + kht * (int64_t)N_K * d_t : NULL;
    for (int j = 0; j < n; ++j) {
        const double logp = s_t[j] - lse_t, logq = s_s[j] - lse_s;
        const double p = exp(logp), q = exp(logq);
        const double ds_s = g * (q - p);
        const double ds_t = g * p * (logp - logq - kl);
        if (dqs) for (int k = 0; k < d_s; ++k) dqs[k] += w->scale_s * ds_s * ks[(int64_t)j * d_s + k];
        if (dks) for (int k = 0; k < d_s; ++k) dks[(int64_t)j * d_s + k] += w->scale_s * ds_s * qs[k];
        if (dqt) for (int k = 0; k < d_t; ++k) dqt[k] += w->scale_t * ds_t * kt[(int64_t)j * d_t + k];
        if (dkt) for (int k = 0; k < d_t; ++k) dkt[(int64_t)j * d_t + k] += w->scale_t * ds_t * qt[k];
    }
}

static void *worker(void *arg)
{
    work_t *w = (work_t *)arg;
    double *s_t = (double *)malloc(sizeof(double) * (size_t)(w->N_K > 0 ? w->N_K : 1));
    double *s_s = (double *)malloc(sizeof(double) * (size_t)(w->N_K > 0 ? w->N_K : 1));
    if (s_t && s_s)
        for (int64_t k = w->r_begin; k < w->r_end; ++k)
            one_row(w, w->rows ? w->rows[k] : k, s_t, s_s);
    free(s_t);
    free(s_s);
    return NULL;
}

static int pick_threads(int nthreads, int64_t nrows)
{
    if (nthreads <= 0) {
        long c = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = c > 0 ? (int)c : 1;
    }
    if (nthreads > 256) nthreads = 256;
    if (nrows < nthreads) nthreads = nrows > 0 ? (int)nrows : 1;
    return nthreads;
}

static int check_shape(int B, int H, int N_Q, int N_K, int d_t, int d_s, int causal, int H_kt, int H_ks)
{
    if (B < 0 || H < 0 || N_Q < 0 || N_K < 0 || d_t <= 0 || d_s <= 0) return 1;
    if (H_kt <= 0 || H_ks <= 0 || (H > 0 && (H % H_kt || H % H_ks))) return 1;
    if (causal && N_Q > N_K) return 1;     /* would leave rows with no visible key */
    if (!causal && N_K == 0 && N_Q > 0) return 1;
    return 0;
}

/* Runs rows [0, nrows) (or the listed rows) over nthreads workers.  When
 * dK is wanted, each worker gets private accumulators, summed in order. */
static int run(work_t proto, int64_t nrows, int nthreads, double *dk_s, double *dk_t)
{
    const int T = pick_threads(nthreads, nrows);
    const int64_t nk_s = (int64_t)proto.B * proto.H_ks * proto.N_K * proto.d_s;
    const int64_t nk_t = (int64_t)proto.B * proto.H_kt * proto.N_K * proto.d_t;
    work_t *ws = (work_t *)calloc((size_t)T, sizeof(work_t));
    pthread_t *th = (pthread_t *)calloc((size_t)T, sizeof(pthread_t));
    if (!ws || !th) { free(ws); free(th); return 2; }
    int err = 0;
    for (int t = 0; t < T; ++t) {
        ws[t] = proto;
        ws[t].r_begin = nrows * t / T;
        ws[t].r_end = nrows * (t + 1) / T;
        ws[t].dk_s_priv = ws[t].dk_t_priv = NULL;
        if (dk_s) { ws[t].dk_s_priv = (double *)calloc((size_t)nk_s, sizeof(double)); if (!ws[t].dk_s_priv) err = 2; }
        if (dk_t) { ws[t].dk_t_priv = (double *)calloc((size_t)nk_t, sizeof(double)); if (!ws[t].dk_t_priv) err = 2; }
    }
    if (!err) {
        for (int t = 0; t < T; ++t) pthread_create(&th[t], NULL, worker, &ws[t]);
        for (int t = 0; t < T; ++t) pthread_join(th[t], NULL);
        if (dk_s) { memset(dk_s, 0, sizeof(double) * (size_t)nk_s);
            for (int t = 0; t < T; ++t) for (int64_t e = 0; e < nk_s; ++e) dk_s[e] += ws[t].dk_s_priv[e]; }
        if (dk_t) { memset(dk_t, 0, sizeof(double) * (size_t)nk_t);
            for (int t = 0; t < T; ++t) for (int64_t e = 0; e < nk_t; ++e) dk_t[e] += ws[t].dk_t_priv[e]; }
    }
    for (int t = 0; t < T; ++t) { free(ws[t].dk_s_priv); free(ws[t].dk_t_priv); }
    free(ws);
    free(th);
    return err;
}

/* Forward: per-row KL and both log-sum-exps.  K_t, K_s have H_kt, H_ks
 * heads; kv_len (per batch, nullable) hides padding keys. */
int streamkl_oracle_fwd(const double *q_t, const double *k_t, const double *q_s, const double *k_s,
                        int B, int H, int N_Q, int N_K, int d_t, int d_s,
                        double scale_t, double scale_s, int causal,
                        int H_kt, int H_ks, const int *kv_len,
                        double *kl, double *lse_t, double *lse_s, int nthreads)
{
    if (check_shape(B, H, N_Q, N_K, d_t, d_s, causal, H_kt, H_ks)) return 1;
    work_t w;
    memset(&w, 0, sizeof w);
    w.q_t = q_t; w.k_t = k_t; w.q_s = q_s; w.k_s = k_s;
    w.B = B; w.H = H; w.N_Q = N_Q; w.N_K = N_K; w.d_t = d_t; w.d_s = d_s; w.causal = causal;
    w.H_kt = H_kt; w.H_ks = H_ks; w.kv_len = kv_len;
    w.scale_t = scale_t; w.scale_s = scale_s;
    w.kl = kl; w.lse_t = lse_t; w.lse_s = lse_s;
    return run(w, (int64_t)B * H * N_Q, nthreads, NULL, NULL);
}

/* Backward: all four gradients for the per-row upstream gradient g
 * ([B,H,N_Q]); any output pointer may be NULL to skip it.  KL and the LSEs
 * are recomputed here, from the inputs alone. */
int streamkl_oracle_bwd(const double *q_t, const double *k_t, const double *q_s, const double *k_s,
                        int B, int H, int N_Q, int N_K, int d_t, int d_s,
                        double scale_t, double scale_s, int causal,
                        int H_kt, int H_ks, const int *kv_len, const double *g,
                        double *dq_s, double *dk_s, double *dq_t, double *dk_t, int nthreads)
{
    if (check_shape(B, H, N_Q, N_K, d_t, d_s, causal, H_kt, H_ks) || !g) return 1;
    work_t w;
    memset(&w, 0, sizeof w);
    w.q_t = q_t; w.k_t = k_t; w.q_s = q_s; w.k_s = k_s;
    w.B = B; w.H = H; w.N_Q = N_Q; w.N_K = N_K; w.d_t = d_t; w.d_s = d_s; w.causal = causal;
    w.H_kt = H_kt; w.H_ks = H_ks; w.kv_len = kv_len;
    w.scale_t = scale_t; w.scale_s = scale_s;
    w.g = g; w.dq_s = dq_s; w.dq_t = dq_t;
    return run(w, (int64_t)B * H * N_Q, nthreads, dk_s, dk_t);
}

/* Selected rows only (flat ids r = (b*H + h)*N_Q + i): KL, LSEs and, if g is
 * given, the rows' dQ.  Outputs are indexed like the full tensors, so a caller
 * passes full-size buffers and reads back the listed rows. */
int streamkl_oracle_rows(const double *q_t, const double *k_t, const double *q_s, const double *k_s,
                         int B, int H, int N_Q, int N_K, int d_t, int d_s,
                         double scale_t, double scale_s, int causal,
                        int H_kt, int H_ks, const int *kv_len,
                         const int64_t *rows, int64_t n_rows, const double *g,
                         double *kl, double *lse_t, double *lse_s,
                         double *dq_s, double *dq_t, int nthreads)
{
    if (check_shape(B, H, N_Q, N_K, d_t, d_s, causal, H_kt, H_ks)) return 1;
    for (int64_t k = 0; k < n_rows; ++k)
        if (rows[k] < 0 || rows[k] >= (int64_t)B * H * N_Q) return 1;
    work_t w;
    memset(&w, 0, sizeof w);
    w.q_t = q_t; w.k_t = k_t; w.q_s = q_s; w.k_s = k_s;
    w.B = B; w.H = H; w.N_Q = N_Q; w.N_K = N_K; w.d_t = d_t; w.d_s = d_s; w.causal = causal;
    w.H_kt = H_kt; w.H_ks = H_ks; w.kv_len = kv_len;
    w.scale_t = scale_t; w.scale_s = scale_s;
    w.kl = kl; w.lse_t = lse_t; w.lse_s = lse_s;
    w.g = g; w.dq_s = dq_s; w.dq_t = dq_t;
    w.rows = rows;
    return run(w, n_rows, nthreads, NULL, NULL);
}

/* Backward restricted to the listed rows: their dQ rows and their
 * contributions to dK (the dK of the rows not listed is left out).  Used to
 * time the oracle on a bounded sample of a large problem. */
int streamkl_oracle_bwd_rows(const double *q_t, const double *k_t, const double *q_s, const double *k_s,
                             int B, int H, int N_Q, int N_K, int d_t, int d_s,
                             double scale_t, double scale_s, int causal,
                        int H_kt, int H_ks, const int *kv_len, const double *g,
                             const int64_t *rows, int64_t n_rows,
                             double *dq_s, double *dk_s, double *dq_t, double *dk_t, int nthreads)
{
    if (check_shape(B, H, N_Q, N_K, d_t, d_s, causal, H_kt, H_ks) || !g) return 1;
    for (int64_t k = 0; k < n_rows; ++k)
        if (rows[k] < 0 || rows[k] >= (int64_t)B * H * N_Q) return 1;
    work_t w;
    memset(&w, 0, sizeof w);
    w.q_t = q_t; w.k_t = k_t; w.q_s = q_s; w.k_s = k_s;
    w.B = B; w.H = H; w.N_Q = N_Q; w.N_K = N_K; w.d_t = d_t; w.d_s = d_s; w.causal = causal;
    w.H_kt = H_kt; w.H_ks = H_ks; w.kv_len = kv_len;
    w.scale_t = scale_t; w.scale_s = scale_s;
    w.g = g; w.dq_s = dq_s; w.dq_t = dq_t;
    w.rows = rows;
    return run(w, n_rows, nthreads, dk_s, dk_t);
}

/* Mean of the per-row KL over every (b, h, i) row. */
double streamkl_oracle_mean(const double *kl, int64_t n)
{
    double s = 0.0;
    for (int64_t k = 0; k < n; ++k) s += kl[k];
    return n > 0 ? s / (double)n : 0.0;
}
