/*
 * oracle.c -- plain, slow fp64 CPU oracle for blockwise softmax attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or
 * calls this file; only the test suite, the package smoke check and the CPU
 * baseline leg of the benchmark load it (through oracle/__init__.py).  It shares
 * no code, header, table or constant with the CUDA path.
 *
 * What it computes follows "上下文并行与 Ring Attention" (hs-black.github.io),
 * section 分块注意力 (online softmax 与 log-sum-exp 合并):
 *   - the attention output of one query against a key set is the plain softmax
 *     average  o = sum_j softmax(x)_j v_j  with  x_j = q.k_j / sqrt(d_h)
 *     (scale passed in by the caller);
 *   - the per-block statistics m_b = max x_j, l_b = sum e^{x_j - m_b},
 *     o_b = (1/l_b) sum e^{x_j - m_b} v_j, and lse_b = m_b + log l_b (natural log);
 *   - the merge of two partials, in the stable form given right after the boxed
 *     identity: M = max(lse_1, lse_2), lse = M + log(e^{lse_1-M} + e^{lse_2-M}),
 *     o = e^{lse_1-lse} o_1 + e^{lse_2-lse} o_2.
 * The causal mask is judged on original token positions (same page, sections
 * 因果掩码带来的负载不均 and 重排 token 的代价): key t is visible to query p iff
 * pos_k(t) <= pos_q(p).  The GQA head map is kv_head = q_head / (Hq / Hkv).
 *
 * Readings taken where the page is silent: a query that sees no key in the
 * given set gets o = 0 and lse = -inf; merging two such partials gives (0, -inf).
 *
 * Everything is scalar fp64, sequential summation in key order, no blocking and
 * no reordering; threads only split independent output rows.  The gradients of
 * the same section's backward paragraph follow at the end of the file.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Document of a position: the index of the last document start <= pos, with
 * doc_starts sorted ascending (section All-Gather 式 CP: several documents packed
 * into one sequence, keys of another document are invisible).  -1 before the
 * first start. */
static int64_t doc_of(const int64_t *doc_starts, int64_t n_docs, int64_t pos)
{
    int64_t lo = 0, hi = n_docs; /* first start > pos */
    while (lo < hi) {
        int64_t mid = (lo + hi) / 2;
        if (doc_starts[mid] <= pos) lo = mid + 1; else hi = mid;
    }
    return lo - 1;
}

/* One query row against all keys of one kv head.
 *   q      : d values of the query
 *   k, v   : key/value rows; row t starts at k + t * kv_row_stride
 *   pos_k  : original position of each key (NULL means t)
 *   docs   : document starts (NULL = one document); a key of another document is
 *            invisible
 *   x      : caller scratch of sk doubles
 * Writes d outputs to o and returns lse. */
static double attend_row(const double *q, int64_t pos_q, const double *k, const double *v,
                         const int64_t *pos_k, int64_t sk, int64_t kv_row_stride, int64_t d,
                         int causal, const int64_t *docs, int64_t n_docs, double scale, double *x,
                         double *o)
{
    double m = -INFINITY;
    int64_t nvis = 0;
    const int64_t dq = docs ? doc_of(docs, n_docs, pos_q) : 0;
    for (int64_t t = 0; t < sk; ++t) {
        int64_t pk = pos_k ? pos_k[t] : t;
        if (causal && pk > pos_q) { x[t] = NAN; continue; }
        if (docs && doc_of(docs, n_docs, pk) != dq) { x[t] = NAN; continue; }
        const double *kr = k + t * kv_row_stride;
        double dot = 0.0;
        for (int64_t e = 0; e < d; ++e) dot += q[e] * kr[e];
        x[t] = scale * dot;
        if (x[t] > m) m = x[t];
        ++nvis;
    }
    for (int64_t e = 0; e < d; ++e) o[e] = 0.0;
    if (nvis == 0) return -INFINITY;
    double l = 0.0;
    for (int64_t t = 0; t < sk; ++t) {
        if (isnan(x[t])) continue;
        double w = exp(x[t] - m);
        l += w;
        const double *vr = v + t * kv_row_stride;
        for (int64_t e = 0; e < d; ++e) o[e] += w * vr[e];
    }
    for (int64_t e = 0; e < d; ++e) o[e] /= l;
    return m + log(l);
}

/* ------------------------------------------------------------------ full problem */

typedef struct {
    const double *q, *k, *v;
    const int64_t *pos_q, *pos_k;
    int64_t b, sq, sk, hq, hkv, d;
    int causal;
    const int64_t *docs;
    int64_t n_docs;
    double scale;
    double *o, *lse;
    /* row selection (rows mode) */
    const int64_t *sel;  /* [n][3] = (batch, q head, query index) */
    const double *q_sel; /* [n][d] */
    int64_t nsel;
    /* work split */
    int64_t begin, end;
} job_t;

static void *full_worker(void *arg)
{
    job_t *j = (job_t *)arg;
    double *x = (double *)malloc(sizeof(double) * (size_t)(j->sk > 0 ? j->sk : 1));
    int64_t g = j->hq / j->hkv;
    for (int64_t r = j->begin; r < j->end; ++r) {
        /* r enumerates (batch, q head, query index) */
        int64_t s = r % j->sq;
        int64_t h = (r / j->sq) % j->hq;
        int64_t bb = r / (j->sq * j->hq);
        int64_t hk = h / g;
        const double *qr = j->q + ((bb * j->sq + s) * j->hq + h) * j->d;
        const double *kb = j->k + (bb * j->sk * j->hkv + hk) * j->d;
        const double *vb = j->v + (bb * j->sk * j->hkv + hk) * j->d;
        int64_t pq = j->pos_q ? j->pos_q[s] : s;
        double *orow = j->o + ((bb * j->sq + s) * j->hq + h) * j->d;
        j->lse[(bb * j->hq + h) * j->sq + s] =
            attend_row(qr, pq, kb, vb, j->pos_k, j->sk, j->hkv * j->d, j->d, j->causal, j->docs,
                       j->n_docs, j->scale, x, orow);
    }
    free(x);
    return NULL;
}

static void *rows_worker(void *arg)
{
    job_t *j = (job_t *)arg;
    double *x = (double *)malloc(sizeof(double) * (size_t)(j->sk > 0 ? j->sk : 1));
    int64_t g = j->hq / j->hkv;
    for (int64_t r = j->begin; r < j->end; ++r) {
        int64_t bb = j->sel[3 * r + 0], h = j->sel[3 * r + 1], pq = j->sel[3 * r + 2];
        int64_t hk = h / g;
        const double *kb = j->k + (bb * j->sk * j->hkv + hk) * j->d;
        const double *vb = j->v + (bb * j->sk * j->hkv + hk) * j->d;
        j->lse[r] = attend_row(j->q_sel + r * j->d, pq, kb, vb, j->pos_k, j->sk, j->hkv * j->d,
                               j->d, j->causal, j->docs, j->n_docs, j->scale, x, j->o + r * j->d);
    }
    free(x);
    return NULL;
}

static int run_jobs(job_t *proto, int64_t nrows, int nthreads, void *(*fn)(void *))
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 1024) nthreads = 1024;
    if (nrows < nthreads) nthreads = nrows > 0 ? (int)nrows : 1;
    pthread_t th[1024];
    job_t jobs[1024];
    int64_t per = (nrows + nthreads - 1) / nthreads;
    int started = 0;
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = *proto;
        jobs[t].begin = t * per < nrows ? t * per : nrows;
        jobs[t].end = (t + 1) * per < nrows ? (t + 1) * per : nrows;
        if (nthreads == 1) { fn(&jobs[t]); continue; }
        if (pthread_create(&th[t], NULL, fn, &jobs[t]) != 0) return -1;
        ++started;
    }
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    return 0;
}

/* Attention of every query row against every key.
 *   q [b, sq, hq, d], k/v [b, sk, hkv, d], o [b, sq, hq, d], lse [b, hq, sq]
 *   pos_q [sq] / pos_k [sk]: original token positions (NULL = identity).
 * Returns 0, or -1 on bad sizes / thread failure. */
int oracle_attention(const double *q, const double *k, const double *v, const int64_t *pos_q,
                     const int64_t *pos_k, int64_t b, int64_t sq, int64_t sk, int64_t hq,
                     int64_t hkv, int64_t d, int causal, double scale, double *o, double *lse,
                     int nthreads)
{
    if (b < 0 || sq < 0 || sk < 0 || hq <= 0 || hkv <= 0 || d <= 0 || hq % hkv) return -1;
    job_t j;
    memset(&j, 0, sizeof j);
    j.q = q; j.k = k; j.v = v; j.pos_q = pos_q; j.pos_k = pos_k;
    j.b = b; j.sq = sq; j.sk = sk; j.hq = hq; j.hkv = hkv; j.d = d;
    j.causal = causal; j.scale = scale; j.o = o; j.lse = lse;
    return run_jobs(&j, b * hq * sq, nthreads, full_worker);
}

/* Attention of selected query rows only (for sampled checks at full size).
 *   sel [n][3] = (batch, q head, original query position); q_sel [n][d]
 *   k/v [b, sk, hkv, d] with original key positions pos_k (NULL = identity)
 *   o_sel [n][d], lse_sel [n]. */
int oracle_attention_rows(const double *q_sel, const int64_t *sel, int64_t n, const double *k,
                          const double *v, const int64_t *pos_k, int64_t b, int64_t sk,
                          int64_t hq, int64_t hkv, int64_t d, int causal, double scale,
                          double *o_sel, double *lse_sel, int nthreads)
{
    if (n < 0 || b <= 0 || sk < 0 || hq <= 0 || hkv <= 0 || d <= 0 || hq % hkv) return -1;
    for (int64_t r = 0; r < n; ++r)
        if (sel[3 * r] < 0 || sel[3 * r] >= b || sel[3 * r + 1] < 0 || sel[3 * r + 1] >= hq)
            return -1;
    job_t j;
    memset(&j, 0, sizeof j);
    j.k = k; j.v = v; j.pos_k = pos_k;
    j.b = b; j.sk = sk; j.hq = hq; j.hkv = hkv; j.d = d;
    j.causal = causal; j.scale = scale; j.o = o_sel; j.lse = lse_sel;
    j.sel = sel; j.q_sel = q_sel; j.nsel = n;
    return run_jobs(&j, n, nthreads, rows_worker);
}

/* Attention with a document mask as well (section All-Gather 式 CP): doc_starts
 * [n_docs] sorted ascending, first entry 0; key t is visible to query p only if
 * both positions fall in the same document (and, causal, pos_k <= pos_q).
 * Otherwise as oracle_attention. */
int oracle_attention_doc(const double *q, const double *k, const double *v, const int64_t *pos_q,
                         const int64_t *pos_k, int64_t b, int64_t sq, int64_t sk, int64_t hq,
                         int64_t hkv, int64_t d, int causal, const int64_t *doc_starts,
                         int64_t n_docs, double scale, double *o, double *lse, int nthreads)
{
    if (b < 0 || sq < 0 || sk < 0 || hq <= 0 || hkv <= 0 || d <= 0 || hq % hkv) return -1;
    if (n_docs < 1 || !doc_starts || doc_starts[0] != 0) return -1;
    for (int64_t i = 1; i < n_docs; ++i)
        if (doc_starts[i] <= doc_starts[i - 1]) return -1;
    job_t j;
    memset(&j, 0, sizeof j);
    j.q = q; j.k = k; j.v = v; j.pos_q = pos_q; j.pos_k = pos_k;
    j.b = b; j.sq = sq; j.sk = sk; j.hq = hq; j.hkv = hkv; j.d = d;
    j.causal = causal; j.docs = doc_starts; j.n_docs = n_docs; j.scale = scale; j.o = o; j.lse = lse;
    return run_jobs(&j, b * hq * sq, nthreads, full_worker);
}

/* Selected rows with the document mask (see oracle_attention_rows). */
int oracle_attention_rows_doc(const double *q_sel, const int64_t *sel, int64_t n, const double *k,
                              const double *v, const int64_t *pos_k, int64_t b, int64_t sk,
                              int64_t hq, int64_t hkv, int64_t d, int causal,
                              const int64_t *doc_starts, int64_t n_docs, double scale,
                              double *o_sel, double *lse_sel, int nthreads)
{
    if (n < 0 || b <= 0 || sk < 0 || hq <= 0 || hkv <= 0 || d <= 0 || hq % hkv) return -1;
    if (n_docs < 1 || !doc_starts || doc_starts[0] != 0) return -1;
    for (int64_t r = 0; r < n; ++r)
        if (sel[3 * r] < 0 || sel[3 * r] >= b || sel[3 * r + 1] < 0 || sel[3 * r + 1] >= hq)
            return -1;
    job_t j;
    memset(&j, 0, sizeof j);
    j.k = k; j.v = v; j.pos_k = pos_k;
    j.b = b; j.sk = sk; j.hq = hq; j.hkv = hkv; j.d = d;
    j.causal = causal; j.docs = doc_starts; j.n_docs = n_docs; j.scale = scale;
    j.o = o_sel; j.lse = lse_sel;
    j.sel = sel; j.q_sel = q_sel; j.nsel = n;
    return run_jobs(&j, n, nthreads, rows_worker);
}

/* Merge of two partials (o_1, lse_1), (o_2, lse_2) for n rows of d values, stable form.
 * Both partials empty (lse = -inf) gives o = 0, lse = -inf. */
void oracle_lse_merge(int64_t n, int64_t d, const double *o1, const double *lse1, const double *o2,
                      const double *lse2, double *o, double *lse)
{
    for (int64_t r = 0; r < n; ++r) {
        double a = lse1[r], c = lse2[r];
        double M = a > c ? a : c;
        if (M == -INFINITY) {
            lse[r] = -INFINITY;
            for (int64_t e = 0; e < d; ++e) o[r * d + e] = 0.0;
            continue;
        }
        double L = M + log(exp(a - M) + exp(c - M));
        double w1 = exp(a - L), w2 = exp(c - L);
        for (int64_t e = 0; e < d; ++e) o[r * d + e] = w1 * o1[r * d + e] + w2 * o2[r * d + e];
        lse[r] = L;
    }
}

/* ------------------------------------------------------------------ backward
 *
 * Same page, last paragraph of section 分块注意力 (the backward pass needs only
 * the lse): with the GLOBAL lse of a query row, the softmax probability of a
 * visible key is p_j = e^{x_j - lse}, whichever block the key sits in, so every
 * key block yields its exact share of the gradients on its own:
 *   dv_j += p_j do,    dx_j = p_j (do . v_j - D),    D = do . o (one scalar per
 *   query row, also global),
 * and through x_j = scale q . k_j (chain rule):
 *   dq += scale dx_j k_j,    dk_j += scale dx_j q.
 * The statistics (lse, D) of each query row are either computed here from the
 * definition over the keys given (whole problem) or passed in (a block of keys
 * against the global statistics: one ring step's contribution).
 *
 * Rows with no visible key (lse = -inf) contribute nothing.  Sums run
 * sequentially: over keys in key order for dq, over (query head, query) in that
 * order for dk and dv; threads split independent output rows only.
 */

typedef struct {
    const double *q, *k, *v, *dout;
    const int64_t *pos_q, *pos_k;
    int64_t b, sq, sk, hq, hkv, d;
    int causal;
    double scale;
    const double *lse_in, *delta_in; /* [b, hq, sq] or NULL (compute them) */
    double *lse, *delta;             /* [b, hq, sq] statistics in use */
    const int64_t *min_pos;          /* [b * hq]: with the causal mask only rows at positions
                                        >= min_pos are needed, without it only heads whose
                                        entry is not INT64_MAX; NULL = every row */
    const int64_t *sel;              /* [n][3] selected rows, or NULL = every row */
    const int64_t *docs;             /* document starts (NULL = one document) */
    int64_t n_docs;
    double *dq;                      /* query pass: [b, sq, hq, d] or [n][d]; NULL = stats only */
    double *dk, *dv;                 /* key pass: [b, sk, hkv, d] or [n][d] */
    int64_t begin, end;
} bwd_job_t;

static double dotd(const double *a, const double *b, int64_t d)
{
    double s = 0.0;
    for (int64_t e = 0; e < d; ++e) s += a[e] * b[e];
    return s;
}

static const double *qrow_of(const bwd_job_t *j, const double *base, int64_t bb, int64_t i, int64_t h)
{
    return base + ((bb * j->sq + i) * j->hq + h) * j->d;
}

static const double *krow_of(const bwd_job_t *j, const double *base, int64_t bb, int64_t t, int64_t hk)
{
    return base + ((bb * j->sk + t) * j->hkv + hk) * j->d;
}

/* Query pass: statistics of the row, then (optionally) its dq. */
static void *bwd_query_worker(void *arg)
{
    bwd_job_t *j = (bwd_job_t *)arg;
    const int64_t d = j->d, g = j->hq / j->hkv;
    double *x = (double *)malloc(sizeof(double) * (size_t)(j->sk > 0 ? j->sk : 1));
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
    for (int64_t r = j->begin; r < j->end; ++r) {
        int64_t bb, h, i;
        if (j->sel) {
            bb = j->sel[3 * r + 0]; h = j->sel[3 * r + 1]; i = j->sel[3 * r + 2];
        } else {
            i = r % j->sq; h = (r / j->sq) % j->hq; bb = r / (j->sq * j->hq);
        }
        const int64_t hk = h / g;
        const int64_t pq = j->pos_q ? j->pos_q[i] : i;
        if (j->min_pos) {
            const int64_t mp = j->min_pos[bb * j->hq + h];
            if (mp == INT64_MAX || (j->causal && pq < mp)) continue;
        }
        const double *qi = qrow_of(j, j->q, bb, i, h);
        const double *doi = qrow_of(j, j->dout, bb, i, h);
        const int64_t srow = (bb * j->hq + h) * j->sq + i;
        double lse, D;
        if (j->lse_in) {
            lse = j->lse_in[srow];
            D = j->delta_in[srow];
        } else {
            lse = attend_row(qi, pq, krow_of(j, j->k, bb, 0, hk), krow_of(j, j->v, bb, 0, hk), j->pos_k,
                             j->sk, j->hkv * d, d, j->causal, j->docs, j->n_docs, j->scale, x, o);
            D = dotd(doi, o, d);
        }
        if (j->lse) { j->lse[srow] = lse; j->delta[srow] = D; }
        if (!j->dq) continue;
        double *dqi = j->sel ? j->dq + r * d : j->dq + ((bb * j->sq + i) * j->hq + h) * d;
        for (int64_t e = 0; e < d; ++e) dqi[e] = 0.0;
        if (lse == -INFINITY) continue;
        const int64_t dq_doc = j->docs ? doc_of(j->docs, j->n_docs, pq) : 0;
        for (int64_t t = 0; t < j->sk; ++t) {
            const int64_t pk = j->pos_k ? j->pos_k[t] : t;
            if (j->causal && pk > pq) continue;
            if (j->docs && doc_of(j->docs, j->n_docs, pk) != dq_doc) continue;
            const double *kt = krow_of(j, j->k, bb, t, hk);
            const double *vt = krow_of(j, j->v, bb, t, hk);
            const double p = exp(j->scale * dotd(qi, kt, d) - lse);
            const double dx = p * (dotd(doi, vt, d) - D);
            for (int64_t e = 0; e < d; ++e) dqi[e] += j->scale * dx * kt[e];
        }
    }
    free(o);
    free(x);
    return NULL;
}

/* Key pass: dk and dv of one key row, summed over the query heads of its group
 * and over every query row that sees it. */
static void *bwd_key_worker(void *arg)
{
    bwd_job_t *j = (bwd_job_t *)arg;
    const int64_t d = j->d, g = j->hq / j->hkv;
    for (int64_t r = j->begin; r < j->end; ++r) {
        int64_t bb, hk, t;
        if (j->sel) {
            bb = j->sel[3 * r + 0]; hk = j->sel[3 * r + 1]; t = j->sel[3 * r + 2];
        } else {
            t = r % j->sk; hk = (r / j->sk) % j->hkv; bb = r / (j->sk * j->hkv);
        }
        double *dkt = j->sel ? j->dk + r * d : j->dk + ((bb * j->sk + t) * j->hkv + hk) * d;
        double *dvt = j->sel ? j->dv + r * d : j->dv + ((bb * j->sk + t) * j->hkv + hk) * d;
        for (int64_t e = 0; e < d; ++e) { dkt[e] = 0.0; dvt[e] = 0.0; }
        const int64_t pk = j->pos_k ? j->pos_k[t] : t;
        const int64_t dk_doc = j->docs ? doc_of(j->docs, j->n_docs, pk) : 0;
        const double *kt = krow_of(j, j->k, bb, t, hk);
        const double *vt = krow_of(j, j->v, bb, t, hk);
        for (int64_t h = hk * g; h < (hk + 1) * g; ++h) {
            for (int64_t i = 0; i < j->sq; ++i) {
                const int64_t pq = j->pos_q ? j->pos_q[i] : i;
                if (j->causal && pk > pq) continue;
                if (j->docs && doc_of(j->docs, j->n_docs, pq) != dk_doc) continue;
                const int64_t srow = (bb * j->hq + h) * j->sq + i;
                const double lse = j->lse[srow], D = j->delta[srow];
                if (lse == -INFINITY) continue;
                const double *qi = qrow_of(j, j->q, bb, i, h);
                const double *doi = qrow_of(j, j->dout, bb, i, h);
                const double p = exp(j->scale * dotd(qi, kt, d) - lse);
                const double dx = p * (dotd(doi, vt, d) - D);
                for (int64_t e = 0; e < d; ++e) {
                    dvt[e] += p * doi[e];
                    dkt[e] += j->scale * dx * qi[e];
                }
            }
        }
    }
    return NULL;
}

static int run_bwd_jobs(const bwd_job_t *proto, int64_t nrows, int nthreads, void *(*fn)(void *))
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 1024) nthreads = 1024;
    if (nrows < nthreads) nthreads = nrows > 0 ? (int)nrows : 1;
    pthread_t th[1024];
    bwd_job_t *jobs = (bwd_job_t *)malloc(sizeof(bwd_job_t) * (size_t)nthreads);
    if (!jobs) return -1;
    int64_t per = (nrows + nthreads - 1) / nthreads;
    int started = 0, rc = 0;
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = *proto;
        jobs[t].begin = t * per < nrows ? t * per : nrows;
        jobs[t].end = (t + 1) * per < nrows ? (t + 1) * per : nrows;
        if (nthreads == 1) { fn(&jobs[t]); continue; }
        if (pthread_create(&th[t], NULL, fn, &jobs[t]) != 0) { rc = -1; break; }
        ++started;
    }
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    free(jobs);
    return rc;
}

static int bwd_dims_ok(int64_t b, int64_t sq, int64_t sk, int64_t hq, int64_t hkv, int64_t d)
{
    return b >= 0 && sq >= 0 && sk >= 0 && hq > 0 && hkv > 0 && d > 0 && hq % hkv == 0;
}

/* Gradients of every input.
 *   q, dout [b, sq, hq, d]; k, v [b, sk, hkv, d]; pos_q [sq] / pos_k [sk] (NULL = identity)
 *   lse_in, delta_in [b, hq, sq]: the rows' global statistics, or both NULL to
 *     compute them from the definition over these keys;
 *   dq [b, sq, hq, d], dk, dv [b, sk, hkv, d] are overwritten;
 *   lse_out, delta_out [b, hq, sq] (may be NULL) receive the statistics used.
 * Returns 0, or -1 on bad sizes / allocation or thread failure. */
static int attention_bwd_impl(const double *q, const double *k, const double *v, const double *dout,
                              const int64_t *pos_q, const int64_t *pos_k, int64_t b, int64_t sq, int64_t sk,
                              int64_t hq, int64_t hkv, int64_t d, int causal, const int64_t *docs,
                              int64_t n_docs, double scale, const double *lse_in, const double *delta_in,
                              double *dq, double *dk, double *dv, double *lse_out, double *delta_out,
                              int nthreads)
{
    if (!bwd_dims_ok(b, sq, sk, hq, hkv, d) || (!lse_in) != (!delta_in)) return -1;
    const int64_t nstat = b * hq * sq;
    double *lse = lse_out, *delta = delta_out, *own = NULL;
    if (!lse || !delta) {
        own = (double *)malloc(sizeof(double) * (size_t)(2 * nstat + 1));
        if (!own) return -1;
        lse = own;
        delta = own + nstat;
    }
    bwd_job_t j;
    memset(&j, 0, sizeof j);
    j.q = q; j.k = k; j.v = v; j.dout = dout; j.pos_q = pos_q; j.pos_k = pos_k;
    j.b = b; j.sq = sq; j.sk = sk; j.hq = hq; j.hkv = hkv; j.d = d;
    j.causal = causal; j.scale = scale; j.lse_in = lse_in; j.delta_in = delta_in;
    j.docs = docs; j.n_docs = n_docs;
    j.lse = lse; j.delta = delta; j.dq = dq; j.dk = dk; j.dv = dv;
    int rc = run_bwd_jobs(&j, nstat, nthreads, bwd_query_worker);
    if (rc == 0) rc = run_bwd_jobs(&j, b * hkv * sk, nthreads, bwd_key_worker);
    free(own);
    return rc;
}

int oracle_attention_bwd(const double *q, const double *k, const double *v, const double *dout,
                         const int64_t *pos_q, const int64_t *pos_k, int64_t b, int64_t sq, int64_t sk,
                         int64_t hq, int64_t hkv, int64_t d, int causal, double scale,
                         const double *lse_in, const double *delta_in, double *dq, double *dk,
                         double *dv, double *lse_out, double *delta_out, int nthreads)
{
    return attention_bwd_impl(q, k, v, dout, pos_q, pos_k, b, sq, sk, hq, hkv, d, causal, NULL, 0, scale,
                              lse_in, delta_in, dq, dk, dv, lse_out, delta_out, nthreads);
}

/* oracle_attention_bwd with the document mask of oracle_attention_doc (section
 * All-Gather 式 CP): a key of another document than the query contributes nothing. */
int oracle_attention_bwd_doc(const double *q, const double *k, const double *v, const double *dout,
                             const int64_t *pos_q, const int64_t *pos_k, int64_t b, int64_t sq, int64_t sk,
                             int64_t hq, int64_t hkv, int64_t d, int causal, const int64_t *doc_starts,
                             int64_t n_docs, double scale, double *dq, double *dk, double *dv, int nthreads)
{
    if (n_docs < 1 || !doc_starts || doc_starts[0] != 0) return -1;
    for (int64_t i = 1; i < n_docs; ++i)
        if (doc_starts[i] <= doc_starts[i - 1]) return -1;
    return attention_bwd_impl(q, k, v, dout, pos_q, pos_k, b, sq, sk, hq, hkv, d, causal, doc_starts, n_docs,
                              scale, NULL, NULL, dq, dk, dv, NULL, NULL, nthreads);
}

/* Gradients at selected rows only (for sampled checks at full size).
 *   sel_q [nq][3] = (batch, q head, query index) -> dq_sel [nq][d]
 *   sel_k [nk][3] = (batch, kv head, key index)  -> dk_sel, dv_sel [nk][d]
 * The statistics are computed from the definition: per selected query row, and
 * for every query row that may see a selected key row (same batch, a query head
 * of the key's group, and with the causal mask a position at or after the key). */
int oracle_attention_bwd_sel(const double *q, const double *k, const double *v, const double *dout,
                             const int64_t *pos_q, const int64_t *pos_k, int64_t b, int64_t sq,
                             int64_t sk, int64_t hq, int64_t hkv, int64_t d, int causal, double scale,
                             const int64_t *sel_q, int64_t nq, double *dq_sel, const int64_t *sel_k,
                             int64_t nk, double *dk_sel, double *dv_sel, int nthreads)
{
    if (!bwd_dims_ok(b, sq, sk, hq, hkv, d) || nq < 0 || nk < 0) return -1;
    const int64_t g = hq / hkv;
    for (int64_t r = 0; r < nq; ++r)
        if (sel_q[3 * r] < 0 || sel_q[3 * r] >= b || sel_q[3 * r + 1] < 0 || sel_q[3 * r + 1] >= hq ||
            sel_q[3 * r + 2] < 0 || sel_q[3 * r + 2] >= sq)
            return -1;
    for (int64_t r = 0; r < nk; ++r)
        if (sel_k[3 * r] < 0 || sel_k[3 * r] >= b || sel_k[3 * r + 1] < 0 || sel_k[3 * r + 1] >= hkv ||
            sel_k[3 * r + 2] < 0 || sel_k[3 * r + 2] >= sk)
            return -1;
    bwd_job_t j;
    memset(&j, 0, sizeof j);
    j.q = q; j.k = k; j.v = v; j.dout = dout; j.pos_q = pos_q; j.pos_k = pos_k;
    j.b = b; j.sq = sq; j.sk = sk; j.hq = hq; j.hkv = hkv; j.d = d;
    j.causal = causal; j.scale = scale;
    int rc = 0;
    if (nq > 0) {
        bwd_job_t jq = j;
        jq.sel = sel_q;
        jq.dq = dq_sel;
        rc = run_bwd_jobs(&jq, nq, nthreads, bwd_query_worker);
    }
    if (rc == 0 && nk > 0) {
        const int64_t nstat = b * hq * sq;
        double *stats = (double *)malloc(sizeof(double) * (size_t)(2 * nstat + 1));
        int64_t *minp = (int64_t *)malloc(sizeof(int64_t) * (size_t)(b * hq + 1));
        if (!stats || !minp) { free(stats); free(minp); return -1; }
        for (int64_t x = 0; x < b * hq; ++x) minp[x] = INT64_MAX;
        for (int64_t r = 0; r < nk; ++r) {
            const int64_t t = sel_k[3 * r + 2];
            const int64_t pk = pos_k ? pos_k[t] : t;
            for (int64_t h = sel_k[3 * r + 1] * g; h < (sel_k[3 * r + 1] + 1) * g; ++h)
                if (pk < minp[sel_k[3 * r] * hq + h]) minp[sel_k[3 * r] * hq + h] = pk;
        }
        bwd_job_t js = j;
        js.lse = stats;
        js.delta = stats + nstat;
        js.min_pos = minp;
        rc = run_bwd_jobs(&js, nstat, nthreads, bwd_query_worker);
        if (rc == 0) {
            bwd_job_t jk = j;
            jk.lse = stats;
            jk.delta = stats + nstat;
            jk.sel = sel_k;
            jk.dk = dk_sel;
            jk.dv = dv_sel;
            rc = run_bwd_jobs(&jk, nk, nthreads, bwd_key_worker);
        }
        free(minp);
        free(stats);
    }
    return rc;
}
