/*
 * KATA causal forward: fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file; only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, table or
 * constant with the CUDA library.
 *
 * What it computes (per head, rows t = 0..T-1), written out as defined:
 *
 *     w_ts = (q_t . k_s)^2                               for s <= t
 *     y_t  = sum_{s<=t} w_ts v_s  /  sum_{s<=t} w_ts      (y_t = 0 if the sum is 0)
 *
 * Sources (page title, section):
 *   - "Kernelized Linear Attention: Breaking the Capacity Wall with Symmetric
 *     Cones" (gist.science summary), Technical summary 2.2, rank-one PSD cone:
 *     the feature is psi(u) = u u^T, whose inner product squares the raw
 *     inner product, <psi(q), psi(k)> = (q.k)^2.
 *   - same page, 2.1, output gating: the normalised denominator acts as a
 *     convex gate between the previous readout and the current value, so the
 *     current token is included (s <= t) and the output is the weighted mean.
 *   - same title, arXiv abstract (fugumt page): "rank-one positive
 *     semi-definite features", "parameter-free convex output gate", "exact
 *     O(T) chunked-state form", "constant-time recurrent inference".
 *
 * Readings where the pages are silent (each is also listed in the design
 * notes): no scale constant (the ratio is invariant to q -> a q, k -> b k);
 * no epsilon in the denominator; a zero denominator gives y = 0.
 *
 * Parity pins: every function here is checked by tests/test_oracle_pins.py
 * against exact rational brute force, closed forms and invariants.
 *
 * Layout of every array: row-major [BH][T][d] (q, k: d = dk; v, y: d = dv).
 * The state is S[BH][dk*dk][dv] with row index i*dk + j, and Z[BH][dk][dk].
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Work splitting over (head, row) items with plain pthreads.          */
/* ------------------------------------------------------------------ */

typedef struct {
    void (*fn)(void *ctx, long item);
    void *ctx;
    long n_items;
    long next;
    pthread_mutex_t lock;
} work_pool;

static void *pool_worker(void *arg) {
    work_pool *p = (work_pool *)arg;
    for (;;) {
        long item;
        pthread_mutex_lock(&p->lock);
        item = p->next++;
        pthread_mutex_unlock(&p->lock);
        if (item >= p->n_items) break;
        p->fn(p->ctx, item);
    }
    return NULL;
}

static void run_items(void (*fn)(void *, long), void *ctx, long n_items, int nthreads) {
    work_pool p;
    p.fn = fn;
    p.ctx = ctx;
    p.n_items = n_items;
    p.next = 0;
    pthread_mutex_init(&p.lock, NULL);
    if (nthreads <= 1 || n_items <= 1) {
        pool_worker(&p);
    } else {
        if (nthreads > 256) nthreads = 256;
        pthread_t th[256];
        for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, pool_worker, &p);
        for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    }
    pthread_mutex_destroy(&p.lock);
}

/* ------------------------------------------------------------------ */
/* One output row from the quadratic definition.                       */
/* ------------------------------------------------------------------ */

/* y_t for head `bh`, row t: the weighted mean of v_0..v_t with weights
 * (q_t . k_s)^2 (gist.science summary 2.2 for the weight, 2.1 for the
 * normalisation).  Returns the denominator. */
static double quadratic_row(const double *q, const double *k, const double *v,
                            long T, int dk, int dv, long bh, long t, double *y) {
    const double *qt = q + (bh * T + t) * dk;
    double den = 0.0;
    for (int e = 0; e < dv; ++e) y[e] = 0.0;
    for (long s = 0; s <= t; ++s) {
        const double *ks = k + (bh * T + s) * dk;
        const double *vs = v + (bh * T + s) * dv;
        double dot = 0.0;
        for (int i = 0; i < dk; ++i) dot += qt[i] * ks[i];
        double w = dot * dot;
        den += w;
        for (int e = 0; e < dv; ++e) y[e] += w * vs[e];
    }
    if (den == 0.0) {
        for (int e = 0; e < dv; ++e) y[e] = 0.0;
    } else {
        for (int e = 0; e < dv; ++e) y[e] /= den;
    }
    return den;
}

typedef struct {
    const double *q, *k, *v;
    double *y, *den;
    long T;
    int dk, dv;
    const long *bh_idx, *t_idx; /* NULL: every row, item = bh*T + t */
} rows_ctx;

static void rows_item(void *c, long item) {
    rows_ctx *x = (rows_ctx *)c;
    long bh, t;
    if (x->bh_idx) {
        bh = x->bh_idx[item];
        t = x->t_idx[item];
    } else {
        bh = item / x->T;
        t = item % x->T;
    }
    double d = quadratic_row(x->q, x->k, x->v, x->T, x->dk, x->dv, bh, t, x->y + item * x->dv);
    if (x->den) x->den[item] = d;
}

/* Every row of every head.  y: [BH][T][dv]; den (nullable): [BH][T]. */
void kata_oracle_forward(const double *q, const double *k, const double *v, double *y,
                         double *den, long BH, long T, int dk, int dv, int nthreads) {
    rows_ctx c = {q, k, v, y, den, T, dk, dv, NULL, NULL};
    run_items(rows_item, &c, BH * T, nthreads);
}

/* Selected rows (bh_idx[r], t_idx[r]) only; y: [nrows][dv]; den: [nrows]. */
void kata_oracle_forward_rows(const double *q, const double *k, const double *v, long T,
                              int dk, int dv, const long *bh_idx, const long *t_idx,
                              long nrows, double *y, double *den, int nthreads) {
    rows_ctx c = {q, k, v, y, den, T, dk, dv, bh_idx, t_idx};
    run_items(rows_item, &c, nrows, nthreads);
}

/* ------------------------------------------------------------------ */
/* State by direct summation (the recurrent-inference state).          */
/* ------------------------------------------------------------------ */

/* After the first n tokens of head bh:
 *   S[(i,j), e] = sum_{s<n} k_si k_sj v_se      (sum of phi(k_s) v_s^T)
 *   Z[i, j]     = sum_{s<n} k_si k_sj           (sum of k_s k_s^T)
 * gist.science summary 2.2 (psi(u) = u u^T, state enlarged without
 * parameters); arXiv abstract ("constant-time recurrent inference"). */
typedef struct {
    const double *k, *v;
    double *S, *Z;
    long T, n;
    int dk, dv;
} state_ctx;

static void state_item(void *c, long bh) {
    state_ctx *x = (state_ctx *)c;
    const int dk = x->dk, dv = x->dv;
    double *S = x->S + bh * (long)dk * dk * dv;
    double *Z = x->Z + bh * (long)dk * dk;
    memset(S, 0, sizeof(double) * (size_t)dk * dk * dv);
    memset(Z, 0, sizeof(double) * (size_t)dk * dk);
    for (long s = 0; s < x->n; ++s) {
        const double *ks = x->k + (bh * x->T + s) * dk;
        const double *vs = x->v + (bh * x->T + s) * dv;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dk; ++j) {
                double f = ks[i] * ks[j];
                Z[i * dk + j] += f;
                double *row = S + ((long)i * dk + j) * dv;
                for (int e = 0; e < dv; ++e) row[e] += f * vs[e];
            }
    }
}

void kata_oracle_state(const double *k, const double *v, long BH, long T, long n, int dk,
                       int dv, double *S, double *Z, int nthreads) {
    state_ctx c = {k, v, S, Z, T, n, dk, dv};
    run_items(state_item, &c, BH, nthreads);
}

/* ------------------------------------------------------------------ */
/* Readout from a state: phi(q)^T S / (q^T Z q).                        */
/* ------------------------------------------------------------------ */

/* Numerator phi(q)^T S (dv values) and denominator q^T Z q, unnormalised. */
static void readout_raw(const double *qt, const double *S, const double *Z, int dk, int dv,
                        double *num, double *den_out) {
    double den = 0.0;
    for (int e = 0; e < dv; ++e) num[e] = 0.0;
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dk; ++j) {
            double f = qt[i] * qt[j];
            den += f * Z[i * dk + j];
            const double *row = S + ((long)i * dk + j) * dv;
            for (int e = 0; e < dv; ++e) num[e] += f * row[e];
        }
    *den_out = den;
}

/* Normalised readout: y = num / den, and y = 0 when den == 0. */
static void readout(const double *qt, const double *S, const double *Z, int dk, int dv,
                    double *y, double *den_out) {
    double den;
    readout_raw(qt, S, Z, dk, dv, y, &den);
    for (int e = 0; e < dv; ++e) y[e] = (den == 0.0) ? 0.0 : y[e] / den;
    if (den_out) *den_out = den;
}

/* Recurrent form: for t = 0..T-1, S += phi(k_t) v_t^T, Z += k_t k_t^T,
 * then y_t = phi(q_t)^T S / (q_t^T Z q_t).  A second, independent route
 * to the same numbers (arXiv abstract, "constant-time recurrent
 * inference"; gist.science summary 1, fixed-size state). */
typedef struct {
    const double *q, *k, *v;
    double *y;
    long T;
    int dk, dv;
} rec_ctx;

static void rec_item(void *c, long bh) {
    rec_ctx *x = (rec_ctx *)c;
    const int dk = x->dk, dv = x->dv;
    double *S = (double *)calloc((size_t)dk * dk * dv, sizeof(double));
    double *Z = (double *)calloc((size_t)dk * dk, sizeof(double));
    for (long t = 0; t < x->T; ++t) {
        const double *kt = x->k + (bh * x->T + t) * dk;
        const double *vt = x->v + (bh * x->T + t) * dv;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dk; ++j) {
                double f = kt[i] * kt[j];
                Z[i * dk + j] += f;
                double *row = S + ((long)i * dk + j) * dv;
                for (int e = 0; e < dv; ++e) row[e] += f * vt[e];
            }
        readout(x->q + (bh * x->T + t) * dk, S, Z, dk, dv, x->y + (bh * x->T + t) * dv, NULL);
    }
    free(S);
    free(Z);
}

void kata_oracle_forward_recurrent(const double *q, const double *k, const double *v,
                                   double *y, long BH, long T, int dk, int dv, int nthreads) {
    rec_ctx c = {q, k, v, y, T, dk, dv};
    run_items(rec_item, &c, BH, nthreads);
}

/* ------------------------------------------------------------------ */
/* Chunked-state form in fp64, any chunk size C >= 1.                   */
/* ------------------------------------------------------------------ */

/* gist.science summary 2.3 (chunked parallelism; "exact chunked-state
 * form"), arXiv abstract ("exact O(T) chunked-state form"): chunk c holds
 * tokens [cC, (c+1)C).  S_c, Z_c are the sums over all tokens before the
 * chunk (the exclusive prefix of the per-chunk sums).  For t in chunk c:
 *   num_t = phi(q_t)^T S_c + sum_{cC <= s <= t} w_ts v_s
 *   den_t = q_t^T Z_c q_t  + sum_{cC <= s <= t} w_ts
 * The per-chunk sums are formed first, then prefix-summed over chunks, as
 * the pages describe (state per chunk, then a scan across chunks). */
typedef struct {
    const double *q, *k, *v;
    double *y;
    long T, C;
    int dk, dv;
} chunk_ctx;

static void chunk_item(void *c, long bh) {
    chunk_ctx *x = (chunk_ctx *)c;
    const int dk = x->dk, dv = x->dv;
    const long T = x->T, C = x->C;
    const long nc = (T + C - 1) / C;
    const size_t ssz = (size_t)dk * dk * dv, zsz = (size_t)dk * dk;
    /* per-chunk sums dS[c], dZ[c] */
    double *dS = (double *)calloc(ssz * nc, sizeof(double));
    double *dZ = (double *)calloc(zsz * nc, sizeof(double));
    for (long ci = 0; ci < nc; ++ci) {
        for (long s = ci * C; s < (ci + 1) * C && s < T; ++s) {
            const double *ks = x->k + (bh * T + s) * dk;
            const double *vs = x->v + (bh * T + s) * dv;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dk; ++j) {
                    double f = ks[i] * ks[j];
                    dZ[ci * zsz + i * dk + j] += f;
                    double *row = dS + ci * ssz + ((size_t)i * dk + j) * dv;
                    for (int e = 0; e < dv; ++e) row[e] += f * vs[e];
                }
        }
    }
    /* exclusive prefix over chunks, in place: dS[c] <- sum_{c' < c} dS[c'] */
    double *run = (double *)calloc(ssz + zsz, sizeof(double));
    for (long ci = 0; ci < nc; ++ci) {
        for (size_t u = 0; u < ssz; ++u) {
            double cur = dS[ci * ssz + u];
            dS[ci * ssz + u] = run[u];
            run[u] += cur;
        }
        for (size_t u = 0; u < zsz; ++u) {
            double cur = dZ[ci * zsz + u];
            dZ[ci * zsz + u] = run[ssz + u];
            run[ssz + u] += cur;
        }
    }
    /* per row: inter-chunk term from the prefix state + intra-chunk term */
    for (long t = 0; t < T; ++t) {
        const long ci = t / C;
        const double *qt = x->q + (bh * T + t) * dk;
        double *yt = x->y + (bh * T + t) * dv;
        double num[512], den_inter;
        readout_raw(qt, dS + ci * ssz, dZ + ci * zsz, dk, dv, num, &den_inter);
        double den = den_inter;
        for (long s = ci * C; s <= t; ++s) {
            const double *ks = x->k + (bh * T + s) * dk;
            const double *vs = x->v + (bh * T + s) * dv;
            double dot = 0.0;
            for (int i = 0; i < dk; ++i) dot += qt[i] * ks[i];
            double w = dot * dot;
            den += w;
            for (int e = 0; e < dv; ++e) num[e] += w * vs[e];
        }
        for (int e = 0; e < dv; ++e) yt[e] = (den == 0.0) ? 0.0 : num[e] / den;
    }
    free(run);
    free(dS);
    free(dZ);
}

/* Requires dv <= 512. */
int kata_oracle_forward_chunked(const double *q, const double *k, const double *v, double *y,
                                long BH, long T, int dk, int dv, long C, int nthreads) {
    if (C < 1 || dv > 512) return 1;
    chunk_ctx c = {q, k, v, y, T, C, dk, dv};
    run_items(chunk_item, &c, BH, nthreads);
    return 0;
}

/* ------------------------------------------------------------------ */
/* One decode step on a given state.                                    */
/* ------------------------------------------------------------------ */

/* For each head: S += phi(k) v^T, Z += k k^T, then
 * y = phi(q)^T S / (q^T Z q), the current token included (gist.science
 * summary 2.1: the gate interpolates between the previous readout and the
 * current value).  q, k: [BH][dk]; v, y: [BH][dv]; S, Z updated in place. */
void kata_oracle_decode_step(const double *q, const double *k, const double *v, double *S,
                             double *Z, double *y, double *den, long BH, int dk, int dv) {
    for (long bh = 0; bh < BH; ++bh) {
        double *Sh = S + bh * (long)dk * dk * dv;
        double *Zh = Z + bh * (long)dk * dk;
        const double *kh = k + bh * dk, *vh = v + bh * dv;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dk; ++j) {
                double f = kh[i] * kh[j];
                Zh[i * dk + j] += f;
                double *row = Sh + ((long)i * dk + j) * dv;
                for (int e = 0; e < dv; ++e) row[e] += f * vh[e];
            }
        readout(q + bh * dk, Sh, Zh, dk, dv, y + bh * dv, den ? den + bh : NULL);
    }
}

/* ------------------------------------------------------------------ */
/* KATA-Mg: several rank-one PSD factors per head.                      */
/* ------------------------------------------------------------------ */

/* gist.science summary, Technical summary 2.3 ("Variantes"): KATA-Mg uses
 * several PSD factors to trade state size against packing efficiency.  The
 * pages name the variant without its formula; the reading taken (listed with
 * the other readings in the design notes): the feature cone is a product of
 * g rank-one PSD cones (2.1: the admissible geometries are the irreducible
 * factors of the Koecher-Vinberg classification, of which a symmetric cone is
 * a product), factor m with its own projection dimension p = dk / g (2.2)
 * acting on coordinates [m p, (m + 1) p) of q and k.  The inner product on a
 * product of cones is the sum of the factors' inner products, so
 *
 *     w_ts = sum_m (q_t^(m) . k_s^(m))^2 ,   y_t = sum_{s<=t} w_ts v_s / sum_{s<=t} w_ts
 *
 * with y_t = 0 when the sum is 0 (as for one factor).  The state is the g
 * blocks S^(m)[(i,j), e] = sum_s k_si k_sj v_se with i, j both in block m, and
 * Z^(m) likewise; g = 1 is the single factor above.  dk must be a multiple
 * of g. */

/* The Mg weight of query row qt and key row ks. */
static double mg_weight(const double *qt, const double *ks, int dk, int g) {
    const int p = dk / g;
    double w = 0.0;
    for (int m = 0; m < g; ++m) {
        double dot = 0.0;
        for (int i = m * p; i < (m + 1) * p; ++i) dot += qt[i] * ks[i];
        w += dot * dot;
    }
    return w;
}

typedef struct {
    const double *q, *k, *v;
    double *y, *den;
    long T;
    int dk, dv, g;
    const long *bh_idx, *t_idx; /* NULL: every row, item = bh*T + t */
} mg_rows_ctx;

static void mg_rows_item(void *c, long item) {
    mg_rows_ctx *x = (mg_rows_ctx *)c;
    long bh, t;
    if (x->bh_idx) {
        bh = x->bh_idx[item];
        t = x->t_idx[item];
    } else {
        bh = item / x->T;
        t = item % x->T;
    }
    const int dk = x->dk, dv = x->dv;
    const double *qt = x->q + (bh * x->T + t) * dk;
    double *y = x->y + item * dv;
    double den = 0.0;
    for (int e = 0; e < dv; ++e) y[e] = 0.0;
    for (long s = 0; s <= t; ++s) {
        const double *vs = x->v + (bh * x->T + s) * dv;
        double w = mg_weight(qt, x->k + (bh * x->T + s) * dk, dk, x->g);
        den += w;
        for (int e = 0; e < dv; ++e) y[e] += w * vs[e];
    }
    for (int e = 0; e < dv; ++e) y[e] = (den == 0.0) ? 0.0 : y[e] / den;
    if (x->den) x->den[item] = den;
}

/* Every row of every head; returns 1 (nothing computed) if g does not divide dk. */
int kata_oracle_forward_mg(const double *q, const double *k, const double *v, double *y,
                           double *den, long BH, long T, int dk, int dv, int g, int nthreads) {
    if (g < 1 || dk % g != 0) return 1;
    mg_rows_ctx c = {q, k, v, y, den, T, dk, dv, g, NULL, NULL};
    run_items(mg_rows_item, &c, BH * T, nthreads);
    return 0;
}

/* Selected rows (bh_idx[r], t_idx[r]); y: [nrows][dv]; den: [nrows]. */
int kata_oracle_forward_mg_rows(const double *q, const double *k, const double *v, long T,
                                int dk, int dv, int g, const long *bh_idx, const long *t_idx,
                                long nrows, double *y, double *den, int nthreads) {
    if (g < 1 || dk % g != 0) return 1;
    mg_rows_ctx c = {q, k, v, y, den, T, dk, dv, g, bh_idx, t_idx};
    run_items(mg_rows_item, &c, nrows, nthreads);
    return 0;
}

/* The Mg state after the first n tokens, in the dense layout of the single
 * factor: S[(i,j), e] = sum_{s<n} k_si k_sj v_se and Z[i, j] = sum_{s<n} k_si k_sj
 * when i and j lie in the same block of p coordinates, and 0 otherwise (the
 * g blocks of the product cone's state, side by side). */
typedef struct {
    const double *k, *v;
    double *S, *Z;
    long T, n;
    int dk, dv, g;
} mg_state_ctx;

static void mg_state_item(void *c, long bh) {
    mg_state_ctx *x = (mg_state_ctx *)c;
    const int dk = x->dk, dv = x->dv, p = dk / x->g;
    double *S = x->S + bh * (long)dk * dk * dv;
    double *Z = x->Z + bh * (long)dk * dk;
    memset(S, 0, sizeof(double) * (size_t)dk * dk * dv);
    memset(Z, 0, sizeof(double) * (size_t)dk * dk);
    for (long s = 0; s < x->n; ++s) {
        const double *ks = x->k + (bh * x->T + s) * dk;
        const double *vs = x->v + (bh * x->T + s) * dv;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dk; ++j) {
                if (i / p != j / p) continue;
                double f = ks[i] * ks[j];
                Z[i * dk + j] += f;
                double *row = S + ((long)i * dk + j) * dv;
                for (int e = 0; e < dv; ++e) row[e] += f * vs[e];
            }
    }
}

int kata_oracle_state_mg(const double *k, const double *v, long BH, long T, long n, int dk,
                         int dv, int g, double *S, double *Z, int nthreads) {
    if (g < 1 || dk % g != 0) return 1;
    mg_state_ctx c = {k, v, S, Z, T, n, dk, dv, g};
    run_items(mg_state_item, &c, BH, nthreads);
    return 0;
}

/* Recurrent Mg form: per token, the block state update then the readout
 * phi(q)^T S / (q^T Z q) over the blocks (zeros elsewhere add nothing); a
 * second route to the Mg outputs. */
typedef struct {
    const double *q, *k, *v;
    double *y;
    long T;
    int dk, dv, g;
} mg_rec_ctx;

static void mg_rec_item(void *c, long bh) {
    mg_rec_ctx *x = (mg_rec_ctx *)c;
    const int dk = x->dk, dv = x->dv, p = dk / x->g;
    double *S = (double *)calloc((size_t)dk * dk * dv, sizeof(double));
    double *Z = (double *)calloc((size_t)dk * dk, sizeof(double));
    for (long t = 0; t < x->T; ++t) {
        const double *kt = x->k + (bh * x->T + t) * dk;
        const double *vt = x->v + (bh * x->T + t) * dv;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dk; ++j) {
                if (i / p != j / p) continue;
                double f = kt[i] * kt[j];
                Z[i * dk + j] += f;
                double *row = S + ((long)i * dk + j) * dv;
                for (int e = 0; e < dv; ++e) row[e] += f * vt[e];
            }
        readout(x->q + (bh * x->T + t) * dk, S, Z, dk, dv, x->y + (bh * x->T + t) * dv, NULL);
    }
    free(S);
    free(Z);
}

int kata_oracle_forward_mg_recurrent(const double *q, const double *k, const double *v,
                                     double *y, long BH, long T, int dk, int dv, int g,
                                     int nthreads) {
    if (g < 1 || dk % g != 0) return 1;
    mg_rec_ctx c = {q, k, v, y, T, dk, dv, g};
    run_items(mg_rec_item, &c, BH, nthreads);
    return 0;
}

/* One Mg decode step: the block state update for token (k, v), then the
 * readout with query q, current token included.  S, Z hold Mg states (zeros
 * outside the blocks) and stay so. */
int kata_oracle_decode_step_mg(const double *q, const double *k, const double *v, double *S,
                               double *Z, double *y, double *den, long BH, int dk, int dv,
                               int g) {
    if (g < 1 || dk % g != 0) return 1;
    const int p = dk / g;
    for (long bh = 0; bh < BH; ++bh) {
        double *Sh = S + bh * (long)dk * dk * dv;
        double *Zh = Z + bh * (long)dk * dk;
        const double *kh = k + bh * dk, *vh = v + bh * dv;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dk; ++j) {
                if (i / p != j / p) continue;
                double f = kh[i] * kh[j];
                Zh[i * dk + j] += f;
                double *row = Sh + ((long)i * dk + j) * dv;
                for (int e = 0; e < dv; ++e) row[e] += f * vh[e];
            }
        readout(q + bh * dk, Sh, Zh, dk, dv, y + bh * dv, den ? den + bh : NULL);
    }
    return 0;
}
