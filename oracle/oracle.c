/*
 * oracle.c -- plain, slow, float64 CPU oracle for the AB-Attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file.  It is used by the test-suite, by the smoke check and by the CPU
 * baseline leg of the benchmark, and it shares no code with the CUDA library.
 *
 * Source of the method: "Accurate Block Attention (AB-Attention)", abstract
 * (paper listing page, Xing Ma query).  The abstract describes three stages:
 *   - IBCS: k-means of the queries inside each query block (no token
 *     permutation), whose centroids score every key/value block;
 *   - SIP: blocks are drawn with probability proportional to those scores and
 *     re-weighted by the inverse inclusion probability, so the pass estimates
 *     dense attention;
 *   - a kernel that packs the small selected key/value blocks into full
 *     tensor-core tiles.
 * The abstract gives no formulas.  Every open detail below is fixed by a
 * stated reading (written next to the code that takes it).
 *
 * Conventions
 *   Q, K, V  bf16 bit patterns, layout [B][H][N][d], widened exactly to double.
 *   row      one query block (beta, h, i); linear id ((beta*H)+h)*nQ + i.
 *   Bq       query block size, Bk key/value block size.
 *   nQ = ceil(N/Bq), nK = ceil(N/Bk).  Tail blocks are partial: rows/keys past
 *   N do not exist (they are neither counted nor attended to).
 *
 * Every entry point returns 0 on success and a negative value on bad input.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* helpers                                                                   */
/* ------------------------------------------------------------------------ */

static double bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

typedef struct {
    int B, H, N, d, Bq, Bk, nQ, nK;
} geom_t;

static int make_geom(geom_t *g, int B, int H, int N, int d, int Bq, int Bk)
{
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || Bq <= 0 || Bk <= 0) return -1;
    g->B = B; g->H = H; g->N = N; g->d = d; g->Bq = Bq; g->Bk = Bk;
    g->nQ = (N + Bq - 1) / Bq;
    g->nK = (N + Bk - 1) / Bk;
    return 0;
}

/* Decode a linear row id into (beta, h, i).  Returns -1 if out of range. */
static int decode_row(const geom_t *g, int64_t row, int *beta, int *h, int *i)
{
    int64_t total = (int64_t)g->B * g->H * g->nQ;
    if (row < 0 || row >= total) return -1;
    *i = (int)(row % g->nQ);
    int64_t bh = row / g->nQ;
    *h = (int)(bh % g->H);
    *beta = (int)(bh / g->H);
    return 0;
}

/* Pointer to token t of head (beta,h) in a [B][H][N][d] tensor. */
static const uint16_t *tok(const uint16_t *X, const geom_t *g, int beta, int h, int t)
{
    return X + (((size_t)beta * g->H + h) * g->N + t) * (size_t)g->d;
}

static double dot_bf(const uint16_t *a, const uint16_t *b, int d)
{
    double s = 0.0;
    for (int k = 0; k < d; ++k) s += bf16_to_f64(a[k]) * bf16_to_f64(b[k]);
    return s;
}

static double dot_fb(const double *a, const uint16_t *b, int d)
{
    double s = 0.0;
    for (int k = 0; k < d; ++k) s += a[k] * bf16_to_f64(b[k]);
    return s;
}

/* Number of valid query rows in query block i. */
static int rows_in_block(const geom_t *g, int i)
{
    int n = g->N - i * g->Bq;
    return n < g->Bq ? n : g->Bq;
}

/* Number of valid keys in key block b. */
static int keys_in_block(const geom_t *g, int b)
{
    int n = g->N - b * g->Bk;
    return n < g->Bk ? n : g->Bk;
}

/* Simple parallel-for over [0, n): worker(ctx, index). */
typedef void (*work_fn)(void *ctx, int64_t index);
typedef struct {
    work_fn fn;
    void *ctx;
    int64_t n;
    int64_t next;
} pool_t;

static void *pool_main(void *arg)
{
    pool_t *p = (pool_t *)arg;
    for (;;) {
        int64_t k = __atomic_fetch_add(&p->next, 1, __ATOMIC_RELAXED);
        if (k >= p->n) break;
        p->fn(p->ctx, k);
    }
    return NULL;
}

static void parallel_for(int64_t n, int nthreads, work_fn fn, void *ctx)
{
    pool_t p = {fn, ctx, n, 0};
    if (nthreads <= 1 || n <= 1) {
        pool_main(&p);
        return;
    }
    if (nthreads > 512) nthreads = 512;
    pthread_t th[512];
    int started = 0;
    for (int t = 0; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, pool_main, &p) != 0) break;
        ++started;
    }
    if (started == 0) pool_main(&p);
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as   */
/* easy as 1, 2, 3", SC 2011).  Ten rounds of the 4x32 Philox S-box with the  */
/* multipliers and Weyl key increments published in that paper.             */
/* ------------------------------------------------------------------------ */

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        uint64_t p0 = (uint64_t)PHILOX_M0 * c0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        k0 += PHILOX_W0;
        k1 += PHILOX_W1;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* ------------------------------------------------------------------------ */
/* O1  dense softmax attention (non-causal "3D full attention" of the        */
/* abstract's problem statement).                                            */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t *Q, *K, *V;
    geom_t g;
    double scale;
    const int64_t *rows;
    double *O, *lse;
    int bad;
} dense_ctx;

static void dense_row(void *vctx, int64_t k)
{
    dense_ctx *c = (dense_ctx *)vctx;
    const geom_t *g = &c->g;
    int beta, h, i;
    if (decode_row(g, c->rows[k], &beta, &h, &i)) { c->bad = 1; return; }
    int n = rows_in_block(g, i), d = g->d, N = g->N;
    double *z = (double *)malloc(sizeof(double) * (size_t)N);
    double *O = c->O + (size_t)k * g->Bq * d;
    memset(O, 0, sizeof(double) * (size_t)g->Bq * d);
    if (c->lse)
        for (int r = 0; r < g->Bq; ++r) c->lse[(size_t)k * g->Bq + r] = -INFINITY;
    for (int r = 0; r < n; ++r) {
        const uint16_t *q = tok(c->Q, g, beta, h, i * g->Bq + r);
        double m = -INFINITY;
        for (int t = 0; t < N; ++t) {
            z[t] = c->scale * dot_bf(q, tok(c->K, g, beta, h, t), d);
            if (z[t] > m) m = z[t];
        }
        double den = 0.0;
        double *o = O + (size_t)r * d;
        for (int t = 0; t < N; ++t) {
            double e = exp(z[t] - m);
            den += e;
            const uint16_t *v = tok(c->V, g, beta, h, t);
            for (int x = 0; x < d; ++x) o[x] += e * bf16_to_f64(v[x]);
        }
        for (int x = 0; x < d; ++x) o[x] /= den;
        if (c->lse) c->lse[(size_t)k * g->Bq + r] = m + log(den);
    }
    free(z);
}

int orc_dense_attention(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                        int B, int H, int N, int d, int Bq, double scale,
                        const int64_t *rows, int64_t nrows, int nthreads,
                        double *O, double *lse)
{
    dense_ctx c;
    memset(&c, 0, sizeof c);
    if (make_geom(&c.g, B, H, N, d, Bq, 1)) return -1;
    if (!Q || !K || !V || !rows || !O || nrows < 0) return -1;
    c.Q = Q; c.K = K; c.V = V; c.scale = scale; c.rows = rows; c.O = O; c.lse = lse;
    parallel_for(nrows, nthreads, dense_row, &c);
    return c.bad ? -2 : 0;
}

/* ------------------------------------------------------------------------ */
/* O2  IBCS part 1: Lloyd k-means of the queries of ONE query block.         */
/*                                                                           */
/* The abstract says the selector clusters the queries of each query block   */
/* on their own and never reorders tokens.  It gives no initialisation, no   */
/* iteration count and no rule for empty clusters; the readings taken here:  */
/*   - C_eff = min(C, n) clusters, n = valid rows of the block;              */
/*   - init: centroid j starts at row floor(j*n/C_eff) (evenly spaced rows,  */
/*     deterministic, no random draw);                                       */
/*   - `iters` rounds of (assign, update); assignment minimises squared      */
/*     Euclidean distance, ties to the smallest centroid index; the update   */
/*     sets each centroid to the mean of its rows, an empty cluster keeps    */
/*     its previous centroid;                                                */
/*   - the cluster sizes n_j are those of the last round's assignment.       */
/* `dist_trace` (nullable, 2*iters values) records the distortion after each */
/* assignment and after each update, for the monotonicity check.             */
/* ------------------------------------------------------------------------ */

static int kmeans_block(const uint16_t *Q, const geom_t *g, int beta, int h, int i,
                        int C, int iters, double *cent /*[C][d]*/,
                        int32_t *count /*[C]*/, int32_t *assign /*[Bq]*/,
                        double *dist_trace)
{
    const int d = g->d;
    const int n = rows_in_block(g, i);
    const int ce = C < n ? C : n;
    double *sum = (double *)calloc((size_t)C * d, sizeof(double));
    if (!sum) return -3;
    for (int j = 0; j < C; ++j) {
        count[j] = 0;
        for (int x = 0; x < d; ++x) cent[(size_t)j * d + x] = 0.0;
    }
    for (int r = 0; r < g->Bq; ++r) assign[r] = -1;
    for (int j = 0; j < ce; ++j) {
        int r = (int)(((int64_t)j * n) / ce);
        const uint16_t *q = tok(Q, g, beta, h, i * g->Bq + r);
        for (int x = 0; x < d; ++x) cent[(size_t)j * d + x] = bf16_to_f64(q[x]);
    }
    for (int it = 0; it < iters; ++it) {
        /* assignment */
        double dist_a = 0.0;
        for (int j = 0; j < ce; ++j) count[j] = 0;
        for (int r = 0; r < n; ++r) {
            const uint16_t *q = tok(Q, g, beta, h, i * g->Bq + r);
            int best = 0;
            double bestd = INFINITY;
            for (int j = 0; j < ce; ++j) {
                double s = 0.0;
                for (int x = 0; x < d; ++x) {
                    double diff = bf16_to_f64(q[x]) - cent[(size_t)j * d + x];
                    s += diff * diff;
                }
                if (s < bestd) { bestd = s; best = j; }
            }
            assign[r] = best;
            count[best] += 1;
            dist_a += bestd;
        }
        /* update */
        memset(sum, 0, sizeof(double) * (size_t)C * d);
        for (int r = 0; r < n; ++r) {
            const uint16_t *q = tok(Q, g, beta, h, i * g->Bq + r);
            double *s = sum + (size_t)assign[r] * d;
            for (int x = 0; x < d; ++x) s[x] += bf16_to_f64(q[x]);
        }
        for (int j = 0; j < ce; ++j) {
            if (count[j] == 0) continue;
            for (int x = 0; x < d; ++x)
                cent[(size_t)j * d + x] = sum[(size_t)j * d + x] / (double)count[j];
        }
        if (dist_trace) {
            double dist_u = 0.0;
            for (int r = 0; r < n; ++r) {
                const uint16_t *q = tok(Q, g, beta, h, i * g->Bq + r);
                const double *c = cent + (size_t)assign[r] * d;
                for (int x = 0; x < d; ++x) {
                    double diff = bf16_to_f64(q[x]) - c[x];
                    dist_u += diff * diff;
                }
            }
            dist_trace[2 * it] = dist_a;
            dist_trace[2 * it + 1] = dist_u;
        }
    }
    if (iters == 0) {
        /* no round: sizes come from one assignment against the seeds */
        for (int r = 0; r < n; ++r) {
            const uint16_t *q = tok(Q, g, beta, h, i * g->Bq + r);
            int best = 0;
            double bestd = INFINITY;
            for (int j = 0; j < ce; ++j) {
                double s = 0.0;
                for (int x = 0; x < d; ++x) {
                    double diff = bf16_to_f64(q[x]) - cent[(size_t)j * d + x];
                    s += diff * diff;
                }
                if (s < bestd) { bestd = s; best = j; }
            }
            assign[r] = best;
            count[best] += 1;
        }
    }
    free(sum);
    return 0;
}

typedef struct {
    const uint16_t *Q;
    geom_t g;
    int C, iters;
    const int64_t *rows;
    double *cent, *trace;
    int32_t *count, *assign;
    int bad;
} km_ctx;

static void km_row(void *vctx, int64_t k)
{
    km_ctx *c = (km_ctx *)vctx;
    int beta, h, i;
    if (decode_row(&c->g, c->rows[k], &beta, &h, &i)) { c->bad = 1; return; }
    if (kmeans_block(c->Q, &c->g, beta, h, i, c->C, c->iters,
                     c->cent + (size_t)k * c->C * c->g.d, c->count + (size_t)k * c->C,
                     c->assign + (size_t)k * c->g.Bq,
                     c->trace ? c->trace + (size_t)k * 2 * c->iters : NULL))
        c->bad = 1;
}

int orc_kmeans(const uint16_t *Q, int B, int H, int N, int d, int Bq, int C, int iters,
               const int64_t *rows, int64_t nrows, int nthreads,
               double *cent, int32_t *count, int32_t *assign, double *trace)
{
    km_ctx c;
    memset(&c, 0, sizeof c);
    if (make_geom(&c.g, B, H, N, d, Bq, 1)) return -1;
    if (C <= 0 || C > Bq || iters < 0 || !Q || !rows || !cent || !count || !assign) return -1;
    c.Q = Q; c.C = C; c.iters = iters; c.rows = rows;
    c.cent = cent; c.count = count; c.assign = assign; c.trace = trace;
    parallel_for(nrows, nthreads, km_row, &c);
    return c.bad ? -2 : 0;
}

/* ------------------------------------------------------------------------ */
/* O3  IBCS part 2: block importance p_{i,b} of every key block b for query  */
/* block i.                                                                  */
/*                                                                           */
/* Each non-empty centroid c_j attends over all valid keys with the          */
/* attention scale; its softmax mass is summed per key block, and the        */
/* centroids are combined with weights n_j / n (the share of the block's     */
/* queries each stands for), so p_{i,.} sums to one.  The scoring rule,      */
/* the temperature (same scale as attention) and the weighting are the       */
/* readings taken where the abstract only says the selector estimates block  */
/* importance from the clustered queries.                                    */
/* ------------------------------------------------------------------------ */

/* Coarse variant (the abstract's other contrast: blocks "scored from coarse */
/* summaries"): each key block b is scored once through its mean key kbar_b  */
/* (the mean of its valid keys), with the block's share of the softmax       */
/* taken as n_b * exp(scale * c.kbar_b) normalised over the blocks (n_b =    */
/* valid keys of b) -- the per-key rule above applied to keys replaced by    */
/* their block means.  Same centroids and weights.                           */

static int block_probs_row(const uint16_t *Q, const uint16_t *K, const geom_t *g,
                           int beta, int h, int i, int C, int iters, double scale, int coarse,
                           double *p /*[nK]*/)
{
    const int d = g->d, N = g->N, nK = g->nK;
    const int n = rows_in_block(g, i);
    double *cent = (double *)malloc(sizeof(double) * (size_t)C * d);
    int32_t *count = (int32_t *)malloc(sizeof(int32_t) * (size_t)C);
    int32_t *assign = (int32_t *)malloc(sizeof(int32_t) * (size_t)g->Bq);
    double *z = (double *)malloc(sizeof(double) * (size_t)N);
    if (!cent || !count || !assign || !z) {
        free(cent); free(count); free(assign); free(z);
        return -3;
    }
    int rc = kmeans_block(Q, g, beta, h, i, C, iters, cent, count, assign, NULL);
    for (int b = 0; b < nK; ++b) p[b] = 0.0;
    if (coarse && rc == 0) {
        double *kbar = (double *)malloc(sizeof(double) * (size_t)nK * d);
        if (!kbar) rc = -3;
        for (int b = 0; rc == 0 && b < nK; ++b) {
            const int nb = keys_in_block(g, b);
            for (int x = 0; x < d; ++x) {
                double sum = 0.0;
                for (int u = 0; u < nb; ++u) sum += bf16_to_f64(tok(K, g, beta, h, b * g->Bk + u)[x]);
                kbar[(size_t)b * d + x] = sum / nb;
            }
        }
        for (int j = 0; rc == 0 && j < C; ++j) {
            if (count[j] == 0) continue;
            const double w = (double)count[j] / (double)n;
            double m = -INFINITY;
            for (int b = 0; b < nK; ++b) {
                double dot = 0.0;
                for (int x = 0; x < d; ++x) dot += cent[(size_t)j * d + x] * kbar[(size_t)b * d + x];
                z[b] = scale * dot + log((double)keys_in_block(g, b));
                if (z[b] > m) m = z[b];
            }
            double Z = 0.0;
            for (int b = 0; b < nK; ++b) {
                z[b] = exp(z[b] - m);
                Z += z[b];
            }
            for (int b = 0; b < nK; ++b) p[b] += w * (z[b] / Z);
        }
        free(kbar);
        free(cent); free(count); free(assign); free(z);
        return rc;
    }
    for (int j = 0; rc == 0 && j < C; ++j) {
        if (count[j] == 0) continue;
        const double w = (double)count[j] / (double)n;
        double m = -INFINITY;
        for (int t = 0; t < N; ++t) {
            z[t] = scale * dot_fb(cent + (size_t)j * d, tok(K, g, beta, h, t), d);
            if (z[t] > m) m = z[t];
        }
        double Z = 0.0;
        for (int t = 0; t < N; ++t) {
            z[t] = exp(z[t] - m);
            Z += z[t];
        }
        for (int b = 0; b < nK; ++b) {
            double mass = 0.0;
            int nb = keys_in_block(g, b);
            for (int u = 0; u < nb; ++u) mass += z[b * g->Bk + u];
            p[b] += w * (mass / Z);
        }
    }
    free(cent); free(count); free(assign); free(z);
    return rc;
}

typedef struct {
    const uint16_t *Q, *K;
    geom_t g;
    int C, iters;
    double scale;
    int coarse;
    const int64_t *rows;
    double *p64;
    float *p32;
    int bad;
} bp_ctx;

static void bp_row(void *vctx, int64_t k)
{
    bp_ctx *c = (bp_ctx *)vctx;
    int beta, h, i;
    if (decode_row(&c->g, c->rows[k], &beta, &h, &i)) { c->bad = 1; return; }
    double *p = c->p64 + (size_t)k * c->g.nK;
    if (block_probs_row(c->Q, c->K, &c->g, beta, h, i, c->C, c->iters, c->scale, c->coarse, p)) {
        c->bad = 1;
        return;
    }
    if (c->p32)
        for (int b = 0; b < c->g.nK; ++b) c->p32[(size_t)k * c->g.nK + b] = (float)p[b];
}

int orc_block_probs(const uint16_t *Q, const uint16_t *K, int B, int H, int N, int d,
                    int Bq, int Bk, int C, int iters, double scale, int coarse,
                    const int64_t *rows, int64_t nrows, int nthreads,
                    double *p64, float *p32)
{
    bp_ctx c;
    memset(&c, 0, sizeof c);
    if (make_geom(&c.g, B, H, N, d, Bq, Bk)) return -1;
    if (C <= 0 || C > Bq || iters < 0 || !Q || !K || !rows || !p64) return -1;
    c.Q = Q; c.K = K; c.C = C; c.iters = iters; c.scale = scale; c.coarse = coarse; c.rows = rows;
    c.p64 = p64; c.p32 = p32;
    parallel_for(nrows, nthreads, bp_row, &c);
    return c.bad ? -2 : 0;
}

/* ------------------------------------------------------------------------ */
/* O4  SIP: Poisson sampling with inclusion probabilities proportional to    */
/* the block estimates, capped at one, with expected size M.                 */
/*                                                                           */
/* The abstract says blocks are drawn in proportion to the estimates and     */
/* re-weighted by the inverse inclusion probability.  Readings taken:        */
/*   - M = floor((budget_bp * nK + 5000) / 10000) blocks per query block     */
/*     (budget in basis points, rounded half up); M >= nK keeps every block  */
/*     with weight one ("keep-all");                                         */
/*   - pi_b = min(1, c * p_b) with c chosen so that sum_b pi_b = M, solved   */
/*     exactly in 48-bit fixed point:  P_b = round-half-even(p_b * 2^48)     */
/*     (p clamped to [0,1], NaN read as 0), then water-filling: with S the   */
/*     saturated set, R = M - |S| and T = sum of P_b outside S, every b      */
/*     outside S with R*P_b >= T joins S; repeat until S stops growing or    */
/*     T = 0.  Outside S, pi_b = R*P_b / T exactly;                          */
/*   - the draw for block b of row (beta,h,i) is word (b mod 4) of           */
/*     Philox4x32-10 at counter (b/4, i, h, beta) and key (seed lo, seed hi);*/
/*     with paired draws the counter is (b/4, floor(i/2), h, beta): query    */
/*     blocks 2j and 2j+1 share every uniform (common random numbers; each   */
/*     row keeps its own pi_b, so its marginal draws are unchanged);         */
/*   - b is taken iff b is in S or U_b * T < R * P_b * 2^32 (exact integer  */
/*     comparison, i.e. U_b / 2^32 < pi_b);                                  */
/*   - log-weight: 0 on S, else fp32 round-to-nearest of -ln(x) with         */
/*     x = double(R*P_b) / double(T) (IEEE double conversions and divide);   */
/*   - output in ascending block order; at most `capacity` entries are kept. */
/* ------------------------------------------------------------------------ */

#define FIX_ONE 281474976710656.0 /* 2^48 */

int64_t orc_budget_blocks(int budget_bp, int nK)
{
    return ((int64_t)budget_bp * nK + 5000) / 10000;
}

static int64_t to_fixed(float pf)
{
    double p = (double)pf;
    if (!(p > 0.0)) return 0; /* negative, zero and NaN */
    if (p > 1.0) p = 1.0;
    return (int64_t)nearbyint(p * FIX_ONE);
}

/* Water-filling for one row.  Fills P[nK], sat[nK] and returns R, T. */
int orc_inclusion(const float *p, int nK, int64_t M, int64_t *P, uint8_t *sat,
                  int64_t *R_out, int64_t *T_out, int32_t *rounds_out)
{
    if (!p || !P || !sat || nK <= 0 || nK > 32767 || M < 0) return -1;
    int64_t inS = 0;
    for (int b = 0; b < nK; ++b) {
        P[b] = to_fixed(p[b]);
        sat[b] = 0;
    }
    int32_t rounds = 0;
    int64_t R = M, T = 0;
    if (M >= nK) {
        for (int b = 0; b < nK; ++b) sat[b] = 1;
        R = 0; T = 0;
    } else {
        for (;;) {
            R = M - inS;
            T = 0;
            for (int b = 0; b < nK; ++b)
                if (!sat[b]) T += P[b];
            if (T == 0 || R <= 0) break;
            int64_t added = 0;
            for (int b = 0; b < nK; ++b)
                if (!sat[b] && R * P[b] >= T) { sat[b] = 1; ++added; }
            ++rounds;
            if (added == 0) break;
            inS += added;
        }
    }
    if (R_out) *R_out = R;
    if (T_out) *T_out = T;
    if (rounds_out) *rounds_out = rounds;
    return 0;
}

/* fp32 rounding of -ln(x); *amb set when the exact value lies so close to a
 * rounding boundary between two floats that a faithful (not correctly
 * rounded) double logarithm could land on either side. */
static float neg_log_f32(double x, int *amb)
{
    long double y = -logl((long double)x);
    float f = (float)y;
    *amb = 0;
    if (y != 0.0L) {
        float lo = f, hi = f;
        if ((long double)f > y) lo = nextafterf(f, -INFINITY);
        else hi = nextafterf(f, INFINITY);
        long double mid = ((long double)lo + (long double)hi) * 0.5L;
        long double gap = fabsl(y - mid);
        if (gap <= fabsl(y) * 0x1p-44L) *amb = 1;
    }
    return f;
}

static int sample_row(const float *p, const geom_t *g, int beta, int h, int i,
                      int budget_bp, uint64_t seed, int paired, int capacity,
                      int32_t *count, int32_t *idx, float *logw, uint8_t *amb,
                      int *overflow)
{
    /* beta and h enter the counter as global indices: the caller adds the
       offsets of a slice of a larger problem */
    const int nK = g->nK;
    int64_t M = orc_budget_blocks(budget_bp, nK);
    int64_t *P = (int64_t *)malloc(sizeof(int64_t) * (size_t)nK);
    uint8_t *sat = (uint8_t *)malloc((size_t)nK);
    if (!P || !sat) { free(P); free(sat); return -3; }
    int64_t R, T;
    orc_inclusion(p, nK, M, P, sat, &R, &T, NULL);
    const uint32_t key[2] = {(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32)};
    uint32_t u4[4] = {0, 0, 0, 0};
    int n = 0;
    *overflow = 0;
    for (int b = 0; b < nK; ++b) {
        if ((b & 3) == 0) {
            const uint32_t ctr[4] = {(uint32_t)(b >> 2), (uint32_t)(paired ? i >> 1 : i), (uint32_t)h,
                                     (uint32_t)beta};
            orc_philox4x32_10(ctr, key, u4);
        }
        const uint32_t U = u4[b & 3];
        int take;
        float lw = 0.0f;
        int a = 0;
        if (sat[b]) {
            take = 1;
        } else {
            unsigned __int128 lhs = (unsigned __int128)U * (unsigned __int128)(uint64_t)T;
            unsigned __int128 rhs = ((unsigned __int128)(uint64_t)(R * P[b])) << 32;
            take = lhs < rhs;
            if (take) lw = neg_log_f32((double)(R * P[b]) / (double)T, &a);
        }
        if (!take) continue;
        if (n < capacity) {
            idx[n] = b;
            logw[n] = lw;
            if (amb) amb[n] = (uint8_t)a;
            ++n;
        } else {
            *overflow = 1;
        }
    }
    *count = n;
    free(P); free(sat);
    return 0;
}

typedef struct {
    const float *p;
    geom_t g;
    const int64_t *rows;
    int budget_bp, capacity, paired, b_off, h_off;
    uint64_t seed;
    int32_t *counts, *idx;
    float *logw;
    uint8_t *amb;
    int bad, overflow;
} smp_ctx;

static void smp_row(void *vctx, int64_t k)
{
    smp_ctx *c = (smp_ctx *)vctx;
    int beta, h, i, of = 0;
    if (decode_row(&c->g, c->rows[k], &beta, &h, &i)) { c->bad = 1; return; }
    size_t o = (size_t)k * c->capacity;
    if (sample_row(c->p + (size_t)k * c->g.nK, &c->g, beta + c->b_off, h + c->h_off, i, c->budget_bp, c->seed,
                   c->paired, c->capacity, c->counts + k, c->idx + o, c->logw + o,
                   c->amb ? c->amb + o : NULL, &of))
        c->bad = 1;
    if (of) __atomic_store_n(&c->overflow, 1, __ATOMIC_RELAXED);
}

/* p is [nrows][nK] (row k belongs to linear row id rows[k]).  b_off, h_off:
 * global index of the tensor's first batch element and head, when it is a
 * slice of a larger problem (0 otherwise).  Returns 1 if some row had more
 * draws than `capacity` (its list is truncated). */
int orc_sample(const float *p, int B, int H, int N, int Bq, int Bk,
               const int64_t *rows, int64_t nrows, int budget_bp, uint64_t seed,
               int capacity, int nthreads,
               int32_t *counts, int32_t *idx, float *logw, uint8_t *amb, int paired,
               int b_off, int h_off)
{
    smp_ctx c;
    memset(&c, 0, sizeof c);
    if (make_geom(&c.g, B, H, N, 1, Bq, Bk)) return -1;
    if (!p || !rows || !counts || !idx || !logw || capacity < 0 || budget_bp < 0) return -1;
    if (b_off < 0 || h_off < 0) return -1;
    c.b_off = b_off; c.h_off = h_off;
    if (c.g.nK > 32767) return -1;
    c.p = p; c.rows = rows; c.budget_bp = budget_bp; c.capacity = capacity; c.seed = seed;
    c.counts = counts; c.idx = idx; c.logw = logw; c.amb = amb; c.paired = paired ? 1 : 0;
    parallel_for(nrows, nthreads, smp_row, &c);
    if (c.bad) return -2;
    return c.overflow ? 1 : 0;
}

/* ------------------------------------------------------------------------ */
/* O4' Top-M truncation, the baseline the abstract contrasts with SIP: keep  */
/* the M blocks with the largest estimate (ranked on the same 48-bit fixed   */
/* point as the sampler, ties to the lower block index), ascending, each     */
/* with log-weight 0 (no reweighting).  M >= nK keeps every block.          */
/* ------------------------------------------------------------------------ */

typedef struct { int64_t P; int32_t b; } rank_t;

static int rank_cmp(const void *x, const void *y)
{
    const rank_t *a = (const rank_t *)x, *c = (const rank_t *)y;
    if (a->P != c->P) return a->P > c->P ? -1 : 1;  /* larger estimate first */
    return a->b < c->b ? -1 : (a->b > c->b);        /* then lower index */
}

static int topk_row(const float *p, int nK, int budget_bp, int capacity, int32_t *count,
                    int32_t *idx, float *logw, int *overflow)
{
    const int64_t M = orc_budget_blocks(budget_bp, nK);
    const int keep = M >= nK ? nK : (int)M;
    rank_t *r = (rank_t *)malloc(sizeof(rank_t) * (size_t)nK);
    uint8_t *take = (uint8_t *)calloc((size_t)nK, 1);
    if (!r || !take) { free(r); free(take); return -3; }
    for (int b = 0; b < nK; ++b) { r[b].P = to_fixed(p[b]); r[b].b = b; }
    qsort(r, (size_t)nK, sizeof(rank_t), rank_cmp);
    for (int k = 0; k < keep; ++k) take[r[k].b] = 1;
    int n = 0;
    *overflow = 0;
    for (int b = 0; b < nK; ++b) {
        if (!take[b]) continue;
        if (n < capacity) { idx[n] = b; logw[n] = 0.0f; ++n; }
        else *overflow = 1;
    }
    *count = n;
    free(r); free(take);
    return 0;
}

typedef struct {
    const float *p;
    int nK, budget_bp, capacity;
    int32_t *counts, *idx;
    float *logw;
    int bad, overflow;
} topk_ctx;

static void topk_job(void *vctx, int64_t k)
{
    topk_ctx *c = (topk_ctx *)vctx;
    int of = 0;
    size_t o = (size_t)k * c->capacity;
    if (topk_row(c->p + (size_t)k * c->nK, c->nK, c->budget_bp, c->capacity, c->counts + k,
                 c->idx + o, c->logw + o, &of))
        c->bad = 1;
    if (of) __atomic_store_n(&c->overflow, 1, __ATOMIC_RELAXED);
}

/* p is [nrows][nK].  Returns 1 if some row kept more blocks than `capacity`. */
int orc_topk(const float *p, int64_t nrows, int nK, int budget_bp, int capacity, int nthreads,
             int32_t *counts, int32_t *idx, float *logw)
{
    if (!p || !counts || !idx || !logw || nK <= 0 || nK > 32767 || capacity < 0 || budget_bp < 0)
        return -1;
    topk_ctx c;
    memset(&c, 0, sizeof c);
    c.p = p; c.nK = nK; c.budget_bp = budget_bp; c.capacity = capacity;
    c.counts = counts; c.idx = idx; c.logw = logw;
    parallel_for(nrows, nthreads, topk_job, &c);
    if (c.bad) return -2;
    return c.overflow ? 1 : 0;
}

/* ------------------------------------------------------------------------ */
/* O5  attention restricted to the drawn blocks, each logit shifted by its   */
/* block's log-weight -ln(pi_b) (multiplying its exponential by 1/pi_b).     */
/* Numerator and denominator are then Horvitz-Thompson estimates of the      */
/* dense ones, and their ratio estimates the dense output (abstract: one     */
/* pass estimates dense attention instead of truncating it).                 */
/*                                                                           */
/* Outputs per valid query row r of the block (rows past `nq_max` skipped):  */
/*   O[r]   = sum e^{l-m} v / sum e^{l-m}   (0 for an empty list)            */
/*   lse[r] = m + ln sum e^{l-m}            (-inf for an empty list)         */
/*   num[r], den[r] (optional): the same sums taken relative to the DENSE    */
/*   row maximum of s*q.k over all keys, for the unbiasedness checks.        */
/* logw is given in double so exact weights can be fed in tests.            */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t *Q, *K, *V;
    geom_t g;
    double scale;
    const int64_t *rows;
    const int32_t *counts, *idx;
    const double *logw;
    int capacity, nq_max;
    double *O, *lse, *num, *den;
    int bad;
} ht_ctx;

static void ht_row(void *vctx, int64_t k)
{
    ht_ctx *c = (ht_ctx *)vctx;
    const geom_t *g = &c->g;
    int beta, h, i;
    if (decode_row(g, c->rows[k], &beta, &h, &i)) { c->bad = 1; return; }
    const int d = g->d, n = rows_in_block(g, i);
    const int L = c->counts[k];
    const int32_t *idx = c->idx + (size_t)k * c->capacity;
    const double *lw = c->logw + (size_t)k * c->capacity;
    if (L < 0 || L > c->capacity) { c->bad = 1; return; }
    for (int s = 0; s < L; ++s)
        if (idx[s] < 0 || idx[s] >= g->nK) { c->bad = 1; return; }
    double *O = c->O + (size_t)k * g->Bq * d;
    memset(O, 0, sizeof(double) * (size_t)g->Bq * d);
    if (c->lse)
        for (int r = 0; r < g->Bq; ++r) c->lse[(size_t)k * g->Bq + r] = -INFINITY;
    if (c->num) memset(c->num + (size_t)k * g->Bq * d, 0, sizeof(double) * (size_t)g->Bq * d);
    if (c->den) memset(c->den + (size_t)k * g->Bq, 0, sizeof(double) * (size_t)g->Bq);
    size_t nl = (size_t)L * g->Bk;
    double *l = (double *)malloc(sizeof(double) * (nl ? nl : 1));
    int *tk = (int *)malloc(sizeof(int) * (nl ? nl : 1));
    if (!l || !tk) { free(l); free(tk); c->bad = 1; return; }
    const int nr = n < c->nq_max ? n : c->nq_max;
    for (int r = 0; r < nr; ++r) {
        const uint16_t *q = tok(c->Q, g, beta, h, i * g->Bq + r);
        size_t cnt = 0;
        double m = -INFINITY;
        for (int s = 0; s < L; ++s) {
            const int b = idx[s];
            const int nb = keys_in_block(g, b);
            for (int u = 0; u < nb; ++u) {
                const int t = b * g->Bk + u;
                l[cnt] = c->scale * dot_bf(q, tok(c->K, g, beta, h, t), d) + lw[s];
                tk[cnt] = t;
                if (l[cnt] > m) m = l[cnt];
                ++cnt;
            }
        }
        double *o = O + (size_t)r * d;
        if (cnt > 0) {
            double sum = 0.0;
            for (size_t e = 0; e < cnt; ++e) {
                double w = exp(l[e] - m);
                sum += w;
                const uint16_t *v = tok(c->V, g, beta, h, tk[e]);
                for (int x = 0; x < d; ++x) o[x] += w * bf16_to_f64(v[x]);
            }
            for (int x = 0; x < d; ++x) o[x] /= sum;
            if (c->lse) c->lse[(size_t)k * g->Bq + r] = m + log(sum);
        }
        if (c->num || c->den) {
            double md = -INFINITY;
            for (int t = 0; t < g->N; ++t) {
                double z = c->scale * dot_bf(q, tok(c->K, g, beta, h, t), d);
                if (z > md) md = z;
            }
            double dsum = 0.0;
            double *nu = c->num ? c->num + ((size_t)k * g->Bq + r) * d : NULL;
            for (size_t e = 0; e < cnt; ++e) {
                double w = exp(l[e] - md);
                dsum += w;
                if (nu) {
                    const uint16_t *v = tok(c->V, g, beta, h, tk[e]);
                    for (int x = 0; x < d; ++x) nu[x] += w * bf16_to_f64(v[x]);
                }
            }
            if (c->den) c->den[(size_t)k * g->Bq + r] = dsum;
        }
    }
    free(l); free(tk);
}

int orc_ht_attention(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                     int B, int H, int N, int d, int Bq, int Bk, double scale,
                     const int64_t *rows, int64_t nrows,
                     const int32_t *counts, const int32_t *idx, const double *logw,
                     int capacity, int nq_max, int nthreads,
                     double *O, double *lse, double *num, double *den)
{
    ht_ctx c;
    memset(&c, 0, sizeof c);
    if (make_geom(&c.g, B, H, N, d, Bq, Bk)) return -1;
    if (!Q || !K || !V || !rows || !counts || !idx || !logw || !O || capacity < 0) return -1;
    c.Q = Q; c.K = K; c.V = V; c.scale = scale; c.rows = rows;
    c.counts = counts; c.idx = idx; c.logw = logw; c.capacity = capacity;
    c.nq_max = nq_max > 0 ? nq_max : Bq;
    c.O = O; c.lse = lse; c.num = num; c.den = den;
    parallel_for(nrows, nthreads, ht_row, &c);
    return c.bad ? -2 : 0;
}

/* ------------------------------------------------------------------------ */
/* Whole path for a set of rows: IBCS probabilities -> fp32 -> SIP draw ->   */
/* weighted attention.  Rows are independent, so each worker runs the       */
/* full chain for one row.                                                   */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t *Q, *K, *V;
    geom_t g;
    int C, iters, budget_bp, b_off, h_off;
    double scale;
    uint64_t seed;
    const int64_t *rows;
    float *p32;
    int32_t *counts, *idx;
    float *logw;
    double *O;
    int bad;
} fwd_ctx;

static void fwd_row(void *vctx, int64_t k)
{
    fwd_ctx *c = (fwd_ctx *)vctx;
    const geom_t *g = &c->g;
    int beta, h, i, of = 0;
    if (decode_row(g, c->rows[k], &beta, &h, &i)) { c->bad = 1; return; }
    const int nK = g->nK;
    double *p = (double *)malloc(sizeof(double) * (size_t)nK);
    double *lwd = (double *)malloc(sizeof(double) * (size_t)nK);
    if (!p || !lwd) { free(p); free(lwd); c->bad = 1; return; }
    float *p32 = c->p32 + (size_t)k * nK;
    int32_t *idx = c->idx + (size_t)k * nK;
    float *logw = c->logw + (size_t)k * nK;
    if (block_probs_row(c->Q, c->K, g, beta, h, i, c->C, c->iters, c->scale, 0, p)) {
        c->bad = 1;
    } else {
        for (int b = 0; b < nK; ++b) p32[b] = (float)p[b];
        if (sample_row(p32, g, beta + c->b_off, h + c->h_off, i, c->budget_bp, c->seed, 0, nK, c->counts + k, idx,
                       logw, NULL, &of))
            c->bad = 1;
        for (int s = 0; s < c->counts[k]; ++s) lwd[s] = (double)logw[s];
        ht_ctx hc;
        memset(&hc, 0, sizeof hc);
        hc.Q = c->Q; hc.K = c->K; hc.V = c->V; hc.g = *g; hc.scale = c->scale;
        hc.rows = c->rows + k; hc.counts = c->counts + k; hc.idx = idx; hc.logw = lwd;
        hc.capacity = nK; hc.nq_max = g->Bq; hc.O = c->O + (size_t)k * g->Bq * g->d;
        ht_row(&hc, 0);
        if (hc.bad) c->bad = 1;
    }
    free(p); free(lwd);
}

/* Outputs per listed row: p32 [nrows][nK], counts [nrows], idx/logw
 * [nrows][nK] (capacity nK), O [nrows][Bq][d].  b_off, h_off: global index
 * of the tensors' first batch element and head (the sampler's counter). */
int orc_forward(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                int B, int H, int N, int d, int Bq, int Bk, int C, int iters,
                int budget_bp, double scale, uint64_t seed,
                const int64_t *rows, int64_t nrows, int nthreads,
                float *p32, int32_t *counts, int32_t *idx, float *logw, double *O,
                int b_off, int h_off)
{
    fwd_ctx c;
    memset(&c, 0, sizeof c);
    if (make_geom(&c.g, B, H, N, d, Bq, Bk)) return -1;
    if (C <= 0 || C > Bq || iters < 0 || budget_bp < 0 || c.g.nK > 32767) return -1;
    if (b_off < 0 || h_off < 0) return -1;
    c.b_off = b_off; c.h_off = h_off;
    if (!Q || !K || !V || !rows || !p32 || !counts || !idx || !logw || !O) return -1;
    c.Q = Q; c.K = K; c.V = V; c.C = C; c.iters = iters; c.budget_bp = budget_bp;
    c.scale = scale; c.seed = seed; c.rows = rows;
    c.p32 = p32; c.counts = counts; c.idx = idx; c.logw = logw; c.O = O;
    parallel_for(nrows, nthreads, fwd_row, &c);
    return c.bad ? -2 : 0;
}
