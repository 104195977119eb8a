/*
 * DART forward path -- float64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the plain, slow, obviously correct
 * definition of what the DART forward path computes. Only tests/, the smoke
 * check and bench.py's CPU-baseline leg may load it. It shares no code, header,
 * constant or helper with the CUDA library, and it never calls into it.
 *
 * Source: "DART: Decoded Attention over Recurrent States for Efficient
 * Long-Context Sequence Modeling" (arXiv 2608.02032):
 *   - token recurrence ........... §2 "State Space Duality", eq (2); App. A eq (15)
 *   - decay products A_{u:v} ..... §2 eq (3); App. A eq (16) (identity when u > v)
 *   - chunk state memory dH[c] ... §3 "Chunk State Memories", eq (5); App. A eq (20)
 *   - state-memory attention ..... §3 "State-Memory Attention", eq (8)-(10)
 *   - normalised score branch .... App. B.1 "Normalization in DART", eq (25)-(27)
 *   - gated residual ............. §3 "Gated Residual Integration", eq (11)
 *   - empty history .............. §3 text after eq (10): R_t = 0 in the first chunk;
 *                                  Algorithm 1 step 16: logsumexp = -inf there.
 *
 * Everything is float64 and written as the definition reads: no blocking, no
 * fusion, no reordering. The only parallelism is over independent (batch, head)
 * pairs (or sampled tokens), one pthread per work item range.
 *
 * Layouts (row-major, contiguous, 0-based tokens and chunks; chunk(t) = t / S):
 *   X, E, Y, R, out : [batch, L, H, P]
 *   B, C, Q         : [batch, L, G, N]      head h reads group h / (H / G)
 *   logA            : [batch, L, H]         a_t = exp(logA_t)
 *   dH, Hend        : [batch, H, M, N, P]   M = ceil(L / S)
 *   lse             : [batch, H, L]
 *   g               : strided, index b*gsb + t*gst + h*gsh
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef int64_t i64;

/* ------------------------------------------------------------------ */
/* parallel-for over independent work items                            */
/* ------------------------------------------------------------------ */

typedef void (*item_fn)(void *ctx, i64 item, double *scratch);

typedef struct {
    item_fn fn;
    void *ctx;
    i64 n_items;
    i64 next;           /* shared counter, taken with __atomic_fetch_add */
    size_t scratch_len; /* doubles of per-thread scratch */
} pool_job;

static void *pool_worker(void *arg) {
    pool_job *job = (pool_job *)arg;
    double *scratch = job->scratch_len ? (double *)malloc(job->scratch_len * sizeof(double)) : NULL;
    for (;;) {
        i64 item = __atomic_fetch_add(&job->next, 1, __ATOMIC_RELAXED);
        if (item >= job->n_items) break;
        job->fn(job->ctx, item, scratch);
    }
    free(scratch);
    return NULL;
}

static void parallel_for(item_fn fn, void *ctx, i64 n_items, size_t scratch_len, int threads) {
    pool_job job = {fn, ctx, n_items, 0, scratch_len};
    if (threads < 1) threads = 1;
    if (threads > 256) threads = 256;
    if (threads == 1 || n_items <= 1) {
        pool_worker(&job);
        return;
    }
    pthread_t tid[256];
    int started = 0;
    for (int i = 0; i < threads; ++i) {
        if (pthread_create(&tid[i], NULL, pool_worker, &job) != 0) break;
        ++started;
    }
    if (started == 0) pool_worker(&job);
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
}

/* ------------------------------------------------------------------ */
/* shapes                                                              */
/* ------------------------------------------------------------------ */

typedef struct {
    i64 Bt, L, H, G, N, P, S, M;
} shape_t;

static shape_t make_shape(i64 Bt, i64 L, i64 H, i64 G, i64 N, i64 P, i64 S) {
    shape_t s = {Bt, L, H, G, N, P, S, (L + S - 1) / S};
    return s;
}

static i64 group_of(const shape_t *s, i64 h) { return h / (s->H / s->G); }
static i64 at_x(const shape_t *s, i64 b, i64 t, i64 h) { return ((b * s->L + t) * s->H + h) * s->P; }
static i64 at_b(const shape_t *s, i64 b, i64 t, i64 g) { return ((b * s->L + t) * s->G + g) * s->N; }
static i64 at_a(const shape_t *s, i64 b, i64 t, i64 h) { return (b * s->L + t) * s->H + h; }
static i64 at_state(const shape_t *s, i64 b, i64 h, i64 c) { return ((b * s->H + h) * s->M + c) * s->N * s->P; }
/* last token of chunk c, e(c) */
static i64 chunk_end(const shape_t *s, i64 c) {
    i64 e = (c + 1) * s->S - 1;
    return e < s->L ? e : s->L - 1;
}

/* ------------------------------------------------------------------ */
/* 1. token recurrence, eq (2):  H_t = a_t H_{t-1} + B_t^T X_t,  Y_t = C_t H_t  */
/* ------------------------------------------------------------------ */

typedef struct {
    shape_t s;
    const double *X, *B, *C, *logA;
    double *Y, *Hend, *Hfinal;
} rec_ctx;

static void recurrence_item(void *vctx, i64 item, double *Hs) {
    rec_ctx *c = (rec_ctx *)vctx;
    const shape_t *s = &c->s;
    i64 b = item / s->H, h = item % s->H, g = group_of(s, h);
    i64 NP = s->N * s->P;
    for (i64 k = 0; k < NP; ++k) Hs[k] = 0.0; /* H_{-1} = 0 */
    for (i64 t = 0; t < s->L; ++t) {
        double a = exp(c->logA[at_a(s, b, t, h)]);
        const double *Bt = c->B + at_b(s, b, t, g);
        const double *Ct = c->C + at_b(s, b, t, g);
        const double *Xt = c->X + at_x(s, b, t, h);
        for (i64 n = 0; n < s->N; ++n)
            for (i64 p = 0; p < s->P; ++p) Hs[n * s->P + p] = a * Hs[n * s->P + p] + Bt[n] * Xt[p];
        double *Yt = c->Y + at_x(s, b, t, h);
        for (i64 p = 0; p < s->P; ++p) {
            double acc = 0.0;
            for (i64 n = 0; n < s->N; ++n) acc += Ct[n] * Hs[n * s->P + p];
            Yt[p] = acc;
        }
        if (c->Hend && t == chunk_end(s, t / s->S))
            memcpy(c->Hend + at_state(s, b, h, t / s->S), Hs, (size_t)NP * sizeof(double));
    }
    if (c->Hfinal) memcpy(c->Hfinal + (b * s->H + h) * NP, Hs, (size_t)NP * sizeof(double));
}

void dart_oracle_recurrence(i64 Bt, i64 L, i64 H, i64 G, i64 N, i64 P, i64 S, const double *X, const double *B,
                            const double *C, const double *logA, double *Y, double *Hend, double *Hfinal,
                            int threads) {
    rec_ctx ctx = {make_shape(Bt, L, H, G, N, P, S), X, B, C, logA, Y, Hend, Hfinal};
    parallel_for(recurrence_item, &ctx, Bt * H, (size_t)(N * P), threads);
}

/* ------------------------------------------------------------------ */
/* 2. chunk state memories by direct summation, eq (5):                */
/*    dH[c] = sum_{s in c} A_{s+1:e(c)} B_s^T X_s,                     */
/*    A_{s+1:e(c)} = exp(sum_{r=s+1}^{e(c)} logA_r)  (empty sum -> 1)  */
/* ------------------------------------------------------------------ */

typedef struct {
    shape_t s;
    const double *X, *B, *logA;
    double *dH;
} cs_ctx;

static void chunk_states_item(void *vctx, i64 item, double *unused) {
    (void)unused;
    cs_ctx *c = (cs_ctx *)vctx;
    const shape_t *s = &c->s;
    i64 b = item / s->H, h = item % s->H, g = group_of(s, h);
    for (i64 ch = 0; ch < s->M; ++ch) {
        double *D = c->dH + at_state(s, b, h, ch);
        for (i64 k = 0; k < s->N * s->P; ++k) D[k] = 0.0;
        i64 first = ch * s->S, e = chunk_end(s, ch);
        for (i64 t = first; t <= e; ++t) {
            double logw = 0.0;
            for (i64 r = t + 1; r <= e; ++r) logw += c->logA[at_a(s, b, r, h)];
            double w = exp(logw);
            const double *Bs = c->B + at_b(s, b, t, g);
            const double *Xs = c->X + at_x(s, b, t, h);
            for (i64 n = 0; n < s->N; ++n)
                for (i64 p = 0; p < s->P; ++p) D[n * s->P + p] += w * Bs[n] * Xs[p];
        }
    }
}

void dart_oracle_chunk_states(i64 Bt, i64 L, i64 H, i64 G, i64 N, i64 P, i64 S, const double *X, const double *B,
                              const double *logA, double *dH, int threads) {
    cs_ctx ctx = {make_shape(Bt, L, H, G, N, P, S), X, B, logA, dH};
    parallel_for(chunk_states_item, &ctx, Bt * H, 0, threads);
}

/* ------------------------------------------------------------------ */
/* 3. state-memory attention, eq (8)-(10), one token at a time:        */
/*    for c < chunk(t):  V = C_t dH[c],  K = dH[c] E_t,                */
/*                       l_c = Q_t K / sqrt(N)                         */
/*    R_t = sum_c softmax_c(l) V_c,  lse_t = log sum_c exp(l_c)        */
/*    no history (chunk(t) = 0): R_t = 0, lse_t = -inf                 */
/* ------------------------------------------------------------------ */

typedef struct {
    i64 N, P;
} np_t;

/* SMA for one query (q, c_read, e) over memories mem[0..k-1] (each N x P). */
static void sma_one(np_t d, const double *q, const double *cr, const double *e, const double *mem, i64 mem_stride,
                    i64 k, double *R, double *lse, double *scratch) {
    double *logit = scratch;      /* k */
    double *V = scratch + k;      /* k x P */
    double *K = V + k * d.P;      /* N */
    if (k == 0) {
        for (i64 p = 0; p < d.P; ++p) R[p] = 0.0;
        *lse = -INFINITY;
        return;
    }
    for (i64 c = 0; c < k; ++c) {
        const double *D = mem + c * mem_stride;
        for (i64 p = 0; p < d.P; ++p) { /* value-side readout C_t dH[c] */
            double acc = 0.0;
            for (i64 n = 0; n < d.N; ++n) acc += cr[n] * D[n * d.P + p];
            V[c * d.P + p] = acc;
        }
        for (i64 n = 0; n < d.N; ++n) { /* key-side readout dH[c] E_t */
            double acc = 0.0;
            for (i64 p = 0; p < d.P; ++p) acc += D[n * d.P + p] * e[p];
            K[n] = acc;
        }
        double l = 0.0;
        for (i64 n = 0; n < d.N; ++n) l += q[n] * K[n];
        logit[c] = l / sqrt((double)d.N);
    }
    /* stable softmax over the k historical chunks (App. C eq (28)) and its logsumexp (eq (32)) */
    double m = logit[0];
    for (i64 c = 1; c < k; ++c) m = logit[c] > m ? logit[c] : m;
    double den = 0.0;
    for (i64 c = 0; c < k; ++c) den += exp(logit[c] - m);
    *lse = m + log(den);
    for (i64 c = 0; c < k; ++c) logit[c] = exp(logit[c] - m) / den; /* now the weights g_{t,c} */
    for (i64 p = 0; p < d.P; ++p) {
        double acc = 0.0;
        for (i64 c = 0; c < k; ++c) acc += logit[c] * V[c * d.P + p];
        R[p] = acc;
    }
}

typedef struct {
    shape_t s;
    const double *Q, *C, *E, *dH;
    const i64 *tokens; /* NULL: every token */
    i64 ntok;
    double *R, *lse;
} sma_ctx;

static void sma_item(void *vctx, i64 item, double *scratch) {
    sma_ctx *c = (sma_ctx *)vctx;
    const shape_t *s = &c->s;
    i64 nt = c->tokens ? c->ntok : s->L;
    i64 bh = item / nt, j = item % nt;
    i64 b = bh / s->H, h = bh % s->H, g = group_of(s, h);
    i64 t = c->tokens ? c->tokens[j] : j;
    np_t d = {s->N, s->P};
    double *R = c->R + ((b * nt + j) * s->H + h) * s->P;
    double *lse = c->lse + (b * s->H + h) * nt + j;
    sma_one(d, c->Q + at_b(s, b, t, g), c->C + at_b(s, b, t, g), c->E + at_x(s, b, t, h),
            c->dH + at_state(s, b, h, 0), s->N * s->P, t / s->S, R, lse, scratch);
}

/* tokens == NULL: R [Bt, L, H, P], lse [Bt, H, L].
 * tokens != NULL: R [Bt, ntok, H, P], lse [Bt, H, ntok] for the listed token indices. */
void dart_oracle_sma(i64 Bt, i64 L, i64 H, i64 G, i64 N, i64 P, i64 S, const double *Q, const double *C,
                     const double *E, const double *dH, const i64 *tokens, i64 ntok, double *R, double *lse,
                     int threads) {
    sma_ctx ctx = {make_shape(Bt, L, H, G, N, P, S), Q, C, E, dH, tokens, ntok, R, lse};
    i64 nt = tokens ? ntok : L;
    i64 M = (L + S - 1) / S;
    parallel_for(sma_item, &ctx, Bt * H * nt, (size_t)(M + M * P + N), threads);
}

/* ------------------------------------------------------------------ */
/* 3b. state-memory attention with the normalised score branch         */
/*     (App. B.1 eq (25)-(27)), one token at a time:                   */
/*     Qb = Q_t / sqrt(mean_n Q_t^2 + eps), Eb likewise over p (eq 25) */
/*     r_{c,n} = (mean_p dH[c]_{n,p}^2 + eps)^(-1/2)                   */
/*     K = r_c (.) (dH[c] Eb),  l_c = Qb K / sqrt(N)         (eq 26-27) */
/*     V = C_t dH[c] (the value side is not normalised); softmax as 3. */
/*     RMSNorm carries no weight (unit weight).                        */
/* ------------------------------------------------------------------ */

static void sma_one_norm(np_t d, double eps, const double *q, const double *cr, const double *e, const double *mem,
                         i64 mem_stride, i64 k, double *R, double *lse, double *scratch) {
    double *logit = scratch;      /* k */
    double *V = scratch + k;      /* k x P */
    double *K = V + k * d.P;      /* N */
    double *qb = K + d.N;         /* N */
    double *eb = qb + d.N;        /* P */
    if (k == 0) {
        for (i64 p = 0; p < d.P; ++p) R[p] = 0.0;
        *lse = -INFINITY;
        return;
    }
    double sq = 0.0;
    for (i64 n = 0; n < d.N; ++n) sq += q[n] * q[n];
    double inv_q = 1.0 / sqrt(sq / (double)d.N + eps);
    for (i64 n = 0; n < d.N; ++n) qb[n] = q[n] * inv_q;
    double se = 0.0;
    for (i64 p = 0; p < d.P; ++p) se += e[p] * e[p];
    double inv_e = 1.0 / sqrt(se / (double)d.P + eps);
    for (i64 p = 0; p < d.P; ++p) eb[p] = e[p] * inv_e;
    for (i64 c = 0; c < k; ++c) {
        const double *D = mem + c * mem_stride;
        for (i64 p = 0; p < d.P; ++p) { /* value-side readout C_t dH[c] */
            double acc = 0.0;
            for (i64 n = 0; n < d.N; ++n) acc += D[n * d.P + p] * cr[n];
            V[c * d.P + p] = acc;
        }
        for (i64 n = 0; n < d.N; ++n) { /* key K_{t,c} = r_c (.) (dH[c] Eb) */
            double acc = 0.0, row_sq = 0.0;
            for (i64 p = 0; p < d.P; ++p) {
                acc += D[n * d.P + p] * eb[p];
                row_sq += D[n * d.P + p] * D[n * d.P + p];
            }
            double r = 1.0 / sqrt(row_sq / (double)d.P + eps);
            K[n] = r * acc;
        }
        double l = 0.0;
        for (i64 n = 0; n < d.N; ++n) l += qb[n] * K[n];
        logit[c] = l * (1.0 / sqrt((double)d.N)); /* eq (27) */
    }
    double m = logit[0];
    for (i64 c = 1; c < k; ++c) m = logit[c] > m ? logit[c] : m;
    double den = 0.0;
    for (i64 c = 0; c < k; ++c) den = den + exp(logit[c] - m);
    *lse = m + log(den);
    for (i64 c = 0; c < k; ++c) logit[c] = exp(logit[c] - m) / den;
    for (i64 p = 0; p < d.P; ++p) {
        double acc = 0.0;
        for (i64 c = 0; c < k; ++c) acc += logit[c] * V[c * d.P + p];
        R[p] = acc;
    }
}

typedef struct {
    sma_ctx base;
    double eps;
} sma_norm_ctx;

static void sma_norm_item(void *vctx, i64 item, double *scratch) {
    sma_norm_ctx *cn = (sma_norm_ctx *)vctx;
    sma_ctx *c = &cn->base;
    const shape_t *s = &c->s;
    i64 nt = c->tokens ? c->ntok : s->L;
    i64 bh = item / nt, j = item % nt;
    i64 b = bh / s->H, h = bh % s->H, g = group_of(s, h);
    i64 t = c->tokens ? c->tokens[j] : j;
    np_t d = {s->N, s->P};
    double *R = c->R + ((b * nt + j) * s->H + h) * s->P;
    double *lse = c->lse + (b * s->H + h) * nt + j;
    i64 history = t / s->S; /* the chunks before chunk(t) */
    sma_one_norm(d, cn->eps, c->Q + at_b(s, b, t, g), c->C + at_b(s, b, t, g), c->E + at_x(s, b, t, h),
                 c->dH + at_state(s, b, h, 0), s->N * s->P, history, R, lse, scratch);
}

/* Layouts as dart_oracle_sma; eps > 0 enters every RMS of eq (25)-(26). */
void dart_oracle_sma_norm(i64 Bt, i64 L, i64 H, i64 G, i64 N, i64 P, i64 S, double eps, const double *Q,
                          const double *C, const double *E, const double *dH, const i64 *tokens, i64 ntok, double *R,
                          double *lse, int threads) {
    sma_norm_ctx ctx = {{make_shape(Bt, L, H, G, N, P, S), Q, C, E, dH, tokens, ntok, R, lse}, eps};
    i64 nt = tokens ? ntok : L;
    i64 M = (L + S - 1) / S;
    parallel_for(sma_norm_item, &ctx, Bt * H * nt, (size_t)(M + M * P + 2 * N + P), threads);
}

/* ------------------------------------------------------------------ */
/* 4. gated residual, eq (11): out_t = Y_t + g_t R_t                   */
/* ------------------------------------------------------------------ */

void dart_oracle_combine(i64 Bt, i64 L, i64 H, i64 P, const double *Y, const double *R, const double *g, i64 gsb,
                         i64 gst, i64 gsh, double *out) {
    for (i64 b = 0; b < Bt; ++b)
        for (i64 t = 0; t < L; ++t)
            for (i64 h = 0; h < H; ++h) {
                double gv = g[b * gsb + t * gst + h * gsh];
                i64 o = ((b * L + t) * H + h) * P;
                for (i64 p = 0; p < P; ++p) out[o + p] = Y[o + p] + gv * R[o + p];
            }
}

/* ------------------------------------------------------------------ */
/* 5. single-token decode: SMA of one new token over every cached      */
/*    chunk memory (all cached chunks are complete, so all are         */
/*    historical), then the gated residual.                            */
/*    Q, C [Bt, G, N]; E, Y, out [Bt, H, P]; cache [Bt, H, cs, N, P];  */
/*    lse [Bt, H]; g index b*gsb + h*gsh.                              */
/* ------------------------------------------------------------------ */

typedef struct {
    i64 Bt, H, G, N, P, n_chunks, chunk_stride;
    const double *Q, *C, *E, *Y, *g;
    i64 gsb, gsh;
    const double *cache;
    double *out, *lse;
} dec_ctx;

static void decode_item(void *vctx, i64 item, double *scratch) {
    dec_ctx *c = (dec_ctx *)vctx;
    i64 b = item / c->H, h = item % c->H, g = h / (c->H / c->G);
    np_t d = {c->N, c->P};
    double *R = scratch;
    double *rest = scratch + c->P;
    const double *mem = c->cache + ((b * c->H + h) * c->chunk_stride) * c->N * c->P;
    double lse;
    sma_one(d, c->Q + (b * c->G + g) * c->N, c->C + (b * c->G + g) * c->N, c->E + (b * c->H + h) * c->P, mem,
            c->N * c->P, c->n_chunks, R, &lse, rest);
    double gv = c->g[b * c->gsb + h * c->gsh];
    for (i64 p = 0; p < c->P; ++p) c->out[(b * c->H + h) * c->P + p] = c->Y[(b * c->H + h) * c->P + p] + gv * R[p];
    c->lse[b * c->H + h] = lse;
}

void dart_oracle_decode(i64 Bt, i64 H, i64 G, i64 N, i64 P, i64 n_chunks, i64 chunk_stride, const double *Q,
                        const double *C, const double *E, const double *Y, const double *g, i64 gsb, i64 gsh,
                        const double *cache, double *out, double *lse, int threads) {
    dec_ctx ctx = {Bt, H, G, N, P, n_chunks, chunk_stride, Q, C, E, Y, g, gsb, gsh, cache, out, lse};
    parallel_for(decode_item, &ctx, Bt * H, (size_t)(P + n_chunks + n_chunks * P + N), threads);
}

/* ------------------------------------------------------------------ */
/* 6. one decode step with its state maintenance (§4 "Inference        */
/*    Cache": the recurrent state and the chunk memories are cached;   */
/*    §2 eq (2) in recurrent form):                                    */
/*      a     = exp(logA)                                              */
/*      state = a state + B^T X        (the full state H_t)            */
/*      acc   = a acc   + B^T X        (the memory of the open chunk,  */
/*                                      eq (5) accumulated token by    */
/*                                      token from zero at its start)  */
/*      Y     = C state                                                */
/*      out   = Y + g R, R over cache chunks [0, n_chunks) (section 5) */
/*    and, when the token is the last of its chunk, cache[n_chunks] =  */
/*    acc and acc = 0.                                                 */
/*    X, E, out [Bt, H, P]; B, C, Q [Bt, G, N]; logA, lse [Bt, H];     */
/*    state, acc [Bt, H, N, P]; cache [Bt, H, cs, N, P].               */
/* ------------------------------------------------------------------ */

void dart_oracle_decode_step(i64 Bt, i64 H, i64 G, i64 N, i64 P, i64 n_chunks, i64 chunk_stride, int close_chunk,
                             const double *X, const double *B, const double *C, const double *Q, const double *E,
                             const double *logA, const double *g, i64 gsb, i64 gsh, double *state, double *acc,
                             double *cache, double *out, double *lse, int threads) {
    double *Y = (double *)malloc((size_t)(Bt * H * P) * sizeof(double));
    for (i64 b = 0; b < Bt; ++b)
        for (i64 h = 0; h < H; ++h) {
            i64 grp = h / (H / G);
            double a = exp(logA[b * H + h]);
            const double *Bv = B + (b * G + grp) * N, *Cv = C + (b * G + grp) * N, *Xv = X + (b * H + h) * P;
            double *st = state + (b * H + h) * N * P, *ac = acc + (b * H + h) * N * P;
            for (i64 n = 0; n < N; ++n)
                for (i64 p = 0; p < P; ++p) {
                    st[n * P + p] = a * st[n * P + p] + Bv[n] * Xv[p];
                    ac[n * P + p] = a * ac[n * P + p] + Bv[n] * Xv[p];
                }
            for (i64 p = 0; p < P; ++p) {
                double y = 0.0;
                for (i64 n = 0; n < N; ++n) y += Cv[n] * st[n * P + p];
                Y[(b * H + h) * P + p] = y;
            }
        }
    dart_oracle_decode(Bt, H, G, N, P, n_chunks, chunk_stride, Q, C, E, Y, g, gsb, gsh, cache, out, lse, threads);
    if (close_chunk)
        for (i64 b = 0; b < Bt; ++b)
            for (i64 h = 0; h < H; ++h) {
                double *ac = acc + (b * H + h) * N * P;
                double *slot = cache + ((b * H + h) * chunk_stride + n_chunks) * N * P;
                for (i64 e = 0; e < N * P; ++e) {
                    slot[e] = ac[e];
                    ac[e] = 0.0;
                }
            }
    free(Y);
}

/* ------------------------------------------------------------------ */
/* 7. SMA backward (§4 "Efficient Training": gradients of the readout  */
/*    by recomputation; App. C eq (32)-(35)). For one token t with      */
/*    k = chunk(t) >= 1, the forward of 3. is, per head,                */
/*      V_c = C_t dH[c],  K_c = dH[c] E_t,  l_c = Q_t . K_c / sqrt(N),  */
/*      w = softmax(l),   R_t = sum_c w_c V_c,                          */
/*    and the gradient dR_t of a loss w.r.t. R_t flows back by the      */
/*    chain rule, with dw_c = dR_t . V_c and the softmax Jacobian       */
/*      dl_c = w_c (dw_c - sum_c' w_c' dw_c') = w_c (dw_c - dR_t . R_t):*/
/*      dC_t    += w_c dH[c] dR_t            (through V_c)              */
/*      ddH[c]  += w_c C_t^T dR_t            (through V_c)              */
/*      dQ_t    += dl_c K_c / sqrt(N)        (through l_c)              */
/*      dE_t    += dl_c dH[c]^T Q_t / sqrt(N)                           */
/*      ddH[c]  += dl_c Q_t^T E_t / sqrt(N)                             */
/*    The weights are recomputed here from scratch (own max and sum).   */
/*    Q and C are shared by the heads of a group, so dQ and dC sum the  */
/*    contributions of every head of the group; one work item is one    */
/*    (batch, group), which owns all the outputs it writes. lse is a    */
/*    statistic of the forward and takes no gradient.                   */
/* ------------------------------------------------------------------ */

typedef struct {
    shape_t s;
    const double *Q, *C, *E, *dH, *dR;
    double *dQ, *dC, *dE, *ddH;
} sma_bwd_ctx;

/* The chain rule for one token t of head h (batch row b), added into dq, dc (N) and de (P) when they are
 * not NULL, and into the chunk memories' gradients dD (M x N x P) when not NULL: every historical chunk,
 * or only chunk `only` when only >= 0. scratch holds M + M P + M N + P doubles. */
static void bwd_token(const sma_bwd_ctx *c, i64 b, i64 h, i64 t, double *dq, double *dc, double *de, double *dD,
                      i64 only, double *scratch) {
    const shape_t *s = &c->s;
    const i64 N = s->N, P = s->P, M = s->M;
    const i64 g = group_of(s, h);
    const i64 k = t / s->S;
    if (k == 0) return; /* R_t = 0 does not depend on any input */
    const double rs = 1.0 / sqrt((double)N);
    double *w = scratch;        /* M: logits, then weights */
    double *V = w + M;          /* M x P */
    double *K = V + M * P;      /* M x N */
    double *Rt = K + M * N;     /* P */
    const double *q = c->Q + at_b(s, b, t, g), *cr = c->C + at_b(s, b, t, g);
    const double *e = c->E + at_x(s, b, t, h), *dr = c->dR + at_x(s, b, t, h);
    /* recompute the forward for this token */
    for (i64 ch = 0; ch < k; ++ch) {
        const double *D = c->dH + at_state(s, b, h, ch);
        for (i64 p = 0; p < P; ++p) {
            double acc = 0.0;
            for (i64 n = 0; n < N; ++n) acc += cr[n] * D[n * P + p];
            V[ch * P + p] = acc;
        }
        double l = 0.0;
        for (i64 n = 0; n < N; ++n) {
            double acc = 0.0;
            for (i64 p = 0; p < P; ++p) acc += D[n * P + p] * e[p];
            K[ch * N + n] = acc;
            l += q[n] * acc;
        }
        w[ch] = l * rs;
    }
    double m = w[0];
    for (i64 ch = 1; ch < k; ++ch) m = w[ch] > m ? w[ch] : m;
    double den = 0.0;
    for (i64 ch = 0; ch < k; ++ch) den += exp(w[ch] - m);
    for (i64 ch = 0; ch < k; ++ch) w[ch] = exp(w[ch] - m) / den;
    for (i64 p = 0; p < P; ++p) {
        double acc = 0.0;
        for (i64 ch = 0; ch < k; ++ch) acc += w[ch] * V[ch * P + p];
        Rt[p] = acc;
    }
    double dRR = 0.0; /* sum_c w_c dw_c = dR_t . R_t */
    for (i64 p = 0; p < P; ++p) dRR += dr[p] * Rt[p];
    /* chain rule, chunk by chunk */
    for (i64 ch = 0; ch < k; ++ch) {
        const double *D = c->dH + at_state(s, b, h, ch);
        double dw = 0.0;
        for (i64 p = 0; p < P; ++p) dw += dr[p] * V[ch * P + p];
        const double dl = w[ch] * (dw - dRR);
        if (dc || dq) {
            for (i64 n = 0; n < N; ++n) {
                double acc = 0.0;
                for (i64 p = 0; p < P; ++p) acc += D[n * P + p] * dr[p];
                if (dc) dc[n] += w[ch] * acc;
                if (dq) dq[n] += dl * rs * K[ch * N + n];
            }
        }
        if (de) {
            for (i64 p = 0; p < P; ++p) {
                double acc = 0.0;
                for (i64 n = 0; n < N; ++n) acc += D[n * P + p] * q[n];
                de[p] += dl * rs * acc;
            }
        }
        if (dD && (only < 0 || only == ch)) {
            double *dd = dD + (only < 0 ? ch * N * P : 0);
            for (i64 n = 0; n < N; ++n)
                for (i64 p = 0; p < P; ++p) dd[n * P + p] += w[ch] * cr[n] * dr[p] + dl * rs * q[n] * e[p];
        }
    }
}

static void sma_bwd_item(void *vctx, i64 item, double *scratch) {
    sma_bwd_ctx *c = (sma_bwd_ctx *)vctx;
    const shape_t *s = &c->s;
    const i64 N = s->N, P = s->P, M = s->M;
    const i64 b = item / s->G, g = item % s->G;
    const i64 hpg = s->H / s->G;
    for (i64 t = 0; t < s->L; ++t) { /* this item's dQ, dC rows start at zero */
        memset(c->dQ + at_b(s, b, t, g), 0, (size_t)N * sizeof(double));
        memset(c->dC + at_b(s, b, t, g), 0, (size_t)N * sizeof(double));
    }
    for (i64 h = g * hpg; h < (g + 1) * hpg; ++h) {
        memset(c->ddH + at_state(s, b, h, 0), 0, (size_t)(M * N * P) * sizeof(double));
        for (i64 t = 0; t < s->L; ++t) memset(c->dE + at_x(s, b, t, h), 0, (size_t)P * sizeof(double));
        for (i64 t = 0; t < s->L; ++t)
            bwd_token(c, b, h, t, c->dQ + at_b(s, b, t, g), c->dC + at_b(s, b, t, g), c->dE + at_x(s, b, t, h),
                      c->ddH + at_state(s, b, h, 0), -1, scratch);
    }
}

/* dQ, dC [Bt, L, G, N]; dE [Bt, L, H, P]; ddH [Bt, H, M, N, P]; every element is written. */
void dart_oracle_sma_bwd(i64 Bt, i64 L, i64 H, i64 G, i64 N, i64 P, i64 S, const double *Q, const double *C,
                         const double *E, const double *dH, const double *dR, double *dQ, double *dC, double *dE,
                         double *ddH, int threads) {
    sma_bwd_ctx ctx = {make_shape(Bt, L, H, G, N, P, S), Q, C, E, dH, dR, dQ, dC, dE, ddH};
    const i64 M = (L + S - 1) / S;
    parallel_for(sma_bwd_item, &ctx, Bt * G, (size_t)(M + M * P + M * N + P), threads);
}

/* Sampled backward, per-token gradients only: for every batch row b and listed token tokens[j],
 * dQs, dCs [Bt, ntok, G, N] and dEs [Bt, ntok, H, P] (item = (b, j), all heads). */
typedef struct {
    sma_bwd_ctx base;
    const i64 *tokens;
    i64 ntok;
} sma_bwd_tok_ctx;

static void sma_bwd_tok_item(void *vctx, i64 item, double *scratch) {
    sma_bwd_tok_ctx *ct = (sma_bwd_tok_ctx *)vctx;
    const sma_bwd_ctx *c = &ct->base;
    const shape_t *s = &c->s;
    const i64 b = item / ct->ntok, j = item % ct->ntok, t = ct->tokens[j];
    for (i64 g = 0; g < s->G; ++g) {
        double *dq = c->dQ + ((b * ct->ntok + j) * s->G + g) * s->N, *dc = c->dC + ((b * ct->ntok + j) * s->G + g) * s->N;
        memset(dq, 0, (size_t)s->N * sizeof(double));
        memset(dc, 0, (size_t)s->N * sizeof(double));
    }
    for (i64 h = 0; h < s->H; ++h) {
        double *de = c->dE + ((b * ct->ntok + j) * s->H + h) * s->P;
        memset(de, 0, (size_t)s->P * sizeof(double));
        const i64 g = group_of(s, h);
        bwd_token(c, b, h, t, c->dQ + ((b * ct->ntok + j) * s->G + g) * s->N,
                  c->dC + ((b * ct->ntok + j) * s->G + g) * s->N, de, NULL, -1, scratch);
    }
}

void dart_oracle_sma_bwd_tokens(i64 Bt, i64 L, i64 H, i64 G, i64 N, i64 P, i64 S, const double *Q, const double *C,
                                const double *E, const double *dH, const double *dR, const i64 *tokens, i64 ntok,
                                double *dQs, double *dCs, double *dEs, int threads) {
    sma_bwd_tok_ctx ctx = {{make_shape(Bt, L, H, G, N, P, S), Q, C, E, dH, dR, dQs, dCs, dEs, NULL}, tokens, ntok};
    const i64 M = (L + S - 1) / S;
    parallel_for(sma_bwd_tok_item, &ctx, Bt * ntok, (size_t)(M + M * P + M * N + P), threads);
}

/* Sampled backward, chunk-memory gradients only: ddHs [n, N, P] for the listed (b, h, c) triples, each
 * summed over every later token (item = one triple). */
typedef struct {
    sma_bwd_ctx base;
    const i64 *trip;
} sma_bwd_ddh_ctx;

static void sma_bwd_ddh_item(void *vctx, i64 item, double *scratch) {
    sma_bwd_ddh_ctx *cd = (sma_bwd_ddh_ctx *)vctx;
    const sma_bwd_ctx *c = &cd->base;
    const shape_t *s = &c->s;
    const i64 b = cd->trip[3 * item], h = cd->trip[3 * item + 1], ch = cd->trip[3 * item + 2];
    double *dd = c->ddH + item * s->N * s->P;
    memset(dd, 0, (size_t)(s->N * s->P) * sizeof(double));
    for (i64 t = (ch + 1) * s->S; t < s->L; ++t) bwd_token(c, b, h, t, NULL, NULL, NULL, dd, ch, scratch);
}

void dart_oracle_sma_bwd_ddh(i64 Bt, i64 L, i64 H, i64 G, i64 N, i64 P, i64 S, const double *Q, const double *C,
                             const double *E, const double *dH, const double *dR, const i64 *triples, i64 n,
                             double *ddHs, int threads) {
    sma_bwd_ddh_ctx ctx = {{make_shape(Bt, L, H, G, N, P, S), Q, C, E, dH, dR, NULL, NULL, NULL, ddHs}, triples};
    const i64 M = (L + S - 1) / S;
    parallel_for(sma_bwd_ddh_item, &ctx, n, (size_t)(M + M * P + M * N + P), threads);
}

/* ------------------------------------------------------------------ */
/* 8. backward of the normalised score branch (App. B.1 eq (25)-(27)), */
/*    by the chain rule with the weights recomputed, for one token t    */
/*    of head h. The forward of 3b. is                                  */
/*      Qb = iq Q_t, iq = (mean_n Q_t^2 + eps)^(-1/2); Eb = ie E_t      */
/*      r_{c,n} = (mean_p dH[c]_{n,p}^2 + eps)^(-1/2)                   */
/*      K_c = r_c (.) (dH[c] Eb), l_c = Qb . K_c / sqrt(N)              */
/*      V_c = C_t dH[c], w = softmax(l), R_t = sum_c w_c V_c            */
/*    With dl_c = w_c (dR_t . V_c - dR_t . R_t) (as in 7.):             */
/*      dQb += dl_c K_c / sqrt(N),                                      */
/*      dEb += dl_c dH[c]^T (r_c (.) Qb) / sqrt(N),                     */
/*      ddH[c]_{n,p} += dl_c Qb_n / sqrt(N) (r_n Eb_p                   */
/*                      - r_n^3 (dH[c] Eb)_n dH[c]_{n,p} / P)           */
/*    (d r_n / d dH_{n,p} = -r_n^3 dH_{n,p} / P), the value path as in  */
/*    7., and through the two RMSNorms                                  */
/*      dQ_t = iq dQb - iq^3 Q_t (Q_t . dQb) / N, dE_t likewise over P. */
/* ------------------------------------------------------------------ */

typedef struct {
    sma_bwd_ctx base;
    double eps;
} sma_bwd_norm_ctx;

static void bwd_token_norm(const sma_bwd_ctx *c, double eps, i64 b, i64 h, i64 t, double *dq, double *dc,
                           double *de, double *dD, double *scratch) {
    const shape_t *s = &c->s;
    const i64 N = s->N, P = s->P, M = s->M;
    const i64 g = group_of(s, h);
    const i64 k = t / s->S;
    if (k == 0) return;
    const double rs = 1.0 / sqrt((double)N);
    double *w = scratch;        /* M */
    double *V = w + M;          /* M x P */
    double *K = V + M * P;      /* M x N: r_c (.) (dH[c] Eb) */
    double *Rt = K + M * N;     /* P */
    double *qb = Rt + P;        /* N */
    double *eb = qb + N;        /* P */
    double *rr = eb + P;        /* M x N: r_{c,n} */
    double *dqb = rr + M * N;   /* N */
    double *deb = dqb + N;      /* P */
    const double *q = c->Q + at_b(s, b, t, g), *cr = c->C + at_b(s, b, t, g);
    const double *e = c->E + at_x(s, b, t, h), *dr = c->dR + at_x(s, b, t, h);
    double sq = 0.0;
    for (i64 n = 0; n < N; ++n) sq += q[n] * q[n];
    const double iq = 1.0 / sqrt(sq / (double)N + eps);
    for (i64 n = 0; n < N; ++n) qb[n] = q[n] * iq;
    double se = 0.0;
    for (i64 p = 0; p < P; ++p) se += e[p] * e[p];
    const double ie = 1.0 / sqrt(se / (double)P + eps);
    for (i64 p = 0; p < P; ++p) eb[p] = e[p] * ie;
    for (i64 ch = 0; ch < k; ++ch) {
        const double *D = c->dH + at_state(s, b, h, ch);
        for (i64 p = 0; p < P; ++p) {
            double acc = 0.0;
            for (i64 n = 0; n < N; ++n) acc += cr[n] * D[n * P + p];
            V[ch * P + p] = acc;
        }
        double l = 0.0;
        for (i64 n = 0; n < N; ++n) {
            double kv = 0.0, rowsq = 0.0;
            for (i64 p = 0; p < P; ++p) {
                kv += D[n * P + p] * eb[p];
                rowsq += D[n * P + p] * D[n * P + p];
            }
            const double r = 1.0 / sqrt(rowsq / (double)P + eps);
            rr[ch * N + n] = r;
            K[ch * N + n] = r * kv;
            l += qb[n] * K[ch * N + n];
        }
        w[ch] = l * rs;
    }
    double m = w[0];
    for (i64 ch = 1; ch < k; ++ch) m = w[ch] > m ? w[ch] : m;
    double den = 0.0;
    for (i64 ch = 0; ch < k; ++ch) den += exp(w[ch] - m);
    for (i64 ch = 0; ch < k; ++ch) w[ch] = exp(w[ch] - m) / den;
    for (i64 p = 0; p < P; ++p) {
        double acc = 0.0;
        for (i64 ch = 0; ch < k; ++ch) acc += w[ch] * V[ch * P + p];
        Rt[p] = acc;
    }
    double dRR = 0.0;
    for (i64 p = 0; p < P; ++p) dRR += dr[p] * Rt[p];
    for (i64 n = 0; n < N; ++n) dqb[n] = 0.0;
    for (i64 p = 0; p < P; ++p) deb[p] = 0.0;
    for (i64 ch = 0; ch < k; ++ch) {
        const double *D = c->dH + at_state(s, b, h, ch);
        double dw = 0.0;
        for (i64 p = 0; p < P; ++p) dw += dr[p] * V[ch * P + p];
        const double a = w[ch] * (dw - dRR) * rs; /* dl_c / sqrt(N) */
        for (i64 n = 0; n < N; ++n) {
            dqb[n] += a * K[ch * N + n];
            if (dc) {
                double acc = 0.0;
                for (i64 p = 0; p < P; ++p) acc += D[n * P + p] * dr[p];
                dc[n] += acc * w[ch];
            }
        }
        for (i64 p = 0; p < P; ++p) {
            double acc = 0.0;
            for (i64 n = 0; n < N; ++n) acc += D[n * P + p] * rr[ch * N + n] * qb[n];
            deb[p] += a * acc;
        }
        if (dD) {
            double *dd = dD + ch * N * P;
            for (i64 n = 0; n < N; ++n) {
                const double r = rr[ch * N + n];
                const double kv = K[ch * N + n] / r; /* (dH[c] Eb)_n */
                for (i64 p = 0; p < P; ++p)
                    dd[n * P + p] += cr[n] * w[ch] * dr[p] +
                                     a * qb[n] * (r * eb[p] - r * r * r * kv * D[n * P + p] / (double)P);
            }
        }
    }
    /* through the RMSNorms of Q_t and E_t */
    if (dq) {
        double qd = 0.0;
        for (i64 n = 0; n < N; ++n) qd += q[n] * dqb[n];
        for (i64 n = 0; n < N; ++n) dq[n] += iq * dqb[n] - iq * iq * iq * q[n] * qd / (double)N;
    }
    if (de) {
        double ed = 0.0;
        for (i64 p = 0; p < P; ++p) ed += e[p] * deb[p];
        for (i64 p = 0; p < P; ++p) de[p] += ie * deb[p] - ie * ie * ie * e[p] * ed / (double)P;
    }
}

static void sma_bwd_norm_item(void *vctx, i64 item, double *scratch) {
    sma_bwd_norm_ctx *cn = (sma_bwd_norm_ctx *)vctx;
    const sma_bwd_ctx *c = &cn->base;
    const shape_t *s = &c->s;
    const i64 N = s->N, P = s->P, M = s->M;
    const i64 b = item / s->G, g = item % s->G;
    const i64 hpg = s->H / s->G;
    for (i64 t = 0; t < s->L; ++t) {
        memset(c->dQ + at_b(s, b, t, g), 0, (size_t)N * sizeof(double));
        memset(c->dC + at_b(s, b, t, g), 0, (size_t)N * sizeof(double));
    }
    for (i64 h = g * hpg; h < (g + 1) * hpg; ++h) {
        memset(c->ddH + at_state(s, b, h, 0), 0, (size_t)(M * N * P) * sizeof(double));
        for (i64 t = 0; t < s->L; ++t) memset(c->dE + at_x(s, b, t, h), 0, (size_t)P * sizeof(double));
        for (i64 t = 0; t < s->L; ++t)
            bwd_token_norm(c, cn->eps, b, h, t, c->dQ + at_b(s, b, t, g), c->dC + at_b(s, b, t, g),
                           c->dE + at_x(s, b, t, h), c->ddH + at_state(s, b, h, 0), scratch);
    }
}

void dart_oracle_sma_bwd_norm(i64 Bt, i64 L, i64 H, i64 G, i64 N, i64 P, i64 S, double eps, const double *Q,
                              const double *C, const double *E, const double *dH, const double *dR, double *dQ,
                              double *dC, double *dE, double *ddH, int threads) {
    sma_bwd_norm_ctx ctx = {{make_shape(Bt, L, H, G, N, P, S), Q, C, E, dH, dR, dQ, dC, dE, ddH}, eps};
    const i64 M = (L + S - 1) / S;
    parallel_for(sma_bwd_norm_item, &ctx, Bt * G, (size_t)(M + M * P + 2 * M * N + 3 * P + 2 * N), threads);
}

/* Sampled backward of the normalised score branch (the gradients of 8. at fewer places), in the layouts
 * of dart_oracle_sma_bwd_tokens and dart_oracle_sma_bwd_ddh. The per-memory mode sums every later token's
 * contribution to all chunk memories of (b, h) into scratch and keeps the listed one. */
typedef struct {
    sma_bwd_tok_ctx tok;
    double eps;
} sma_bwd_norm_tok_ctx;

static void sma_bwd_norm_tok_item(void *vctx, i64 item, double *scratch) {
    sma_bwd_norm_tok_ctx *cn = (sma_bwd_norm_tok_ctx *)vctx;
    const sma_bwd_tok_ctx *ct = &cn->tok;
    const sma_bwd_ctx *c = &ct->base;
    const shape_t *s = &c->s;
    const i64 b = item / ct->ntok, j = item % ct->ntok, t = ct->tokens[j];
    for (i64 g = 0; g < s->G; ++g) {
        memset(c->dQ + ((b * ct->ntok + j) * s->G + g) * s->N, 0, (size_t)s->N * sizeof(double));
        memset(c->dC + ((b * ct->ntok + j) * s->G + g) * s->N, 0, (size_t)s->N * sizeof(double));
    }
    for (i64 h = 0; h < s->H; ++h) {
        double *de = c->dE + ((b * ct->ntok + j) * s->H + h) * s->P;
        memset(de, 0, (size_t)s->P * sizeof(double));
        const i64 g = group_of(s, h);
        bwd_token_norm(c, cn->eps, b, h, t, c->dQ + ((b * ct->ntok + j) * s->G + g) * s->N,
                       c->dC + ((b * ct->ntok + j) * s->G + g) * s->N, de, NULL, scratch);
    }
}

void dart_oracle_sma_bwd_norm_tokens(i64 Bt, i64 L, i64 H, i64 G, i64 N, i64 P, i64 S, double eps, const double *Q,
                                     const double *C, const double *E, const double *dH, const double *dR,
                                     const i64 *tokens, i64 ntok, double *dQs, double *dCs, double *dEs,
                                     int threads) {
    sma_bwd_norm_tok_ctx ctx = {{{make_shape(Bt, L, H, G, N, P, S), Q, C, E, dH, dR, dQs, dCs, dEs, NULL}, tokens,
                                 ntok},
                                eps};
    const i64 M = (L + S - 1) / S;
    parallel_for(sma_bwd_norm_tok_item, &ctx, Bt * ntok, (size_t)(M + M * P + 2 * M * N + 3 * P + 2 * N), threads);
}

typedef struct {
    sma_bwd_ddh_ctx dd;
    double eps;
} sma_bwd_norm_ddh_ctx;

static void sma_bwd_norm_ddh_item(void *vctx, i64 item, double *scratch) {
    sma_bwd_norm_ddh_ctx *cn = (sma_bwd_norm_ddh_ctx *)vctx;
    const sma_bwd_ctx *c = &cn->dd.base;
    const shape_t *s = &c->s;
    const i64 b = cn->dd.trip[3 * item], h = cn->dd.trip[3 * item + 1], ch = cn->dd.trip[3 * item + 2];
    const i64 M = s->M, NP = s->N * s->P;
    double *all = scratch;                        /* M x N x P: every memory of (b, h) */
    double *tok = scratch + M * NP;               /* the per-token scratch of bwd_token_norm */
    memset(all, 0, (size_t)(M * NP) * sizeof(double));
    for (i64 t = (ch + 1) * s->S; t < s->L; ++t) bwd_token_norm(c, cn->eps, b, h, t, NULL, NULL, NULL, all, tok);
    memcpy(c->ddH + item * NP, all + ch * NP, (size_t)NP * sizeof(double));
}

void dart_oracle_sma_bwd_norm_ddh(i64 Bt, i64 L, i64 H, i64 G, i64 N, i64 P, i64 S, double eps, const double *Q,
                                  const double *C, const double *E, const double *dH, const double *dR,
                                  const i64 *triples, i64 n, double *ddHs, int threads) {
    sma_bwd_norm_ddh_ctx ctx = {{{make_shape(Bt, L, H, G, N, P, S), Q, C, E, dH, dR, NULL, NULL, NULL, ddHs}, triples},
                                eps};
    const i64 M = (L + S - 1) / S;
    parallel_for(sma_bwd_norm_ddh_item, &ctx, n, (size_t)(M * N * P + M + M * P + 2 * M * N + 3 * P + 2 * N), threads);
}
