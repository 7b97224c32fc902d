/*
 * qsa_oracle.c -- plain, slow CPU oracle for Qwen Sparse Attention (QSA).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA path and must never be linked into
 * it.
 *
 * Sources (web pages on the method):
 *   [SGL]  "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section
 *          "Qwen Sparse Attention: Retrieve Coarsely, Attend Precisely"
 *          (compression ratio 4; FP32 averaging; pooled key rotated with the
 *          first token's position; score equation s_{t,b}; best 512 blocks,
 *          expansion to 2048 positions plus the 0-3 tail tokens, at most 2051;
 *          original uncompressed K/V for the softmax; one BF16 compressed key
 *          per four tokens; four-slot raw-key ring).
 *   [LBL]  "Qwen3.8-Flash-Next, Layer by Layer", section "Token mixing: a
 *          fixed state and a selective cache" (4 query heads, 1 key head of
 *          128 dimensions; blocks of four tokens; best 512 blocks).
 *   [ARCH] flozi.net architecture guide, "How a token moves through the
 *          model", item 2 "QSA's two stages" (RoPE after key pooling;
 *          512 complete blocks plus any incomplete tail block).
 *   [MTP]  "Qwen3.8-Flash-Next: Day-0 Support in SGLang", section "IndexShare
 *          MTP: Reusing the QSA Selection Across Draft Steps" (the selection
 *          of the last accepted row is frozen for the draft loop; each draft
 *          step reads it plus the positions drafted since).
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes of the repository):
 *   - score rule: identity by default, ReLU of [SGL]'s equation behind a flag;
 *     optional per-head weights applied outside the nonlinearity;
 *   - key normalisation (named, not defined, by the pages): optional
 *     unit-weight RMS normalisation (eps 1e-6) of the FP32 mean, off by default;
 *   - RoPE: rotate-half pairs (i, i + R/2), inv_freq_i = base^(-2i/R),
 *     angle = (pos / pos_scale) * inv_freq_i;
 *   - visibility: block b is visible to the query at position t iff
 *     4b + 3 <= t; the tail is positions 4*floor((t+1)/4) .. t;
 *   - ties in top-k go to the lower block index; fewer than k visible blocks
 *     means all of them;
 *   - IndexShare draft step at position t with the selection frozen at the
 *     capture row t_c <= t: the blocks selected for t_c plus every position
 *     from t_c's first incomplete-block position 4*floor((t_c+1)/4) through t
 *     (t_c's own tail and the positions drafted since, a contiguous range);
 *   - attention logits scaled by the caller's `scale` (1/sqrt(d) by default);
 *     q head h reads kv head floor(h * Hkv / Hq); one selection per query is
 *     shared by every head (the score has no head index).
 *
 * Arithmetic: fp64 everywhere the pages do not fix a precision.  The pages fix
 * FP32 for the 4-key average and BF16 for the stored pooled key; the oracle
 * follows both.  The rotated indexer query is rounded to the storage type
 * (BF16, or FP32 in fp32 mode), the operand precision of the kernel it
 * checks.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fPIC -shared -pthread -lm
 * (no -ffast-math: the FP32 average must be evaluated exactly as written).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define IDX_HEADS 4   /* [LBL]: 4 indexer query heads */
#define IDX_DIM 128   /* [LBL]: 128-dimensional indexer heads */
#define BLK 4         /* [SGL]: compression ratio 4 (c4) */

/* ------------------------------------------------------------------------- */
/* Rounding                                                                   */
/* ------------------------------------------------------------------------- */

/* Round a double to the nearest bfloat16 value (ties to even), directly from
 * the double (no intermediate float, so no double rounding).  bfloat16 has an
 * 8-bit significand and float's exponent range. */
double oracle_round_bf16(double x)
{
    if (x == 0.0 || isnan(x) || isinf(x)) return x;
    int e;
    frexp(x, &e);               /* x = m * 2^e, 0.5 <= |m| < 1 */
    int ex = e - 1;             /* x = 1.f * 2^ex */
    if (ex < -126) ex = -126;   /* subnormal range: fixed quantum */
    double quantum = ldexp(1.0, ex - 7);
    double n = nearbyint(x / quantum);   /* default mode: ties to even */
    double y = n * quantum;
    const double bf16_max = ldexp(255.0, 127 - 7);   /* 0x7F7F */
    if (fabs(y) > bf16_max) y = copysign(INFINITY, x);
    return y;
}

/* Round a double to the nearest FP8 E4M3 value (ties to even), directly from
 * the double, saturating to +-448.  E4M3 (the FP8 format of the pages' FP8
 * indexer-key cache, "--attention-config.indexer_kv_dtype fp8"): 1 sign bit,
 * 4 exponent bits with bias 7, 3 mantissa bits; normal values 2^-6 .. 448,
 * subnormals k * 2^-9; no infinities. */
double oracle_round_e4m3(double x)
{
    if (x == 0.0 || isnan(x)) return x;
    if (isinf(x)) return copysign(448.0, x);
    int e;
    frexp(x, &e);               /* x = m * 2^e, 0.5 <= |m| < 1 */
    int ex = e - 1;             /* x = 1.f * 2^ex */
    if (ex < -6) ex = -6;       /* subnormal range: fixed quantum 2^-9 */
    double quantum = ldexp(1.0, ex - 3);
    double y = nearbyint(x / quantum) * quantum;   /* ties to even */
    if (fabs(y) > 448.0) y = copysign(448.0, x);
    return y;
}

/* store: 0 = FP32, 1 = BF16, 2 = FP8 E4M3 */
static double round_store(double x, int store_bf16)
{
    if (store_bf16 == 2) return oracle_round_e4m3(x);
    return store_bf16 ? oracle_round_bf16(x) : (double)(float)x;
}

/* ------------------------------------------------------------------------- */
/* RoPE (rotate-half), fp64                                                   */
/* ------------------------------------------------------------------------- */

typedef struct {
    double base;
    double pos_scale;
    int rotary_dim;
} orope_t;

/* Rotate x[0..dim) in place for position `pos`: pairs (i, i + R/2) for
 * i < R/2 are turned by the angle (pos / pos_scale) * base^(-2i/R); dims at
 * and above R are left alone. */
static void rope_rotate(double *x, double pos, const orope_t *r)
{
    int half = r->rotary_dim / 2;
    for (int i = 0; i < half; ++i) {
        double inv_freq = pow(r->base, -(2.0 * i) / (double)r->rotary_dim);
        double ang = (pos / r->pos_scale) * inv_freq;
        double c = cos(ang), s = sin(ang);
        double a = x[i], b = x[i + half];
        x[i] = a * c - b * s;
        x[i + half] = b * c + a * s;
    }
}

/* Public wrapper (used by the pins): rotate n rows of `dim` values, row i at
 * position pos[i], result in fp64. */
void oracle_rope_rows(const float *x, int64_t n, int dim, const int64_t *pos,
                      double base, double pos_scale, int rotary_dim, double *out)
{
    orope_t r = {base, pos_scale, rotary_dim};
    for (int64_t i = 0; i < n; ++i) {
        for (int j = 0; j < dim; ++j) out[i * dim + j] = x[i * dim + j];
        rope_rotate(out + i * dim, (double)pos[i], &r);
    }
}

/* ------------------------------------------------------------------------- */
/* Step 1-4: micro-block key pooling ([SGL], [ARCH])                          */
/* ------------------------------------------------------------------------- */

/* One compressed key from four raw keys k0..k3 (each IDX_DIM floats) whose
 * first token sits at position `pos`:
 *   mean in FP32 (((k0 + k1) + k2) + k3) * 0.25,
 *   optional RMS normalisation (fp64, eps 1e-6, unit weight),
 *   RoPE at the first token's position (fp64),
 *   rounded to the stored type. */
static void pool_one(const float *k0, const float *k1, const float *k2, const float *k3,
                     double pos, const orope_t *r, int rmsnorm, int store_bf16, float *out)
{
    double x[IDX_DIM];
    for (int i = 0; i < IDX_DIM; ++i) {
        float s = k0[i];
        s = s + k1[i];
        s = s + k2[i];
        s = s + k3[i];
        float m = s * 0.25f;
        x[i] = (double)m;
    }
    if (rmsnorm) {
        double ss = 0.0;
        for (int i = 0; i < IDX_DIM; ++i) ss += x[i] * x[i];
        double inv = 1.0 / sqrt(ss / IDX_DIM + 1e-6);
        for (int i = 0; i < IDX_DIM; ++i) x[i] *= inv;
    }
    rope_rotate(x, pos, r);
    for (int i = 0; i < IDX_DIM; ++i) out[i] = (float)round_store(x[i], store_bf16);
}

/* Prefill pooling: k_raw holds n_tok raw indexer keys [n_tok][128] whose
 * first token is at position pos0 (a multiple of 4).  Writes n_tok/4
 * compressed keys [n_tok/4][128]; block j starts at position pos0 + 4j. */
void oracle_pool_keys(const float *k_raw, int64_t n_tok, int64_t pos0,
                      double base, double pos_scale, int rotary_dim,
                      int rmsnorm, int store_bf16, float *k_pool)
{
    orope_t r = {base, pos_scale, rotary_dim};
    int64_t nblk = n_tok / BLK;
    for (int64_t j = 0; j < nblk; ++j) {
        const float *k = k_raw + j * BLK * IDX_DIM;
        pool_one(k, k + IDX_DIM, k + 2 * IDX_DIM, k + 3 * IDX_DIM,
                 (double)(pos0 + BLK * j), &r, rmsnorm, store_bf16, k_pool + j * IDX_DIM);
    }
}

/* Decode pooling for one sequence ([SGL]: four-slot per-request ring of raw
 * keys of the unfinished block).  seq_len counts tokens including the new
 * one, whose position is p = seq_len - 1.  The new raw key goes to ring slot
 * p mod 4; when it completes its block (seq_len mod 4 == 0) the ring is
 * pooled into compressed key seq_len/4 - 1, rotated at position seq_len - 4. */
void oracle_pool_decode(const float *k_new, float *ring /*[4][128]*/, float *k_pool /*[cap][128]*/,
                        int64_t seq_len, double base, double pos_scale, int rotary_dim,
                        int rmsnorm, int store_bf16)
{
    orope_t r = {base, pos_scale, rotary_dim};
    int64_t p = seq_len - 1;
    memcpy(ring + (p % BLK) * IDX_DIM, k_new, sizeof(float) * IDX_DIM);
    if (seq_len % BLK == 0) {
        int64_t b = seq_len / BLK - 1;
        pool_one(ring, ring + IDX_DIM, ring + 2 * IDX_DIM, ring + 3 * IDX_DIM,
                 (double)(seq_len - BLK), &r, rmsnorm, store_bf16, k_pool + b * IDX_DIM);
    }
}

/* ------------------------------------------------------------------------- */
/* Step 5: rotated indexer query                                               */
/* ------------------------------------------------------------------------- */

/* q_raw [4][128] for the query at position t -> q_hat [4][128], rotated at t
 * and rounded to the operand type. */
static void rotate_query(const float *q_raw, double t, const orope_t *r, int store_bf16,
                         double *q_hat)
{
    for (int h = 0; h < IDX_HEADS; ++h) {
        double x[IDX_DIM];
        for (int i = 0; i < IDX_DIM; ++i) x[i] = q_raw[h * IDX_DIM + i];
        rope_rotate(x, t, r);
        for (int i = 0; i < IDX_DIM; ++i) q_hat[h * IDX_DIM + i] = round_store(x[i], store_bf16 ? 1 : 0);
    }
}

/* ------------------------------------------------------------------------- */
/* Step 6: block scores ([SGL] score equation)                                */
/* ------------------------------------------------------------------------- */

/* s_b = (1/sqrt(128)) * sum_h w_h * phi(<q_hat_h, kbar_b>) for b < nb, with
 * phi = ReLU when relu != 0 and the identity otherwise; w = 1 when w4 is
 * NULL. */
static void index_scores(const double *q_hat, const float *k_pool, int64_t nb,
                         const float *w4, int relu, double *s)
{
    const double inv_sqrt = 1.0 / sqrt((double)IDX_DIM);
    for (int64_t b = 0; b < nb; ++b) {
        const float *kb = k_pool + b * IDX_DIM;
        double acc = 0.0;
        for (int h = 0; h < IDX_HEADS; ++h) {
            double d = 0.0;
            for (int i = 0; i < IDX_DIM; ++i) d += q_hat[h * IDX_DIM + i] * (double)kb[i];
            if (relu && d < 0.0) d = 0.0;
            acc += (w4 ? (double)w4[h] : 1.0) * d;
        }
        s[b] = acc * inv_sqrt;
    }
}

/* ------------------------------------------------------------------------- */
/* Step 7: top-k selection                                                    */
/* ------------------------------------------------------------------------- */

typedef struct {
    double s;
    int64_t b;
} scored_t;

/* Order: higher score first; equal scores -> lower block index first. */
static int cmp_rank(const void *x, const void *y)
{
    const scored_t *a = (const scored_t *)x, *c = (const scored_t *)y;
    if (a->s > c->s) return -1;
    if (a->s < c->s) return 1;
    return (a->b < c->b) ? -1 : (a->b > c->b);
}

static int cmp_i32(const void *x, const void *y)
{
    int32_t a = *(const int32_t *)x, b = *(const int32_t *)y;
    return (a > b) - (a < b);
}

/* Select the min(k, n) best of scores s[0..n): sort all (score, b) pairs by
 * (score desc, b asc), keep the first min(k, n), return them sorted by block
 * index ascending in sel[0..k) padded with -1.  kth / next receive the k-th
 * and (k+1)-th best scores (NAN where they do not exist).  Returns nsel. */
int oracle_topk(const double *s, int64_t n, int k, int32_t *sel, double *kth, double *next)
{
    scored_t *v = (scored_t *)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
    for (int64_t b = 0; b < n; ++b) { v[b].s = s[b]; v[b].b = b; }
    qsort(v, (size_t)n, sizeof(scored_t), cmp_rank);
    int nsel = (int)(n < k ? n : k);
    for (int i = 0; i < nsel; ++i) sel[i] = (int32_t)v[i].b;
    qsort(sel, (size_t)nsel, sizeof(int32_t), cmp_i32);
    for (int i = nsel; i < k; ++i) sel[i] = -1;
    if (kth) *kth = (n >= k && k > 0) ? v[k - 1].s : NAN;
    if (next) *next = (n > k) ? v[k].s : NAN;
    free(v);
    return nsel;
}

/* ------------------------------------------------------------------------- */
/* Step 8: sparse attention over the original K/V ([SGL])                     */
/* ------------------------------------------------------------------------- */

/* Number of complete blocks visible to the query at position t. */
static int64_t visible_blocks(int64_t t) { return (t + 1) / BLK; }

/* Attention of one query at position t over the positions
 *   P(t) = {4b .. 4b+3 : b in sel[0..nsel)}  U  {tail_from .. t},
 * where tail_from = 4*nb(t) for a query that selected its own blocks ([SGL]),
 * or 4*nb(t_c) for an IndexShare draft step using the selection of row t_c
 * ([MTP]).  q [Hq][d] (already rotated), k/v cache rows indexed by position
 * [pos][Hkv][d].  out [Hq][d] fp64; lse [Hq] natural-log log-sum-exp of the
 * scaled logits (may be NULL). */
static void attend(const float *q, const float *kc, const float *vc, int64_t t, int64_t tail_from,
                   const int32_t *sel, int nsel, int Hq, int Hkv, int d, double scale,
                   double *out, double *lse)
{
    int64_t ntail = t + 1 - tail_from;
    if (ntail < 0) ntail = 0;
    int64_t npos = (int64_t)nsel * BLK + ntail;
    int64_t *pos = (int64_t *)malloc(sizeof(int64_t) * (size_t)(npos > 0 ? npos : 1));
    int64_t m = 0;
    for (int i = 0; i < nsel; ++i)
        for (int j = 0; j < BLK; ++j) pos[m++] = (int64_t)sel[i] * BLK + j;
    for (int64_t j = 0; j < ntail; ++j) pos[m++] = tail_from + j;

    double *logit = (double *)malloc(sizeof(double) * (size_t)(npos > 0 ? npos : 1));
    for (int h = 0; h < Hq; ++h) {
        int g = (int)(((int64_t)h * Hkv) / Hq);
        const float *qh = q + (int64_t)h * d;
        double mx = -INFINITY;
        for (int64_t i = 0; i < npos; ++i) {
            const float *kr = kc + (pos[i] * Hkv + g) * d;
            double acc = 0.0;
            for (int e = 0; e < d; ++e) acc += (double)qh[e] * (double)kr[e];
            logit[i] = acc * scale;
            if (logit[i] > mx) mx = logit[i];
        }
        double denom = 0.0;
        for (int64_t i = 0; i < npos; ++i) denom += exp(logit[i] - mx);
        double *oh = out + (int64_t)h * d;
        for (int e = 0; e < d; ++e) oh[e] = 0.0;
        for (int64_t i = 0; i < npos; ++i) {
            double p = exp(logit[i] - mx) / denom;
            const float *vr = vc + (pos[i] * Hkv + g) * d;
            for (int e = 0; e < d; ++e) oh[e] += p * (double)vr[e];
        }
        if (lse) lse[h] = mx + log(denom);
    }
    free(logit);
    free(pos);
}

/* Textbook causal softmax attention of the query at position t over every
 * position 0..t (used to pin the sparse path where it must coincide). */
static void attend_dense(const float *q, const float *kc, const float *vc, int64_t t,
                         int Hq, int Hkv, int d, double scale, double *out)
{
    double *logit = (double *)malloc(sizeof(double) * (size_t)(t + 1));
    for (int h = 0; h < Hq; ++h) {
        int g = (int)(((int64_t)h * Hkv) / Hq);
        const float *qh = q + (int64_t)h * d;
        double mx = -INFINITY;
        for (int64_t j = 0; j <= t; ++j) {
            const float *kr = kc + (j * Hkv + g) * d;
            double acc = 0.0;
            for (int e = 0; e < d; ++e) acc += (double)qh[e] * (double)kr[e];
            logit[j] = acc * scale;
            if (logit[j] > mx) mx = logit[j];
        }
        double denom = 0.0;
        for (int64_t j = 0; j <= t; ++j) denom += exp(logit[j] - mx);
        double *oh = out + (int64_t)h * d;
        for (int e = 0; e < d; ++e) oh[e] = 0.0;
        for (int64_t j = 0; j <= t; ++j) {
            double p = exp(logit[j] - mx) / denom;
            const float *vr = vc + (j * Hkv + g) * d;
            for (int e = 0; e < d; ++e) oh[e] += p * (double)vr[e];
        }
    }
    free(logit);
}

/* ------------------------------------------------------------------------- */
/* Row drivers (threads only distribute independent query rows)               */
/* ------------------------------------------------------------------------- */

typedef struct {
    /* indexer */
    const float *q_idx;     /* raw [n_q][4][128], row i at position q0 + i */
    const float *k_pool;    /* [nblk][128] */
    const float *head_w;    /* [n_q][4] or NULL */
    int relu, store_bf16, top_k;
    orope_t rope;
    /* attention */
    const float *q;         /* [n_q][Hq][d], rotated */
    const float *k, *v;     /* [L][Hkv][d], rows by position */
    int Hq, Hkv, d;
    double scale;
    int64_t q0;
    /* work list */
    const int64_t *rows;    /* query row indices (relative to q0) */
    int64_t nrows;
    /* stage-isolated attention: selection given as input */
    const int32_t *sel_in;  /* [nrows][top_k] or NULL */
    const int32_t *nsel_in; /* [nrows] */
    /* outputs (any may be NULL) */
    int32_t *sel;           /* [nrows][top_k] */
    int32_t *nsel;          /* [nrows] */
    double *kth, *next;     /* [nrows] */
    double *scores;         /* [nrows][score_cap] or NULL */
    int64_t score_cap;
    double *out;            /* [nrows][Hq][d] */
    double *lse;            /* [nrows][Hq] */
    int dense;              /* 1: textbook dense causal attention instead */
    /* threading */
    int nthreads;
    int tid;
} job_t;

static void run_row(const job_t *J, int64_t r)
{
    int64_t i = J->rows[r];
    int64_t t = J->q0 + i;
    int64_t nb = visible_blocks(t);
    int32_t *sel = NULL;
    int nsel = 0;
    int32_t *sel_own = NULL;

    if (J->dense) {
        attend_dense(J->q + i * J->Hq * J->d, J->k, J->v, t, J->Hq, J->Hkv, J->d, J->scale,
                     J->out + r * J->Hq * J->d);
        return;
    }
    if (J->sel_in) {
        sel = (int32_t *)(J->sel_in + r * J->top_k);
        nsel = J->nsel_in[r];
    } else if (J->q_idx) {
        double q_hat[IDX_HEADS * IDX_DIM];
        rotate_query(J->q_idx + i * IDX_HEADS * IDX_DIM, (double)t, &J->rope, J->store_bf16, q_hat);
        double *s = (double *)malloc(sizeof(double) * (size_t)(nb > 0 ? nb : 1));
        index_scores(q_hat, J->k_pool, nb, J->head_w ? J->head_w + i * IDX_HEADS : NULL, J->relu, s);
        if (J->scores)
            for (int64_t b = 0; b < nb && b < J->score_cap; ++b) J->scores[r * J->score_cap + b] = s[b];
        sel_own = (int32_t *)malloc(sizeof(int32_t) * (size_t)J->top_k);
        double kth, nxt;
        nsel = oracle_topk(s, nb, J->top_k, sel_own, &kth, &nxt);
        if (J->kth) J->kth[r] = kth;
        if (J->next) J->next[r] = nxt;
        if (J->sel) memcpy(J->sel + r * J->top_k, sel_own, sizeof(int32_t) * (size_t)J->top_k);
        if (J->nsel) J->nsel[r] = nsel;
        sel = sel_own;
        free(s);
    }
    if (J->out && J->q)
        attend(J->q + i * J->Hq * J->d, J->k, J->v, t, BLK * visible_blocks(t), sel, nsel, J->Hq, J->Hkv, J->d, J->scale,
               J->out + r * J->Hq * J->d, J->lse ? J->lse + r * J->Hq : NULL);
    free(sel_own);
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    for (int64_t r = J->tid; r < J->nrows; r += J->nthreads) run_row(J, r);
    return NULL;
}

static void run_job(job_t *J)
{
    int nt = J->nthreads < 1 ? 1 : J->nthreads;
    if (nt > 256) nt = 256;
    pthread_t th[256];
    job_t jobs[256];
    for (int i = 0; i < nt; ++i) {
        jobs[i] = *J;
        jobs[i].nthreads = nt;
        jobs[i].tid = i;
    }
    for (int i = 1; i < nt; ++i) pthread_create(&th[i], NULL, worker, &jobs[i]);
    worker(&jobs[0]);
    for (int i = 1; i < nt; ++i) pthread_join(th[i], NULL);
}

/* Prefill QSA for the listed query rows (relative index i, position q0 + i):
 * rotate the indexer query, score every visible complete block, select the
 * top-k, attend over the selected blocks plus the tail.  Pass q == NULL to
 * stop after the selection; pass q_idx == NULL with sel_in/nsel_in to run the
 * attention alone on a given selection. */
void oracle_prefill_rows(const float *q_idx, const float *k_pool, const float *head_w,
                         int relu, int store_bf16, int top_k,
                         double base, double pos_scale, int rotary_dim,
                         const float *q, const float *k, const float *v,
                         int Hq, int Hkv, int d, double scale, int64_t q0,
                         const int64_t *rows, int64_t nrows,
                         const int32_t *sel_in, const int32_t *nsel_in,
                         int32_t *sel, int32_t *nsel, double *kth, double *next,
                         double *scores, int64_t score_cap,
                         double *out, double *lse, int nthreads)
{
    job_t J;
    memset(&J, 0, sizeof J);
    J.q_idx = q_idx; J.k_pool = k_pool; J.head_w = head_w;
    J.relu = relu; J.store_bf16 = store_bf16; J.top_k = top_k;
    J.rope.base = base; J.rope.pos_scale = pos_scale; J.rope.rotary_dim = rotary_dim;
    J.q = q; J.k = k; J.v = v; J.Hq = Hq; J.Hkv = Hkv; J.d = d; J.scale = scale; J.q0 = q0;
    J.rows = rows; J.nrows = nrows; J.sel_in = sel_in; J.nsel_in = nsel_in;
    J.sel = sel; J.nsel = nsel; J.kth = kth; J.next = next;
    J.scores = scores; J.score_cap = score_cap; J.out = out; J.lse = lse;
    J.nthreads = nthreads;
    run_job(&J);
}

/* Textbook dense causal attention for the listed rows (position q0 + i). */
void oracle_dense_rows(const float *q, const float *k, const float *v, int Hq, int Hkv, int d,
                       double scale, int64_t q0, const int64_t *rows, int64_t nrows,
                       double *out, int nthreads)
{
    job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.Hq = Hq; J.Hkv = Hkv; J.d = d; J.scale = scale; J.q0 = q0;
    J.rows = rows; J.nrows = nrows; J.out = out; J.dense = 1; J.nthreads = nthreads;
    run_job(&J);
}

/* ------------------------------------------------------------------------- */
/* Decode step for a batch of independent sequences                           */
/* ------------------------------------------------------------------------- */

typedef struct {
    const float *q_idx;      /* [B][4][128] raw indexer query of the new token */
    const float *k_pool;     /* [B][pool_stride][128] compressed keys (complete blocks) */
    int64_t pool_stride;
    const float *head_w;     /* [B][4] or NULL */
    const float *q;          /* [B][Hq][d] rotated query of the new token */
    const float *k, *v;      /* [B][kv_stride][Hkv][d] caches incl. the new token */
    int64_t kv_stride;
    const int32_t *seq_len;  /* [B], tokens including the new one */
    const int32_t *cap_len;  /* [B] or NULL: IndexShare, the selection is that of row cap_len - 1 */
    int relu, store_bf16, top_k, Hq, Hkv, d;
    double scale;
    orope_t rope;
    int32_t *sel, *nsel;
    double *kth, *next, *out, *lse;
    double *scores;          /* [B][score_cap] or NULL: the block scores, as ranked */
    int64_t score_cap;
    int64_t B;
    int nthreads, tid;
} djob_t;

static void decode_one(const djob_t *J, int64_t bi)
{
    int64_t t = (int64_t)J->seq_len[bi] - 1;
    /* row whose selection is used: the new token itself, or the IndexShare
     * capture row ([MTP]); q_idx is that row's indexer query */
    int64_t t_sel = J->cap_len ? (int64_t)J->cap_len[bi] - 1 : t;
    int64_t nb = visible_blocks(t_sel);
    double q_hat[IDX_HEADS * IDX_DIM];
    rotate_query(J->q_idx + bi * IDX_HEADS * IDX_DIM, (double)t_sel, &J->rope, J->store_bf16, q_hat);
    double *s = (double *)malloc(sizeof(double) * (size_t)(nb > 0 ? nb : 1));
    index_scores(q_hat, J->k_pool + bi * J->pool_stride * IDX_DIM, nb,
                 J->head_w ? J->head_w + bi * IDX_HEADS : NULL, J->relu, s);
    if (J->scores)
        for (int64_t b = 0; b < nb && b < J->score_cap; ++b) J->scores[bi * J->score_cap + b] = s[b];
    int32_t *sel = J->sel + bi * J->top_k;
    double kth, nxt;
    int nsel = oracle_topk(s, nb, J->top_k, sel, &kth, &nxt);
    free(s);
    J->nsel[bi] = nsel;
    if (J->kth) J->kth[bi] = kth;
    if (J->next) J->next[bi] = nxt;
    if (J->out && J->q) {
        int64_t kvoff = bi * J->kv_stride * J->Hkv * J->d;
        attend(J->q + bi * J->Hq * J->d, J->k + kvoff, J->v + kvoff, t, BLK * nb, sel, nsel,
               J->Hq, J->Hkv, J->d, J->scale, J->out + bi * J->Hq * J->d,
               J->lse ? J->lse + bi * J->Hq : NULL);
    }
}

static void *dworker(void *arg)
{
    djob_t *J = (djob_t *)arg;
    for (int64_t b = J->tid; b < J->B; b += J->nthreads) decode_one(J, b);
    return NULL;
}

/* One QSA decode step for B sequences: score all floor(seq_len/4) compressed
 * blocks, select the top-k, attend over them plus the tail (the new token's
 * incomplete block).  The caller has already run oracle_pool_decode.
 * With cap_len (IndexShare draft step, [MTP]): the selection is the one of row
 * cap_len - 1 (q_idx is that row's indexer query, scored over the blocks it
 * sees), and the attention at row seq_len - 1 reads those blocks plus every
 * position from 4*floor(cap_len/4) through seq_len - 1. */
void oracle_decode(const float *q_idx, const float *k_pool, int64_t pool_stride, const float *head_w,
                   const float *q, const float *k, const float *v, int64_t kv_stride,
                   const int32_t *seq_len, const int32_t *cap_len, int64_t B, int relu, int store_bf16, int top_k,
                   int Hq, int Hkv, int d, double scale, double base, double pos_scale, int rotary_dim,
                   int32_t *sel, int32_t *nsel, double *kth, double *next,
                   double *out, double *lse, double *scores, int64_t score_cap, int nthreads)
{
    djob_t J;
    memset(&J, 0, sizeof J);
    J.q_idx = q_idx; J.k_pool = k_pool; J.pool_stride = pool_stride; J.head_w = head_w;
    J.q = q; J.k = k; J.v = v; J.kv_stride = kv_stride; J.seq_len = seq_len; J.cap_len = cap_len;
    J.relu = relu; J.store_bf16 = store_bf16; J.top_k = top_k; J.Hq = Hq; J.Hkv = Hkv; J.d = d;
    J.scale = scale; J.rope.base = base; J.rope.pos_scale = pos_scale; J.rope.rotary_dim = rotary_dim;
    J.sel = sel; J.nsel = nsel; J.kth = kth; J.next = next; J.out = out; J.lse = lse; J.B = B;
    J.scores = scores; J.score_cap = score_cap;
    int nt = nthreads < 1 ? 1 : (nthreads > 256 ? 256 : nthreads);
    pthread_t th[256];
    djob_t jobs[256];
    for (int i = 0; i < nt; ++i) { jobs[i] = J; jobs[i].nthreads = nt; jobs[i].tid = i; }
    for (int i = 1; i < nt; ++i) pthread_create(&th[i], NULL, dworker, &jobs[i]);
    dworker(&jobs[0]);
    for (int i = 1; i < nt; ++i) pthread_join(th[i], NULL);
}
