/*
 * kda_oracle.c -- plain, slow, fp64 CPU oracle for Kimi Delta Attention (KDA).
 *
 * TEST INFRASTRUCTURE. This file is the independent checker for libkda. Only the
 * test suite, the smoke check and the benchmark's CPU-baseline leg may load it.
 * It shares no code, header or constant with the CUDA library, and the CUDA
 * library never calls it.
 *
 * Sources (web pages about the AliceAI-Foundation-80B-A3B-Base model):
 *  [P1] "Яндекс открыл веса AliceAI-Foundation-80B-A3B-Base: MoE-модель,
 *       обученная с нуля" (sarnas.ru), section "Что именно изменилось":
 *       KDA keeps a fixed-size state; for a new token it reads the value the
 *       state holds for the token's key, compares it with the new value and
 *       writes back only the difference; it forgets with a separate
 *       coefficient per row of the state matrix (Gated DeltaNet uses one).
 *  [P4] "两天两篇深度拆解抢跑 CSDN ..." (m.lqnn.cn/news/205170), section
 *       "KDA 与 Gated Attention：每 4 层只留 1 层全注意力": q/k/v each go
 *       through a kernel-4 causal convolution whose cache is updated per
 *       step; the recurrence is  state = state * exp(gate) + delta  with
 *       delta = prediction residual times sigmoid(beta); beta lies in (0,1).
 *  [P5] "80B 参数只花 3B 算力 ..." (m.lqnn.cn/news/255115), section
 *       "二、第一关：配置文件": conv kernel >= 2, chunk size > 0.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - the read-out that forms the residual uses the state AFTER the per-row
 *    decay (decay, read, correct, emit);
 *  - the output o_t = scale * S_t^T q_t reads the state AFTER the write;
 *  - the per-row gate is the log-decay g (<= 0) given per key channel;
 *  - the conv has no bias, tap K-1 multiplies the current token, positions
 *    before the sequence start come from the conv cache (oldest first) or 0;
 *  - SiLU follows the conv on q, k and v; q and k are then L2-normalised per
 *    head vector as x / sqrt(sum x^2 + eps).
 *
 * Layouts (row-major, token-major):
 *  q, k, g : [T_tot, H, dk]     v, o : [T_tot, H, dv]     beta : [T_tot, H]
 *  h0, ht  : [N, H, dk, dv]  (row i = key channel i, column j = value channel j)
 *  cu_seqlens : [N+1], sequence n covers tokens [cu[n], cu[n+1]).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Work splitting over (sequence, head) pairs: every pair is independent.    */
/* ------------------------------------------------------------------------ */

typedef void (*pair_fn)(void* ctx, int64_t pair);

typedef struct {
    pair_fn fn;
    void* ctx;
    int64_t npairs;
    int nthreads;
    int tid;
} pair_job;

static void* pair_worker(void* arg) {
    pair_job* job = (pair_job*)arg;
    for (int64_t p = job->tid; p < job->npairs; p += job->nthreads) job->fn(job->ctx, p);
    return NULL;
}

static void run_pairs(pair_fn fn, void* ctx, int64_t npairs, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((int64_t)nthreads > npairs) nthreads = (int)(npairs > 0 ? npairs : 1);
    pthread_t th[256];
    pair_job jobs[256];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].fn = fn; jobs[t].ctx = ctx; jobs[t].npairs = npairs;
        jobs[t].nthreads = nthreads; jobs[t].tid = t;
    }
    for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, pair_worker, &jobs[t]);
    pair_worker(&jobs[0]);
    for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
}

/* ------------------------------------------------------------------------ */
/* KDA recurrence, token by token ([P1], [P4]).                              */
/* ------------------------------------------------------------------------ */

typedef struct {
    const double *q, *k, *v, *g, *beta, *h0;
    double *ht, *o;
    const int64_t* cu;
    double scale;
    int H, dk, dv;
} kda_ctx;

static void kda_pair(void* vctx, int64_t pair) {
    const kda_ctx* c = (const kda_ctx*)vctx;
    const int H = c->H, dk = c->dk, dv = c->dv;
    const int64_t n = pair / H;
    const int h = (int)(pair % H);
    const int64_t bos = c->cu[n], eos = c->cu[n + 1];

    double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
    double* u = (double*)malloc(sizeof(double) * (size_t)dv);
    const size_t sbase = ((size_t)n * H + h) * (size_t)dk * dv;
    if (c->h0) memcpy(S, c->h0 + sbase, sizeof(double) * (size_t)dk * dv);
    else memset(S, 0, sizeof(double) * (size_t)dk * dv);

    for (int64_t t = bos; t < eos; ++t) {
        const double* qt = c->q + ((size_t)t * H + h) * dk;
        const double* kt = c->k + ((size_t)t * H + h) * dk;
        const double* gt = c->g + ((size_t)t * H + h) * dk;
        const double* vt = c->v + ((size_t)t * H + h) * dv;
        const double bt = c->beta[(size_t)t * H + h];
        double* ot = c->o + ((size_t)t * H + h) * dv;

        /* forget: row i (key channel i) is scaled by its own gate exp(g_i) */
        for (int i = 0; i < dk; ++i) {
            const double a = exp(gt[i]);
            for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= a;
        }
        /* read the value the decayed state holds for k_t; residual u = v - S^T k */
        for (int j = 0; j < dv; ++j) {
            double r = 0.0;
            for (int i = 0; i < dk; ++i) r += S[(size_t)i * dv + j] * kt[i];
            u[j] = vt[j] - r;
        }
        /* write back only the correction, scaled by beta in (0,1) */
        for (int i = 0; i < dk; ++i) {
            const double bk = bt * kt[i];
            for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += bk * u[j];
        }
        /* output reads the updated state */
        for (int j = 0; j < dv; ++j) {
            double r = 0.0;
            for (int i = 0; i < dk; ++i) r += S[(size_t)i * dv + j] * qt[i];
            ot[j] = c->scale * r;
        }
    }
    if (c->ht) memcpy(c->ht + sbase, S, sizeof(double) * (size_t)dk * dv);
    free(u);
    free(S);
}

/* o, ht are written; h0 and ht may be NULL (zero initial state / not returned). */
void kda_oracle_fwd(const double* q, const double* k, const double* v, const double* g,
                    const double* beta, double scale, const double* h0, double* ht, double* o,
                    const int64_t* cu_seqlens, int N, int H, int dk, int dv, int nthreads) {
    kda_ctx c;
    c.q = q; c.k = k; c.v = v; c.g = g; c.beta = beta; c.h0 = h0; c.ht = ht; c.o = o;
    c.cu = cu_seqlens; c.scale = scale; c.H = H; c.dk = dk; c.dv = dv;
    run_pairs(kda_pair, &c, (int64_t)N * H, nthreads);
}

/* ------------------------------------------------------------------------ */
/* Transition of a stretch of tokens ([P1], [P4]). Each token maps the state */
/* affinely: S -> (I - beta k k^T) diag(exp(g)) S + beta k v^T. Composing    */
/* the maps of a stretch gives S_end = M S_start + (S_end started from 0),   */
/* with M the product of the linear parts (I - beta k k^T) diag(exp(g)), the */
/* latest token's on the left. This routine forms M by that product, one     */
/* token at a time. A prefill split into stretches (context parallelism)     */
/* joins them with it.                                                       */
/* ------------------------------------------------------------------------ */

typedef struct {
    const double *k, *g, *beta;
    double* m;
    const int64_t* cu;
    int H, dk;
} trans_ctx;

static void trans_pair(void* vctx, int64_t pair) {
    const trans_ctx* c = (const trans_ctx*)vctx;
    const int H = c->H, dk = c->dk;
    const int64_t n = pair / H;
    const int h = (int)(pair % H);
    double* M = (double*)calloc((size_t)dk * dk, sizeof(double));
    double* w = (double*)malloc(sizeof(double) * (size_t)dk);
    for (int i = 0; i < dk; ++i) M[(size_t)i * dk + i] = 1.0;
    for (int64_t t = c->cu[n]; t < c->cu[n + 1]; ++t) {
        const double* kt = c->k + ((size_t)t * H + h) * dk;
        const double* gt = c->g + ((size_t)t * H + h) * dk;
        const double bt = c->beta[(size_t)t * H + h];
        /* left-multiply by diag(exp(g)): row r of M scales by exp(g_r) */
        for (int r = 0; r < dk; ++r) {
            const double decay = exp(gt[r]);
            for (int col = 0; col < dk; ++col) M[(size_t)r * dk + col] *= decay;
        }
        /* left-multiply by (I - beta k k^T): M -= beta k (k^T M) */
        for (int col = 0; col < dk; ++col) {
            double acc = 0.0;
            for (int r = 0; r < dk; ++r) acc += kt[r] * M[(size_t)r * dk + col];
            w[col] = acc;
        }
        for (int r = 0; r < dk; ++r)
            for (int col = 0; col < dk; ++col) M[(size_t)r * dk + col] -= bt * kt[r] * w[col];
    }
    memcpy(c->m + (size_t)pair * dk * dk, M, sizeof(double) * (size_t)dk * dk);
    free(w);
    free(M);
}

/* m : [N, H, dk, dk], the transition of every (sequence, head). */
void kda_oracle_transition(const double* k, const double* g, const double* beta, double* m,
                           const int64_t* cu_seqlens, int N, int H, int dk, int nthreads) {
    trans_ctx c;
    c.k = k; c.g = g; c.beta = beta; c.m = m; c.cu = cu_seqlens; c.H = H; c.dk = dk;
    run_pairs(trans_pair, &c, (int64_t)N * H, nthreads);
}

/* ------------------------------------------------------------------------ */
/* Scalar-gated DeltaNet in Householder form, written independently of the   */
/* KDA loop above: S <- exp(alpha) (I - beta k k^T) S + beta k v^T,          */
/* o = scale S^T q. [P1] contrasts KDA's per-row gate with this scalar gate.  */
/* ------------------------------------------------------------------------ */

typedef struct {
    const double *q, *k, *v, *alpha, *beta, *h0;
    double *ht, *o;
    const int64_t* cu;
    double scale;
    int H, dk, dv;
} gdn_ctx;

static void gdn_pair(void* vctx, int64_t pair) {
    const gdn_ctx* c = (const gdn_ctx*)vctx;
    const int H = c->H, dk = c->dk, dv = c->dv;
    const int64_t n = pair / H;
    const int h = (int)(pair % H);
    double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
    double* kS = (double*)malloc(sizeof(double) * (size_t)dv);
    const size_t sbase = ((size_t)n * H + h) * (size_t)dk * dv;
    if (c->h0) memcpy(S, c->h0 + sbase, sizeof(double) * (size_t)dk * dv);
    else memset(S, 0, sizeof(double) * (size_t)dk * dv);

    for (int64_t t = c->cu[n]; t < c->cu[n + 1]; ++t) {
        const double* qt = c->q + ((size_t)t * H + h) * dk;
        const double* kt = c->k + ((size_t)t * H + h) * dk;
        const double* vt = c->v + ((size_t)t * H + h) * dv;
        const double at = exp(c->alpha[(size_t)t * H + h]);
        const double bt = c->beta[(size_t)t * H + h];
        double* ot = c->o + ((size_t)t * H + h) * dv;
        /* kS = k^T S (row vector over value channels) */
        for (int j = 0; j < dv; ++j) {
            double r = 0.0;
            for (int i = 0; i < dk; ++i) r += kt[i] * S[(size_t)i * dv + j];
            kS[j] = r;
        }
        /* S = a * (S - beta k (k^T S)) + beta k v^T */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                S[(size_t)i * dv + j] =
                    at * (S[(size_t)i * dv + j] - bt * kt[i] * kS[j]) + bt * kt[i] * vt[j];
        for (int j = 0; j < dv; ++j) {
            double r = 0.0;
            for (int i = 0; i < dk; ++i) r += qt[i] * S[(size_t)i * dv + j];
            ot[j] = c->scale * r;
        }
    }
    if (c->ht) memcpy(c->ht + sbase, S, sizeof(double) * (size_t)dk * dv);
    free(kS);
    free(S);
}

/* alpha, beta : [T_tot, H] (one scalar log-decay per token and head). */
void kda_oracle_gdn_fwd(const double* q, const double* k, const double* v, const double* alpha,
                        const double* beta, double scale, const double* h0, double* ht, double* o,
                        const int64_t* cu_seqlens, int N, int H, int dk, int dv, int nthreads) {
    gdn_ctx c;
    c.q = q; c.k = k; c.v = v; c.alpha = alpha; c.beta = beta; c.h0 = h0; c.ht = ht; c.o = o;
    c.cu = cu_seqlens; c.scale = scale; c.H = H; c.dk = dk; c.dv = dv;
    run_pairs(gdn_pair, &c, (int64_t)N * H, nthreads);
}

/* ------------------------------------------------------------------------ */
/* Short causal depthwise convolution with cache, then SiLU ([P4], [P5]).    */
/* ------------------------------------------------------------------------ */

/*
 * x, y       : [T_tot, C]      (C = H * d channels, channel-contiguous per token)
 * w          : [C, K]          tap K-1 multiplies the current token
 * cache_in   : [N, C, K-1] or NULL; the K-1 inputs preceding each sequence,
 *              oldest first. NULL means a zero history.
 * cache_out  : [N, C, K-1] or NULL; the last K-1 inputs of the extended
 *              sequence (cache_in followed by x), oldest first.
 * y[t,c] = silu( sum_{j=0}^{K-1} w[c,j] * x[t-(K-1)+j, c] ),  silu(z) = z / (1 + exp(-z)).
 */
void kda_oracle_conv_silu(const double* x, const double* w, const double* cache_in, double* y,
                          double* cache_out, const int64_t* cu_seqlens, int N, int C, int K) {
    const int P = K - 1;
    double* ext = NULL;
    for (int n = 0; n < N; ++n) {
        const int64_t bos = cu_seqlens[n], eos = cu_seqlens[n + 1];
        const int64_t L = eos - bos;
        ext = (double*)realloc(ext, sizeof(double) * (size_t)(L + P));
        for (int c = 0; c < C; ++c) {
            /* the extended input: history (oldest first) then the sequence */
            for (int p = 0; p < P; ++p)
                ext[p] = cache_in ? cache_in[((size_t)n * C + c) * P + p] : 0.0;
            for (int64_t t = 0; t < L; ++t) ext[P + t] = x[(size_t)(bos + t) * C + c];
            for (int64_t t = 0; t < L; ++t) {
                double z = 0.0;
                for (int j = 0; j < K; ++j) z += w[(size_t)c * K + j] * ext[t + j];
                y[(size_t)(bos + t) * C + c] = z / (1.0 + exp(-z));
            }
            if (cache_out)
                for (int p = 0; p < P; ++p)
                    cache_out[((size_t)n * C + c) * P + p] = ext[L + p];
        }
    }
    free(ext);
}

/* In place: each d-vector x[t, h, :] becomes x / sqrt(sum x^2 + eps). */
void kda_oracle_l2norm(double* x, int64_t rows, int d, double eps) {
    for (int64_t r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int i = 0; i < d; ++i) ss += x[(size_t)r * d + i] * x[(size_t)r * d + i];
        const double inv = 1.0 / sqrt(ss + eps);
        for (int i = 0; i < d; ++i) x[(size_t)r * d + i] *= inv;
    }
}

/* ------------------------------------------------------------------------ */
/* Gate activation ([P4]: the gate is computed from a_log_bias and dt_bias;  */
/* delta is the residual times sigmoid(beta)).                               */
/* ------------------------------------------------------------------------ */

/*
 * The pages name only the inputs of the gate. Reading: per token t, head h and key channel c,
 *     g[t, h, c] = -exp(A_log[h]) * softplus(x[t, h, c] + dt_bias[h * dk + c]),
 *     softplus(z) = log(1 + exp(z)),
 * so g <= 0 and exp(g) is the per-row forgetting factor of [P1].
 * x, g : [T_tot, H, dk];  A_log : [H];  dt_bias : [H * dk].
 */
void kda_oracle_gate(const double* x, const double* A_log, const double* dt_bias, double* g,
                     int64_t T_tot, int H, int dk) {
    for (int64_t t = 0; t < T_tot; ++t)
        for (int h = 0; h < H; ++h) {
            const double a = exp(A_log[h]);
            for (int c = 0; c < dk; ++c) {
                const size_t i = ((size_t)t * H + h) * dk + c;
                const double z = x[i] + dt_bias[(size_t)h * dk + c];
                const double sp = z > 30.0 ? z + log1p(exp(-z)) : log1p(exp(z));
                g[i] = -a * sp;
            }
        }
}

/* beta = sigmoid(b_raw), elementwise over n values ([P4]). */
void kda_oracle_sigmoid(const double* b_raw, double* beta, int64_t n) {
    for (int64_t i = 0; i < n; ++i) beta[i] = 1.0 / (1.0 + exp(-b_raw[i]));
}

/* ------------------------------------------------------------------------ */
/* Gated RMSNorm of the output ([P1], "Отвергнутые решения": every norm but   */
/* the QK norms is a gated RMSNorm).                                         */
/* ------------------------------------------------------------------------ */

/*
 * Reading: per token and head, over the dv output channels,
 *     y = o / sqrt(mean(o^2) + eps) * w * sigmoid(z),
 * with a weight w [dv] shared by the heads and a gate z of o's shape.
 * o, z, y : [rows, dv].
 */
void kda_oracle_gated_rmsnorm(const double* o, const double* z, const double* w, double* y,
                              int64_t rows, int dv, double eps) {
    for (int64_t r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int j = 0; j < dv; ++j) ss += o[(size_t)r * dv + j] * o[(size_t)r * dv + j];
        const double inv = 1.0 / sqrt(ss / dv + eps);
        for (int j = 0; j < dv; ++j) {
            const size_t i = (size_t)r * dv + j;
            y[i] = o[i] * inv * w[j] * (1.0 / (1.0 + exp(-z[i])));
        }
    }
}
