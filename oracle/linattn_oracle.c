/*
 * Reference oracle for kernelised causal linear attention read as a
 * fast-weight recurrence.  TEST INFRASTRUCTURE ONLY: this file is compiled
 * into its own shared library and is called by the test-suite, by the smoke
 * check and by the CPU-baseline leg of the benchmark.  The product path (the
 * CUDA library) never links, loads or calls it, and this file includes nothing
 * from the product.
 *
 * Everything is plain scalar IEEE double arithmetic in the order the
 * definitions are written, multithreaded over independent (batch, head)
 * pairs only.  Inputs arrive already widened to double (bf16 and fp32 widen
 * exactly), so both sides of a parity test see the same numbers.
 *
 * Sources (page title, section):
 *   [FW]  "attention is also an FFN" fast-weight article, kwkr.cn/news/587576
 *   [LN]  linear-attention note, tqpw.cn/news/561043
 *   [BSA] "Beyond self-attention: what comes after the Transformer",
 *         datadaily.news/zh/attention-mechanism-alternatives-transformers
 *
 * Layouts (row-major, contiguous):
 *   q, k      [B, H, N, dk]       v, y  [B, H, N, dv]
 *   S         [B, H, dk, dv]      z     [B, H, dk]
 *   lambda    [H] (NULL means lambda = 1 for every head)
 *
 * Every function here is pinned by tests that do not call back into it:
 * brute-force O(N^2) weights, exact rational arithmetic, closed forms and
 * the convex-hull invariant (tests/test_oracle.py).
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* Feature map phi(x) = elu(x) + 1 with ELU alpha = 1:
 * x + 1 for x > 0 and exp(x) otherwise ([FW] §4.1 feature_map; [LN] §4.1,
 * "elu(x)+1", alpha = 1.0; [BSA] linear-attention section).  exp(x) is taken
 * directly rather than as (exp(x) - 1) + 1. */
static double phi(double x) { return x > 0.0 ? x + 1.0 : exp(x); }

void oracle_feature_map(long n, const double *x, double *out) {
    for (long i = 0; i < n; ++i) out[i] = phi(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Work splitting over (batch, head) pairs.                                 */

typedef void (*pair_fn)(void *ctx, long pair);

typedef struct {
    pair_fn fn;
    void *ctx;
    long begin, end;
} span_t;

static void *run_span(void *arg) {
    span_t *s = (span_t *)arg;
    for (long p = s->begin; p < s->end; ++p) s->fn(s->ctx, p);
    return NULL;
}

static int resolve_threads(int nthreads) {
    if (nthreads > 0) return nthreads;
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

static void for_each_pair(long npairs, int nthreads, pair_fn fn, void *ctx) {
    int nt = resolve_threads(nthreads);
    if (nt > npairs) nt = (int)npairs;
    if (nt <= 1) {
        for (long p = 0; p < npairs; ++p) fn(ctx, p);
        return;
    }
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * nt);
    span_t *spans = (span_t *)malloc(sizeof(span_t) * nt);
    long per = npairs / nt, extra = npairs % nt, at = 0;
    for (int t = 0; t < nt; ++t) {
        long len = per + (t < extra ? 1 : 0);
        spans[t].fn = fn;
        spans[t].ctx = ctx;
        spans[t].begin = at;
        spans[t].end = at + len;
        at += len;
        pthread_create(&tid[t], NULL, run_span, &spans[t]);
    }
    for (int t = 0; t < nt; ++t) pthread_join(tid[t], NULL);
    free(spans);
    free(tid);
}

/* ------------------------------------------------------------------------ */
/* Causal recurrence.                                                       */
/*
 * For every (b, h), with lambda_h (1 when lambda is NULL), starting from
 * S_0, z_0 (zeros unless an initial state is given; [FW] §4.1 init_state,
 * [LN] §6 init_state):
 *     S_i = lambda S_{i-1} + phi(k_i) v_i^T       ([FW] §2.1, §3.2)
 *     z_i = lambda z_{i-1} + phi(k_i)             ([FW] §4.2)
 *     y_i = phi(q_i)^T S_i / (phi(q_i)^T z_i + eps)   ([FW] §4.2; [LN] §3)
 * Token i is included in its own output: decay, then add, then read
 * ([FW] §2.1 defines S_i as the sum over j <= i).
 */
typedef struct {
    int H, N, dk, dv;
    const double *q, *k, *v, *lam, *S0, *z0;
    double eps;
    double *y, *S_out, *z_out;
} causal_ctx;

static void causal_pair(void *vctx, long pair) {
    const causal_ctx *c = (const causal_ctx *)vctx;
    const int N = c->N, dk = c->dk, dv = c->dv;
    const int h = (int)(pair % c->H);
    const double lam = c->lam ? c->lam[h] : 1.0;
    const double *q = c->q + (size_t)pair * N * dk;
    const double *k = c->k + (size_t)pair * N * dk;
    const double *v = c->v + (size_t)pair * N * dv;
    double *y = c->y ? c->y + (size_t)pair * N * dv : NULL;

    double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
    double *z = (double *)calloc((size_t)dk, sizeof(double));
    double *fq = (double *)malloc(sizeof(double) * dk);
    double *fk = (double *)malloc(sizeof(double) * dk);
    if (c->S0) memcpy(S, c->S0 + (size_t)pair * dk * dv, sizeof(double) * dk * dv);
    if (c->z0) memcpy(z, c->z0 + (size_t)pair * dk, sizeof(double) * dk);

    for (int i = 0; i < N; ++i) {
        const double *qi = q + (size_t)i * dk;
        const double *ki = k + (size_t)i * dk;
        const double *vi = v + (size_t)i * dv;
        for (int a = 0; a < dk; ++a) {
            fq[a] = phi(qi[a]);
            fk[a] = phi(ki[a]);
        }
        /* state update: decay, then add the outer product phi(k_i) v_i^T */
        for (int a = 0; a < dk; ++a) {
            double *Sa = S + (size_t)a * dv;
            for (int b = 0; b < dv; ++b) Sa[b] = lam * Sa[b] + fk[a] * vi[b];
            z[a] = lam * z[a] + fk[a];
        }
        /* read: numerator phi(q_i)^T S_i and denominator phi(q_i)^T z_i + eps */
        if (y) {
            double den = 0.0;
            for (int a = 0; a < dk; ++a) den += fq[a] * z[a];
            den += c->eps;
            double *yi = y + (size_t)i * dv;
            for (int b = 0; b < dv; ++b) {
                double num = 0.0;
                for (int a = 0; a < dk; ++a) num += fq[a] * S[(size_t)a * dv + b];
                yi[b] = num / den;
            }
        }
    }
    if (c->S_out) memcpy(c->S_out + (size_t)pair * dk * dv, S, sizeof(double) * dk * dv);
    if (c->z_out) memcpy(c->z_out + (size_t)pair * dk, z, sizeof(double) * dk);
    free(fk);
    free(fq);
    free(z);
    free(S);
}

/* Causal forward over N tokens.  S0/z0 may be NULL (zero initial state);
 * y, S_out and z_out may each be NULL when not wanted.  Returns 0, or -1 on
 * a bad argument. */
int oracle_causal(int B, int H, int N, int dk, int dv,
                  const double *q, const double *k, const double *v,
                  const double *lam, double eps,
                  const double *S0, const double *z0,
                  double *y, double *S_out, double *z_out, int nthreads) {
    if (B < 0 || H < 0 || N < 0 || dk <= 0 || dv <= 0) return -1;
    if (N > 0 && (!q || !k || !v)) return -1;
    causal_ctx c = {H, N, dk, dv, q, k, v, lam, S0, z0, eps, y, S_out, z_out};
    for_each_pair((long)B * H, nthreads, causal_pair, &c);
    return 0;
}

/* One decode step ([FW] §4.1 forward_step; [LN] §6 forward_autoregressive):
 * q, k, v are [B, H, d]; S [B, H, dk, dv] and z [B, H, dk] are updated in
 * place; y [B, H, dv] receives the read-out.  It is the recurrence above
 * applied to a single token from the given state. */
int oracle_decode_step(int B, int H, int dk, int dv,
                       const double *q, const double *k, const double *v,
                       const double *lam, double eps,
                       double *S, double *z, double *y, int nthreads) {
    if (!S || !z) return -1;
    return oracle_causal(B, H, 1, dk, dv, q, k, v, lam, eps, S, z, y, S, z, nthreads);
}

/* ------------------------------------------------------------------------ */
/* Global (non-causal) form ([LN] §3 after the sum swap, §6 forward; [BSA]
 * linear-attention section):
 *     KV = sum_n phi(k_n) v_n^T      [dk, dv]
 *     ks = sum_n phi(k_n)            [dk]
 *     y_i = phi(q_i)^T KV / (phi(q_i)^T ks + eps)
 * Every query sees every key; there is no decay (the sum has no order). */
typedef struct {
    int Nq, Nk, dk, dv;
    const double *q, *k, *v;
    double eps;
    double *y, *KV, *ks;
    const unsigned char *pad;   /* [B, Nk], nonzero: the key is padding, or NULL */
    int H;
} global_ctx;

static void global_pair(void *vctx, long pair) {
    const global_ctx *c = (const global_ctx *)vctx;
    const int Nq = c->Nq, Nk = c->Nk, dk = c->dk, dv = c->dv;
    const double *q = c->q + (size_t)pair * Nq * dk;
    const double *k = c->k + (size_t)pair * Nk * dk;
    const double *v = c->v + (size_t)pair * Nk * dv;
    double *KV = (double *)calloc((size_t)dk * dv, sizeof(double));
    double *ks = (double *)calloc((size_t)dk, sizeof(double));
    double *f = (double *)malloc(sizeof(double) * dk);

    const unsigned char *pad = c->pad ? c->pad + (size_t)(pair / c->H) * Nk : NULL;
    for (int n = 0; n < Nk; ++n) {
        if (pad && pad[n]) continue;   /* a padding key enters neither sum */
        const double *kn = k + (size_t)n * dk;
        const double *vn = v + (size_t)n * dv;
        for (int a = 0; a < dk; ++a) f[a] = phi(kn[a]);
        for (int a = 0; a < dk; ++a) {
            for (int b = 0; b < dv; ++b) KV[(size_t)a * dv + b] += f[a] * vn[b];
            ks[a] += f[a];
        }
    }
    if (c->y) {
        for (int i = 0; i < Nq; ++i) {
            const double *qi = q + (size_t)i * dk;
            for (int a = 0; a < dk; ++a) f[a] = phi(qi[a]);
            double den = 0.0;
            for (int a = 0; a < dk; ++a) den += f[a] * ks[a];
            den += c->eps;
            double *yi = c->y + ((size_t)pair * Nq + i) * dv;
            for (int b = 0; b < dv; ++b) {
                double num = 0.0;
                for (int a = 0; a < dk; ++a) num += f[a] * KV[(size_t)a * dv + b];
                yi[b] = num / den;
            }
        }
    }
    if (c->KV) memcpy(c->KV + (size_t)pair * dk * dv, KV, sizeof(double) * dk * dv);
    if (c->ks) memcpy(c->ks + (size_t)pair * dk, ks, sizeof(double) * dk);
    free(f);
    free(ks);
    free(KV);
}

/* Cross form: Nq queries attend to Nk keys/values of another sequence
 * (the linear-attention note's multi-head module, §6, takes target and source
 * lengths); Nq = Nk = N is the self form above. */
int oracle_global_cross(int B, int H, int Nq, int Nk, int dk, int dv,
                        const double *q, const double *k, const double *v, double eps,
                        double *y, double *KV, double *ks, int nthreads) {
    if (B < 0 || H < 0 || Nq < 0 || Nk < 0 || dk <= 0 || dv <= 0) return -1;
    if ((Nq > 0 && !q) || (Nk > 0 && (!k || !v))) return -1;
    global_ctx c = {Nq, Nk, dk, dv, q, k, v, eps, y, KV, ks, NULL, H};
    for_each_pair((long)B * H, nthreads, global_pair, &c);
    return 0;
}

/* Cross form with a key padding mask: the linear-attention note's module
 * forward (§6) takes key_padding_mask (its example leaves it out); a key
 * marked as padding (pad[b][n] != 0, one row per sequence b shared by its
 * heads) is not attended to, so it is left out of both sums KV and ks. */
int oracle_global_masked(int B, int H, int Nq, int Nk, int dk, int dv,
                         const double *q, const double *k, const double *v,
                         const unsigned char *pad, double eps,
                         double *y, double *KV, double *ks, int nthreads) {
    if (B < 0 || H <= 0 || Nq < 0 || Nk < 0 || dk <= 0 || dv <= 0) return -1;
    if ((Nq > 0 && !q) || (Nk > 0 && (!k || !v))) return -1;
    global_ctx c = {Nq, Nk, dk, dv, q, k, v, eps, y, KV, ks, pad, H};
    for_each_pair((long)B * H, nthreads, global_pair, &c);
    return 0;
}

int oracle_global(int B, int H, int N, int dk, int dv,
                  const double *q, const double *k, const double *v, double eps,
                  double *y, double *KV, double *ks, int nthreads) {
    return oracle_global_cross(B, H, N, N, dk, dv, q, k, v, eps, y, KV, ks, nthreads);
}

int oracle_num_threads(int nthreads) { return resolve_threads(nthreads); }
