/*
 * attn_oracle_bwd.c -- fp64 CPU reference for the gradients of exact attention.
 *
 * TEST INFRASTRUCTURE ONLY, like attn_oracle.c: only the tests may use it; it
 * shares no code with the CUDA library.
 *
 * Forward (the definition of attn_oracle.c): S = scale * Q K^T with masked
 * entries -inf, P = softmax(S) row by row, O = P V.  Given dO = dLoss/dO, the
 * chain rule through these three steps gives, for one query head:
 *
 *   dV = P^T dO                      (O = P V)
 *   dP = dO V^T
 *   dS = P o (dP - D),  D_i = sum_j P_ij dP_ij      (softmax Jacobian, row i)
 *   dQ = scale * dS K,  dK = scale * dS^T Q        (S = scale * Q K^T)
 *
 * "FlashAttention technical analysis" (jsqmd.com/news/722897), section 3.3:
 * the backward pass works from P, which the fused forward does not keep and
 * recomputes block by block from Q, K and the saved per-row statistics; this
 * file is the unfused definition, so it materialises P of one head at a time.
 * Masked entries have P = 0 and therefore dS = 0.  With grouped K/V heads the
 * K/V gradients of a K/V head are the sums over the query heads that read it.
 * A row with no unmasked key has P = 0: it contributes nothing and gets dQ = 0.
 *
 * Variants (oracle_attention_bwd_mod), the same readings as the forward
 * oracle's oracle_attention_fwd_mod: the score is
 *   s_ij = c(x_ij) + mask_ij,  x_ij = scale * <q_i, k_j>,
 * with c(x) = cap * tanh(x / cap) under soft-capping (else c(x) = x), an
 * additive mask added after it, and the 2-D neighbourhood / window masks
 * setting s_ij = -inf outside the query's grid rectangle.  The chain rule
 * through c gives dL/dx_ij = dS_ij * c'(x_ij), c'(x) = 1 - tanh^2(x / cap);
 * dQ and dK then follow from x as above.  The mask has no parameter to
 * differentiate.
 *
 * Every step is fp64; units of work are (batch, K/V head) pairs spread over
 * POSIX threads, each computed by the plain sequence below.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    const double *q, *k, *v, *dout;
    double *dq, *dk, *dv;
    int B, Hq, Hkv, Nq, Nk, d;
    double scale;
    int is_causal;
    const int32_t *key_lens;
    const int32_t *units; /* optional subset of b * Hkv + hkv */
    int n_units;
    const double *mask;                /* additive mask or NULL */
    int64_t mask_sb, mask_sh, mask_sq; /* its element strides */
    double softcap;                    /* 0: off */
    int m2_kind, m2_w, m2_size, m2_shift;
} bwd_args;

/* Whether the 2-D mask lets query i see key j (the forward oracle's rule). */
static int bwd_allowed_2d(const bwd_args *a, int i, int j)
{
    if (a->m2_kind == 0) return 1;
    const int W = a->m2_w;
    const int ri = i / W, ci = i % W, rj = j / W, cj = j % W;
    if (a->m2_kind == 1) {
        const int dr = ri > rj ? ri - rj : rj - ri;
        const int dc = ci > cj ? ci - cj : cj - ci;
        return dr < a->m2_size && dc < a->m2_size;
    }
    if (a->m2_kind == 2) {
        const int w = a->m2_size, sh = a->m2_shift;
        return (ri + sh) / w == (rj + sh) / w && (ci + sh) / w == (cj + sh) / w;
    }
    return 1;
}

typedef struct {
    const bwd_args *a;
    int first, last;
    int status;
} bwd_job;

/* One (batch, K/V head) pair: every query head of its group. */
static int bwd_unit(const bwd_args *a, int b, int hk, double *P, double *dP, double *C)
{
    const int Nq = a->Nq, Nk = a->Nk, d = a->d;
    const int group = a->Hq / a->Hkv;
    const int len = a->key_lens ? a->key_lens[b] : Nk;
    const double *K = a->k + ((int64_t)b * a->Hkv + hk) * (int64_t)Nk * d;
    const double *V = a->v + ((int64_t)b * a->Hkv + hk) * (int64_t)Nk * d;
    double *dK = a->dk + ((int64_t)b * a->Hkv + hk) * (int64_t)Nk * d;
    double *dV = a->dv + ((int64_t)b * a->Hkv + hk) * (int64_t)Nk * d;
    memset(dK, 0, sizeof(double) * (size_t)Nk * d);
    memset(dV, 0, sizeof(double) * (size_t)Nk * d);
    for (int g = 0; g < group; ++g) {
        const int h = hk * group + g;
        const int64_t qh = ((int64_t)b * a->Hq + h) * (int64_t)Nq * d;
        const double *Q = a->q + qh, *dO = a->dout + qh;
        double *dQ = a->dq + qh;
        /* P: scores, masks, row softmax (two passes); C: the derivative c'(x) of the
         * score variant (1 without soft-capping) */
        for (int i = 0; i < Nq; ++i) {
            double *p = P + (int64_t)i * Nk;
            double *c = C + (int64_t)i * Nk;
            const double *mrow = a->mask
                ? a->mask + (int64_t)b * a->mask_sb + (int64_t)h * a->mask_sh + (int64_t)i * a->mask_sq
                : NULL;
            double M = -INFINITY;
            for (int j = 0; j < Nk; ++j) {
                c[j] = 1.0;
                if (j >= len || (a->is_causal && j > i) || !bwd_allowed_2d(a, i, j)) {
                    p[j] = -INFINITY;
                    continue;
                }
                double dot = 0.0;
                for (int t = 0; t < d; ++t) dot += Q[(int64_t)i * d + t] * K[(int64_t)j * d + t];
                p[j] = a->scale * dot;
                if (a->softcap > 0.0) {
                    const double th = tanh(p[j] / a->softcap);
                    p[j] = a->softcap * th;
                    c[j] = 1.0 - th * th;
                }
                if (mrow) p[j] += mrow[j];
                if (p[j] > M) M = p[j];
            }
            if (M == -INFINITY) {
                for (int j = 0; j < Nk; ++j) p[j] = 0.0;
                continue;
            }
            double L = 0.0;
            for (int j = 0; j < Nk; ++j) {
                p[j] = exp(p[j] - M);
                L += p[j];
            }
            for (int j = 0; j < Nk; ++j) p[j] /= L;
        }
        /* dP = dO V^T; D_i = sum_j P_ij dP_ij; dS = P o (dP - D) (stored in dP) */
        for (int i = 0; i < Nq; ++i) {
            const double *p = P + (int64_t)i * Nk;
            double *dp = dP + (int64_t)i * Nk;
            double D = 0.0;
            for (int j = 0; j < Nk; ++j) {
                double s = 0.0;
                for (int t = 0; t < d; ++t) s += dO[(int64_t)i * d + t] * V[(int64_t)j * d + t];
                dp[j] = s;
                D += p[j] * s;
            }
            for (int j = 0; j < Nk; ++j) dp[j] = p[j] * (dp[j] - D);
            /* through the score variant: dL/dx = dS * c'(x) */
            const double *c = C + (int64_t)i * Nk;
            for (int j = 0; j < Nk; ++j) dp[j] *= c[j];
        }
        /* dQ = scale * dS K */
        for (int i = 0; i < Nq; ++i)
            for (int t = 0; t < d; ++t) {
                double s = 0.0;
                for (int j = 0; j < Nk; ++j) s += dP[(int64_t)i * Nk + j] * K[(int64_t)j * d + t];
                dQ[(int64_t)i * d + t] = a->scale * s;
            }
        /* dK += scale * dS^T Q;  dV += P^T dO */
        for (int j = 0; j < Nk; ++j)
            for (int t = 0; t < d; ++t) {
                double sk = 0.0, sv = 0.0;
                for (int i = 0; i < Nq; ++i) {
                    sk += dP[(int64_t)i * Nk + j] * Q[(int64_t)i * d + t];
                    sv += P[(int64_t)i * Nk + j] * dO[(int64_t)i * d + t];
                }
                dK[(int64_t)j * d + t] += a->scale * sk;
                dV[(int64_t)j * d + t] += sv;
            }
    }
    return 0;
}

static void *bwd_worker(void *p)
{
    bwd_job *job = (bwd_job *)p;
    const bwd_args *a = job->a;
    double *P = (double *)malloc(sizeof(double) * (size_t)a->Nq * (size_t)a->Nk);
    double *dP = (double *)malloc(sizeof(double) * (size_t)a->Nq * (size_t)a->Nk);
    double *C = (double *)malloc(sizeof(double) * (size_t)a->Nq * (size_t)a->Nk);
    if (!P || !dP || !C) {
        free(P); free(dP); free(C);
        job->status = -2;
        return NULL;
    }
    for (int u = job->first; u < job->last; ++u) {
        const int id = a->units ? a->units[u] : u;
        bwd_unit(a, id / a->Hkv, id % a->Hkv, P, dP, C);
    }
    free(P); free(dP); free(C);
    job->status = 0;
    return NULL;
}

/*
 * oracle_attention_bwd_mod -- oracle_attention_bwd with the score and mask
 * variants: mask (fp64, element (b, h, i, j) at b*mask_sb + h*mask_sh +
 * i*mask_sq + j, or NULL), softcap (0: off), m2_kind (0 none, 1 neighbourhood
 * of radius m2_size, 2 windows of side m2_size displaced by m2_shift) on a
 * grid of m2_w tokens per row.
 */
int oracle_attention_bwd_mod(const double *q, const double *k, const double *v, const double *dout,
                             double *dq, double *dk, double *dv,
                             int B, int Hq, int Hkv, int Nq, int Nk, int d,
                             double scale, int is_causal, const int32_t *key_lens,
                             const double *mask, int64_t mask_sb, int64_t mask_sh, int64_t mask_sq,
                             double softcap, int m2_kind, int m2_w, int m2_size, int m2_shift,
                             const int32_t *units, int n_units, int n_threads);

/*
 * oracle_attention_bwd
 *   q, dout [B, Hq, Nq, d]; k, v [B, Hkv, Nk, d]: fp64, contiguous.
 *   dq [B, Hq, Nq, d], dk / dv [B, Hkv, Nk, d]: fp64 outputs.
 *   key_lens [B] or NULL; is_causal as in the forward.
 *   units: if non-NULL, only these (b * Hkv + hkv) pairs are computed (all
 *   query heads of each); the other outputs are left untouched.
 * Returns 0, -1 on invalid arguments, -2 on allocation failure.
 */
int oracle_attention_bwd(const double *q, const double *k, const double *v, const double *dout,
                         double *dq, double *dk, double *dv,
                         int B, int Hq, int Hkv, int Nq, int Nk, int d,
                         double scale, int is_causal, const int32_t *key_lens,
                         const int32_t *units, int n_units, int n_threads)
{
    return oracle_attention_bwd_mod(q, k, v, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, is_causal, key_lens,
                                    NULL, 0, 0, 0, 0.0, 0, 1, 1, 0, units, n_units, n_threads);
}

int oracle_attention_bwd_mod(const double *q, const double *k, const double *v, const double *dout,
                             double *dq, double *dk, double *dv,
                             int B, int Hq, int Hkv, int Nq, int Nk, int d,
                             double scale, int is_causal, const int32_t *key_lens,
                             const double *mask, int64_t mask_sb, int64_t mask_sh, int64_t mask_sq,
                             double softcap, int m2_kind, int m2_w, int m2_size, int m2_shift,
                             const int32_t *units, int n_units, int n_threads)
{
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return -1;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0 || Hq % Hkv != 0) return -1;
    if (key_lens)
        for (int b = 0; b < B; ++b)
            if (key_lens[b] < 0 || key_lens[b] > Nk) return -1;
    if (softcap < 0.0 || m2_kind < 0 || m2_kind > 2 || (m2_kind && (m2_w <= 0 || m2_size <= 0 || m2_shift < 0)))
        return -1;
    const int total = units ? n_units : B * Hkv;
    if (units)
        for (int u = 0; u < n_units; ++u)
            if (units[u] < 0 || units[u] >= B * Hkv) return -1;
    if (total <= 0) return -1;
    bwd_args a = {q, k, v, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, is_causal, key_lens, units, n_units,
                  mask, mask_sb, mask_sh, mask_sq, softcap, m2_kind, m2_w, m2_size, m2_shift};
    if (n_threads <= 0) n_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > total) n_threads = total;
    bwd_job *jobs = (bwd_job *)calloc((size_t)n_threads, sizeof(bwd_job));
    pthread_t *tids = (pthread_t *)calloc((size_t)n_threads, sizeof(pthread_t));
    if (!jobs || !tids) {
        free(jobs); free(tids);
        return -2;
    }
    for (int t = 0; t < n_threads; ++t) {
        jobs[t].a = &a;
        jobs[t].first = (int)((int64_t)total * t / n_threads);
        jobs[t].last = (int)((int64_t)total * (t + 1) / n_threads);
        jobs[t].status = -2;
        if (t == 0) continue;
        if (pthread_create(&tids[t], NULL, bwd_worker, &jobs[t]) != 0) {
            bwd_worker(&jobs[t]);
            tids[t] = 0;
        }
    }
    bwd_worker(&jobs[0]);
    int status = 0;
    for (int t = 1; t < n_threads; ++t)
        if (tids[t]) pthread_join(tids[t], NULL);
    for (int t = 0; t < n_threads; ++t)
        if (jobs[t].status != 0) status = jobs[t].status;
    free(jobs); free(tids);
    return status;
}
