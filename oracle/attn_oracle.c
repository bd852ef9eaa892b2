/*
 * attn_oracle.c -- fp64 CPU reference for the exact attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link or call
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg use it.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes is the plain, unfused definition of scaled dot-product
 * attention, in the order the pages give it:
 *
 *   "Flash Attention in a production Stable-Diffusion service" (xxmr.cn/news/81028),
 *   section 2.3: S = Q K^T; S = S / sqrt(d_k); S = S + attn_mask;
 *   S = softmax(S, -1); O = S V   (dropout is 0 at inference).
 *
 *   "FlashAttention technical analysis" (jsqmd.com/news/722897), section 2.1:
 *   the three steps QK^T -> softmax -> PV; section 6.2, "precision problems":
 *   the two-pass stable softmax m = max(x), l = sum(exp(x - m)),
 *   softmax = exp(x - m) / l.
 *
 * Readings where the pages are silent (stated once here, applied below):
 *   - the scale multiplies the raw dot product; a mask is added after scaling;
 *   - a key j of batch b is masked when j >= key_len[b] (padding) or, with
 *     is_causal, when j > i (top-left alignment, query i sees keys 0..i);
 *   - a masked score is -infinity, so its probability is exactly 0;
 *   - grouped K/V heads: query head h reads K/V head h / (Hq / Hkv);
 *   - LSE is the natural-log log-sum-exp of the scaled (and masked) scores,
 *     LSE_i = M_i + ln L_i;
 *   - a row with no unmasked key returns O = 0 and LSE = -infinity.
 *
 * Score and mask variants (oracle_attention_fwd_mod):
 *   - soft-capping, the score_mod example of the PyTorch attention article
 *     (atyun.com/61003.html, "Score Mod example: soft-capping with tanh"):
 *     the scaled dot product x = scale * <q_i, k_j> becomes cap * tanh(x / cap);
 *     an additive mask, if any, is added after it (a score_mod acts on the
 *     score, masking comes after);
 *   - 2-D neighbourhood, the mask_mod example of the same article: token n of
 *     a row-major grid with W tokens per row sits at (n / W, n % W); query i
 *     sees key j iff |r_i - r_j| < R and |c_i - c_j| < R;
 *   - 2-D windows, the window attention of "Flash Attention in a production
 *     Stable-Diffusion service" (xxmr.cn/news/81028) section 3.2: the grid is
 *     cut into non-overlapping w x w windows, displaced by `shift` tokens in
 *     both directions (0 = plain, w / 2 = the shifted variant; border windows
 *     are partial, no cyclic wrap), and query i sees key j iff both lie in the
 *     same window: (r_i + shift) / w == (r_j + shift) / w and the same for
 *     the columns.
 *
 * Every arithmetic step is fp64 on the bf16 input values (converted exactly
 * to double by the caller).  Rows are spread over POSIX threads; a row's own
 * arithmetic is the plain sequence below, never blocked or reordered.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <unistd.h>

typedef struct {
    const double *q, *k, *v;
    double *out, *lse;
    int B, Hq, Hkv, Nq, Nk, d;
    double scale;
    int is_causal;
    const int32_t *key_lens;
    const double *mask;
    int64_t mask_sb, mask_sh, mask_sq; /* element strides of the mask */
    double softcap;                    /* 0: off */
    int m2_kind;                       /* 0 none, 1 neighbourhood, 2 windows */
    int m2_w, m2_size, m2_shift;       /* grid width, R or w, window shift */
    const int32_t *rows;               /* optional subset of query rows */
    int n_rows;
    int64_t n_units;                   /* B * Hq * (rows per head) */
    int n_threads;
} oracle_args;

typedef struct {
    const oracle_args *a;
    int64_t first, last; /* [first, last) in unit index space */
    int status;
} oracle_job;

/* Whether the 2-D mask lets query i see key j. */
static int allowed_2d(const oracle_args *a, int i, int j)
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

/* One query row of one head: the three steps of the definition. */
static void oracle_row(const oracle_args *a, int b, int h, int i, double *s)
{
    const int group = a->Hq / a->Hkv;
    const int hk = h / group;
    const int d = a->d;
    const double *qi = a->q + (((int64_t)b * a->Hq + h) * a->Nq + i) * d;
    const double *kh = a->k + ((int64_t)b * a->Hkv + hk) * (int64_t)a->Nk * d;
    const double *vh = a->v + ((int64_t)b * a->Hkv + hk) * (int64_t)a->Nk * d;
    double *oi = a->out + (((int64_t)b * a->Hq + h) * a->Nq + i) * d;
    const int len = a->key_lens ? a->key_lens[b] : a->Nk;
    const double *mrow = a->mask
        ? a->mask + (int64_t)b * a->mask_sb + (int64_t)h * a->mask_sh + (int64_t)i * a->mask_sq
        : NULL;

    /* Step 1: scores s_ij = scale * <q_i, k_j>, soft-capped if asked, (+ mask_ij);
     * masked keys -> -inf. */
    for (int j = 0; j < a->Nk; ++j) {
        if (j >= len || (a->is_causal && j > i) || !allowed_2d(a, i, j)) {
            s[j] = -INFINITY;
            continue;
        }
        double dot = 0.0;
        for (int t = 0; t < d; ++t) dot += qi[t] * kh[(int64_t)j * d + t];
        s[j] = a->scale * dot;
        if (a->softcap > 0.0) s[j] = a->softcap * tanh(s[j] / a->softcap);
        if (mrow) s[j] += mrow[j];
    }

    /* Step 2: two-pass softmax: M = max_j s_ij, then L = sum_j exp(s_ij - M). */
    double M = -INFINITY;
    for (int j = 0; j < a->Nk; ++j)
        if (s[j] > M) M = s[j];
    if (M == -INFINITY) { /* no unmasked key */
        for (int t = 0; t < d; ++t) oi[t] = 0.0;
        if (a->lse) a->lse[((int64_t)b * a->Hq + h) * a->Nq + i] = -INFINITY;
        return;
    }
    double L = 0.0;
    for (int j = 0; j < a->Nk; ++j) {
        s[j] = exp(s[j] - M); /* s now holds the unnormalised p_ij */
        L += s[j];
    }

    /* Step 3: O_i = (sum_j p_ij v_j) / L; LSE_i = M + ln L. */
    for (int t = 0; t < d; ++t) oi[t] = 0.0;
    for (int j = 0; j < a->Nk; ++j) {
        if (s[j] == 0.0) continue; /* exact zero weight adds nothing */
        const double *vj = vh + (int64_t)j * d;
        for (int t = 0; t < d; ++t) oi[t] += s[j] * vj[t];
    }
    for (int t = 0; t < d; ++t) oi[t] /= L;
    if (a->lse) a->lse[((int64_t)b * a->Hq + h) * a->Nq + i] = M + log(L);
}

static void *oracle_worker(void *p)
{
    oracle_job *job = (oracle_job *)p;
    const oracle_args *a = job->a;
    double *s = (double *)malloc(sizeof(double) * (size_t)(a->Nk > 0 ? a->Nk : 1));
    if (!s) {
        job->status = -2;
        return NULL;
    }
    const int per_head = a->rows ? a->n_rows : a->Nq;
    for (int64_t u = job->first; u < job->last; ++u) {
        const int64_t bh = u / per_head;
        const int r = (int)(u % per_head);
        const int b = (int)(bh / a->Hq);
        const int h = (int)(bh % a->Hq);
        const int i = a->rows ? a->rows[r] : r;
        oracle_row(a, b, h, i, s);
    }
    free(s);
    job->status = 0;
    return NULL;
}

/*
 * oracle_attention_fwd_mod
 *   q   [B, Hq, Nq, d], k/v [B, Hkv, Nk, d], out [B, Hq, Nq, d]: fp64, contiguous.
 *   lse [B, Hq, Nq] fp64 or NULL.
 *   key_lens [B] (0 <= len <= Nk) or NULL; mask fp64 with element strides
 *   (sb, sh, sq) and a contiguous last dimension, or NULL.
 *   rows: if non-NULL, only these query indices (in every head) are computed.
 *   n_threads <= 0 uses every online core.
 *   softcap > 0 applies cap * tanh(x / cap) to the scaled score (0: off);
 *   m2_kind 1 (neighbourhood, m2_size = R) or 2 (windows, m2_size = w,
 *   m2_shift) on a grid of m2_w tokens per row; 0: no 2-D mask.
 * Returns 0 on success, -1 on invalid arguments, -2 on allocation failure.
 */
int oracle_attention_fwd_mod(const double *q, const double *k, const double *v,
                             double *out, double *lse,
                             int B, int Hq, int Hkv, int Nq, int Nk, int d,
                             double scale, int is_causal,
                             const int32_t *key_lens,
                             const double *mask, int64_t mask_sb, int64_t mask_sh, int64_t mask_sq,
                             double softcap, int m2_kind, int m2_w, int m2_size, int m2_shift,
                             const int32_t *rows, int n_rows, int n_threads)
{
    if (!q || !k || !v || !out) return -1;
    if (!(softcap >= 0.0)) return -1;
    if (m2_kind < 0 || m2_kind > 2) return -1;
    if (m2_kind != 0 && (m2_w <= 0 || m2_size <= 0 || m2_shift < 0)) return -1;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0) return -1;
    if (Hq % Hkv != 0) return -1;
    if (rows) {
        if (n_rows <= 0) return -1;
        for (int r = 0; r < n_rows; ++r)
            if (rows[r] < 0 || rows[r] >= Nq) return -1;
    }
    if (key_lens)
        for (int b = 0; b < B; ++b)
            if (key_lens[b] < 0 || key_lens[b] > Nk) return -1;

    oracle_args a;
    a.q = q; a.k = k; a.v = v; a.out = out; a.lse = lse;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.d = d;
    a.scale = scale; a.is_causal = is_causal;
    a.key_lens = key_lens;
    a.mask = mask; a.mask_sb = mask_sb; a.mask_sh = mask_sh; a.mask_sq = mask_sq;
    a.softcap = softcap; a.m2_kind = m2_kind; a.m2_w = m2_w; a.m2_size = m2_size; a.m2_shift = m2_shift;
    a.rows = rows; a.n_rows = n_rows;
    a.n_units = (int64_t)B * Hq * (rows ? n_rows : Nq);

    if (n_threads <= 0) n_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (n_threads < 1) n_threads = 1;
    if ((int64_t)n_threads > a.n_units) n_threads = (int)a.n_units;
    a.n_threads = n_threads;

    oracle_job *jobs = (oracle_job *)calloc((size_t)n_threads, sizeof(oracle_job));
    pthread_t *tids = (pthread_t *)calloc((size_t)n_threads, sizeof(pthread_t));
    if (!jobs || !tids) {
        free(jobs); free(tids);
        return -2;
    }
    int status = 0;
    int started = 0;
    for (int t = 0; t < n_threads; ++t) {
        jobs[t].a = &a;
        jobs[t].first = a.n_units * t / n_threads;
        jobs[t].last = a.n_units * (t + 1) / n_threads;
        jobs[t].status = -2;
        if (t == 0) continue; /* the calling thread takes job 0 */
        if (pthread_create(&tids[t], NULL, oracle_worker, &jobs[t]) != 0) {
            oracle_worker(&jobs[t]); /* fall back to running it inline */
            tids[t] = 0;
        } else {
            ++started;
        }
    }
    oracle_worker(&jobs[0]);
    for (int t = 1; t < n_threads; ++t)
        if (tids[t]) pthread_join(tids[t], NULL);
    for (int t = 0; t < n_threads; ++t)
        if (jobs[t].status != 0) status = jobs[t].status;
    (void)started;
    free(jobs);
    free(tids);
    return status;
}

/* The plain definition: no soft-cap, no 2-D mask. */
int oracle_attention_fwd(const double *q, const double *k, const double *v,
                         double *out, double *lse,
                         int B, int Hq, int Hkv, int Nq, int Nk, int d,
                         double scale, int is_causal,
                         const int32_t *key_lens,
                         const double *mask, int64_t mask_sb, int64_t mask_sh, int64_t mask_sq,
                         const int32_t *rows, int n_rows, int n_threads)
{
    return oracle_attention_fwd_mod(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, is_causal, key_lens,
                                    mask, mask_sb, mask_sh, mask_sq, 0.0, 0, 0, 0, 0, rows, n_rows, n_threads);
}

/* Number of threads oracle_attention_fwd would use for n_threads <= 0. */
int oracle_default_threads(void)
{
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n < 1 ? 1 : (int)n;
}
