/*
 * attn_oracle.c -- plain, slow, fp64 CPU oracle for the fused attention forward pass and the
 * K channel-mean pre-pass.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's CPU-baseline
 * arm may load this file's library. It shares no code, header, table or helper with the CUDA
 * path and must never be used to produce a product result.
 *
 * What it computes (the pages name the operation -- the Triton MHA forward "_attn_fwd" with
 * sq, sk, d_head_qk, d_v, HQ/HK and the causal flag, "Tune MHA config & small-head pipeline
 * pathology", Technical Details and the tables after Final status -- but never write the
 * formula out; this is the standard scaled-dot-product attention it names):
 *
 *   for batch bi, query head h < hq, query row i < sq, with kv head g = h / (hq / hk):
 *     J      = { j < sk : !causal  or  j <= i + sk - sq }          (bottom-right causal mask)
 *     s_j    = scale * sum_c Q[bi,i,h,c] * K[bi,j,g,c]             (j in J)
 *     m      = max_J s_j,   l = sum_J exp(s_j - m)
 *     O[bi,i,h,:]  = sum_J exp(s_j - m) * V[bi,j,g,:] / l
 *     LSE[bi,h,i]  = m + ln(l)
 *   An empty J gives O = 0 and LSE = -inf.
 *
 * Sliding window and attention sink (the "GPT-OSS sink+sliding-window" shapes of "Tune MHA
 * config & small-head pipeline pathology", Source of shapes; the pages define neither, and
 * this is the usual reading -- a left window relative to the row's diagonal key, and a
 * per-head logit that joins the softmax denominator without a value):
 *     J      = J  intersected with  { j >= i + sk - sq - window }     (window >= 0)
 *     with sink sigma_h:  m = max(max_J s_j, sigma_h),
 *                         l = sum_J exp(s_j - m) + exp(sigma_h - m),
 *     O and LSE as above; an empty J then gives O = 0 and LSE = sigma_h.
 *
 * K channel mean ("[HIP] Mha v4: run the K-smoothing gate as one HIP call", Summary and the
 * commit message: per-(batch*head) moments of K over its key axis, folded per head):
 *     mean[bi,g,c] = (1/sk) * sum_s K[bi,s,g,c]      (fp64 sum, rounded once to fp32)
 *     K'[bi,s,g,c] = bf16_rne(K[bi,s,g,c] - mean[bi,g,c])
 *
 * Inputs are exchanged as raw bf16 bit patterns (uint16), BSHD and contiguous:
 *   Q [b,sq,hq,dqk], K [b,sk,hk,dqk], V [b,sk,hk,dv], O [b,sq,hq,dv], LSE [b,hq,sq].
 * The *_f64 entry points take the same layouts as fp64 values instead (used for the FP8
 * recipe, whose inputs are E4M3 codes times per-head scales, decoded by the Python side).
 * Every sum is a plain left-to-right loop in double precision.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 -> double: a bf16 value is the top 16 bits of an IEEE binary32. */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* double -> bf16, round to nearest, ties to even, with one rounding step.
 * The spacing of bf16 values around |x| is 2^(e-8) for |x| = m*2^e, 0.5 <= m < 1, and never
 * finer than the subnormal spacing 2^-133. Scaling by a power of two is exact, nearbyint()
 * rounds ties to even in the default rounding mode. */
uint16_t oracle_bf16_rne(double x)
{
    if (isnan(x)) return (uint16_t)0x7FC0;
    int neg = signbit(x) ? 1 : 0;
    double ax = fabs(x);
    uint16_t sign = neg ? (uint16_t)0x8000 : (uint16_t)0;
    if (isinf(ax)) return (uint16_t)(sign | 0x7F80);
    if (ax == 0.0) return sign;
    int e;
    (void)frexp(ax, &e);
    int qexp = e - 8;
    if (qexp < -133) qexp = -133;
    double r = nearbyint(ldexp(ax, -qexp));
    double y = ldexp(r, qexp);
    if (y >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80);
    float f = (float)y; /* exact: y has at most 8 significant bits and is in float range */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (uint16_t)((u >> 16) & 0x7FFF));
}

typedef struct {
    const uint16_t *q, *k, *v;
    const double *qf, *kf, *vf; /* fp64 inputs instead of q, k, v when non-NULL */
    int64_t b, hq, hk, sq, sk, dqk, dv;
    int causal;
    double scale;
    int64_t window;       /* left window (keys before the diagonal), < 0: none */
    const double *sinks;  /* per query head sink logit, or NULL */
    const int64_t *rows; /* nrows triples (bi, h, i), or NULL for every row in BSHD order */
    int64_t nrows;
    double *o, *lse;
    int64_t next; /* guarded by lock */
    pthread_mutex_t lock;
} attn_job;

/* Input element idx of one of the three tensors: bf16 bits or an fp64 value. */
static double in_val(const uint16_t *bits, const double *vals, int64_t idx)
{
    return vals ? vals[idx] : bf16_value(bits[idx]);
}

/* One output row, straight from the definition above. s holds sk doubles, qd holds dqk. */
static void attn_row(const attn_job *a, int64_t bi, int64_t h, int64_t i, double *s, double *qd,
                     double *o_row, double *lse_out)
{
    int64_t group = a->hq / a->hk;
    int64_t g = h / group;
    const int64_t diag = i + a->sk - a->sq; /* the row's diagonal key */
    int64_t hi = a->sk - 1;                 /* allowed keys: lo .. hi */
    if (a->causal && diag < hi) hi = diag;
    int64_t lo = 0;
    if (a->window >= 0 && diag - a->window > lo) lo = diag - a->window;
    const int has_sink = a->sinks != NULL;
    const double sink = has_sink ? a->sinks[h] : 0.0;
    if (hi < lo) {
        for (int64_t c = 0; c < a->dv; ++c) o_row[c] = 0.0;
        *lse_out = has_sink ? sink : -INFINITY;
        return;
    }
    const int64_t n = hi - lo + 1;
    const int64_t qoff = ((bi * a->sq + i) * a->hq + h) * a->dqk;
    for (int64_t c = 0; c < a->dqk; ++c) qd[c] = in_val(a->q, a->qf, qoff + c);

    for (int64_t j = 0; j < n; ++j) {
        const int64_t koff = ((bi * a->sk + lo + j) * a->hk + g) * a->dqk;
        double dot = 0.0;
        for (int64_t c = 0; c < a->dqk; ++c) dot += qd[c] * in_val(a->k, a->kf, koff + c);
        s[j] = a->scale * dot;
    }
    double m = s[0];
    for (int64_t j = 1; j < n; ++j)
        if (s[j] > m) m = s[j];
    if (has_sink && sink > m) m = sink;
    double l = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        s[j] = exp(s[j] - m); /* s now holds the unnormalised weights */
        l += s[j];
    }
    if (has_sink) l += exp(sink - m);
    for (int64_t c = 0; c < a->dv; ++c) o_row[c] = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        const int64_t voff = ((bi * a->sk + lo + j) * a->hk + g) * a->dv;
        for (int64_t c = 0; c < a->dv; ++c) o_row[c] += s[j] * in_val(a->v, a->vf, voff + c);
    }
    for (int64_t c = 0; c < a->dv; ++c) o_row[c] /= l;
    *lse_out = m + log(l);
}

static void *attn_worker(void *arg)
{
    attn_job *a = (attn_job *)arg;
    double *s = (double *)malloc(sizeof(double) * (size_t)(a->sk > 0 ? a->sk : 1));
    double *qd = (double *)malloc(sizeof(double) * (size_t)a->dqk);
    if (!s || !qd) {
        free(s);
        free(qd);
        return (void *)1;
    }
    const int64_t chunk = 16;
    for (;;) {
        pthread_mutex_lock(&a->lock);
        int64_t r0 = a->next;
        a->next += chunk;
        pthread_mutex_unlock(&a->lock);
        if (r0 >= a->nrows) break;
        int64_t r1 = r0 + chunk < a->nrows ? r0 + chunk : a->nrows;
        for (int64_t r = r0; r < r1; ++r) {
            int64_t bi, h, i;
            double *o_row, *lse_out;
            if (a->rows) {
                bi = a->rows[3 * r];
                h = a->rows[3 * r + 1];
                i = a->rows[3 * r + 2];
                o_row = a->o + r * a->dv;
                lse_out = a->lse + r;
            } else { /* r enumerates BSHD output rows: r = (bi*sq + i)*hq + h */
                h = r % a->hq;
                i = (r / a->hq) % a->sq;
                bi = r / (a->hq * a->sq);
                o_row = a->o + r * a->dv;
                lse_out = a->lse + (bi * a->hq + h) * a->sq + i;
            }
            attn_row(a, bi, h, i, s, qd, o_row, lse_out);
        }
    }
    free(s);
    free(qd);
    return NULL;
}

static int run_attn(attn_job *a, int nthreads)
{
    if (a->hk <= 0 || a->hq % a->hk != 0 || a->dqk <= 0 || a->dv <= 0) return 1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 1024) nthreads = 1024;
    pthread_t tid[1024];
    a->next = 0;
    pthread_mutex_init(&a->lock, NULL);
    int started = 0, rc = 0;
    for (int t = 0; t < nthreads; ++t) {
        if (pthread_create(&tid[t], NULL, attn_worker, a) != 0) break;
        ++started;
    }
    if (started == 0) rc = (attn_worker(a) != NULL);
    for (int t = 0; t < started; ++t) {
        void *ret = NULL;
        pthread_join(tid[t], &ret);
        if (ret) rc = 1;
    }
    pthread_mutex_destroy(&a->lock);
    return rc;
}

/* Selected rows with a left window (< 0: none) and per-head sinks (NULL: none):
 * rows[3r..3r+2] = (bi, h, i); o is [nrows, dv], lse is [nrows]. */
int oracle_attn_rows_ex(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t b,
                        int64_t hq, int64_t hk, int64_t sq, int64_t sk, int64_t dqk, int64_t dv,
                        int causal, double scale, int64_t window, const double *sinks,
                        const int64_t *rows, int64_t nrows, double *o, double *lse, int nthreads)
{
    attn_job a = {q, k, v, NULL, NULL, NULL, b, hq, hk, sq, sk, dqk, dv, causal, scale, window,
                  sinks, rows, nrows, o, lse};
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[3 * r] < 0 || rows[3 * r] >= b || rows[3 * r + 1] < 0 ||
            rows[3 * r + 1] >= hq || rows[3 * r + 2] < 0 || rows[3 * r + 2] >= sq)
            return 2;
    return run_attn(&a, nthreads);
}

/* Selected rows, no window, no sink. */
int oracle_attn_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t b,
                     int64_t hq, int64_t hk, int64_t sq, int64_t sk, int64_t dqk, int64_t dv,
                     int causal, double scale, const int64_t *rows, int64_t nrows, double *o,
                     double *lse, int nthreads)
{
    return oracle_attn_rows_ex(q, k, v, b, hq, hk, sq, sk, dqk, dv, causal, scale, -1, NULL,
                               rows, nrows, o, lse, nthreads);
}

/* Every row, with a left window (< 0: none) and per-head sinks (NULL: none). */
int oracle_attn_full_ex(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t b,
                        int64_t hq, int64_t hk, int64_t sq, int64_t sk, int64_t dqk, int64_t dv,
                        int causal, double scale, int64_t window, const double *sinks, double *o,
                        double *lse, int nthreads)
{
    attn_job a = {q, k, v, NULL, NULL, NULL, b, hq, hk, sq, sk, dqk, dv, causal, scale, window,
                  sinks, NULL, b * sq * hq, o, lse};
    return run_attn(&a, nthreads);
}

/* Every row from fp64 inputs (no window, no sink). */
int oracle_attn_full_f64(const double *q, const double *k, const double *v, int64_t b,
                         int64_t hq, int64_t hk, int64_t sq, int64_t sk, int64_t dqk, int64_t dv,
                         int causal, double scale, double *o, double *lse, int nthreads)
{
    attn_job a = {NULL, NULL, NULL, q, k, v, b, hq, hk, sq, sk, dqk, dv, causal, scale, -1, NULL,
                  NULL, b * sq * hq, o, lse};
    return run_attn(&a, nthreads);
}

/* Selected rows from fp64 inputs (no window, no sink). */
int oracle_attn_rows_f64(const double *q, const double *k, const double *v, int64_t b,
                         int64_t hq, int64_t hk, int64_t sq, int64_t sk, int64_t dqk, int64_t dv,
                         int causal, double scale, const int64_t *rows, int64_t nrows, double *o,
                         double *lse, int nthreads)
{
    attn_job a = {NULL, NULL, NULL, q, k, v, b, hq, hk, sq, sk, dqk, dv, causal, scale, -1, NULL,
                  rows, nrows, o, lse};
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[3 * r] < 0 || rows[3 * r] >= b || rows[3 * r + 1] < 0 ||
            rows[3 * r + 1] >= hq || rows[3 * r + 2] < 0 || rows[3 * r + 2] >= sq)
            return 2;
    return run_attn(&a, nthreads);
}

/* Every row: o is BSHD [b,sq,hq,dv], lse is [b,hq,sq]. */
int oracle_attn_full(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t b,
                     int64_t hq, int64_t hk, int64_t sq, int64_t sk, int64_t dqk, int64_t dv,
                     int causal, double scale, double *o, double *lse, int nthreads)
{
    return oracle_attn_full_ex(q, k, v, b, hq, hk, sq, sk, dqk, dv, causal, scale, -1, NULL, o,
                               lse, nthreads);
}

/* Channel mean of K over its sequence axis: mean64/mean32 are [b,hk,d]. */
int oracle_k_mean(const uint16_t *k, int64_t b, int64_t hk, int64_t sk, int64_t d,
                  double *mean64, float *mean32)
{
    if (sk <= 0) return 1;
    for (int64_t bi = 0; bi < b; ++bi)
        for (int64_t g = 0; g < hk; ++g)
            for (int64_t c = 0; c < d; ++c) {
                double sum = 0.0;
                for (int64_t s = 0; s < sk; ++s) sum += bf16_value(k[((bi * sk + s) * hk + g) * d + c]);
                double mean = sum / (double)sk;
                int64_t idx = (bi * hk + g) * d + c;
                if (mean64) mean64[idx] = mean;
                if (mean32) mean32[idx] = (float)mean;
            }
    return 0;
}

/* K' = bf16_rne(K - mean), with the fp32 mean broadcast over the sequence axis. */
/* K-smoothing gate. The pages run it as "per-(batch*head, chunk) moments over the same
 * strided sample, then a per-head fold and gate" with a threshold and a stride they do not
 * print ("[HIP] Mha v4: run the K-smoothing gate as one HIP call", commit message; "below 2048
 * keys a full ... copy of K"). Reading:
 *   sample   keys s = 0, stride, 2*stride, ... < sk with stride = ceil(sk / 2048) (every key
 *            when sk <= 2048); n = the number of sampled keys
 *   moments  mu_c = (1/n) sum_s K[bi,s,g,c],   e_c = (1/n) sum_s K[bi,s,g,c]^2
 *   ratio    r = sum_c mu_c^2 / sum_c e_c        (the share of K's energy in its channel mean;
 *            0 when K is all zero)
 *   gate     r >= threshold
 *   output   mean = gate ? mu (rounded to fp32) : 0, per (bi, g, c)
 * Everything in double precision; mean32 is the fp32 rounding of the output mean. */
int oracle_k_gate(const uint16_t *k, int64_t b, int64_t hk, int64_t sk, int64_t d,
                  double threshold, double *mean64, float *mean32, double *ratio, int *gate)
{
    if (sk <= 0 || d <= 0) return 1;
    const int64_t stride = (sk + 2047) / 2048;
    const int64_t n = (sk + stride - 1) / stride;
    double *mu = (double *)malloc(sizeof(double) * (size_t)d);
    if (!mu) return 1;
    for (int64_t bi = 0; bi < b; ++bi)
        for (int64_t g = 0; g < hk; ++g) {
            double num = 0.0, den = 0.0;
            for (int64_t c = 0; c < d; ++c) {
                double sum = 0.0, sq = 0.0;
                for (int64_t t = 0; t < n; ++t) {
                    const double x = bf16_value(k[((bi * sk + t * stride) * hk + g) * d + c]);
                    sum += x;
                    sq += x * x;
                }
                mu[c] = sum / (double)n;
                num += mu[c] * mu[c];
                den += sq / (double)n;
            }
            const double r = den > 0.0 ? num / den : 0.0;
            const int on = r >= threshold;
            if (ratio) ratio[bi * hk + g] = r;
            if (gate) gate[bi * hk + g] = on;
            for (int64_t c = 0; c < d; ++c) {
                const int64_t idx = (bi * hk + g) * d + c;
                if (mean64) mean64[idx] = on ? mu[c] : 0.0;
                if (mean32) mean32[idx] = on ? (float)mu[c] : 0.0f;
            }
        }
    free(mu);
    return 0;
}

int oracle_k_sub(const uint16_t *k, const float *mean32, uint16_t *kout, int64_t b, int64_t hk,
                 int64_t sk, int64_t d)
{
    for (int64_t bi = 0; bi < b; ++bi)
        for (int64_t s = 0; s < sk; ++s)
            for (int64_t g = 0; g < hk; ++g)
                for (int64_t c = 0; c < d; ++c) {
                    int64_t idx = ((bi * sk + s) * hk + g) * d + c;
                    double x = bf16_value(k[idx]) - (double)mean32[(bi * hk + g) * d + c];
                    kout[idx] = oracle_bf16_rne(x);
                }
    return 0;
}
