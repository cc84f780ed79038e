/*
 * FP64 CPU oracle for the Flint sink-aware GQA attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check of the
 * package entry module and the CPU-baseline leg of the benchmark may build,
 * load or call this file.  It shares no code with the CUDA path.
 *
 * It is the plain definition, written out in double precision with no
 * blocking, fusion or reordering:
 *
 *   1. per-head RMSNorm in weight form (HF discussion on RecursiveSI/flint,
 *      "What was unusually easy": plain RMSNorm, not the 1+w variant;
 *      FlintConfig.rms_norm_eps = 1e-6; "Query/key normalization precedes
 *      RoPE", flint model page, section "Model Architecture"):
 *          n = x / sqrt(mean(x^2) + eps) * w
 *   2. on sliding layers only, NeoX RoPE over all 128 channels
 *      (FlintAttention._apply_rope: "rotate corresponding channels in the two
 *      halves of each head"; FlintConfig: "sliding layers rotate all head
 *      channels"), channel i against channel i+64 with inverse frequency
 *      theta^(-2i/128) at the token's document-local position;
 *   3. logits s_ij = q~_i . k~_j / sqrt(128) over the keys j a query may see:
 *      same document (or batch row), j <= i, and on sliding layers
 *      i - j <= window - 1 (the window counts the current token: flint model
 *      page, "Model Architecture"; HF discussion item 4);
 *   4. the learned sink is one extra softmax column with zero value, in
 *      natural-logit units, not scaled by 1/sqrt(d) (HF discussion,
 *      "learned-sink semantics" and item 5; _FlintSinkParameters.forward
 *      returns unscaled sink logits):
 *          Z = e^sink + sum_j e^s_ij,  out = sum_j e^s_ij v_j / Z,
 *          lse = ln Z;
 *   5. a padded query sees only the sink (FlintAttention.forward,
 *      attention_mask: padded queries and keys are excluded, the sink remains
 *      valid): out = 0, lse = sink.
 *
 * Query head h reads key/value head h / 8 (32 query heads, 4 KV heads).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define HQ 32
#define HKV 4
#define HD 128
#define HALF 64

/* ---- rounding of normalised Q/K, used only for precision-floor studies ---- */

/* Round a double to the nearest BF16 (8 significant bits, 8-bit exponent),
 * ties to even; written from the IEEE-754 definition via frexp.  Values are
 * the ones a normalised head row can take (finite, far from the BF16 range
 * limits). */
static double round_sig(double x, int sig_bits, int min_exp) {
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    double m = frexp(x, &e);           /* x = m * 2^e, 0.5 <= |m| < 1 */
    if (e - 1 < min_exp) e = min_exp + 1; /* subnormal: fixed quantum */
    double q = ldexp(1.0, e - sig_bits); /* spacing of representable values */
    double r = x / q;
    double fl = floor(r);
    double diff = r - fl;
    double res;
    if (diff > 0.5) res = fl + 1.0;
    else if (diff < 0.5) res = fl;
    else res = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    (void)m;
    return res * q;
}

double flint_oracle_round_bf16(double x) { return round_sig(x, 8, -126); }
double flint_oracle_round_fp16(double x) { return round_sig(x, 11, -14); }

/* ---- step 1: RMSNorm, weight form ---- */
void flint_oracle_rmsnorm(const double *x, const double *w, double eps, double *y) {
    double ss = 0.0;
    for (int c = 0; c < HD; ++c) ss += x[c] * x[c];
    double r = 1.0 / sqrt(ss / HD + eps);
    for (int c = 0; c < HD; ++c) y[c] = x[c] * r * w[c];
}

/* ---- step 2: NeoX rotary embedding at integer position pos ---- */
void flint_oracle_rope(const double *x, int64_t pos, double theta, double *y) {
    for (int i = 0; i < HALF; ++i) {
        double f = pow(theta, -2.0 * (double)i / (double)HD);
        double a = (double)pos * f;
        double c = cos(a), s = sin(a);
        double x0 = x[i], x1 = x[i + HALF];
        y[i] = x0 * c - x1 * s;
        y[i + HALF] = x1 * c + x0 * s;
    }
}

/* ---- segment bookkeeping: which tokens share a document / batch row ---- */

/* Packed THD input (FlintAttention.forward, attn_kwargs: shared THD
 * boundaries): tokens [cu[d], cu[d+1]) form document d; tokens at or beyond
 * cu[ndocs] are padding.  Returns 0, or -1 if cu is not a valid boundary list. */
int flint_oracle_doc_ids_thd(int64_t T, const int32_t *cu, int32_t ndocs, int32_t *doc) {
    if (ndocs < 0 || cu[0] != 0 || cu[ndocs] > T) return -1;
    for (int64_t t = 0; t < T; ++t) doc[t] = -1;
    for (int32_t d = 0; d < ndocs; ++d) {
        if (cu[d + 1] < cu[d]) return -1;
        for (int64_t t = cu[d]; t < cu[d + 1]; ++t) doc[t] = d;
    }
    return 0;
}

/* Batch layout with a binary attention mask [B,S], 1 = valid token
 * (FlintAttention.forward, attention_mask).  Token b*S+j belongs to row b if
 * valid, else it is padding. */
int flint_oracle_doc_ids_padmask(int32_t B, int32_t S, const uint8_t *mask, int32_t *doc) {
    for (int64_t b = 0; b < B; ++b)
        for (int64_t j = 0; j < S; ++j)
            doc[b * S + j] = mask[b * S + j] ? (int32_t)b : -1;
    return 0;
}

/* ---- steps 3-5 ---- */

typedef struct {
    int64_t T;
    const double *q, *k, *v, *wq, *wk, *sinks;
    const int32_t *pos, *doc;
    int32_t window, use_rope;
    double theta, eps;
    int32_t qk_round;
    int64_t nrows;
    const int64_t *rows;
    double *out, *lse;
    const double *kt;        /* normalised (and rotated) keys, [T,4,128] */
    const int64_t *posv;     /* effective position per token */
    int64_t next;            /* work counter */
    pthread_mutex_t mu;
} job_t;

static double apply_round(double x, int mode) {
    if (mode == 1) return flint_oracle_round_bf16(x);
    if (mode == 2) return flint_oracle_round_fp16(x);
    return x;
}

/* Normalise (and rotate) one head row: steps 1 and 2. */
static void prep_row(const double *x, const double *w, int64_t pos, const job_t *J, double *y) {
    double n[HD];
    flint_oracle_rmsnorm(x, w, J->eps, n);
    if (J->use_rope) flint_oracle_rope(n, pos, J->theta, y);
    else memcpy(y, n, sizeof(n));
    for (int c = 0; c < HD; ++c) y[c] = apply_round(y[c], J->qk_round);
}

static int visible(const job_t *J, int64_t i, int64_t j) {
    if (J->doc[j] < 0 || J->doc[j] != J->doc[i]) return 0;
    if (j > i) return 0;
    if (J->window > 0 && i - j > (int64_t)J->window - 1) return 0;
    return 1;
}

static void one_row(job_t *J, int64_t r, double *s_buf) {
    const int64_t i = J->rows ? J->rows[r] : r;
    double *out = J->out + r * (int64_t)HQ * HD;
    double *lse = J->lse + r * (int64_t)HQ;
    if (J->doc[i] < 0) {           /* padded query: only the sink is valid */
        for (int h = 0; h < HQ; ++h) {
            lse[h] = J->sinks[h];
            for (int c = 0; c < HD; ++c) out[h * HD + c] = 0.0;
        }
        return;
    }
    int64_t j0 = 0;
    if (J->window > 0 && i - ((int64_t)J->window - 1) > 0) j0 = i - ((int64_t)J->window - 1);
    const double scale = 1.0 / sqrt((double)HD);
    for (int h = 0; h < HQ; ++h) {
        const int g = h / (HQ / HKV);
        double qt[HD];
        prep_row(J->q + (i * HQ + h) * HD, J->wq, J->posv[i], J, qt);
        double sink = J->sinks[h];
        double M = sink;
        int64_t n = 0;
        for (int64_t j = j0; j <= i; ++j) {
            if (!visible(J, i, j)) continue;
            const double *kt = J->kt + (j * HKV + g) * HD;
            double dot = 0.0;
            for (int c = 0; c < HD; ++c) dot += qt[c] * kt[c];
            double s = dot * scale;
            s_buf[j - j0] = s;
            if (s > M || isnan(M)) M = s;
            ++n;
        }
        double *o = out + h * HD;
        for (int c = 0; c < HD; ++c) o[c] = 0.0;
        if (isinf(M) && M > 0) {   /* sink = +inf: all mass on the sink */
            lse[h] = INFINITY;
            continue;
        }
        if (isinf(M) && M < 0) {   /* sink = -inf and no visible key */
            lse[h] = -INFINITY;
            continue;
        }
        double Z = exp(sink - M);
        for (int64_t j = j0; j <= i; ++j) {
            if (!visible(J, i, j)) continue;
            double p = exp(s_buf[j - j0] - M);
            Z += p;
            const double *vv = J->v + (j * HKV + g) * HD;
            for (int c = 0; c < HD; ++c) o[c] += p * vv[c];
        }
        for (int c = 0; c < HD; ++c) o[c] /= Z;
        lse[h] = M + log(Z);
        (void)n;
    }
}

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    int64_t span = J->window > 0 ? J->window : J->T;
    double *s_buf = (double *)malloc(sizeof(double) * (size_t)(span + 1));
    for (;;) {
        pthread_mutex_lock(&J->mu);
        int64_t r0 = J->next;
        J->next += 16;
        pthread_mutex_unlock(&J->mu);
        if (r0 >= J->nrows) break;
        int64_t r1 = r0 + 16 < J->nrows ? r0 + 16 : J->nrows;
        for (int64_t r = r0; r < r1; ++r) one_row(J, r, s_buf);
    }
    free(s_buf);
    return NULL;
}

typedef struct { job_t *J; int64_t t0, t1; } kjob_t;

static void *kworker(void *arg) {
    kjob_t *K = (kjob_t *)arg;
    job_t *J = K->J;
    for (int64_t t = K->t0; t < K->t1; ++t)
        for (int g = 0; g < HKV; ++g)
            prep_row(J->k + (t * HKV + g) * HD, J->wk, J->posv[t], J,
                     (double *)J->kt + (t * HKV + g) * HD);
    return NULL;
}

/*
 * q [T,32,128], k/v [T,4,128], wq/wk [128], sinks [32] (all FP64).
 * pos [T] or NULL (NULL: position = index within the token's segment).
 * doc [T]: segment id per token, -1 for padding (see flint_oracle_doc_ids_*).
 * window <= 0: full causal; else the window length counting the current token.
 * qk_round: 0 = exact, 1 = round normalised Q/K to BF16, 2 = to FP16.
 * rows [nrows] query tokens (NULL: all T, nrows = T).
 * out [nrows,32,128], lse [nrows,32].  nthreads <= 0: all online cores.
 */
int flint_oracle_attn_fwd(int64_t T, const double *q, const double *k, const double *v,
                          const double *wq, const double *wk, const double *sinks,
                          const int32_t *pos, const int32_t *doc,
                          int32_t window, int32_t use_rope, double theta, double eps,
                          int32_t qk_round, int64_t nrows, const int64_t *rows,
                          double *out, double *lse, int32_t nthreads) {
    if (T < 0 || nrows < 0) return -1;
    if (!rows) nrows = T;
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows ? rows[r] : r;
        if (i < 0 || i >= T) return -1;
    }
    if (nthreads <= 0) nthreads = (int32_t)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;

    int64_t *posv = (int64_t *)malloc(sizeof(int64_t) * (size_t)(T > 0 ? T : 1));
    double *kt = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * HKV * HD);
    if (!posv || !kt) { free(posv); free(kt); return -2; }
    /* default positions: index within the segment (first token of each
     * segment is position 0) */
    for (int64_t t = 0; t < T; ++t) {
        if (pos) posv[t] = pos[t];
        else posv[t] = (t > 0 && doc[t - 1] == doc[t]) ? posv[t - 1] + 1 : 0;
    }

    job_t J;
    memset(&J, 0, sizeof(J));
    J.T = T; J.q = q; J.k = k; J.v = v; J.wq = wq; J.wk = wk; J.sinks = sinks;
    J.pos = pos; J.doc = doc; J.window = window; J.use_rope = use_rope;
    J.theta = theta; J.eps = eps; J.qk_round = qk_round;
    J.nrows = nrows; J.rows = rows; J.out = out; J.lse = lse;
    J.kt = kt; J.posv = posv; J.next = 0;
    pthread_mutex_init(&J.mu, NULL);

    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    kjob_t *kj = (kjob_t *)malloc(sizeof(kjob_t) * (size_t)nthreads);
    for (int i = 0; i < nthreads; ++i) {
        kj[i].J = &J;
        kj[i].t0 = T * i / nthreads;
        kj[i].t1 = T * (i + 1) / nthreads;
        pthread_create(&th[i], NULL, kworker, &kj[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &J);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);

    pthread_mutex_destroy(&J.mu);
    free(th); free(kj); free(posv); free(kt);
    return 0;
}
