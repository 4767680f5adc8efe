/*
 * diffattn_oracle.c — fp64 CPU oracle for differential attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no source with the CUDA library.
 *
 * It is a plain, slow statement of what the operator computes: every
 * attention row is materialised in double precision, one query row at a
 * time, with no tiling, no online softmax and no reordering.  Inputs are
 * read as float (bf16 and fp32 values are both exactly representable in
 * float) and widened to double on load.
 *
 * Sources (web pages; cited by page title and section):
 *   [G]  "Differential Transformer", Ultralytics glossary, section
 *        "Cómo funciona la atención diferencial" (same text in the Turkish
 *        edition, "Diferansiyel Dikkat Nasıl Çalışır").
 *   [L]  "Atención Diferencial (V2)", ai-engineering.academy lesson:
 *        "El piso de ruido de softmax", "La idea diferencial",
 *        "V1 vs V2: la diferencia", "Implementación" steps 1-3, and
 *        step 4 "medición de la cancelación de ruido" (signal-to-noise).
 *
 * Readings of points the pages leave open (each one is listed with its
 * reason in the design notes):
 *   - the score scale is 1/sqrt(d) with d the width of ONE branch's query;
 *   - V1 branch r uses columns [(r-1)d, rd) of the head's 2d-wide Q and K;
 *   - lambda is one scalar per head (V1) or per query-head pair (V2), any
 *     sign, never clamped;
 *   - the per-head "GroupNorm" is an RMS normalisation over the d_v output
 *     features of one head row, eps inside the square root, optional
 *     per-feature gain, then a multiply by (1 - lambda_init);
 *   - causal means key j is visible to query i iff j <= i (square prefill);
 *   - V2 pair p is query heads (2p, 2p+1), the even head positive, both
 *     reading KV head (2p) / (Hq / Hkv);
 *   - decode attends every one of the first len_b cache entries.
 *
 * Parity status: every function here is pinned by the not-gpu tests
 * (worked example of [G], closed forms, invariants and library routines).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG -1
#define ORACLE_ERR_NOMEM -2

/* lambda_init for 1-based layer l: 0.8 - 0.6 exp(-0.3 (l - 1)).
 * [G] gives this starting value per layer.  NaN for l < 1. */
double oracle_lambda_init(int layer)
{
    if (layer < 1) return NAN;
    return 0.8 - 0.6 * exp(-0.3 * (double)(layer - 1));
}

/* lambda_h = exp(lq1_h . lk1_h) - exp(lq2_h . lk2_h) + lambda_init(l).
 * [L] "La idea diferencial" (re-parameterised per-head scalar, may be
 * negative); [G] (four small learned vectors, per-layer initial value).
 * Vectors are [n_heads, dim], row-major. */
int oracle_lambda_from_params(const float *lq1, const float *lk1,
                              const float *lq2, const float *lk2,
                              int n_heads, int dim, int layer,
                              double *lambda_out)
{
    if (!lq1 || !lk1 || !lq2 || !lk2 || !lambda_out) return ORACLE_ERR_ARG;
    if (n_heads < 1 || dim < 1 || layer < 1) return ORACLE_ERR_ARG;
    double linit = oracle_lambda_init(layer);
    for (int h = 0; h < n_heads; ++h) {
        double dot1 = 0.0, dot2 = 0.0;
        for (int c = 0; c < dim; ++c) {
            dot1 += (double)lq1[(size_t)h * dim + c] * (double)lk1[(size_t)h * dim + c];
            dot2 += (double)lq2[(size_t)h * dim + c] * (double)lk2[(size_t)h * dim + c];
        }
        lambda_out[h] = exp(dot1) - exp(dot2) + linit;
    }
    return ORACLE_OK;
}

/* Sliding window: of the n visible keys 0..n-1 (causal prefix or cache
 * entries), only the last `window` stay visible; window <= 0 keeps all.
 * [L] "Úselo" names hybrids of differential and sliding-window attention;
 * the reading is that query i then sees keys j with i - window < j <= i in
 * both branches, and a decode query the last `window` cache entries.
 * Returns the first visible key. */
static int64_t window_start(int64_t n, int window)
{
    return (window > 0 && n > (int64_t)window) ? n - (int64_t)window : 0;
}

/* softmax of one row with the row maximum subtracted first
 * ([L] "Implementación", step 1).  In place on x[0..n). */
static void softmax_row(double *x, int64_t n)
{
    double m = x[0];
    for (int64_t j = 1; j < n; ++j)
        if (x[j] > m) m = x[j];
    double s = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        x[j] = exp(x[j] - m);
        s += x[j];
    }
    for (int64_t j = 0; j < n; ++j) x[j] /= s;
}

/*
 * One query row of differential attention over keys 0..n_keys-1:
 *   a1 = softmax(q1 . k1_j / sqrt(d)),  a2 = softmax(q2 . k2_j / sqrt(d))
 *   w_j = a1_j - lambda a2_j,           o_c = sum_j w_j v_j[c]
 * [G] (two softmax maps, combined as (map1 - lambda map2) x V);
 * [L] "La idea diferencial" (A_1, A_2, DiffAttn), step 3.
 * Key j of branch r is at kr + j * k_stride; value j at v + j * v_stride.
 * a1, a2 are scratch rows of n_keys doubles; w (optional) receives w_j.
 */
static void diff_attention_row(const float *q1, const float *q2,
                               const float *k1, const float *k2, int64_t k_stride,
                               const float *v, int64_t v_stride,
                               int64_t n_keys, int d, int dv, double lambda,
                               double *a1, double *a2, double *w_out, double *o)
{
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    for (int64_t j = 0; j < n_keys; ++j) {
        const float *k1j = k1 + j * k_stride;
        const float *k2j = k2 + j * k_stride;
        double s1 = 0.0, s2 = 0.0;
        for (int c = 0; c < d; ++c) {
            s1 += (double)q1[c] * (double)k1j[c];
            s2 += (double)q2[c] * (double)k2j[c];
        }
        a1[j] = s1 * inv_sqrt_d;
        a2[j] = s2 * inv_sqrt_d;
    }
    softmax_row(a1, n_keys);
    softmax_row(a2, n_keys);
    for (int c = 0; c < dv; ++c) o[c] = 0.0;
    for (int64_t j = 0; j < n_keys; ++j) {
        double wj = a1[j] - lambda * a2[j];
        if (w_out) w_out[j] = wj;
        const float *vj = v + j * v_stride;
        for (int c = 0; c < dv; ++c) o[c] += wj * (double)vj[c];
    }
}

/* Per-head normalisation of one output row, then the (1 - lambda_init)
 * scale: y_c = o_c / sqrt(mean_c o_c^2 + eps) * g_c * (1 - lambda_init).
 * [G] (each head normalised on its own, "GroupNorm", then scaled by one
 * minus the initial lambda); [L] "V1 vs V2" calls it a per-head RMSNorm. */
static void head_rms_norm(double *o, int dv, const float *g, double eps,
                          double lambda_init)
{
    double ss = 0.0;
    for (int c = 0; c < dv; ++c) ss += o[c] * o[c];
    double inv_rms = 1.0 / sqrt(ss / (double)dv + eps);
    for (int c = 0; c < dv; ++c) {
        double gc = g ? (double)g[c] : 1.0;
        o[c] = o[c] * inv_rms * gc * (1.0 - lambda_init);
    }
}

/*
 * V1 differential attention, selected output rows.
 *   q, k : [B, N, H, 2d]  (branch 1 = first d columns, branch 2 = last d)
 *   v    : [B, N, H, dv]
 *   lambda: [H] (double)
 *   rows : flattened output-row indices r = (b*N + i)*H + h, n_rows of them
 *   out  : [n_rows, dv] (double)
 *   weights (optional): [n_rows, N] receives w_j for visible keys and 0 for
 *            masked ones.
 * [G] (halves of the query/key projections; values twice as wide).
 */
int oracle_v1_rows(const float *q, const float *k, const float *v,
                   int B, int N, int H, int d, int dv,
                   const double *lambda, int causal, int window,
                   int apply_norm, const float *norm_weight, double eps,
                   double lambda_init,
                   const int64_t *rows, int64_t n_rows,
                   double *out, double *weights)
{
    if (!q || !k || !v || !lambda || !rows || !out) return ORACLE_ERR_ARG;
    if (B < 1 || N < 1 || H < 1 || d < 1 || dv < 1) return ORACLE_ERR_ARG;
    double *a1 = (double *)malloc(sizeof(double) * (size_t)N);
    double *a2 = (double *)malloc(sizeof(double) * (size_t)N);
    if (!a1 || !a2) { free(a1); free(a2); return ORACLE_ERR_NOMEM; }
    const int64_t row_qk = 2LL * d;          /* elements per (token, head) of Q/K */
    const int64_t tok_qk = (int64_t)H * row_qk;
    const int64_t tok_v = (int64_t)H * dv;
    int rc = ORACLE_OK;
    for (int64_t t = 0; t < n_rows; ++t) {
        int64_t r = rows[t];
        if (r < 0 || r >= (int64_t)B * N * H) { rc = ORACLE_ERR_ARG; break; }
        int h = (int)(r % H);
        int64_t bi = r / H;
        int i = (int)(bi % N);
        int b = (int)(bi / N);
        int64_t n_keys = causal ? (int64_t)i + 1 : (int64_t)N;
        const float *qrow = q + ((int64_t)b * N + i) * tok_qk + (int64_t)h * row_qk;
        const float *kb = k + (int64_t)b * N * tok_qk + (int64_t)h * row_qk;
        const float *vb = v + (int64_t)b * N * tok_v + (int64_t)h * dv;
        double *w = weights ? weights + t * (int64_t)N : NULL;
        if (w) for (int64_t j = 0; j < N; ++j) w[j] = 0.0;
        double *o = out + t * (int64_t)dv;
        const int64_t first = window_start(n_keys, window);
        kb += first * tok_qk;
        vb += first * tok_v;
        if (w) w += first;
        diff_attention_row(qrow, qrow + d, kb, kb + d, tok_qk, vb, tok_v,
                           n_keys - first, d, dv, lambda[h], a1, a2, w, o);
        if (apply_norm) head_rms_norm(o, dv, norm_weight, eps, lambda_init);
    }
    free(a1);
    free(a2);
    return rc;
}

/*
 * V2 differential attention, selected output rows.
 *   q : [B, N, Hq, d];  k, v : [B, N, Hkv, d];  lambda : [Hq/2]
 *   pair p = query heads (2p, 2p+1); both read KV head (2p)/(Hq/Hkv).
 *   rows : r = (b*N + i)*(Hq/2) + p;  out : [n_rows, d]; no normalisation.
 * [L] "V1 vs V2: la diferencia" (twice the query heads, KV heads kept, head
 * width kept, no per-head RMSNorm) and "Ejercicios" 5 (GQA with 8 KV heads).
 */
int oracle_v2_rows(const float *q, const float *k, const float *v,
                   int B, int N, int Hq, int Hkv, int d,
                   const double *lambda, int causal, int window,
                   const int64_t *rows, int64_t n_rows,
                   double *out, double *weights)
{
    if (!q || !k || !v || !lambda || !rows || !out) return ORACLE_ERR_ARG;
    if (B < 1 || N < 1 || Hq < 2 || Hkv < 1 || d < 1) return ORACLE_ERR_ARG;
    if (Hq % 2 != 0 || Hq % Hkv != 0 || (Hq / Hkv) % 2 != 0) return ORACLE_ERR_ARG;
    const int P = Hq / 2, group = Hq / Hkv;
    double *a1 = (double *)malloc(sizeof(double) * (size_t)N);
    double *a2 = (double *)malloc(sizeof(double) * (size_t)N);
    if (!a1 || !a2) { free(a1); free(a2); return ORACLE_ERR_NOMEM; }
    const int64_t tok_q = (int64_t)Hq * d, tok_kv = (int64_t)Hkv * d;
    int rc = ORACLE_OK;
    for (int64_t t = 0; t < n_rows; ++t) {
        int64_t r = rows[t];
        if (r < 0 || r >= (int64_t)B * N * P) { rc = ORACLE_ERR_ARG; break; }
        int p = (int)(r % P);
        int64_t bi = r / P;
        int i = (int)(bi % N);
        int b = (int)(bi / N);
        int g = (2 * p) / group;
        int64_t n_keys = causal ? (int64_t)i + 1 : (int64_t)N;
        const float *qa = q + ((int64_t)b * N + i) * tok_q + (int64_t)(2 * p) * d;
        const float *qb = q + ((int64_t)b * N + i) * tok_q + (int64_t)(2 * p + 1) * d;
        const float *kb = k + (int64_t)b * N * tok_kv + (int64_t)g * d;
        const float *vb = v + (int64_t)b * N * tok_kv + (int64_t)g * d;
        double *w = weights ? weights + t * (int64_t)N : NULL;
        if (w) for (int64_t j = 0; j < N; ++j) w[j] = 0.0;
        const int64_t first = window_start(n_keys, window);
        kb += first * tok_kv;
        vb += first * tok_kv;
        if (w) w += first;
        diff_attention_row(qa, qb, kb, kb, tok_kv, vb, tok_kv, n_keys - first, d, d,
                           lambda[p], a1, a2, w, out + t * (int64_t)d);
    }
    free(a1);
    free(a2);
    return rc;
}

/*
 * V2 single-token decode against a KV cache, selected (batch, pair) rows.
 *   q : [B, Hq, d];  k_cache, v_cache : [B, max_len, Hkv, d]
 *   lens : [B] number of valid cache entries (NULL: all max_len)
 *   rows : r = b*(Hq/2) + p;  out : [n_rows, d]
 * The query attends cache entries 0..len_b-1 (the new token's K/V already
 * appended).  [L] "V1 vs V2" (KV cache read once per decode step in V2).
 */
int oracle_v2_decode_rows(const float *q, const float *k_cache, const float *v_cache,
                          const int *lens, int max_len, int window,
                          int B, int Hq, int Hkv, int d, const double *lambda,
                          const int64_t *rows, int64_t n_rows, double *out)
{
    if (!q || !k_cache || !v_cache || !lambda || !rows || !out) return ORACLE_ERR_ARG;
    if (B < 1 || max_len < 1 || Hq < 2 || Hkv < 1 || d < 1) return ORACLE_ERR_ARG;
    if (Hq % 2 != 0 || Hq % Hkv != 0 || (Hq / Hkv) % 2 != 0) return ORACLE_ERR_ARG;
    const int P = Hq / 2, group = Hq / Hkv;
    double *a1 = (double *)malloc(sizeof(double) * (size_t)max_len);
    double *a2 = (double *)malloc(sizeof(double) * (size_t)max_len);
    if (!a1 || !a2) { free(a1); free(a2); return ORACLE_ERR_NOMEM; }
    const int64_t tok_kv = (int64_t)Hkv * d;
    int rc = ORACLE_OK;
    for (int64_t t = 0; t < n_rows; ++t) {
        int64_t r = rows[t];
        if (r < 0 || r >= (int64_t)B * P) { rc = ORACLE_ERR_ARG; break; }
        int p = (int)(r % P), b = (int)(r / P), g = (2 * p) / group;
        int64_t len = lens ? lens[b] : max_len;
        if (len < 1 || len > max_len) { rc = ORACLE_ERR_ARG; break; }
        const float *qa = q + ((int64_t)b * Hq + 2 * p) * d;
        const float *kb = k_cache + (int64_t)b * max_len * tok_kv + (int64_t)g * d;
        const float *vb = v_cache + (int64_t)b * max_len * tok_kv + (int64_t)g * d;
        const int64_t first = window_start(len, window);
        kb += first * tok_kv;
        vb += first * tok_kv;
        diff_attention_row(qa, qa + d, kb, kb, tok_kv, vb, tok_kv, len - first, d, d,
                           lambda[p], a1, a2, NULL, out + t * (int64_t)d);
    }
    free(a1);
    free(a2);
    return rc;
}

/*
 * V1 single-token decode against an MHA cache, selected (batch, head) rows.
 *   q : [B, H, 2d];  k_cache : [B, max_len, H, 2d];  v_cache : [B, max_len, H, dv]
 *   rows : r = b*H + h;  out : [n_rows, dv]; optional per-head norm as in V1.
 */
int oracle_v1_decode_rows(const float *q, const float *k_cache, const float *v_cache,
                          const int *lens, int max_len, int window,
                          int B, int H, int d, int dv, const double *lambda,
                          int apply_norm, const float *norm_weight, double eps,
                          double lambda_init,
                          const int64_t *rows, int64_t n_rows, double *out)
{
    if (!q || !k_cache || !v_cache || !lambda || !rows || !out) return ORACLE_ERR_ARG;
    if (B < 1 || max_len < 1 || H < 1 || d < 1 || dv < 1) return ORACLE_ERR_ARG;
    double *a1 = (double *)malloc(sizeof(double) * (size_t)max_len);
    double *a2 = (double *)malloc(sizeof(double) * (size_t)max_len);
    if (!a1 || !a2) { free(a1); free(a2); return ORACLE_ERR_NOMEM; }
    const int64_t tok_k = (int64_t)H * 2 * d, tok_v = (int64_t)H * dv;
    int rc = ORACLE_OK;
    for (int64_t t = 0; t < n_rows; ++t) {
        int64_t r = rows[t];
        if (r < 0 || r >= (int64_t)B * H) { rc = ORACLE_ERR_ARG; break; }
        int h = (int)(r % H), b = (int)(r / H);
        int64_t len = lens ? lens[b] : max_len;
        if (len < 1 || len > max_len) { rc = ORACLE_ERR_ARG; break; }
        const float *qr = q + ((int64_t)b * H + h) * 2 * d;
        const float *kb = k_cache + (int64_t)b * max_len * tok_k + (int64_t)h * 2 * d;
        const float *vb = v_cache + (int64_t)b * max_len * tok_v + (int64_t)h * dv;
        double *o = out + t * (int64_t)dv;
        const int64_t first = window_start(len, window);
        kb += first * tok_k;
        vb += first * tok_v;
        diff_attention_row(qr, qr + d, kb, kb + d, tok_k, vb, tok_v, len - first, d, dv,
                           lambda[h], a1, a2, NULL, o);
        if (apply_norm) head_rms_norm(o, dv, norm_weight, eps, lambda_init);
    }
    free(a1);
    free(a2);
    return rc;
}

/*
 * Signal-to-noise ratio of one attention-weight row ([L] step 4 asks for the
 * ratio at a signal position in a signal-plus-noise query but fixes no
 * formula).  Reading: the weight at the signal position divided by the
 * root-mean-square weight over every other position,
 *     snr = w[pos] / sqrt( (1/(n-1)) * sum_{j != pos} w[j]^2 ),
 * so a map that puts no weight off the signal has infinite ratio.
 */
int oracle_snr(const double *w, int64_t n, int64_t pos, double *out)
{
    if (!w || !out || n < 2 || pos < 0 || pos >= n) return ORACLE_ERR_ARG;
    double ss = 0.0;
    for (int64_t j = 0; j < n; ++j)
        if (j != pos) ss += w[j] * w[j];
    const double rms = sqrt(ss / (double)(n - 1));
    *out = rms > 0.0 ? w[pos] / rms : (w[pos] > 0.0 ? INFINITY : (w[pos] < 0.0 ? -INFINITY : NAN));
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------
 * Backward pass (gradients of a scalar loss with respect to every input).
 * The pages give the forward only; the gradients below are those of that
 * forward, obtained with the chain rule step by step (the "reading" is
 * only that lambda, and in V1 the norm gain g, are trainable: the glossary
 * page calls lambda learned, from four re-parameterised vectors).
 * ------------------------------------------------------------------------ */

/* One query row: given d(loss)/d(o) for the pre-norm output o (= do), the
 * row's softmax maps a1, a2 (over n_keys keys starting at k1/k2/v), add the
 * row's contributions to dq (this row), dk, dv (those keys) and return
 * d(loss)/d(lambda) of this row.
 *   o = sum_j (a1_j - lambda a2_j) v_j          (forward, [G])
 *   dv_j   += (a1_j - lambda a2_j) do
 *   dlambda = -sum_c do_c (sum_j a2_j v_j[c])
 *   branch r with do_r = do (r = 1) or -lambda do (r = 2):
 *     dp_j = do_r . v_j,   D = sum_j a_r,j dp_j,   ds_j = a_r,j (dp_j - D)
 *     dq_r += sum_j ds_j k_r,j / sqrt(d),   dk_r,j += ds_j q_r / sqrt(d)
 */
static double diff_attention_row_bwd(const float *q1, const float *q2,
                                     const float *k1, const float *k2, int64_t k_stride,
                                     const float *v, int64_t v_stride, int64_t n_keys,
                                     int d, int dv, double lambda,
                                     const double *a1, const double *a2, const double *dout,
                                     double *dq1, double *dq2,
                                     double *dk1, double *dk2, int64_t dk_stride,
                                     double *dvv, int64_t dv_stride)
{
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    double dlam = 0.0;
    for (int64_t j = 0; j < n_keys; ++j) {
        const float *vj = v + j * v_stride;
        double dp = 0.0;
        for (int c = 0; c < dv; ++c) dp += dout[c] * (double)vj[c];
        dlam -= a2[j] * dp;
        double wj = a1[j] - lambda * a2[j];
        double *dvj = dvv + j * dv_stride;
        for (int c = 0; c < dv; ++c) dvj[c] += wj * dout[c];
    }
    for (int r = 0; r < 2; ++r) {
        const double *a = r == 0 ? a1 : a2;
        const double coef = r == 0 ? 1.0 : -lambda;
        const float *qr = r == 0 ? q1 : q2;
        const float *kr = r == 0 ? k1 : k2;
        double *dqr = r == 0 ? dq1 : dq2;
        double *dkr = r == 0 ? dk1 : dk2;
        double D = 0.0;
        for (int64_t j = 0; j < n_keys; ++j) {
            const float *vj = v + j * v_stride;
            double dp = 0.0;
            for (int c = 0; c < dv; ++c) dp += coef * dout[c] * (double)vj[c];
            D += a[j] * dp;
        }
        for (int64_t j = 0; j < n_keys; ++j) {
            const float *vj = v + j * v_stride;
            double dp = 0.0;
            for (int c = 0; c < dv; ++c) dp += coef * dout[c] * (double)vj[c];
            const double ds = a[j] * (dp - D) * inv_sqrt_d;
            const float *kj = kr + j * k_stride;
            double *dkj = dkr + j * dk_stride;
            for (int c = 0; c < d; ++c) {
                dqr[c] += ds * (double)kj[c];
                dkj[c] += ds * (double)qr[c];
            }
        }
    }
    return dlam;
}

/* The two softmax maps of one row (as in diff_attention_row, without V). */
static void softmax_maps(const float *q1, const float *q2, const float *k1, const float *k2,
                         int64_t k_stride, int64_t n_keys, int d, double *a1, double *a2)
{
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    for (int64_t j = 0; j < n_keys; ++j) {
        double s1 = 0.0, s2 = 0.0;
        for (int c = 0; c < d; ++c) {
            s1 += (double)q1[c] * (double)k1[j * k_stride + c];
            s2 += (double)q2[c] * (double)k2[j * k_stride + c];
        }
        a1[j] = s1 * inv_sqrt_d;
        a2[j] = s2 * inv_sqrt_d;
    }
    softmax_row(a1, n_keys);
    softmax_row(a2, n_keys);
}

/*
 * V1 backward over the whole problem.  Inputs as oracle_v1_rows plus
 * dout [B, N, H, dv] (gradient of the loss with respect to the output).
 * Outputs (double, overwritten): dq, dk [B, N, H, 2d]; dvv [B, N, H, dv];
 * dlambda [H] (summed over batch and rows); dnorm_weight [dv] (may be NULL;
 * only with apply_norm).  With the norm,
 *   y = o * g * c / r,  r = sqrt(mean(o^2) + eps),  c = 1 - lambda_init
 *   do_k = (c / r) * (g_k dy_k - o_k * sum_m(g_m dy_m o_m) / (dv r^2))
 *   dg_k += dy_k o_k c / r.
 */
int oracle_v1_bwd(const float *q, const float *k, const float *v, const float *dout,
                  int B, int N, int H, int d, int dv, const double *lambda,
                  int causal, int window, int apply_norm, const float *norm_weight,
                  double eps, double lambda_init,
                  double *dq, double *dk, double *dvv, double *dlambda, double *dnorm_weight)
{
    if (!q || !k || !v || !dout || !lambda || !dq || !dk || !dvv || !dlambda)
        return ORACLE_ERR_ARG;
    if (B < 1 || N < 1 || H < 1 || d < 1 || dv < 1) return ORACLE_ERR_ARG;
    double *a1 = (double *)malloc(sizeof(double) * (size_t)N);
    double *a2 = (double *)malloc(sizeof(double) * (size_t)N);
    double *o = (double *)malloc(sizeof(double) * (size_t)dv);
    double *g_o = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!a1 || !a2 || !o || !g_o) { free(a1); free(a2); free(o); free(g_o); return ORACLE_ERR_NOMEM; }
    const int64_t row_qk = 2LL * d, tok_qk = (int64_t)H * row_qk, tok_v = (int64_t)H * dv;
    for (int64_t t = 0; t < (int64_t)B * N * tok_qk; ++t) { dq[t] = 0.0; dk[t] = 0.0; }
    for (int64_t t = 0; t < (int64_t)B * N * tok_v; ++t) dvv[t] = 0.0;
    for (int h = 0; h < H; ++h) dlambda[h] = 0.0;
    if (dnorm_weight) for (int c = 0; c < dv; ++c) dnorm_weight[c] = 0.0;
    const double cpost = 1.0 - lambda_init;
    for (int b = 0; b < B; ++b)
        for (int i = 0; i < N; ++i)
            for (int h = 0; h < H; ++h) {
                int64_t n_keys = causal ? (int64_t)i + 1 : (int64_t)N;
                const int64_t first = window_start(n_keys, window);
                const int64_t tq = ((int64_t)b * N + i) * tok_qk + (int64_t)h * row_qk;
                const int64_t k0 = ((int64_t)b * N + first) * tok_qk + (int64_t)h * row_qk;
                const int64_t v0 = ((int64_t)b * N + first) * tok_v + (int64_t)h * dv;
                const int64_t nk = n_keys - first;
                softmax_maps(q + tq, q + tq + d, k + k0, k + k0 + d, tok_qk, nk, d, a1, a2);
                const float *dy = dout + ((int64_t)b * N + i) * tok_v + (int64_t)h * dv;
                double *gro = g_o;   /* d(loss)/d(o) */
                if (apply_norm) {
                    for (int c = 0; c < dv; ++c) {
                        double s = 0.0;
                        for (int64_t j = 0; j < nk; ++j)
                            s += (a1[j] - lambda[h] * a2[j]) * (double)v[v0 + j * tok_v + c];
                        o[c] = s;
                    }
                    double ss = 0.0;
                    for (int c = 0; c < dv; ++c) ss += o[c] * o[c];
                    const double r = sqrt(ss / (double)dv + eps);
                    double gdo = 0.0;
                    for (int c = 0; c < dv; ++c) {
                        const double gc = norm_weight ? (double)norm_weight[c] : 1.0;
                        gdo += gc * (double)dy[c] * o[c];
                    }
                    for (int c = 0; c < dv; ++c) {
                        const double gc = norm_weight ? (double)norm_weight[c] : 1.0;
                        gro[c] = (cpost / r) * (gc * (double)dy[c] - o[c] * gdo / ((double)dv * r * r));
                        if (dnorm_weight) dnorm_weight[c] += (double)dy[c] * o[c] * cpost / r;
                    }
                } else {
                    for (int c = 0; c < dv; ++c) gro[c] = (double)dy[c];
                }
                dlambda[h] += diff_attention_row_bwd(
                    q + tq, q + tq + d, k + k0, k + k0 + d, tok_qk, v + v0, tok_v, nk, d, dv,
                    lambda[h], a1, a2, gro, dq + tq, dq + tq + d, dk + k0, dk + k0 + d, tok_qk,
                    dvv + v0, tok_v);
            }
    free(a1); free(a2); free(o); free(g_o);
    return ORACLE_OK;
}

/*
 * V2 backward over the whole problem.  Inputs as oracle_v2_rows plus
 * dout [B, N, Hq/2, d].  Outputs (double, overwritten): dq [B, N, Hq, d];
 * dk, dvv [B, N, Hkv, d] (summed over the pairs that share a KV head);
 * dlambda [Hq/2] (summed over batch and rows).
 */
int oracle_v2_bwd(const float *q, const float *k, const float *v, const float *dout,
                  int B, int N, int Hq, int Hkv, int d, const double *lambda,
                  int causal, int window,
                  double *dq, double *dk, double *dvv, double *dlambda)
{
    if (!q || !k || !v || !dout || !lambda || !dq || !dk || !dvv || !dlambda)
        return ORACLE_ERR_ARG;
    if (B < 1 || N < 1 || Hq < 2 || Hkv < 1 || d < 1) return ORACLE_ERR_ARG;
    if (Hq % 2 != 0 || Hq % Hkv != 0 || (Hq / Hkv) % 2 != 0) return ORACLE_ERR_ARG;
    const int P = Hq / 2, group = Hq / Hkv;
    double *a1 = (double *)malloc(sizeof(double) * (size_t)N);
    double *a2 = (double *)malloc(sizeof(double) * (size_t)N);
    double *gro = (double *)malloc(sizeof(double) * (size_t)d);
    if (!a1 || !a2 || !gro) { free(a1); free(a2); free(gro); return ORACLE_ERR_NOMEM; }
    const int64_t tok_q = (int64_t)Hq * d, tok_kv = (int64_t)Hkv * d, tok_o = (int64_t)P * d;
    for (int64_t t = 0; t < (int64_t)B * N * tok_q; ++t) dq[t] = 0.0;
    for (int64_t t = 0; t < (int64_t)B * N * tok_kv; ++t) { dk[t] = 0.0; dvv[t] = 0.0; }
    for (int p = 0; p < P; ++p) dlambda[p] = 0.0;
    for (int b = 0; b < B; ++b)
        for (int i = 0; i < N; ++i)
            for (int p = 0; p < P; ++p) {
                const int g = (2 * p) / group;
                int64_t n_keys = causal ? (int64_t)i + 1 : (int64_t)N;
                const int64_t first = window_start(n_keys, window);
                const int64_t nk = n_keys - first;
                const int64_t qa = ((int64_t)b * N + i) * tok_q + (int64_t)(2 * p) * d;
                const int64_t qb = qa + d;
                const int64_t k0 = ((int64_t)b * N + first) * tok_kv + (int64_t)g * d;
                softmax_maps(q + qa, q + qb, k + k0, k + k0, tok_kv, nk, d, a1, a2);
                const float *dy = dout + ((int64_t)b * N + i) * tok_o + (int64_t)p * d;
                for (int c = 0; c < d; ++c) gro[c] = (double)dy[c];
                dlambda[p] += diff_attention_row_bwd(
                    q + qa, q + qb, k + k0, k + k0, tok_kv, v + k0, tok_kv, nk, d, d,
                    lambda[p], a1, a2, gro, dq + qa, dq + qb, dk + k0, dk + k0, tok_kv,
                    dvv + k0, tok_kv);
            }
    free(a1); free(a2); free(gro);
    return ORACLE_OK;
}

/* Gradients of the four lambda vectors from d(loss)/d(lambda):
 *   lambda = exp(lq1.lk1) - exp(lq2.lk2) + lambda_init   ([G], [L])
 *   dlq1 = dl e1 lk1, dlk1 = dl e1 lq1, dlq2 = -dl e2 lk2, dlk2 = -dl e2 lq2. */
int oracle_lambda_params_bwd(const float *lq1, const float *lk1, const float *lq2,
                             const float *lk2, int H, int dim, const double *dlambda,
                             double *dlq1, double *dlk1, double *dlq2, double *dlk2)
{
    if (!lq1 || !lk1 || !lq2 || !lk2 || !dlambda || !dlq1 || !dlk1 || !dlq2 || !dlk2 ||
        H < 1 || dim < 1)
        return ORACLE_ERR_ARG;
    for (int h = 0; h < H; ++h) {
        double dot1 = 0.0, dot2 = 0.0;
        for (int c = 0; c < dim; ++c) {
            dot1 += (double)lq1[h * dim + c] * (double)lk1[h * dim + c];
            dot2 += (double)lq2[h * dim + c] * (double)lk2[h * dim + c];
        }
        const double e1 = exp(dot1) * dlambda[h], e2 = exp(dot2) * dlambda[h];
        for (int c = 0; c < dim; ++c) {
            dlq1[h * dim + c] = e1 * (double)lk1[h * dim + c];
            dlk1[h * dim + c] = e1 * (double)lq1[h * dim + c];
            dlq2[h * dim + c] = -e2 * (double)lk2[h * dim + c];
            dlk2[h * dim + c] = -e2 * (double)lq2[h * dim + c];
        }
    }
    return ORACLE_OK;
}
