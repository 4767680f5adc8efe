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
