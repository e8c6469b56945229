/*
 * CPU oracle for LAMP (look-ahead mixed-precision) attention.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
 * CPU-baseline / reference legs load this library. The CUDA library never calls,
 * links or includes anything here, and this file includes nothing from it.
 *
 * Plain single-threaded C. Every float operation below is one IEEE binary32
 * operation (built with -O2 -ffp-contract=off, no fast-math); everything the
 * method leaves open in precision (criterion, softmax, P.V) is done in double.
 * Loops run in the order the method states them; nothing is blocked or fused.
 *
 * Sources: "LAMP: Look-Ahead Mixed-Precision Inference of Large Language
 * Models", technical summary on gist.science (paper 2601.21623; the Korean and
 * Dutch pages carry the same content):
 *   [Impl]   section "Implementation strategy", steps 1-3: evaluate g in low
 *            precision; estimate the condition number from that baseline output
 *            and pick the sparse index set q; recompute only the selected
 *            components of g in higher precision (e.g. FP32) before f.
 *   [Theory] section "Theoretical basis", item 2 (min ||q||_0 s.t. kappa(q) <= tau)
 *            and item 3, softmax bullet: recompute the key-query product y_j
 *            when 2 z_j (1 - z_j) |y_j| > tau, z the softmax probabilities.
 *   [Exp]    section "Experimental results": PS(mu), a simulated float with mu
 *            mantissa bits; relaxed relative-threshold LAMP, which drops the
 *            dependence on the normalising constant so that softmax stays
 *            one-pass (FlashAttention style).
 *   [Target] section "Main contributions", item 3: the method is applied to the
 *            KQ dot products of attention.
 * Readings where the pages are silent (each one listed with its reason in the
 * design notes):
 *   - PS(mu) keeps binary32's exponent range and subnormals; mu counts the
 *     explicit fraction bits (mu = 23 is binary32); rounding is to nearest,
 *     ties to even, after every binary32 add, starting from acc = +0.
 *   - the score scale (default fl(1/sqrt(d))) multiplies the finished sum once,
 *     in binary32, and is not re-rounded to PS(mu).
 *   - the strict criterion uses the low-precision scores; the relaxed one
 *     replaces z_j by exp(y_j - M) with M the running maximum of the
 *     low-precision scores over 64-key tiles from key 0, and bounds 1 - z_j by 1.
 *   - causal masking is bottom-right aligned: key j is valid for query row i
 *     when j <= i + (n_k - n_q).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define LAMP_ORACLE_RELAXED_TILE 64

enum { ORACLE_STRICT = 0, ORACLE_RELAXED = 1, ORACLE_GIVEN_MASK = 2 };

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bfloat16 bit pattern -> binary32 (exact widening). */
static float bf16_to_f32(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/*
 * PS(mu) rounding [Exp]: round a binary32 value to mu explicit fraction bits,
 * to nearest with ties to even, keeping binary32's exponent range. On the bit
 * pattern this is the usual bias-and-mask: add half an ulp of the target
 * format minus one, plus the lowest kept bit (so that ties go to the even
 * neighbour), then clear the s = 23 - mu dropped bits. A carry out of the
 * fraction moves the value to the next binade (and to infinity past the
 * largest finite value), as round-to-nearest requires. Infinities and NaNs are
 * returned unchanged.
 */
float lamp_oracle_round_ps(float x, int mu)
{
    int s = 23 - mu;
    if (s <= 0) return x;
    uint32_t u = bits_from_f32(x);
    if (((u >> 23) & 0xFFu) == 0xFFu) return x;
    u += (1u << (s - 1)) - 1u + ((u >> s) & 1u);
    u &= ~((1u << s) - 1u);
    return f32_from_bits(u);
}

/* Elementwise PS(mu) rounding of n binary32 values. */
void lamp_oracle_round_ps_array(const float *x, float *y, int64_t n, int mu)
{
    for (int64_t i = 0; i < n; ++i) y[i] = lamp_oracle_round_ps(x[i], mu);
}

/*
 * Low-precision baseline of g [Impl step 1, Exp]: the key-query product
 * accumulated in PS(mu). acc starts at +0; for k = 0..d-1 the product q_k*k_k
 * (one binary32 multiply) is added to acc (one binary32 add) and the sum is
 * rounded to PS(mu). The finished sum is scaled once.
 */
float lamp_oracle_ps_dot(const uint16_t *q, const uint16_t *k, int d, int mu, float scale)
{
    float acc = 0.0f;
    for (int t = 0; t < d; ++t) {
        float p = bf16_to_f32(q[t]) * bf16_to_f32(k[t]);
        float x = acc + p;
        acc = lamp_oracle_round_ps(x, mu);
    }
    return scale * acc;
}

/* Higher-precision recompute of one component [Impl step 3]: the same sequential
 * sum in binary32 (one multiply and one add per step), then the same scaling. */
float lamp_oracle_fp32_dot(const uint16_t *q, const uint16_t *k, int d, float scale)
{
    float acc = 0.0f;
    for (int t = 0; t < d; ++t) {
        float p = bf16_to_f32(q[t]) * bf16_to_f32(k[t]);
        acc = acc + p;
    }
    return scale * acc;
}

/*
 * Strict look-ahead criterion [Theory item 3] for one row of n valid
 * low-precision scores ps[0..n-1], in double:
 *   m = max ps, a = lowest index attaining it, e_j = exp(ps_j - m),
 *   S_rest = sum_{j != a} e_j (ascending j), S = 1 + S_rest, z_j = e_j / S,
 *   1 - z_j = S_rest / S for j = a and (S - e_j) / S otherwise,
 *   c_j = 2 z_j (1 - z_j) |ps_j|.
 * Writing 1 - z through S_rest avoids the cancellation of 1 - z near z = 1
 * (only the row maximum can have z > 1/2).
 */
void lamp_oracle_strict_criterion(const float *ps, int n, double *c)
{
    if (n <= 0) return;
    int a = 0;
    for (int j = 1; j < n; ++j)
        if (ps[j] > ps[a]) a = j;
    double m = (double)ps[a];
    double s_rest = 0.0;
    for (int j = 0; j < n; ++j)
        if (j != a) s_rest += exp((double)ps[j] - m);
    double S = 1.0 + s_rest;
    for (int j = 0; j < n; ++j) {
        double e = (j == a) ? 1.0 : exp((double)ps[j] - m);
        double z = e / S;
        double omz = (j == a) ? s_rest / S : (S - e) / S;
        c[j] = 2.0 * z * omz * fabs((double)ps[j]);
    }
}

/*
 * Relaxed relative-threshold criterion [Exp, relaxed LAMP], in double: keys are
 * taken in tiles of 64 from key 0; M_t is the maximum of the low-precision
 * scores over tiles 0..t; c_j = 2 exp(ps_j - M_t(j)) |ps_j|. No normalising
 * constant is needed, so the test can be made while the row is streamed.
 */
void lamp_oracle_relaxed_criterion(const float *ps, int n, double *c)
{
    double M = -INFINITY;
    for (int t0 = 0; t0 < n; t0 += LAMP_ORACLE_RELAXED_TILE) {
        int t1 = t0 + LAMP_ORACLE_RELAXED_TILE < n ? t0 + LAMP_ORACLE_RELAXED_TILE : n;
        for (int j = t0; j < t1; ++j)
            if ((double)ps[j] > M) M = (double)ps[j];
        for (int j = t0; j < t1; ++j)
            c[j] = 2.0 * exp((double)ps[j] - M) * fabs((double)ps[j]);
    }
}

/*
 * f = softmax of the mixed row followed by P.V, in double:
 *   m' = max y, p_j = exp(y_j - m'), l = sum p_j (ascending), P_j = p_j / l,
 *   out_c = sum_j P_j V_jc (ascending j), lse = m' + ln l.
 * A row with no valid key gives out = 0 and lse = -inf.
 */
void lamp_oracle_softmax_pv(const float *y, int n, const uint16_t *V, int d,
                            double *out, double *lse, double *P)
{
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    if (n <= 0) { if (lse) *lse = -INFINITY; return; }
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) if ((double)y[j] > m) m = (double)y[j];
    double l = 0.0;
    for (int j = 0; j < n; ++j) l += exp((double)y[j] - m);
    for (int j = 0; j < n; ++j) {
        double pj = exp((double)y[j] - m) / l;
        if (P) P[j] = pj;
        for (int c = 0; c < d; ++c) out[c] += pj * (double)bf16_to_f32(V[(size_t)j * d + c]);
    }
    if (lse) *lse = m + log(l);
}

/*
 * One query row of LAMP attention [Impl steps 1-3, then f].
 *   q: d bf16; K, V: n_k x d bf16 of the row's head; keys 0..n_valid-1 valid.
 *   variant: 0 strict, 1 relaxed, 2 given mask (mask_in row, for the
 *   random-selection control); q_j = [c_j > tau] for 0 and 1.
 * Outputs (each may be NULL): ps, y32, mixed (n_k floats; -inf past n_valid),
 * mask (ceil(n_k/32) words, bit j%32 of word j/32, invalid keys 0), crit (n_k
 * doubles; 0 past n_valid), out (d doubles), lse, nsel (selected count).
 */
int lamp_oracle_row(const uint16_t *q, const uint16_t *K, const uint16_t *V,
                    int n_k, int d, int n_valid, float scale, int mu, double tau,
                    int variant, const uint32_t *mask_in,
                    float *ps, float *y32, float *mixed, uint32_t *mask,
                    double *crit, double *out, double *lse, long long *nsel)
{
    if (n_valid < 0 || n_valid > n_k || d <= 0 || mu < 1 || mu > 23) return -1;
    if (variant < 0 || variant > 2) return -1;
    if (variant == ORACLE_GIVEN_MASK && !mask_in) return -1;
    int nwords = (n_k + 31) / 32;
    float *a_ps = (float *)malloc(sizeof(float) * (size_t)(n_k > 0 ? n_k : 1));
    float *a_y32 = (float *)malloc(sizeof(float) * (size_t)(n_k > 0 ? n_k : 1));
    float *a_mix = (float *)malloc(sizeof(float) * (size_t)(n_k > 0 ? n_k : 1));
    double *a_c = (double *)malloc(sizeof(double) * (size_t)(n_k > 0 ? n_k : 1));
    double *a_out = (double *)malloc(sizeof(double) * (size_t)d);
    if (!a_ps || !a_y32 || !a_mix || !a_c || !a_out) {
        free(a_ps); free(a_y32); free(a_mix); free(a_c); free(a_out);
        return -2;
    }
    /* step 1: low-precision baseline; the FP32 value is also formed here so that
     * the caller can compare it, but only selected entries enter the mixed row */
    for (int j = 0; j < n_valid; ++j) {
        a_ps[j] = lamp_oracle_ps_dot(q, K + (size_t)j * d, d, mu, scale);
        a_y32[j] = lamp_oracle_fp32_dot(q, K + (size_t)j * d, d, scale);
    }
    /* step 2: look-ahead selection */
    if (variant == ORACLE_STRICT) lamp_oracle_strict_criterion(a_ps, n_valid, a_c);
    else if (variant == ORACLE_RELAXED) lamp_oracle_relaxed_criterion(a_ps, n_valid, a_c);
    else for (int j = 0; j < n_valid; ++j) a_c[j] = 0.0;
    long long count = 0;
    if (mask) for (int w = 0; w < nwords; ++w) mask[w] = 0u;
    /* step 3: recompute the selected components, keep the rest */
    for (int j = 0; j < n_valid; ++j) {
        int sel;
        if (variant == ORACLE_GIVEN_MASK) sel = (int)((mask_in[j >> 5] >> (j & 31)) & 1u);
        else sel = a_c[j] > tau;
        a_mix[j] = sel ? a_y32[j] : a_ps[j];
        if (sel) {
            ++count;
            if (mask) mask[j >> 5] |= 1u << (j & 31);
        }
    }
    /* f: softmax and P.V on the mixed row */
    double l_lse;
    lamp_oracle_softmax_pv(a_mix, n_valid, V, d, a_out, &l_lse, NULL);
    for (int j = n_valid; j < n_k; ++j) {
        a_ps[j] = -INFINITY; a_y32[j] = -INFINITY; a_mix[j] = -INFINITY; a_c[j] = 0.0;
    }
    if (ps) memcpy(ps, a_ps, sizeof(float) * (size_t)n_k);
    if (y32) memcpy(y32, a_y32, sizeof(float) * (size_t)n_k);
    if (mixed) memcpy(mixed, a_mix, sizeof(float) * (size_t)n_k);
    if (crit) memcpy(crit, a_c, sizeof(double) * (size_t)n_k);
    if (out) memcpy(out, a_out, sizeof(double) * (size_t)d);
    if (lse) *lse = l_lse;
    if (nsel) *nsel = count;
    free(a_ps); free(a_y32); free(a_mix); free(a_c); free(a_out);
    return 0;
}

/* Number of valid keys of query row i (bottom-right causal alignment). */
static int valid_keys(int64_t i, int64_t n_q, int64_t n_k, int causal)
{
    if (!causal) return (int)n_k;
    int64_t v = i + 1 + (n_k - n_q);
    if (v < 0) v = 0;
    if (v > n_k) v = n_k;
    return (int)v;
}

/*
 * A list of query rows of a [B, H, n_q, d] problem. dims = {B, H, n_q, n_k, d};
 * rows holds flat row ids (b*H + h)*n_q + i (NULL: all rows in order). Outputs
 * are stored per listed row: ps/y32/mixed [nrows][n_k], mask [nrows][nwords],
 * crit [nrows][n_k], out [nrows][d], lse [nrows], nsel [nrows]; any may be NULL.
 * mask_in (variant 2) is the full [B, H, n_q, nwords] mask.
 */
int lamp_oracle_rows(const int64_t *dims, int causal,
                     const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                     float scale, int mu, double tau, int variant, const uint32_t *mask_in,
                     const int64_t *rows, int64_t nrows,
                     float *ps, float *y32, float *mixed, uint32_t *mask,
                     double *crit, double *out, double *lse, long long *nsel)
{
    int64_t B = dims[0], H = dims[1], n_q = dims[2], n_k = dims[3], d = dims[4];
    int64_t nwords = (n_k + 31) / 32;
    int64_t total = B * H * n_q;
    if (!rows) nrows = total;
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t row = rows ? rows[r] : r;
        if (row < 0 || row >= total) return -1;
        int64_t bh = row / n_q, i = row % n_q;
        int nv = valid_keys(i, n_q, n_k, causal);
        int rc = lamp_oracle_row(Q + (size_t)row * d, K + (size_t)bh * n_k * d,
                                 V + (size_t)bh * n_k * d, (int)n_k, (int)d, nv, scale, mu,
                                 tau, variant, mask_in ? mask_in + (size_t)row * nwords : NULL,
                                 ps ? ps + (size_t)r * n_k : NULL,
                                 y32 ? y32 + (size_t)r * n_k : NULL,
                                 mixed ? mixed + (size_t)r * n_k : NULL,
                                 mask ? mask + (size_t)r * nwords : NULL,
                                 crit ? crit + (size_t)r * n_k : NULL,
                                 out ? out + (size_t)r * d : NULL,
                                 lse ? lse + r : NULL, nsel ? nsel + r : NULL);
        if (rc) return rc;
    }
    return 0;
}

/*
 * KL(softmax(y_ref) || softmax(y_x)) over the first n entries of two score
 * rows, in double (the accuracy measure of [Exp], taken here per attention row).
 */
double lamp_oracle_row_kl(const float *y_ref, const float *y_x, int n)
{
    if (n <= 0) return 0.0;
    double mr = -INFINITY, mx = -INFINITY;
    for (int j = 0; j < n; ++j) {
        if ((double)y_ref[j] > mr) mr = (double)y_ref[j];
        if ((double)y_x[j] > mx) mx = (double)y_x[j];
    }
    double lr = 0.0, lx = 0.0;
    for (int j = 0; j < n; ++j) {
        lr += exp((double)y_ref[j] - mr);
        lx += exp((double)y_x[j] - mx);
    }
    double log_lr = log(lr), log_lx = log(lx), kl = 0.0;
    for (int j = 0; j < n; ++j) {
        double lp = (double)y_ref[j] - mr - log_lr;
        double lq = (double)y_x[j] - mx - log_lx;
        double p = exp(lp);
        if (p > 0.0) kl += p * (lp - lq);
    }
    return kl;
}

/* Row KL for nrows rows of stride n_k with n_valid[r] valid entries each. */
void lamp_oracle_kl_rows(const float *y_ref, const float *y_x, const int32_t *n_valid,
                         int64_t nrows, int64_t n_k, double *kl)
{
    for (int64_t r = 0; r < nrows; ++r)
        kl[r] = lamp_oracle_row_kl(y_ref + (size_t)r * n_k, y_x + (size_t)r * n_k, n_valid[r]);
}
