/*
 * CPU oracle for LAMP on LayerNorm after a PS(mu) linear map.
 *
 * TEST INFRASTRUCTURE ONLY, like lamp_oracle.c (compiled into the same library):
 * only the tests, the smoke check and the benchmark's CPU-baseline / reference
 * legs load it. The CUDA library never calls, links or includes anything here.
 *
 * Sources: "LAMP: Look-Ahead Mixed-Precision Inference of Large Language
 * Models", technical summary on gist.science (paper 2601.21623):
 *   [Theory] section "Theoretical basis": the recompute set q solves
 *            min ||q||_0 s.t. kappa(q) <= tau (item 2); for layer normalisation
 *            a nearly sparsest solution is found greedily by sorting the input
 *            magnitudes (item 3, second bullet).
 *   [Impl]   section "Implementation strategy": g in low precision, selection
 *            from that baseline output, recompute of the selected components of
 *            g in FP32 before f.
 * Readings where the pages are silent (each listed with its reason in the
 * design notes):
 *   - g is the linear map y = scale * x W^T of the activation oracle
 *     (lamp_oracle_act.c), accumulated in PS(mu) like the attention scores.
 *   - f is LayerNorm over the N outputs of a row without the affine part:
 *     f(y) = (y - mean(y)) / sqrt(var(y) + eps), var the biased variance.
 *   - kappa(q) is the norm-wise bound of f's first-order response to relative
 *     errors of the components that are not recomputed: f's Jacobian is
 *     (I - 11^T/N - zz^T/N) / sigma with z the normalised row, a projection
 *     over sigma, so its 2-norm is 1/sigma and
 *         ||f(y + e) - f(y)||_2 <~ ||(1 - q) o y||_2 / sigma  (unit relative errors);
 *     kappa(q) = ||(1 - q) o y_hat||_2 / sigma_hat, at the low-precision row.
 *   - min ||q||_0 s.t. kappa(q) <= tau is then solved exactly by recomputing the
 *     k largest magnitudes, k the smallest count that meets the bound (the
 *     greedy by sorted magnitude); equal magnitudes go in ascending index
 *     order. The sum of squares of the unselected outputs is accumulated from
 *     the smallest magnitude upward. tau < 0 (no feasible q) recomputes all.
 * Precision: everything after the linear map is in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

float lamp_oracle_ps_dot(const uint16_t *q, const uint16_t *k, int d, int mu, float scale);
float lamp_oracle_fp32_dot(const uint16_t *q, const uint16_t *k, int d, float scale);

/* LayerNorm of n values, no affine part, in double: mean and biased variance
 * summed in ascending index order. Returns sigma = sqrt(var + eps). */
double lamp_oracle_layernorm(const double *y, int64_t n, double eps, double *out)
{
    double mean = 0.0, var = 0.0;
    for (int64_t j = 0; j < n; ++j) mean += y[j];
    mean /= (double)n;
    for (int64_t j = 0; j < n; ++j) var += (y[j] - mean) * (y[j] - mean);
    var /= (double)n;
    double sigma = sqrt(var + eps);
    if (out)
        for (int64_t j = 0; j < n; ++j) out[j] = (y[j] - mean) / sigma;
    return sigma;
}

/* Descending magnitude, ties by ascending index. */
typedef struct { double mag; int64_t j; } MagKey;

static int by_magnitude_desc(const void *a, const void *b)
{
    const MagKey *x = (const MagKey *)a, *y = (const MagKey *)b;
    if (x->mag != y->mag) return x->mag > y->mag ? -1 : 1;
    return x->j < y->j ? -1 : (x->j > y->j);
}

/*
 * Greedy selection for one row [Theory item 3]: sel[j] = 1 for the k largest
 * |y_hat_j|, k the smallest count with sqrt(sum of the other squares) <= tau *
 * sigma_hat. Returns k. rest_out (nullable) receives that sum of squares.
 */
int64_t lamp_oracle_ln_select(const float *ps, int64_t n, double eps, double tau, int32_t *sel,
                              double *rest_out)
{
    double *y = (double *)malloc((size_t)n * sizeof(double));
    MagKey *key = (MagKey *)malloc((size_t)n * sizeof(MagKey));
    for (int64_t j = 0; j < n; ++j) {
        y[j] = (double)ps[j];
        key[j].mag = fabs(y[j]);
        key[j].j = j;
    }
    double sigma = lamp_oracle_layernorm(y, n, eps, NULL);
    qsort(key, (size_t)n, sizeof(MagKey), by_magnitude_desc);
    /* unselected = the m smallest (the tail of the descending order); the
     * largest m whose sum of squares, accumulated from the smallest, meets the bound */
    int64_t m = 0;
    double acc = 0.0, rest = 0.0;
    if (tau >= 0.0) {
        for (int64_t t = n - 1; t >= 0; --t) {
            double next = acc + key[t].mag * key[t].mag;
            if (!(sqrt(next) <= tau * sigma)) break;
            acc = next;
            ++m;
        }
        rest = acc;
    }
    int64_t k = n - m;
    for (int64_t j = 0; j < n; ++j) sel[j] = 0;
    for (int64_t t = 0; t < k; ++t) sel[key[t].j] = 1;
    if (rest_out) *rest_out = rest;
    free(key);
    free(y);
    return k;
}

/*
 * The values of tau at which the greedy count of one row changes:
 * t[m - 1] = sqrt(sum of the m smallest squares) / sigma_hat for m = 1 .. n
 * (non-decreasing). The row recomputes n - #{m : t[m-1] <= tau} outputs.
 */
void lamp_oracle_ln_thresholds(const float *ps, int64_t n, double eps, double *t)
{
    double *y = (double *)malloc((size_t)n * sizeof(double));
    MagKey *key = (MagKey *)malloc((size_t)n * sizeof(MagKey));
    for (int64_t j = 0; j < n; ++j) {
        y[j] = (double)ps[j];
        key[j].mag = fabs(y[j]);
        key[j].j = j;
    }
    double sigma = lamp_oracle_layernorm(y, n, eps, NULL);
    qsort(key, (size_t)n, sizeof(MagKey), by_magnitude_desc);
    double acc = 0.0;
    for (int64_t m = 1; m <= n; ++m) {
        acc += key[n - m].mag * key[n - m].mag;
        t[m - 1] = sqrt(acc) / sigma;
    }
    free(key);
    free(y);
}

/*
 * Rows of LAMP LayerNorm(scale * x W^T) [Impl steps 1-3].
 *   dims    = {M, N, K}; x bf16 [M, K], W bf16 [N, K]
 *   variant = 0: the greedy selection; 2: caller mask_in [M][ceil(N/32)]
 * Outputs per evaluated row r (any pointer may be NULL): ps[r][N], mixed[r][N],
 * out[r][N] (double), mask[r][ceil(N/32)], nsel[r], sigma_hat[r] and rest[r]
 * (the selection's sigma and unselected sum of squares).
 */
int lamp_oracle_linear_ln_rows(const int64_t *dims, const uint16_t *x, const uint16_t *W, float scale,
                               int mu, double tau, double eps, int variant, const uint32_t *mask_in,
                               const int64_t *rows, int64_t nrows, float *ps, float *mixed, double *out,
                               uint32_t *mask, int64_t *nsel, double *sigma_hat, double *rest)
{
    int64_t N = dims[1], K = dims[2];
    int64_t nw = (N + 31) / 32;
    if (variant != 0 && variant != 2) return -1;
    float *yl = (float *)malloc((size_t)N * sizeof(float));
    double *ym = (double *)malloc((size_t)N * sizeof(double));
    double *o = (double *)malloc((size_t)N * sizeof(double));
    int32_t *sel = (int32_t *)malloc((size_t)N * sizeof(int32_t));
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows[r];
        const uint16_t *xi = x + i * K;
        /* step 1: the low-precision row of g */
        for (int64_t j = 0; j < N; ++j) yl[j] = lamp_oracle_ps_dot(xi, W + j * K, (int)K, mu, scale);
        /* step 2: the look-ahead selection from that row */
        double rr = 0.0;
        int64_t count;
        if (variant == 0) {
            count = lamp_oracle_ln_select(yl, N, eps, tau, sel, &rr);
        } else {
            count = 0;
            for (int64_t j = 0; j < N; ++j) {
                sel[j] = (int32_t)((mask_in[i * nw + j / 32] >> (j % 32)) & 1u);
                count += sel[j];
            }
        }
        if (sigma_hat) {
            double *yd = o;  /* scratch */
            for (int64_t j = 0; j < N; ++j) yd[j] = (double)yl[j];
            sigma_hat[r] = lamp_oracle_layernorm(yd, N, eps, NULL);
        }
        if (rest) rest[r] = rr;
        /* step 3: recompute the selected outputs in binary32, then f */
        if (mask) memset(mask + r * nw, 0, (size_t)nw * sizeof(uint32_t));
        for (int64_t j = 0; j < N; ++j) {
            float y = sel[j] ? lamp_oracle_fp32_dot(xi, W + j * K, (int)K, scale) : yl[j];
            ym[j] = (double)y;
            if (ps) ps[r * N + j] = yl[j];
            if (mixed) mixed[r * N + j] = y;
            if (mask && sel[j]) mask[r * nw + j / 32] |= 1u << (j % 32);
        }
        lamp_oracle_layernorm(ym, N, eps, o);
        if (out) memcpy(out + r * N, o, (size_t)N * sizeof(double));
        if (nsel) nsel[r] = count;
    }
    free(sel);
    free(o);
    free(ym);
    free(yl);
    return 0;
}
