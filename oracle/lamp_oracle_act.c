/*
 * CPU oracle for LAMP on an elementwise activation: GELU after a PS(mu) linear map.
 *
 * TEST INFRASTRUCTURE ONLY, like lamp_oracle.c (compiled into the same library):
 * only the tests, the smoke check and the benchmark's CPU-baseline / reference
 * legs load it. The CUDA library never calls, links or includes anything here.
 *
 * Sources: "LAMP: Look-Ahead Mixed-Precision Inference of Large Language
 * Models", technical summary on gist.science (paper 2601.21623):
 *   [Theory] section "Theoretical basis": the error of a composition f(g(x)) is
 *            bounded through the condition number of the outer function f and
 *            the rounding error of the inner g (item 1); the recompute set q
 *            solves min ||q||_0 s.t. kappa(q) <= tau with a component-wise or
 *            norm-wise condition number (item 2); for activation functions the
 *            Jacobian is diagonal, so the sensitive components are found
 *            directly (item 3, first bullet).
 *   [Impl]   section "Implementation strategy": g in low precision, selection
 *            from that baseline output, recompute of the selected components of
 *            g in FP32 before f.
 * Readings where the pages are silent (each listed with its reason in the
 * design notes):
 *   - g is a linear map y = scale * x W^T (x [M, K], W [N, K], the weight layout
 *     of a linear layer) accumulated in PS(mu) exactly like the attention
 *     scores: sequential over k, one binary32 multiply and add per step, PS(mu)
 *     rounding after every add from acc = +0, the scale applied once at the end.
 *   - f is GELU in its tanh form, the activation of GPT-2 (the model the pages
 *     evaluate): f(y) = y/2 (1 + tanh(c (y + a y^3))), c = sqrt(2/pi),
 *     a = 0.044715.
 *   - the condition number is the component-wise relative one of a diagonal
 *     Jacobian, kappa_j = |y_j f'(y_j) / f(y_j)| (its limit 1 at y_j = 0), taken
 *     at the low-precision output; component j is recomputed when
 *     kappa_j > tau. Then max_j (1 - q_j) kappa_j <= tau holds with the fewest
 *     recomputed components, which is the pages' optimisation problem solved in
 *     closed form for a diagonal Jacobian.
 *   - kappa of a non-finite low-precision output is +inf (always recomputed
 *     unless tau = +inf).
 * Precision: everything after the scores (kappa, the activation) is in double.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

float lamp_oracle_ps_dot(const uint16_t *q, const uint16_t *k, int d, int mu, float scale);
float lamp_oracle_fp32_dot(const uint16_t *q, const uint16_t *k, int d, float scale);

#define GELU_A 0.044715

static double gelu_c(void) { return sqrt(2.0 / acos(-1.0)); }

/* GELU, tanh form, in double. */
double lamp_oracle_gelu(double y)
{
    double u = gelu_c() * (y + GELU_A * y * y * y);
    return 0.5 * y * (1.0 + tanh(u));
}

/*
 * kappa(y) = |y f'(y) / f(y)| for the tanh-form GELU, in double.
 * Write f(y) = y h(y) with h = (1 + tanh u) / 2 and u = c (y + a y^3). Then
 * y f'(y) / f(y) = 1 + y h'(y) / h(y), and h'/h = u' (1 - tanh^2 u) / (1 + tanh u)
 * = u' (1 - tanh u), with u' = c (1 + 3 a y^2). The factor 1 - tanh u is taken as
 * 2 / (1 + e^{2u}), which loses nothing when tanh u is close to -1 or +1 (very
 * negative inputs, where f(y) underflows while kappa stays finite). At y = 0 the
 * expression is 1, the limit of y f'/f there.
 */
double lamp_oracle_gelu_kappa(double y)
{
    if (!isfinite(y)) return INFINITY;
    double c = gelu_c();
    double u = c * (y + GELU_A * y * y * y);
    double du = c * (1.0 + 3.0 * GELU_A * y * y);
    double one_minus_t = 2.0 / (1.0 + exp(2.0 * u));
    return fabs(1.0 + y * du * one_minus_t);
}

/*
 * Rows of LAMP GELU(scale * x W^T) [Impl steps 1-3].
 *   dims     = {M, N, K}; x bf16 [M, K], W bf16 [N, K] (row-major bit patterns)
 *   variant  = 0: kappa test (q_j = [kappa_j > tau]); 2: caller mask_in [M][ceil(N/32)]
 *   rows     = the row indices to evaluate (nrows of them)
 * Outputs per evaluated row r (any pointer may be NULL):
 *   ps[r][N], mixed[r][N] (binary32), kappa[r][N], out[r][N] (double),
 *   mask[r][ceil(N/32)] (bit j%32 of word j/32), nsel[r].
 * Returns 0, or -1 on an unknown variant.
 */
int lamp_oracle_linear_gelu_rows(const int64_t *dims, const uint16_t *x, const uint16_t *W, float scale,
                                 int mu, double tau, int variant, const uint32_t *mask_in,
                                 const int64_t *rows, int64_t nrows, float *ps, float *mixed,
                                 double *kappa, uint32_t *mask, double *out, int64_t *nsel)
{
    int64_t M = dims[0], N = dims[1], K = dims[2];
    int64_t nw = (N + 31) / 32;
    if (variant != 0 && variant != 2) return -1;
    (void)M;
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows[r];
        const uint16_t *xi = x + i * K;
        int64_t count = 0;
        if (mask) memset(mask + r * nw, 0, (size_t)nw * sizeof(uint32_t));
        for (int64_t j = 0; j < N; ++j) {
            const uint16_t *wj = W + j * K;
            /* step 1: the low-precision output of g */
            float yl = lamp_oracle_ps_dot(xi, wj, (int)K, mu, scale);
            /* step 2: the look-ahead selection from that output */
            double kj = lamp_oracle_gelu_kappa((double)yl);
            int sel;
            if (variant == 0)
                sel = kj > tau;
            else
                sel = (int)((mask_in[i * nw + j / 32] >> (j % 32)) & 1u);
            /* step 3: recompute the selected components in binary32, then f */
            float y = sel ? lamp_oracle_fp32_dot(xi, wj, (int)K, scale) : yl;
            count += sel;
            if (ps) ps[r * N + j] = yl;
            if (mixed) mixed[r * N + j] = y;
            if (kappa) kappa[r * N + j] = kj;
            if (out) out[r * N + j] = lamp_oracle_gelu((double)y);
            if (mask && sel) mask[r * nw + j / 32] |= 1u << (j % 32);
        }
        if (nsel) nsel[r] = count;
    }
    return 0;
}
