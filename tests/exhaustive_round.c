/* Exhaustive check of the oracle's PS(mu) rounding against an independent
 * definition: the nearest value of the PS(mu) grid, computed in double with
 * frexp/ldexp and nearbyint (ties to even). Used by the CPU test suite. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

float lamp_oracle_round_ps(float x, int mu);

static float grid_nearest(float x, int mu)
{
    if (!isfinite(x) || x == 0.0f) return x;
    double ax = fabs((double)x);
    int E;
    frexp(ax, &E);
    E -= 1;                    /* ax in [2^E, 2^(E+1)) */
    if (E < -126) E = -126;    /* subnormals share the quantum of the lowest binade */
    double quantum = ldexp(1.0, E - mu);
    double r = nearbyint(ax / quantum) * quantum;
    if (r >= ldexp(1.0, 128)) r = INFINITY;
    return (float)(x < 0 ? -r : r);
}

int main(int argc, char **argv)
{
    int mu = atoi(argv[1]);
    long long bad = 0;
    #pragma omp parallel for reduction(+:bad) schedule(static)
    for (long long hi = 0; hi < 65536; ++hi) {
        for (uint32_t lo = 0; lo < 65536; ++lo) {
            uint32_t u = ((uint32_t)hi << 16) | lo, a, b;
            float x; memcpy(&x, &u, 4);
            float r1 = lamp_oracle_round_ps(x, mu), r2 = grid_nearest(x, mu);
            memcpy(&a, &r1, 4); memcpy(&b, &r2, 4);
            if (a != b) ++bad;
        }
    }
    printf("%lld\n", bad);
    return 0;
}
