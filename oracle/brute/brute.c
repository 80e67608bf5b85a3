/*
 * Exhaustive low-rank binary factorisation of tiny matrices (oracle side).
 *
 * TEST INFRASTRUCTURE ONLY: used by the oracle's pins, never by the CUDA library.
 *
 * For an m x n matrix W and rank r in {1, 2} it finds
 *     min over U in {+-1}^{m x r}, V in {+-1}^{n x r}, real s1 (m), s2 (n) of
 *         || W - diag(s1) U V^T diag(s2) ||_F^2
 * by enumerating sign patterns and fitting the scales by alternating least
 * squares from several starts.  This is the problem the low-rank binary form of
 * the NanoQuant pages poses (summary page, "Motivation": W ~ s1 U V^T s2); its
 * optimum lower-bounds the squared error of any method that returns that form,
 * LB-ADMM included.
 *
 * Symmetries used (they only shrink the search, they never exclude an optimum):
 *   - flipping row i of U together with the sign of s1_i leaves the product
 *     unchanged, so column 0 of U is fixed to +1; likewise column 0 of V;
 *   - for r = 2, flipping column 1 of both U and V leaves U V^T unchanged, so
 *     U[0][1] is fixed to +1.
 * Scales are real (either sign) so the search is over a superset of the
 * positive-scale form: the result is still a lower bound.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define BF_MAX 8

/* Deterministic start values (a small LCG; the fit does not depend on its quality). */
static double lcg_uniform(uint64_t *state) {
    *state = *state * 6364136223846793005ULL + 1442695040888963407ULL;
    return (double)(*state >> 11) * (1.0 / 9007199254740992.0);
}

/* Alternating least squares for min sum_ij (W_ij - s1_i s2_j P_ij)^2 with P fixed. */
static double fit_scales(const double *W, const double *P, int m, int n, const double *s2_init,
                         int sweeps, double *s1, double *s2) {
    double prev = INFINITY;
    memcpy(s2, s2_init, sizeof(double) * (size_t)n);
    double err = 0.0;
    for (int it = 0; it < sweeps; ++it) {
        for (int i = 0; i < m; ++i) {
            double num = 0.0, den = 0.0;
            for (int j = 0; j < n; ++j) {
                double c = s2[j] * P[i * n + j];
                num += W[i * n + j] * c;
                den += c * c;
            }
            s1[i] = den > 0.0 ? num / den : 0.0;
        }
        for (int j = 0; j < n; ++j) {
            double num = 0.0, den = 0.0;
            for (int i = 0; i < m; ++i) {
                double c = s1[i] * P[i * n + j];
                num += W[i * n + j] * c;
                den += c * c;
            }
            s2[j] = den > 0.0 ? num / den : 0.0;
        }
        err = 0.0;
        for (int i = 0; i < m; ++i)
            for (int j = 0; j < n; ++j) {
                double d = W[i * n + j] - s1[i] * s2[j] * P[i * n + j];
                err += d * d;
            }
        if (prev - err <= 1e-15 * (1.0 + err)) break;
        prev = err;
    }
    return err;
}

/*
 * Returns the minimal squared Frobenius error, or -1 on bad arguments.
 * best_U (m*r), best_V (n*r) receive the optimal +-1 patterns (row-major),
 * best_s1 (m), best_s2 (n) the fitted scales.  Any output pointer may be NULL.
 * ``starts`` random starts are used in addition to the all-ones start.
 */
double nq_brute_min_sq_error(const double *W, int m, int n, int r, int starts, int sweeps,
                             double *best_U, double *best_V, double *best_s1, double *best_s2) {
    if (m < 1 || n < 1 || m > BF_MAX || n > BF_MAX || r < 1 || r > 2 || starts < 0 || sweeps < 1)
        return -1.0;
    double P[BF_MAX * BF_MAX], s1[BF_MAX], s2[BF_MAX], init[BF_MAX];
    double U[BF_MAX * 2], V[BF_MAX * 2];
    double best = INFINITY;
    /* free bits: column 1 of U except row 0 (m-1 bits) and column 1 of V (n bits) */
    const int ubits = (r == 2) ? m - 1 : 0;
    const int vbits = (r == 2) ? n : 0;
    const uint64_t npat = 1ULL << (ubits + vbits);
    uint64_t rng = 0x243F6A8885A308D3ULL;
    for (uint64_t pat = 0; pat < npat; ++pat) {
        for (int i = 0; i < m; ++i) {
            U[i * r] = 1.0;
            if (r == 2) U[i * 2 + 1] = (i == 0) ? 1.0 : (((pat >> (i - 1)) & 1ULL) ? -1.0 : 1.0);
        }
        for (int j = 0; j < n; ++j) {
            V[j * r] = 1.0;
            if (r == 2) V[j * 2 + 1] = ((pat >> (ubits + j)) & 1ULL) ? -1.0 : 1.0;
        }
        for (int i = 0; i < m; ++i)
            for (int j = 0; j < n; ++j) {
                double p = 0.0;
                for (int k = 0; k < r; ++k) p += U[i * r + k] * V[j * r + k];
                P[i * n + j] = p;
            }
        for (int s = 0; s <= starts; ++s) {
            for (int j = 0; j < n; ++j) init[j] = (s == 0) ? 1.0 : 2.0 * lcg_uniform(&rng) - 1.0;
            double e = fit_scales(W, P, m, n, init, sweeps, s1, s2);
            if (e < best) {
                best = e;
                if (best_U) memcpy(best_U, U, sizeof(double) * (size_t)(m * r));
                if (best_V) memcpy(best_V, V, sizeof(double) * (size_t)(n * r));
                if (best_s1) memcpy(best_s1, s1, sizeof(double) * (size_t)m);
                if (best_s2) memcpy(best_s2, s2, sizeof(double) * (size_t)n);
            }
        }
    }
    return best;
}
