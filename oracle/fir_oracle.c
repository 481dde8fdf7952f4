/*
 * fir_oracle.c -- plain fp64 CPU oracle for the gated, grouped, depthwise causal FIR.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check in __graft_entry__.py and
 * the CPU-baseline leg of bench.py may load this library.  It shares no code, header, table
 * or helper with the CUDA path in gated_causal_fir_b200/, and it never sees a value that the
 * CUDA path produced.
 *
 * Source: the StripedHyena 2 page "04. Hardware-aware convolution kernels"
 * (imamachi-n.github.io, homemade-llm, stripedhyena2/hardware-algorithms):
 *   - Sec. 1, causal FIR as a sum: y_t = sum_{k<=t} h_{t-k} x_k, with h_k = 0 outside [0, l_h);
 *   - Sec. 2, block convolution: yhat_n = sum_k H_{n-k} xhat_k over l_b x l_b sub-blocks of the
 *     lower-triangular Toeplitz matrix; blocks beyond the filter support are zero;
 *   - Sec. 3, the worked example (l = 6, l_h = 4, l_b = 3), which fixes the sub-block index rule
 *     H_m[i][j] = h_{m*l_b + i - j}, and the two-stage form Yhat_n = H0 Xhat_n + H1 Xhat_{n-1}
 *     with Xhat_{-1} = 0.
 * The gate y = q * (h_g conv (k * v)), with every d_g consecutive channels sharing filter h_g,
 * is the operator form of Hyena-SE / Hyena-MR (StripedHyena 2 overview page, Sec. 3 operator
 * table: SE/MR are gated convolutions with short / medium explicit filters).
 *
 * Everything is fp64.  Callers pass the exact fp64 upcast of their (bf16 or fp32) inputs, so
 * k*v is exact and the only rounding is fp64 summation, in tap order j = 0, 1, ...
 *
 * Parity pins (tests/test_oracle_pins.py): worked example (symbolic H0/H1 and integer-exact
 * two-stage == direct), dense Toeplitz product, numpy.convolve, scipy.signal.lfilter, torch
 * conv1d, impulse, shift, linearity, causality, closed form of a geometric filter, grouping
 * and batch independence.  No function below is "parity unpinned".
 */
#include <stdint.h>
#include <stddef.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Return codes shared by every oracle entry point. */
#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1

/*
 * Direct definition (page 04, Sec. 1 sum, gated as in the Hyena-SE/MR operator):
 *
 *   y[b,t,c] = q[b,t,c] * sum_{j=0}^{min(l_h-1, t)} h[c / d_g, j] * (k[b,t-j,c] * v[b,t-j,c])
 *
 * q, k, v, y: [B, L, D] row-major (channels contiguous).  h: [D / d_g, l_h] row-major, h[g,0]
 * multiplies the current token.  Every sequence b starts from zero history.
 * nthreads <= 0 lets OpenMP choose.
 */
int oracle_gated_fir_f64(const double *q, const double *k, const double *v, const double *h,
                         double *y, int64_t B, int64_t L, int64_t D, int64_t d_g, int64_t l_h,
                         int nthreads)
{
    if (!q || !k || !v || !h || !y) return ORACLE_BAD_ARG;
    if (B < 0 || L < 0 || D < 1 || d_g < 1 || D % d_g != 0 || l_h < 1) return ORACLE_BAD_ARG;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    const int64_t rows = B * L;
    #pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < rows; ++row) {
        const int64_t b = row / L;
        const int64_t t = row % L;
        const int64_t jmax = (l_h - 1 < t) ? l_h - 1 : t;
        for (int64_t c = 0; c < D; ++c) {
            const double *hg = h + (c / d_g) * l_h;
            double s = 0.0;
            for (int64_t j = 0; j <= jmax; ++j) {
                const int64_t src = (b * L + (t - j)) * D + c;
                s += hg[j] * (k[src] * v[src]);
            }
            y[row * D + c] = q[row * D + c] * s;
        }
    }
    return ORACLE_OK;
}

/*
 * The same direct definition for a list of output rows only: for i < n_rows with
 * rows[i] = b * L + t,  y_rows[i * D + c] = y[b, t, c]  of oracle_gated_fir_f64, computed with
 * the same products in the same tap order.  Lets a test check sampled rows of sequences whose
 * full oracle (O(L l_h D)) would take too long, e.g. filters as long as the sequence.
 */
int oracle_gated_fir_rows_f64(const double *q, const double *k, const double *v, const double *h,
                              const int64_t *rows, int64_t n_rows, double *y_rows, int64_t B,
                              int64_t L, int64_t D, int64_t d_g, int64_t l_h, int nthreads)
{
    if (!q || !k || !v || !h || (!rows && n_rows > 0) || (!y_rows && n_rows > 0))
        return ORACLE_BAD_ARG;
    if (B < 0 || L < 0 || D < 1 || d_g < 1 || D % d_g != 0 || l_h < 1 || n_rows < 0)
        return ORACLE_BAD_ARG;
    for (int64_t i = 0; i < n_rows; ++i)
        if (rows[i] < 0 || rows[i] >= B * L) return ORACLE_BAD_ARG;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    #pragma omp parallel for schedule(static)
    for (int64_t ic = 0; ic < n_rows * D; ++ic) {
        const int64_t i = ic / D, c = ic % D;
        const int64_t row = rows[i];
        const int64_t b = row / L;
        const int64_t t = row % L;
        const int64_t last = (l_h - 1 < t) ? l_h - 1 : t;
        const double *hg = h + (c / d_g) * l_h;
        double acc = 0.0;
        for (int64_t tap = 0; tap <= last; ++tap) {
            const int64_t at = (b * L + (t - tap)) * D + c;
            acc += hg[tap] * (k[at] * v[at]);
        }
        y_rows[ic] = q[row * D + c] * acc;
    }
    return ORACLE_OK;
}

/*
 * Sub-blocks of the lower-triangular Toeplitz matrix (page 04, Sec. 2 and the Sec. 3 worked
 * example): H[m][i][j] = h[m*l_b + i - j] when that index lies in [0, l_h), else 0,
 * for m = 0 .. S-1.  H: [S, l_b, l_b] row-major.
 */
int oracle_toeplitz_blocks_f64(const double *h, int64_t l_h, int64_t l_b, int64_t S, double *H)
{
    if (!h || !H || l_h < 1 || l_b < 1 || S < 1) return ORACLE_BAD_ARG;
    for (int64_t m = 0; m < S; ++m)
        for (int64_t i = 0; i < l_b; ++i)
            for (int64_t j = 0; j < l_b; ++j) {
                const int64_t idx = m * l_b + i - j;
                H[(m * l_b + i) * l_b + j] = (idx >= 0 && idx < l_h) ? h[idx] : 0.0;
            }
    return ORACLE_OK;
}

/*
 * Block convolution of one channel with S stages (page 04, Sec. 2 block sum, truncated to the
 * S sub-blocks H_0 .. H_{S-1}; S = 2 is the Sec. 3 two-stage form):
 *
 *   Yhat_n = sum_{m=0}^{S-1} H_m Xhat_{n-m},   Xhat_{<0} = 0,
 *
 * over the ceil(L / l_b) chunks of x; the tail chunk is zero-padded on read and clipped on
 * write.  Used by the tests to check the pages' two-stage statements against the direct sum.
 */
int oracle_block_conv_f64(const double *h, int64_t l_h, int64_t l_b, int64_t S,
                          const double *x, int64_t L, double *y)
{
    if (!h || !x || !y || l_h < 1 || l_b < 1 || S < 1 || L < 0) return ORACLE_BAD_ARG;
    const int64_t nchunks = (L + l_b - 1) / l_b;
    for (int64_t n = 0; n < nchunks; ++n) {
        for (int64_t i = 0; i < l_b; ++i) {
            const int64_t t = n * l_b + i;
            if (t >= L) break;
            double s = 0.0;
            for (int64_t m = 0; m < S; ++m) {
                const int64_t src_chunk = n - m;
                if (src_chunk < 0) continue;           /* Xhat_{<0} = 0 */
                for (int64_t jj = 0; jj < l_b; ++jj) {
                    const int64_t src = src_chunk * l_b + jj;
                    if (src >= L) continue;             /* zero-padded tail chunk */
                    const int64_t idx = m * l_b + i - jj;  /* H_m[i][jj] */
                    if (idx >= 0 && idx < l_h) s += h[idx] * x[src];
                }
            }
            y[t] = s;
        }
    }
    return ORACLE_OK;
}

/* Number of threads OpenMP would use (reported as the oracle's core count). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Backward of the gated FIR (the gradients the page's Sec. 7 two-pass backward computes):
 * given dy = dL/dy for y = q * z, z = h_g conv x, x = k * v,
 *
 *   dq[b,t,c] = dy[b,t,c] * z[b,t,c]
 *   dz[b,t,c] = dy[b,t,c] * q[b,t,c]
 *   dx[b,t,c] = sum_{j=0}^{min(l_h-1, L-1-t)} h[c/d_g, j] * dz[b,t+j,c]   (transposed Toeplitz)
 *   dk = dx * v,  dv = dx * k
 *   dh[g, j]  = sum_{b, t >= j, c in g} dz[b,t,c] * x[b,t-j,c]
 *
 * written straight from those sums (no blocking).  dh: [D / d_g, l_h].
 */
int oracle_gated_fir_bwd_f64(const double *q, const double *k, const double *v, const double *h,
                             const double *dy, double *dq, double *dk, double *dv, double *dh,
                             int64_t B, int64_t L, int64_t D, int64_t d_g, int64_t l_h,
                             int nthreads)
{
    if (!q || !k || !v || !h || !dy || !dq || !dk || !dv || !dh) return ORACLE_BAD_ARG;
    if (B < 0 || L < 0 || D < 1 || d_g < 1 || D % d_g != 0 || l_h < 1) return ORACLE_BAD_ARG;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    const int64_t rows = B * L;
    #pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < rows; ++row) {
        const int64_t b = row / L;
        const int64_t t = row % L;
        for (int64_t c = 0; c < D; ++c) {
            const double *hg = h + (c / d_g) * l_h;
            double z = 0.0, dx = 0.0;
            for (int64_t j = 0; j < l_h && j <= t; ++j) {
                const int64_t src = (b * L + (t - j)) * D + c;
                z += hg[j] * (k[src] * v[src]);
            }
            for (int64_t j = 0; j < l_h && t + j < L; ++j) {
                const int64_t src = (b * L + (t + j)) * D + c;
                dx += hg[j] * (dy[src] * q[src]);
            }
            const int64_t e = row * D + c;
            dq[e] = dy[e] * z;
            dk[e] = dx * v[e];
            dv[e] = dx * k[e];
        }
    }
    const int64_t G = D / d_g;
    #pragma omp parallel for schedule(static)
    for (int64_t gj = 0; gj < G * l_h; ++gj) {
        const int64_t g = gj / l_h, j = gj % l_h;
        double s = 0.0;
        for (int64_t b = 0; b < B; ++b)
            for (int64_t t = j; t < L; ++t)
                for (int64_t c = g * d_g; c < (g + 1) * d_g; ++c) {
                    const int64_t e = (b * L + t) * D + c;
                    const int64_t src = (b * L + (t - j)) * D + c;
                    s += (dy[e] * q[e]) * (k[src] * v[src]);
                }
        dh[gj] = s;
    }
    return ORACLE_OK;
}
