/*
 * oracle/loops.c -- plain fp64 loops for the S4 oracle.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library links or calls this
 * file; only tests/, the smoke check and the benchmark's CPU-baseline leg may.
 *
 * Each routine is the textbook definition written out with no blocking or
 * reordering, so it can be checked by eye against the pages:
 *   - causal convolution y = K * u + D u  ("The S4 kernel, from scratch", §1
 *     and §5 "Two views, kept in sync"; glossary page "Structured state-space
 *     sequence model and S4", section "One linear layer, two computational
 *     views");
 *   - the kernel by dense powers K_k = C A^k v, summed over periods for the
 *     aliased kernel ("The S4 kernel, from scratch", §4 and its "Aliasing"
 *     paragraph);
 *   - the recurrence x_t = A x_{t-1} + B u_t, y_t = Re(C x_t) + D u_t
 *     ("The S4 kernel, from scratch", §5).
 */
#include <complex.h>
#include <math.h>
#include <stdint.h>

/* y[r, t] = sum_{s=0}^{t} K[h_r, s] * u[r, t-s] + D[h_r] * u[r, t]
 * u, y: [rows, L] row-major; K: [H, L]; row_h[r] = channel of row r. */
void oracle_causal_conv(const double *u, const double *K, const double *D,
                        const int64_t *row_h, int64_t rows, int64_t L, double *y)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        const double *ur = u + r * L;
        const double *Kh = K + row_h[r] * L;
        double *yr = y + r * L;
        for (int64_t t = 0; t < L; ++t) {
            double acc = 0.0;
            for (int64_t s = 0; s <= t; ++s)
                acc += Kh[s] * ur[t - s];
            yr[t] = acc + D[row_h[r]] * ur[t];
        }
    }
}

/* The same sum at selected output times only: yo[r, i] = y[r, ts[i]]. */
void oracle_causal_conv_at(const double *u, const double *K, const double *D,
                           const int64_t *row_h, int64_t rows, int64_t L,
                           const int64_t *ts, int64_t nt, double *yo)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        const double *ur = u + r * L;
        const double *Kh = K + row_h[r] * L;
        for (int64_t i = 0; i < nt; ++i) {
            int64_t t = ts[i];
            double acc = 0.0;
            for (int64_t s = 0; s <= t; ++s)
                acc += Kh[s] * ur[t - s];
            yo[r * nt + i] = acc + D[row_h[r]] * ur[t];
        }
    }
}

/* Dense powers, per channel h (A: [H,N,N] row-major, v0, C: [H,N]):
 *   K[h, k mod L] += C . A^(k) v0   for k = 0 .. periods*L - 1,
 * i.e. the first `periods` periods of the aliased sum. Iteration stops early,
 * after a whole period, once that period's largest term is below
 * rel_tol * (largest accumulated |K|). K_re/K_im: [H, L]. Returns in
 * periods_used[h] how many periods were summed. */
void oracle_power_kernel(const double complex *A, const double complex *v0,
                         const double complex *C, int64_t H, int64_t N, int64_t L,
                         int64_t max_periods, double rel_tol,
                         double *K_re, double *K_im, int64_t *periods_used)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t h = 0; h < H; ++h) {
        const double complex *Ah = A + h * N * N;
        const double complex *Ch = C + h * N;
        double *Kr = K_re + h * L, *Ki = K_im + h * L;
        double complex v[512], w[512];
        for (int64_t n = 0; n < N; ++n) v[n] = v0[h * N + n];
        for (int64_t k = 0; k < L; ++k) { Kr[k] = 0.0; Ki[k] = 0.0; }
        double kmax = 0.0;
        int64_t p;
        for (p = 0; p < max_periods; ++p) {
            double pmax = 0.0;
            for (int64_t k = 0; k < L; ++k) {
                double complex acc = 0.0;
                for (int64_t n = 0; n < N; ++n) acc += Ch[n] * v[n];
                Kr[k] += creal(acc);
                Ki[k] += cimag(acc);
                if (cabs(acc) > pmax) pmax = cabs(acc);
                for (int64_t i = 0; i < N; ++i) {
                    double complex s = 0.0;
                    for (int64_t j = 0; j < N; ++j) s += Ah[i * N + j] * v[j];
                    w[i] = s;
                }
                for (int64_t n = 0; n < N; ++n) v[n] = w[n];
            }
            for (int64_t k = 0; k < L; ++k) {
                double a = fabs(Kr[k]);
                if (a > kmax) kmax = a;
            }
            if (pmax <= rel_tol * kmax) { ++p; break; }
        }
        periods_used[h] = p;
    }
}

/* Dense recurrence per row r (channel h_r), state x in/out [rows, N]:
 *   x_t = A x_{t-1} + B u_t ;  y_t = Re(C . x_t) + D u_t. */
void oracle_recurrence_dense(const double complex *A, const double complex *B,
                             const double complex *C, const double *D,
                             const int64_t *row_h, int64_t rows, int64_t N,
                             const double *u, int64_t T, double complex *x, double *y)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t h = row_h[r];
        const double complex *Ah = A + h * N * N, *Bh = B + h * N, *Ch = C + h * N;
        double complex *xr = x + r * N;
        double complex w[512];
        for (int64_t t = 0; t < T; ++t) {
            double ut = u[r * T + t];
            for (int64_t i = 0; i < N; ++i) {
                double complex s = 0.0;
                for (int64_t j = 0; j < N; ++j) s += Ah[i * N + j] * xr[j];
                w[i] = s + Bh[i] * ut;
            }
            double complex acc = 0.0;
            for (int64_t n = 0; n < N; ++n) { xr[n] = w[n]; acc += Ch[n] * xr[n]; }
            y[r * T + t] = creal(acc) + D[h] * ut;
        }
    }
}

/* Diagonal recurrence over the stored half of a conjugate-closed system:
 *   x_t = a x_{t-1} + b u_t (elementwise) ;  y_t = 2 Re(sum_n c_n x_t[n]) + D u_t. */
void oracle_recurrence_diag(const double complex *a, const double complex *b,
                            const double complex *c, const double *D,
                            const int64_t *row_h, int64_t rows, int64_t Nh,
                            const double *u, int64_t T, double complex *x, double *y)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t h = row_h[r];
        const double complex *ah = a + h * Nh, *bh = b + h * Nh, *ch = c + h * Nh;
        double complex *xr = x + r * Nh;
        for (int64_t t = 0; t < T; ++t) {
            double ut = u[r * T + t];
            double complex acc = 0.0;
            for (int64_t n = 0; n < Nh; ++n) {
                xr[n] = ah[n] * xr[n] + bh[n] * ut;
                acc += ch[n] * xr[n];
            }
            y[r * T + t] = 2.0 * creal(acc) + D[h] * ut;
        }
    }
}
