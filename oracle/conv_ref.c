/* Plain C fp64 oracle for the SSM long convolution -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline arm may
 * load this.  It shares no code with the CUDA library.  Loops are written as
 * the definitions read; OpenMP only splits independent rows across threads.
 *
 * oracle_causal_conv: H3 summary ("Hungry Hungry Hippos", arXiv 2212.14052v3),
 *   section 2 "Convolutional view" -- with zero initial state the output is a
 *   linear convolution of the input with the filter plus the D residual:
 *     y[r, t] = sum_{s<=t} f[h(r), t-s] * u[r, s] + D[h(r)] * u[r, t],
 *   row r = b*H + h of a B x H x L array.
 * oracle_ssm_recurrence: section 2 "State space models" / "Recurrent view":
 *     x_t = A x_{t-1} + B u_t,  y_t = 2 Re(sum_n C_n x_{t,n}) + D u_t
 *   (2 Re = conjugate-pair convention for a complex diagonal A, real u).
 */
#include <complex.h>
#include <stdint.h>

int oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_causal_conv(const double* u, const double* f, const double* D, double* y,
                        int64_t rows, int64_t H, int64_t L) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < rows; ++r) {
    const int64_t h = r % H;
    const double* ur = u + r * L;
    const double* fh = f + h * L;
    double* yr = y + r * L;
    for (int64_t t = 0; t < L; ++t) {
      double acc = 0.0;
      for (int64_t s = 0; s <= t; ++s) acc += fh[t - s] * ur[s];
      yr[t] = acc + D[h] * ur[t];
    }
  }
}

/* A, Bc, Cc: H x N complex (interleaved re, im); x0/x_out: rows x N complex
 * (x0 may be NULL = zero state; x_out may be NULL). */
void oracle_ssm_recurrence(const double* u, const double* A, const double* Bc, const double* Cc,
                           const double* D, const double* x0, double* y, double* x_out,
                           int64_t rows, int64_t H, int64_t N, int64_t L) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < rows; ++r) {
    const int64_t h = r % H;
    double complex x[1024];
    for (int64_t n = 0; n < N; ++n)
      x[n] = x0 ? x0[2 * (r * N + n)] + I * x0[2 * (r * N + n) + 1] : 0.0;
    for (int64_t t = 0; t < L; ++t) {
      const double ut = u[r * L + t];
      double acc = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        const double complex a = A[2 * (h * N + n)] + I * A[2 * (h * N + n) + 1];
        const double complex b = Bc[2 * (h * N + n)] + I * Bc[2 * (h * N + n) + 1];
        const double complex c = Cc[2 * (h * N + n)] + I * Cc[2 * (h * N + n) + 1];
        x[n] = a * x[n] + b * ut;
        acc += 2.0 * creal(c * x[n]);
      }
      y[r * L + t] = acc + D[h] * ut;
    }
    if (x_out)
      for (int64_t n = 0; n < N; ++n) {
        x_out[2 * (r * N + n)] = creal(x[n]);
        x_out[2 * (r * N + n) + 1] = cimag(x[n]);
      }
  }
}
