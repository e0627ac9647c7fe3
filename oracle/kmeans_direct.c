/*
 * k-means assignment in the direct form, for the fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by oracle/sparsepr_oracle.py through ctypes.  It
 * shares nothing with the CUDA library.
 *
 * Definition ("Partition the Support, Reconstruct the Residual", S4.1 and App. C:
 * Lloyd's k-means on the response coordinates; the pages give no formula for the
 * distance, so the plain one is used): the label of point x is
 *     argmin_c  sum_j (x_j - c_j)^2
 * with the sum taken over ascending j, each term added by one correctly rounded fused
 * multiply-add (acc <- fma(t, t, acc), t = x_j - c_j, acc starting at 0), and ties going
 * to the lowest centre index (the first strict improvement over the running minimum,
 * which starts at the largest finite double).  Every (point, centre) pair is computed
 * independently; the loops below only choose which pairs run side by side.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>

#define CB 8 /* centres evaluated side by side (independent sums) */

static void assign_rows(const double* X, const double* CT, int64_t n0, int64_t n1, int64_t k,
                        int64_t r, int64_t* labels) {
  for (int64_t i = n0; i < n1; ++i) {
    const double* x = X + i * r;
    double best = DBL_MAX;
    int64_t bi = 0;
    int64_t c0 = 0;
    for (; c0 + CB <= k; c0 += CB) {
      double acc[CB];
      for (int u = 0; u < CB; ++u) acc[u] = 0.0;
      for (int64_t j = 0; j < r; ++j) {
        const double xj = x[j];
        const double* cj = CT + j * k + c0;
        for (int u = 0; u < CB; ++u) {
          const double t = xj - cj[u];
          acc[u] = fma(t, t, acc[u]);
        }
      }
      for (int u = 0; u < CB; ++u)
        if (acc[u] < best) {
          best = acc[u];
          bi = c0 + u;
        }
    }
    for (; c0 < k; ++c0) {
      double acc = 0.0;
      for (int64_t j = 0; j < r; ++j) {
        const double t = x[j] - CT[j * k + c0];
        acc = fma(t, t, acc);
      }
      if (acc < best) {
        best = acc;
        bi = c0;
      }
    }
    labels[i] = bi;
  }
}

__attribute__((target("avx2,fma"))) static void assign_rows_fma(const double* X, const double* CT,
                                                                int64_t n0, int64_t n1, int64_t k,
                                                                int64_t r, int64_t* labels) {
  /* the same source; compiled with hardware FMA, which rounds exactly as fma() */
  for (int64_t i = n0; i < n1; ++i) {
    const double* x = X + i * r;
    double best = DBL_MAX;
    int64_t bi = 0;
    int64_t c0 = 0;
    for (; c0 + CB <= k; c0 += CB) {
      double acc[CB];
      for (int u = 0; u < CB; ++u) acc[u] = 0.0;
      for (int64_t j = 0; j < r; ++j) {
        const double xj = x[j];
        const double* cj = CT + j * k + c0;
        for (int u = 0; u < CB; ++u) {
          const double t = xj - cj[u];
          acc[u] = __builtin_fma(t, t, acc[u]);
        }
      }
      for (int u = 0; u < CB; ++u)
        if (acc[u] < best) {
          best = acc[u];
          bi = c0 + u;
        }
    }
    for (; c0 < k; ++c0) {
      double acc = 0.0;
      for (int64_t j = 0; j < r; ++j) {
        const double t = x[j] - CT[j * k + c0];
        acc = __builtin_fma(t, t, acc);
      }
      if (acc < best) {
        best = acc;
        bi = c0;
      }
    }
    labels[i] = bi;
  }
}

/*
 * X: [n, r] row-major points; CT: [r, k] centres stored transposed (column c = centre c);
 * labels: [n] output.  Rows are split over OpenMP threads.
 */
void oracle_assign_direct(const double* X, const double* CT, int64_t n, int64_t k, int64_t r,
                          int64_t* labels) {
  const int hw = __builtin_cpu_supports("avx2") && __builtin_cpu_supports("fma");
#pragma omp parallel
  {
#ifdef _OPENMP
    extern int omp_get_thread_num(void);
    extern int omp_get_num_threads(void);
    const int64_t t = omp_get_thread_num(), nt = omp_get_num_threads();
#else
    const int64_t t = 0, nt = 1;
#endif
    const int64_t n0 = n * t / nt, n1 = n * (t + 1) / nt;
    if (hw)
      assign_rows_fma(X, CT, n0, n1, k, r, labels);
    else
      assign_rows(X, CT, n0, n1, k, r, labels);
  }
}
