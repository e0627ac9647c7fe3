// One-sided (Hestenes) Jacobi in shared memory, used by the small per-head solvers:
// the eigen-weighted factors and the probe fit (linalg.cu) and the O3 affine-fit
// diagnostic (diagnostics.cu).
#pragma once

#include "common.cuh"

namespace spr {

// ---------------------------------------------------------------------------------
// One-sided Jacobi: orthogonalise the `ncols` columns (length `rows` <= 128, column-major
// with stride `rows`) of G in shared memory.  Parallel round-robin ordering: in each
// round the column pairs are disjoint; each pair is handled by 16 lanes (half a warp),
// so 1024 threads take all 64 pairs of a round at once.  Only a.b is summed per pair: the
// squared column norms are computed at the start of each sweep and then carried through
// the rotations (|a'|^2 = |a|^2 - t a.b, |b'|^2 = |b|^2 + t a.b for the rotation that
// zeroes a.b).  A pair counts as orthogonal when |a.b| <= 1e-14 |a||b| or
// |a.b| <= 1e-15 ||G||_F^2: the second (absolute) test ends the sweeps when only columns
// near the null space still carry rounding-level overlap, which no relative test can
// remove.  Bounded sweeps.  `nrm` is shared scratch of at least ncols doubles.
__device__ inline void hestenes(double* G, int rows, int ncols, int* flag, double* red, double* nrm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  // sixteen lanes per column pair (two pairs per warp)
  const int sub = lane & 15, grp = 2 * warp + (lane >> 4), ngrp = 2 * nwarps;
  const unsigned gmask = 0xffffu << (lane & 16);
  double f = 0.0;
  for (int e = threadIdx.x; e < rows * ncols; e += blockDim.x) f += G[e] * G[e];
  const double abs_tol = 1e-15 * block_sum(f, red);
  const int nn = ncols + (ncols & 1);   // pad to even with a phantom column
  const int npairs = nn / 2;
  constexpr int kPer = kMaxD / 16;      // rows per lane
  for (int sweep = 0; sweep < 30; ++sweep) {
    // fresh squared norms
    for (int j = warp; j < ncols; j += nwarps) {
      double s = 0.0;
      for (int i = lane; i < rows; i += 32) s += G[j * rows + i] * G[j * rows + i];
      s = warp_sum(s);
      if (lane == 0) nrm[j] = s;
    }
    if (threadIdx.x == 0) *flag = 0;
    __syncthreads();
    for (int round = 0; round < nn - 1; ++round) {
      for (int k = grp; k < npairs; k += ngrp) {
        // circle method: position 0 fixed, the others rotate by `round`
        const int pa = k, pb = nn - 1 - k;
        int ia = 0, ib = 0;
        if (pa != 0) {
          int v = pa - 1 + round;
          if (v >= nn - 1) v -= nn - 1;
          ia = 1 + v;
        }
        if (pb != 0) {
          int v = pb - 1 + round;
          if (v >= nn - 1) v -= nn - 1;
          ib = 1 + v;
        }
        if (ia >= ncols || ib >= ncols) continue;     // uniform over the 16 lanes
        double* a = G + (long long)ia * rows;
        double* b = G + (long long)ib * rows;
        double g0 = 0.0, g1 = 0.0;            // two chains: half the dependent latency
#pragma unroll
        for (int q = 0; q < kPer; q += 2) {
          const int i = sub + 16 * q;
          if (i < rows) g0 = fma(a[i], b[i], g0);
          if (i + 16 < rows) g1 = fma(a[i + 16], b[i + 16], g1);
        }
        double ga = g0 + g1;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) ga += __shfl_xor_sync(gmask, ga, o);
        const double al = nrm[ia], be = nrm[ib];
        if (ga == 0.0 || ga * ga <= 1e-28 * (al * be) || fabs(ga) <= abs_tol) continue;
        // t = tan of the angle that zeroes a.b: with u = |b|^2 - |a|^2 and v = 2 a.b,
        // t = sign(u) v / (|u| + sqrt(u^2 + v^2)) (the smaller root of t^2 v + 2tu - v = 0)
        const double u = be - al, v = 2.0 * ga;
        const double t = copysign(1.0, u) * v / (fabs(u) + sqrt(fma(u, u, v * v)));
        const double c = rsqrt(fma(t, t, 1.0)), s = c * t;
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
          const int i = sub + 16 * q;
          if (i < rows) {
            const double x = a[i], y = b[i];
            a[i] = c * x - s * y;
            b[i] = s * x + c * y;
          }
        }
        if (sub == 0) {
          nrm[ia] = al - t * ga;
          nrm[ib] = be + t * ga;
          *flag = 1;
        }
      }
      __syncthreads();
    }
    const int rotated = *flag;
    __syncthreads();
    if (!rotated) break;
  }
}

}  // namespace spr
