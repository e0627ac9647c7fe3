// Small dense linear algebra of SparsePR, one CTA per head, fp64:
//   key response metric M_K (paper S4.1, App. B.1), the query metric M_Q of the centred
//   K/V centroids (App. B.2), their eigenvalue-weighted factors F_K / F_Q, and the
//   probe fit: coverage-weighted statistics, weighted ridge B_lambda and the residual
//   subspace Psi_r (paper S4.2, App. A.3, App. D.2; review page step 4).
//
// Eigenvectors and singular vectors come from one-sided (Hestenes) Jacobi: rotating
// column pairs of a matrix G until all columns are mutually orthogonal.  For a
// symmetric PSD metric M, the converged columns of M V are lambda_j v_j, so their norms
// are the eigenvalues and their directions the eigenvectors (no rotation accumulation
// needed).  For the residual subspace, orthogonalising the columns of Y^T (one column
// per probe) leaves columns sigma_k u_k with u_k the right singular vectors of Y.
#include <cmath>

#include "common.cuh"
#include "jacobi.cuh"

namespace spr {
namespace {

constexpr int kLinThreads = 1024;

// ---------------------------------------------------------------------------------
// M_K = (1/M_s') sum_s q_s^T q_s over rows floor(s*N_q/M_s) (all rows if M_s >= N_q).
// One block per K/V head.  With G query heads per K/V head (GQA, paper App. C) the rows
// are those of the G heads concatenated in head order, G*M_s of them: sample s is row
// c = floor(s*N_q/M_s) of the concatenation (the same index as floor(s*G*N_q/(G*M_s))),
// i.e. row c mod N_q of query head G*hk + c / N_q.
__global__ void __launch_bounds__(kLinThreads) key_metric_kernel(Dims m, const void* Q, double* MK) {
  extern __shared__ float rows[];   // [64][d]
  const int h = blockIdx.x, d = m.d;
  const int Ms = m.G * (m.Ms < m.Nq ? m.Ms : m.Nq);
  double acc[16];
  for (int k = 0; k < 16; ++k) acc[k] = 0.0;
  const int entries = d * d;
  for (int s0 = 0; s0 < Ms; s0 += 64) {
    const int ns = (Ms - s0) < 64 ? (Ms - s0) : 64;
    __syncthreads();
    for (int e = threadIdx.x; e < ns * d; e += blockDim.x) {
      const int s = s0 + e / d, j = e % d;
      const long long c = (m.Ms >= m.Nq) ? s : ((long long)s * m.Nq) / m.Ms;
      const long long qh = (long long)h * m.G + c / m.Nq;
      rows[e] = load_as_float(Q, (qh * m.Nq + c % m.Nq) * d + j, m.dtype);
    }
    __syncthreads();
    for (int k = 0; k < 16; ++k) {
      const int e = threadIdx.x + k * blockDim.x;
      if (e >= entries) break;
      const int i = e / d, j = e % d;
      double a = acc[k];
      for (int s = 0; s < ns; ++s) a += (double)rows[s * d + i] * (double)rows[s * d + j];
      acc[k] = a;
    }
  }
  for (int k = 0; k < 16; ++k) {
    const int e = threadIdx.x + k * blockDim.x;
    if (e >= entries) break;
    MK[(long long)h * entries + e] = acc[k] / (double)Ms;
  }
}

// rank of column j when columns are ordered by decreasing key, ties by index
__device__ __forceinline__ int desc_rank(const double* key, int n, int j) {
  const double v = key[j];
  int r = 0;
  for (int k = 0; k < n; ++k) r += (key[k] > v) || (key[k] == v && k < j);
  return r;
}

// Eigen-weighted factor of a symmetric PSD metric (paper S4.1, App. B.1):
// F = [u_1 sqrt(l_1/mean) ... u_r sqrt(l_r/mean)], mean over the r kept eigenvalues.
__global__ void __launch_bounds__(kLinThreads) eigen_factor_kernel(Dims m, const double* Mall,
                                                                   int r, double* lam_out,
                                                                   double* F64, float* F32,
                                                                   int* err, int err_bit,
                                                                   const int* only) {
  extern __shared__ double G[];          // [d][d] column-major
  __shared__ double norm[kMaxD], lam[kMaxD], red[32], hnrm[kMaxD];
  __shared__ int rank[kMaxD];
  __shared__ int flag;
  const int h = blockIdx.x, d = m.d;
  if (only && only[h] == 0) return;      // warm plan: this head's factor is already updated
  const double* Mh = Mall + (long long)h * d * d;
  for (int e = threadIdx.x; e < d * d; e += blockDim.x) G[e] = Mh[e];  // symmetric
  __syncthreads();
  hestenes(G, d, d, &flag, red, hnrm);
  // The metrics are Gram matrices (symmetric PSD), so the converged column norms are the
  // eigenvalues; negative eigenvalues exist only at rounding level, where |lambda| and
  // the clamp to zero differ by far less than any distance that decides a label.
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int j = warp; j < d; j += nwarps) {
    double s = 0.0;
    for (int i = lane; i < d; i += 32) s += G[j * d + i] * G[j * d + i];
    s = warp_sum(s);
    if (lane == 0) {
      norm[j] = sqrt(s);
      lam[j] = norm[j];
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < d; j += blockDim.x) rank[j] = desc_rank(lam, d, j);
  __syncthreads();
  double part = 0.0;
  for (int j = threadIdx.x; j < d; j += blockDim.x)
    if (rank[j] < r) part += lam[j];
  const double mean = block_sum(part, red) / (double)r;
  const bool ok = mean > 0.0 && isfinite(mean);
  if (!ok && threadIdx.x == 0) atomicOr(err, err_bit);
  for (int j = threadIdx.x; j < d; j += blockDim.x)
    if (rank[j] < r) lam_out[(long long)h * r + rank[j]] = lam[j];
  for (int e = threadIdx.x; e < d * d; e += blockDim.x) {
    const int j = e / d, i = e % d;   // column j, row i
    const int k = rank[j];
    if (k >= r) continue;
    double v = 0.0;
    if (ok && norm[j] > 0.0) v = G[j * d + i] / norm[j] * sqrt(lam[j] / mean);
    F64[((long long)h * d + i) * r + k] = v;
    F32[((long long)h * d + i) * r + k] = (float)v;
  }
}

// ---------------------------------------------------------------------------------
// Probe fit.  x_p = sparse output of probe p, R_p = exact output - x_p,
// w_p = |G_a|/m_a (review page step 4).  Unit-sum weights give mu_x, mu_R and
// s = sqrt(weighted variance + 1e-6) (App. A.3, App. D.3); unit-mean weights omega weigh
// the ridge objective (App. A.3).  With A = Omega^{1/2} X_bar and Y = Omega^{1/2} R_bar,
// B = (A^T A + lambda I)^-1 A^T Y = A^T (A A^T + lambda I)^-1 Y; the smaller system is
// solved by Cholesky.  Psi_r = leading r right singular vectors of Y (App. D.2).
// The correction is folded as B' = diag(1/s) B P, c = mu_R - (mu_x / s) B P.

// In-place Cholesky of an n x n SPD matrix (row-major, smem). Returns false if not PD.
__device__ bool cholesky(double* L, int n, int* bad) {
  if (threadIdx.x == 0) *bad = 0;
  __syncthreads();
  for (int k = 0; k < n; ++k) {
    if (threadIdx.x == 0) {
      const double dkk = L[k * n + k];
      if (!(dkk > 0.0) || !isfinite(dkk)) *bad = 1;
      L[k * n + k] = dkk > 0.0 ? sqrt(dkk) : 1.0;
    }
    __syncthreads();
    const double piv = L[k * n + k];
    for (int i = k + 1 + threadIdx.x; i < n; i += blockDim.x) L[i * n + k] /= piv;
    __syncthreads();
    const int rem = n - k - 1;
    for (int e = threadIdx.x; e < rem * rem; e += blockDim.x) {
      const int i = k + 1 + e / rem, j = k + 1 + e % rem;
      if (j <= i) L[i * n + j] -= L[i * n + k] * L[j * n + k];
    }
    __syncthreads();
  }
  return *bad == 0;
}

// Solve (L L^T) Z = Z in place for `ncols` right-hand-side columns of Z (n x ldz,
// row-major, global); one thread per column.
__device__ void cholesky_solve(const double* L, int n, double* Z, int ldz, int ncols) {
  for (int c = threadIdx.x; c < ncols; c += blockDim.x) {
    for (int i = 0; i < n; ++i) {
      double v = Z[(long long)i * ldz + c];
      for (int k = 0; k < i; ++k) v -= L[i * n + k] * Z[(long long)k * ldz + c];
      Z[(long long)i * ldz + c] = v / L[i * n + i];
    }
    for (int i = n - 1; i >= 0; --i) {
      double v = Z[(long long)i * ldz + c];
      for (int k = i + 1; k < n; ++k) v -= L[k * n + i] * Z[(long long)k * ldz + c];
      Z[(long long)i * ldz + c] = v / L[i * n + i];
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------------
// Warm update of an eigenvalue-weighted factor (paper App. C: later calls refresh the
// metric factors by two subspace iterations started from the previous factors, with a
// Cholesky factorisation).  Each iteration: Z = M F, L L^T = F^T Z, F <- Z L^-T, so that
// F F^T = M F (F^T M F)^-1 F^T M, a function of span(F) alone that equals the
// eigen-weighted U_r Lambda_r U_r^T when the span is the leading eigenspace.  The result
// is scaled to unit mean eigenvalue (trace F^T F = r).  F and Z live in shared memory
// with rows padded to r + 1 doubles; M is read from global memory (L2-resident).  A head
// whose saved state does not match the plan, or whose F^T M F is not positive definite,
// is flagged in `cold` and left to the full eigendecomposition.
__global__ void __launch_bounds__(kLinThreads) subspace_factor_kernel(
    Dims m, const double* Mall, const int* hdr, const double* Fprev, int r, double* lam_out,
    double* F64, float* F32, int* cold, int* err) {
  extern __shared__ double sm[];
  __shared__ double red[32];
  __shared__ int bad;
  const int h = blockIdx.x, d = m.d, rs = r + 1;
  double* Fs = sm;                 // [d][rs]
  double* Zs = Fs + d * rs;        // [d][rs]
  double* G = Zs + d * rs;         // [r][r]
  if (!state_matches(hdr, m)) {
    if (threadIdx.x == 0) {
      cold[h] = 1;
      atomicOr(err, kErrWarmState);
    }
    return;
  }
  const double* Mh = Mall + (long long)h * d * d;
  const double* Fp = Fprev + (long long)h * d * r;
  for (int e = threadIdx.x; e < d * r; e += blockDim.x) Fs[(e / r) * rs + e % r] = Fp[e];
  for (int step = 0; step < 2; ++step) {
    __syncthreads();
    for (int e = threadIdx.x; e < d * r; e += blockDim.x) {      // Z = M F
      const int i = e / r, k = e % r;
      double v = 0.0;
      for (int j = 0; j < d; ++j) v += Mh[i * d + j] * Fs[j * rs + k];
      Zs[i * rs + k] = v;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < r * r; e += blockDim.x) {      // G = F^T Z
      const int a = e / r, c = e % r;
      double v = 0.0;
      for (int i = 0; i < d; ++i) v += Fs[i * rs + a] * Zs[i * rs + c];
      G[e] = v;
    }
    __syncthreads();
    if (!cholesky(G, r, &bad)) {                                  // uniform across the block
      if (threadIdx.x == 0) cold[h] = 1;
      return;
    }
    // F L^T = Z, column by column: F_k = Z_k / L_kk, then Z_c -= F_k L_ck for c > k
    for (int k = 0; k < r; ++k) {
      const double piv = G[k * r + k];
      for (int i = threadIdx.x; i < d; i += blockDim.x) Fs[i * rs + k] = Zs[i * rs + k] / piv;
      __syncthreads();
      const int rem = r - k - 1;
      for (int e = threadIdx.x; e < d * rem; e += blockDim.x) {
        const int i = e / rem, c = k + 1 + e % rem;
        Zs[i * rs + c] -= Fs[i * rs + k] * G[c * r + k];
      }
      __syncthreads();
    }
  }
  double part = 0.0;
  for (int e = threadIdx.x; e < d * r; e += blockDim.x) {
    const double f = Fs[(e / r) * rs + e % r];
    part += f * f;
  }
  const double mean = block_sum(part, red) / (double)r;
  if (!(mean > 0.0) || !isfinite(mean)) {
    if (threadIdx.x == 0) cold[h] = 1;
    return;
  }
  const double sc = 1.0 / sqrt(mean);
  for (int e = threadIdx.x; e < d * r; e += blockDim.x) {
    const double v = Fs[(e / r) * rs + e % r] * sc;
    F64[(long long)h * d * r + e] = v;
    F32[(long long)h * d * r + e] = (float)v;
  }
  // the columns are not eigenvectors: the eigenvalue export is left at zero
  for (int k = threadIdx.x; k < r; k += blockDim.x) lam_out[(long long)h * r + k] = 0.0;
}

__global__ void __launch_bounds__(kLinThreads) fit_kernel(Dims m, Buffers b) {
  extern __shared__ double S[];   // max(n*n, M*d) doubles
  __shared__ double red[32];
  __shared__ double sig[kMaxM];
  __shared__ double hnrm[kMaxM];
  __shared__ int srank[kMaxM];
  __shared__ int flag, bad;
  const int h = blockIdx.x, d = m.d, M = m.M;
  const long long hd = (long long)h * d;
  double* A = b.fitA + (long long)h * M * d;   // [M][d]
  double* Y = b.fitY + (long long)h * M * d;   // [M][d]
  double* Z = b.fitZ + (long long)h * (M > d ? M : d) * d;
  const int* probes = b.probes + (long long)h * M;
  const double* w = b.wP + (long long)h * M;

  // weights
  double wsum = 0.0;
  for (int p = 0; p < M; ++p) wsum += w[p];   // every thread, same order
  // x (sparse output at the probe rows) and R = dense - sparse, staged in A and Y
  for (int e = threadIdx.x; e < M * d; e += blockDim.x) {
    const int p = e / d, j = e % d;
    const int pos = b.invQ[(long long)h * m.Nq + probes[p]];
    const double x = (double)b.Osp[((long long)h * m.Nq + pos) * d + j];
    const double dn = (double)b.Odense[((long long)h * M + p) * d + j];
    A[e] = x;
    Y[e] = dn - x;
    if (!isfinite(x) || !isfinite(dn)) atomicOr(b.err, kErrNonFinite);
  }
  __syncthreads();
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    double mx = 0.0, mr = 0.0;
    for (int p = 0; p < M; ++p) {
      const double wt = w[p] / wsum;
      mx += wt * A[p * d + j];
      mr += wt * Y[p * d + j];
    }
    double var = 0.0;
    for (int p = 0; p < M; ++p) {
      const double t = A[p * d + j] - mx;
      var += (w[p] / wsum) * t * t;
    }
    b.muX[hd + j] = mx;
    b.muR[hd + j] = mr;
    b.sX[hd + j] = sqrt(var + 1e-6);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < M * d; e += blockDim.x) {
    const int p = e / d, j = e % d;
    const double om = sqrt((double)M * w[p] / wsum);
    A[e] = om * (A[e] - b.muX[hd + j]) / b.sX[hd + j];
    Y[e] = om * (Y[e] - b.muR[hd + j]);
  }
  __syncthreads();

  // ---- ridge: solve the smaller of the dual (M x M) and primal (d x d) systems
  double* Bh = b.Bm + (long long)h * d * d;
  const bool dual = M <= d;
  const int n = dual ? M : d;
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int i = e / n, j = e % n;
    double g = 0.0;
    if (dual) for (int k = 0; k < d; ++k) g += A[i * d + k] * A[j * d + k];
    else      for (int k = 0; k < M; ++k) g += A[k * d + i] * A[k * d + j];
    S[e] = g + (i == j ? m.lambda : 0.0);
  }
  for (int e = threadIdx.x; e < n * d; e += blockDim.x) {
    const int i = e / d, j = e % d;
    if (dual) {
      Z[e] = Y[e];
    } else {
      double g = 0.0;
      for (int k = 0; k < M; ++k) g += A[k * d + i] * Y[k * d + j];
      Z[e] = g;
    }
  }
  __syncthreads();
  const bool pd = cholesky(S, n, &bad);
  if (!pd && threadIdx.x == 0) atomicOr(b.err, kErrNonFinite);
  cholesky_solve(S, n, Z, d, d);
  for (int e = threadIdx.x; e < d * d; e += blockDim.x) {
    double v = 0.0;
    if (pd) {
      if (dual) {
        const int i = e / d, j = e % d;
        for (int p = 0; p < M; ++p) v += A[p * d + i] * Z[p * d + j];
      } else {
        v = Z[e];
      }
    }
    Bh[e] = v;
  }
  __syncthreads();

  // ---- residual subspace: orthogonalise the columns of Y^T (column p = Y[p][:])
  double* Ph = b.Pm + (long long)h * d * d;
  int reff;
  if (m.r == 0) {
    reff = d;
    for (int e = threadIdx.x; e < d * d; e += blockDim.x) Ph[e] = (e / d == e % d) ? 1.0 : 0.0;
  } else {
    for (int e = threadIdx.x; e < M * d; e += blockDim.x) S[e] = Y[e];
    __syncthreads();
    hestenes(S, d, M, &flag, red, hnrm);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    for (int p = warp; p < M; p += nwarps) {
      double s2 = 0.0;
      for (int i = lane; i < d; i += 32) s2 += S[p * d + i] * S[p * d + i];
      s2 = warp_sum(s2);
      if (lane == 0) sig[p] = sqrt(s2);
    }
    __syncthreads();
    for (int p = threadIdx.x; p < M; p += blockDim.x) srank[p] = desc_rank(sig, M, p);
    __syncthreads();
    double smax = 0.0;
    for (int p = 0; p < M; ++p) smax = sig[p] > smax ? sig[p] : smax;
    int keep = 0;
    if (smax > 0.0)
      for (int p = 0; p < M; ++p) keep += sig[p] > 1e-10 * smax;
    reff = m.r < keep ? m.r : keep;
    for (int p = threadIdx.x; p < M; p += blockDim.x) b.sig[(long long)h * kMaxM + srank[p]] = sig[p];
    // P = sum over kept columns of u u^T
    for (int e = threadIdx.x; e < d * d; e += blockDim.x) {
      const int i = e / d, j = e % d;
      double v = 0.0;
      for (int p = 0; p < M; ++p)
        if (srank[p] < reff) v += S[p * d + i] * S[p * d + j] / (sig[p] * sig[p]);
      Ph[e] = v;
    }
  }
  if (threadIdx.x == 0) b.reff[h] = reff;
  __syncthreads();

  // ---- fold: BP = B P (into Z), B' = diag(1/s) BP, c = mu_R - (mu_x/s) BP
  for (int e = threadIdx.x; e < d * d; e += blockDim.x) {
    const int i = e / d, j = e % d;
    double v = 0.0;
    for (int k = 0; k < d; ++k) v += Bh[i * d + k] * Ph[k * d + j];
    Z[e] = v;
    b.Bp[(long long)h * d * d + e] = (float)(v / b.sX[hd + i]);
  }
  __syncthreads();
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    double v = b.muR[hd + j];
    for (int i = 0; i < d; ++i) v -= (b.muX[hd + i] / b.sX[hd + i]) * Z[i * d + j];
    b.cvec[hd + j] = (float)v;
  }
}

// Probe fit with every operand in shared memory (dual form, M <= d, and A, Y, S and the
// M x M Gram fit): the same computation as fit_kernel, with B P formed as (B Psi) Psi^T
// so no d x d product is needed.
__global__ void __launch_bounds__(kLinThreads) fit_smem_kernel(Dims m, Buffers b) {
  extern __shared__ double sm[];
  __shared__ double red[32];
  __shared__ double sig[kMaxM];
  __shared__ double u[kMaxM];          // Jacobi norm scratch, then the fold's u
  __shared__ int srank[kMaxM];
  __shared__ int flag, bad;
  const int h = blockIdx.x, d = m.d, M = m.M;
  const long long hd = (long long)h * d;
  double* A = sm;                 // [M][d] standardised, weighted features; later W = B Psi
  double* Y = A + M * d;          // [M][d] centred, weighted residuals; then Z = G^-1 Y
  double* S = Y + M * d;          // [M][d] columns of Y^T orthogonalised; then Psi
  double* G = S + M * d;          // [M][M] A A^T + lambda I, then its Cholesky factor
  const int* probes = b.probes + (long long)h * M;
  const double* w = b.wP + (long long)h * M;
  double wsum = 0.0;
  for (int p = 0; p < M; ++p) wsum += w[p];
  for (int e = threadIdx.x; e < M * d; e += blockDim.x) {
    const int p = e / d, j = e % d;
    const int pos = b.invQ[(long long)h * m.Nq + probes[p]];
    const double x = (double)b.Osp[((long long)h * m.Nq + pos) * d + j];
    const double dn = (double)b.Odense[((long long)h * M + p) * d + j];
    A[e] = x;
    Y[e] = dn - x;
    if (!isfinite(x) || !isfinite(dn)) atomicOr(b.err, kErrNonFinite);
  }
  __syncthreads();
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    double mx = 0.0, mr = 0.0;
    for (int p = 0; p < M; ++p) {
      const double wt = w[p] / wsum;
      mx += wt * A[p * d + j];
      mr += wt * Y[p * d + j];
    }
    double var = 0.0;
    for (int p = 0; p < M; ++p) {
      const double t = A[p * d + j] - mx;
      var += (w[p] / wsum) * t * t;
    }
    b.muX[hd + j] = mx;
    b.muR[hd + j] = mr;
    b.sX[hd + j] = sqrt(var + 1e-6);
  }
  __syncthreads();
  const double* mux = b.muX + hd;
  const double* mur = b.muR + hd;
  const double* sdv = b.sX + hd;
  for (int e = threadIdx.x; e < M * d; e += blockDim.x) {
    const int p = e / d, j = e % d;
    const double om = sqrt((double)M * w[p] / wsum);
    A[e] = om * (A[e] - mux[j]) / sdv[j];
    Y[e] = om * (Y[e] - mur[j]);
    S[e] = Y[e];
  }
  __syncthreads();

  // ---- residual subspace from the columns of Y^T
  double* Ph = b.Pm + (long long)h * d * d;
  int reff = d;
  if (m.r > 0) {
    hestenes(S, d, M, &flag, red, u);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    for (int p = warp; p < M; p += nwarps) {
      double s2 = 0.0;
      for (int i = lane; i < d; i += 32) s2 += S[p * d + i] * S[p * d + i];
      s2 = warp_sum(s2);
      if (lane == 0) sig[p] = sqrt(s2);
    }
    __syncthreads();
    for (int p = threadIdx.x; p < M; p += blockDim.x) srank[p] = desc_rank(sig, M, p);
    __syncthreads();
    double smax = 0.0;
    for (int p = 0; p < M; ++p) smax = sig[p] > smax ? sig[p] : smax;
    int keep = 0;
    if (smax > 0.0)
      for (int p = 0; p < M; ++p) keep += sig[p] > 1e-10 * smax;
    reff = m.r < keep ? m.r : keep;
    for (int p = threadIdx.x; p < M; p += blockDim.x) b.sig[(long long)h * kMaxM + srank[p]] = sig[p];
    // the kept columns, normalised in place, are the leading right singular vectors
    for (int e = threadIdx.x; e < M * d; e += blockDim.x) {
      const int p = e / d;
      if (srank[p] < reff) S[e] /= sig[p];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < d * d; e += blockDim.x) {
      const int i = e / d, j = e % d;
      double v = 0.0;
      for (int p = 0; p < M; ++p)
        if (srank[p] < reff) v += S[p * d + i] * S[p * d + j];
      Ph[e] = v;
    }
  } else {
    for (int e = threadIdx.x; e < d * d; e += blockDim.x) Ph[e] = (e / d == e % d) ? 1.0 : 0.0;
  }
  if (threadIdx.x == 0) b.reff[h] = reff;
  __syncthreads();

  // ---- ridge, dual form: G = A A^T + lambda I, Z = G^-1 Y (in place), B = A^T Z
  for (int e = threadIdx.x; e < M * M; e += blockDim.x) {
    const int i = e / M, j = e % M;
    double g = 0.0;
    for (int k = 0; k < d; ++k) g += A[i * d + k] * A[j * d + k];
    G[e] = g + (i == j ? m.lambda : 0.0);
  }
  __syncthreads();
  const bool pd = cholesky(G, M, &bad);
  if (!pd && threadIdx.x == 0) atomicOr(b.err, kErrNonFinite);
  cholesky_solve(G, M, Y, d, d);
  double* Bh = b.Bm + (long long)h * d * d;
  for (int e = threadIdx.x; e < d * d; e += blockDim.x) {
    const int i = e / d, j = e % d;
    double v = 0.0;
    if (pd)
      for (int p = 0; p < M; ++p) v += A[p * d + i] * Y[p * d + j];
    Bh[e] = v;
  }
  __syncthreads();

  // ---- fold: B' = diag(1/s) B P, c = mu_R - (mu_x / s) B P, with B P = (B Psi) Psi^T
  float* Bp = b.Bp + (long long)h * d * d;
  if (m.r > 0) {
    double* W = A;                 // [d][M]: column p holds B psi_p for kept p
    for (int e = threadIdx.x; e < d * M; e += blockDim.x) {
      const int i = e / M, p = e % M;
      double v = 0.0;
      if (srank[p] < reff)
        for (int j = 0; j < d; ++j) v += Bh[i * d + j] * S[p * d + j];
      W[e] = v;
    }
    __syncthreads();
    for (int p = threadIdx.x; p < M; p += blockDim.x) {
      double v = 0.0;
      for (int i = 0; i < d; ++i) v += (mux[i] / sdv[i]) * W[i * M + p];
      u[p] = v;
    }
    for (int e = threadIdx.x; e < d * d; e += blockDim.x) {
      const int i = e / d, j = e % d;
      double v = 0.0;
      for (int p = 0; p < M; ++p)
        if (srank[p] < reff) v += W[i * M + p] * S[p * d + j];
      Bp[e] = (float)(v / sdv[i]);
    }
    __syncthreads();
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
      double v = mur[j];
      for (int p = 0; p < M; ++p)
        if (srank[p] < reff) v -= u[p] * S[p * d + j];
      b.cvec[hd + j] = (float)v;
    }
  } else {
    for (int e = threadIdx.x; e < d * d; e += blockDim.x) Bp[e] = (float)(Bh[e] / sdv[e / d]);
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
      double v = mur[j];
      for (int i = 0; i < d; ++i) v -= (mux[i] / sdv[i]) * Bh[i * d + j];
      b.cvec[hd + j] = (float)v;
    }
  }
}

// Semantic reference partition: F_K = F_Q = I (d x d) for every K/V head, so the
// coordinates are the raw rows; no eigenvalues.
__global__ void identity_factor_kernel(Dims m, double* FK64, float* FK, double* FQ64, float* FQ,
                                       double* lamK, double* lamQ) {
  const int h = blockIdx.x, d = m.d;
  for (int e = threadIdx.x; e < d * d; e += blockDim.x) {
    const double v = (e / d == e % d) ? 1.0 : 0.0;
    const long long o = (long long)h * d * d + e;
    FK64[o] = v; FK[o] = (float)v; FQ64[o] = v; FQ[o] = (float)v;
  }
  for (int k = threadIdx.x; k < d; k += blockDim.x) {
    lamK[(long long)h * d + k] = 0.0;
    lamQ[(long long)h * d + k] = 0.0;
  }
}

}  // namespace

sparsepr_status launch_identity_factors(const Plan& p, cudaStream_t st) {
  identity_factor_kernel<<<p.dm.Hk, 256, 0, st>>>(p.dm, p.b.FK64, p.b.FK, p.b.FQ64, p.b.FQ, p.b.lamK, p.b.lamQ);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

sparsepr_status launch_key_metric(const Plan& p, cudaStream_t st) {
  const size_t smem = 64 * p.dm.d * sizeof(float);
  key_metric_kernel<<<p.dm.Hk, kLinThreads, smem, st>>>(p.dm, p.Q, p.b.MK);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

sparsepr_status launch_eigen_factor(const Plan& p, bool query, cudaStream_t st) {
  const size_t smem = (size_t)p.dm.d * p.dm.d * sizeof(double);
  SPR_CUDA_OK(cudaFuncSetAttribute(eigen_factor_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const int* only = p.warm ? p.b.warmCold + (query ? p.dm.H : 0) : nullptr;
  // both metrics belong to the K/V head (M_Q is built from its groups' centroids)
  if (query)
    eigen_factor_kernel<<<p.dm.Hk, kLinThreads, smem, st>>>(p.dm, p.b.MQ, p.dm.rQ, p.b.lamQ, p.b.FQ64, p.b.FQ, p.b.err, kErrEigQ, only);
  else
    eigen_factor_kernel<<<p.dm.Hk, kLinThreads, smem, st>>>(p.dm, p.b.MK, p.dm.rK, p.b.lamK, p.b.FK64, p.b.FK, p.b.err, kErrEigK, only);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

// Warm plans: the subspace update from the saved factor, then the full eigendecomposition
// for the heads it flagged (a launch whose other blocks return at once).
sparsepr_status launch_warm_factor(const Plan& p, bool query, cudaStream_t st) {
  const Dims& m = p.dm;
  const int r = query ? m.rQ : m.rK;
  const StateLayout L = state_layout(m);
  const char* base = static_cast<const char*>(p.warm);
  const size_t smem = (size_t)(2 * m.d * (r + 1) + r * r) * sizeof(double);
  SPR_CUDA_OK(cudaFuncSetAttribute(subspace_factor_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  int* cold = p.b.warmCold + (query ? m.H : 0);
  SPR_CUDA_OK(cudaMemsetAsync(cold, 0, sizeof(int) * m.H, st));
  subspace_factor_kernel<<<m.Hk, kLinThreads, smem, st>>>(
      m, query ? p.b.MQ : p.b.MK, reinterpret_cast<const int*>(base),
      reinterpret_cast<const double*>(base + (query ? L.FQ : L.FK)), r,
      query ? p.b.lamQ : p.b.lamK, query ? p.b.FQ64 : p.b.FK64, query ? p.b.FQ : p.b.FK, cold, p.b.err);
  SPR_LAUNCH_OK();
  return launch_eigen_factor(p, query, st);
}

// Restricted estimators (paper App. D.3, Table 4), one CTA per head: the statistics of
// the full fit, then B = 0 (mean only), B = a I with
// a = sum_pj w_p xb_pj Rb_pj / (sum_pj w_p xb_pj^2 + lambda d) (scalar), or B = diag(b) with
// b_j = sum_p w_p xb_pj Rb_pj / (sum_p w_p xb_pj^2 + lambda) (diagonal); omega-weighted
// sums over the probes, no projection (P = I), folded as B' = diag(b / s), c = mu_R - mu_x b / s.
__global__ void __launch_bounds__(kLinThreads) fit_simple_kernel(Dims m, Buffers b) {
  __shared__ double num[kMaxD], den[kMaxD], red[32];
  const int h = blockIdx.x, d = m.d, M = m.M;
  const long long hd = (long long)h * d;
  const int* probes = b.probes + (long long)h * M;
  const double* w = b.wP + (long long)h * M;
  double wsum = 0.0;
  for (int p = 0; p < M; ++p) wsum += w[p];
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    double mx = 0.0, mr = 0.0;
    for (int p = 0; p < M; ++p) {
      const int pos = b.invQ[(long long)h * m.Nq + probes[p]];
      const double x = (double)b.Osp[((long long)h * m.Nq + pos) * d + j];
      const double dn = (double)b.Odense[((long long)h * M + p) * d + j];
      if (!isfinite(x) || !isfinite(dn)) atomicOr(b.err, kErrNonFinite);
      mx += (w[p] / wsum) * x;
      mr += (w[p] / wsum) * (dn - x);
    }
    double var = 0.0;
    for (int p = 0; p < M; ++p) {
      const int pos = b.invQ[(long long)h * m.Nq + probes[p]];
      const double t = (double)b.Osp[((long long)h * m.Nq + pos) * d + j] - mx;
      var += (w[p] / wsum) * t * t;
    }
    const double sd = sqrt(var + 1e-6);
    double nu = 0.0, de = 0.0;
    for (int p = 0; p < M; ++p) {
      const int pos = b.invQ[(long long)h * m.Nq + probes[p]];
      const double x = (double)b.Osp[((long long)h * m.Nq + pos) * d + j];
      const double dn = (double)b.Odense[((long long)h * M + p) * d + j];
      const double om = (double)M * w[p] / wsum;
      const double xb = (x - mx) / sd, rb = (dn - x) - mr;
      nu += om * xb * rb;
      de += om * xb * xb;
    }
    num[j] = nu;
    den[j] = de;
    b.muX[hd + j] = mx;
    b.muR[hd + j] = mr;
    b.sX[hd + j] = sd;
  }
  __syncthreads();
  double pn = 0.0, pd = 0.0;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    pn += num[j];
    pd += den[j];
  }
  const double snum = block_sum(pn, red), sden = block_sum(pd, red);
  const double a = snum / (sden + m.lambda * d);
  double* Bh = b.Bm + (long long)h * d * d;
  double* Ph = b.Pm + (long long)h * d * d;
  float* Bp = b.Bp + (long long)h * d * d;
  for (int e = threadIdx.x; e < d * d; e += blockDim.x) {
    const int i = e / d, j = e % d;
    double v = 0.0;
    if (i == j)
      v = m.estimator == SPARSEPR_EST_SCALAR ? a
        : m.estimator == SPARSEPR_EST_DIAGONAL ? num[j] / (den[j] + m.lambda) : 0.0;
    Bh[e] = v;
    Ph[e] = i == j ? 1.0 : 0.0;
    Bp[e] = (float)(v / b.sX[hd + i]);
  }
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    const double bj = m.estimator == SPARSEPR_EST_SCALAR ? a
                    : m.estimator == SPARSEPR_EST_DIAGONAL ? num[j] / (den[j] + m.lambda) : 0.0;
    b.cvec[hd + j] = (float)(b.muR[hd + j] - b.muX[hd + j] / b.sX[hd + j] * bj);
  }
  if (threadIdx.x == 0) b.reff[h] = d;
}

sparsepr_status launch_fit(const Plan& p, cudaStream_t st) {
  const int d = p.dm.d, M = p.dm.M;
  if (p.dm.estimator != SPARSEPR_EST_RIDGE) {
    fit_simple_kernel<<<p.dm.H, kLinThreads, 0, st>>>(p.dm, p.b);
    SPR_LAUNCH_OK();
    return SPARSEPR_OK;
  }
  // shared-memory path when the dual form applies and A, Y, S (M x d each) and the
  // M x M Gram fit next to the kernel's static arrays
  const size_t fast_smem = (size_t)(3 * M * d + M * M) * sizeof(double);
  cudaFuncAttributes fa{};
  int dev = 0, optin = 0;
  SPR_CUDA_OK(cudaFuncGetAttributes(&fa, fit_smem_kernel));
  SPR_CUDA_OK(cudaGetDevice(&dev));
  SPR_CUDA_OK(cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
  if (M <= d && fa.sharedSizeBytes + fast_smem <= (size_t)optin) {
    SPR_CUDA_OK(cudaFuncSetAttribute(fit_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fast_smem));
    fit_smem_kernel<<<p.dm.H, kLinThreads, fast_smem, st>>>(p.dm, p.b);
    SPR_LAUNCH_OK();
    return SPARSEPR_OK;
  }
  const int n = M <= d ? M : d;
  const size_t smem = (size_t)((n * n > M * d) ? n * n : M * d) * sizeof(double);
  SPR_CUDA_OK(cudaFuncSetAttribute(fit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  fit_kernel<<<p.dm.H, kLinThreads, smem, st>>>(p.dm, p.b);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

}  // namespace spr
