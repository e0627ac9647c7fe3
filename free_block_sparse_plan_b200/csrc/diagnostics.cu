// Diagnostics of "Partition the Support, Reconstruct the Residual" S3 (observations O1 and
// O3); measurement tools for a partition, off the attention call's hot path.
//
// O1 support densities: for a query row i, D_i(alpha) is the smallest set of keys whose
// dense attention weights reach the fraction alpha of the row's mass, keys taken by
// decreasing weight with the lowest index first among equal weights; tau_i = |D_i| / N_k,
// and a pool of rows has the pooled density |union of their D_i| / N_k.  Everything in
// fp64: logits tau q.k (the products of the stored values are exact, the dot product is
// summed over ascending channels), weights exp(l - max).
//
//   support_weights_kernel  one block per (row, head): logits, row maximum, weights and
//                           their sum Z (fixed-order reductions: deterministic);
//   support_select_kernel   one block per (row, head): the threshold theta, the largest
//                           weight such that the weights >= theta hold at least
//                           alpha Z (1 - 1e-15), found by bisection over the bit patterns
//                           of positive doubles (ordered like their values); then
//                           |D_i| = #{w > theta} + the fewest weights equal to theta that
//                           complete the mass (added one at a time, as a sorted running
//                           sum does), and D_i's keys are marked in the pool's key map (the
//                           lowest-index keys among those equal to theta);
//   support_union_kernel    one block per (pool, head): keys marked in the pool's map.
//
// O3 oracle affine fit (S3 O3, App. D.5): the least-squares fit R ~ 1 b + O_sp B of the
// residual R = O_dense - O_sp over all rows of a head.  With X the sparse output centred
// and its non-zero columns scaled to unit norm, and R_c the centred residual, the fit is
// the projection of R_c on the span of X's columns whose singular values exceed 1e-10
// times the largest.  Here the span comes from the eigendecomposition of the Gram matrix
// G = X^T X (one-sided Jacobi; eigenvalue lambda = sigma^2, kept when above 1e-20
// lambda_max): the fitted squared norm is sum_j |C^T v_j|^2 / lambda_j with C = X^T R_c,
// and the remaining error |R_c|^2 minus that.  Forming G squares X's condition number, so
// directions with sigma below about 1e-8 sigma_max are at rounding level here, where an
// SVD of X resolves them; the fit of a well-conditioned X is unaffected.
//   affine_means_kernel     one thread per (column, side, head): column means of O_sp and
//                           R, and the residual's centred and plain squared column norms;
//   affine_gram_kernel      one block per (column tile, head): X^T X and X^T R_c, every
//                           entry summed by one thread over all rows in row order;
//   affine_solve_kernel     one block per head: scaling, Jacobi eigendecomposition, fit.
#include "common.cuh"
#include "jacobi.cuh"

namespace spr {
namespace {

constexpr int kSupThreads = 256;
constexpr int kSelThreads = 1024;

struct SupArgs {
  int H, Nq, Nk, d, dtype, G, nrows, npools;
  const void* Q;
  const void* K;
  const int* rows;        // [H][nrows]
  const int* pool;        // [H][nrows]
  double alpha;
  double* w;              // [H][nrows][Nk] weights
  double* Z;              // [H][nrows]
  unsigned char* mark;    // [H][npools][Nk]
  int* sizes;             // [H][nrows]
  int* pooled;            // [H][npools]
};

__device__ __forceinline__ double load_d(const void* p, long long i, int dtype) {
  return (double)load_as_float(p, i, dtype);
}

__global__ void __launch_bounds__(kSupThreads) support_weights_kernel(SupArgs g) {
  __shared__ double q[kMaxD];
  __shared__ double red[kSupThreads / 32];
  const int i = blockIdx.x, h = blockIdx.y;
  int row = g.rows[(long long)h * g.nrows + i];
  row = row < 0 ? 0 : (row >= g.Nq ? g.Nq - 1 : row);
  for (int k = threadIdx.x; k < g.d; k += blockDim.x) q[k] = load_d(g.Q, ((long long)h * g.Nq + row) * g.d + k, g.dtype);
  __syncthreads();
  const double tau = 1.0 / sqrt((double)g.d);
  const long long kb = (long long)(h / g.G) * g.Nk * g.d;
  double* w = g.w + ((long long)h * g.nrows + i) * g.Nk;
  double mx = -INFINITY;
  for (int j = threadIdx.x; j < g.Nk; j += blockDim.x) {
    double s = 0.0;
    for (int k = 0; k < g.d; ++k) s = fma(q[k], load_d(g.K, kb + (long long)j * g.d + k, g.dtype), s);
    const double l = tau * s;
    w[j] = l;
    mx = fmax(mx, l);
  }
  for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = red[0];
  for (int k = 1; k < (int)(blockDim.x >> 5); ++k) mx = fmax(mx, red[k]);
  double part = 0.0;
  for (int j = threadIdx.x; j < g.Nk; j += blockDim.x) {
    const double e = exp(w[j] - mx);
    w[j] = e;
    part += e;
  }
  const double z = block_sum(part, red);
  if (threadIdx.x == 0) g.Z[(long long)h * g.nrows + i] = z;
}

// Sum of the weights >= theta (fixed-order reduction) and, when asked, their count.
__device__ double mass_at_least(const double* w, int n, double theta, double* red) {
  double s = 0.0;
  for (int j = threadIdx.x; j < n; j += blockDim.x)
    if (w[j] >= theta) s += w[j];
  return block_sum(s, red);
}

__global__ void __launch_bounds__(kSelThreads) support_select_kernel(SupArgs g) {
  __shared__ double red[kSelThreads / 32];
  __shared__ long long redl[kSelThreads / 32];
  __shared__ int sh[32];
  __shared__ long long s_need;
  const int i = blockIdx.x, h = blockIdx.y;
  const double* w = g.w + ((long long)h * g.nrows + i) * g.Nk;
  const double target = g.alpha * g.Z[(long long)h * g.nrows + i] * (1.0 - 1e-15);
  // bisection over the bit patterns of non-negative doubles: S(lo) >= target > S(hi)
  long long lo = 0;                                            // theta = +0: every weight
  long long hi = __double_as_longlong(1.0) + 1;                // above the largest weight (1)
  while (hi - lo > 1) {
    const long long mid = lo + (hi - lo) / 2;
    const double s = mass_at_least(w, g.Nk, __longlong_as_double(mid), red);
    if (s >= target) lo = mid; else hi = mid;
  }
  const double theta = __longlong_as_double(lo);
  // weights above theta: their mass G < target and their count; then the weights equal
  // to theta join one at a time until the mass reaches the target
  double sg = 0.0;
  long long cg = 0, ce = 0;
  for (int j = threadIdx.x; j < g.Nk; j += blockDim.x) {
    if (w[j] > theta) { sg += w[j]; ++cg; }
    else if (w[j] == theta) ++ce;
  }
  const double G = block_sum(sg, red);
  cg = block_sum_ll(cg, redl);
  ce = block_sum_ll(ce, redl);
  if (threadIdx.x == 0) {
    long long need = 0;
    double acc = G;                                  // G < target: at least one joins
    while (acc < target && need < ce) { acc += theta; ++need; }
    g.sizes[(long long)h * g.nrows + i] = (int)(cg + need);
    s_need = need;
  }
  __syncthreads();
  const long long need = s_need;
  // mark D_i: every weight above theta, and the `need` lowest-index weights equal to it
  // (a row whose pool id is outside [0, npools) marks nothing)
  const int pool = g.pool[(long long)h * g.nrows + i];
  if (pool < 0 || pool >= g.npools) return;
  unsigned char* mk = g.mark + ((long long)h * g.npools + pool) * g.Nk;
  long long run = 0;
  for (int j0 = 0; j0 < g.Nk; j0 += blockDim.x) {
    const int j = j0 + threadIdx.x;
    const bool in = j < g.Nk;
    const double v = in ? w[j] : 0.0;
    const int eq = (in && v == theta) ? 1 : 0;
    int tot;
    const int ex = block_exclusive_scan(eq, sh, &tot);
    if (in && (v > theta || (eq && run + ex < need))) mk[j] = 1;
    run += tot;
    __syncthreads();
  }
}

__global__ void __launch_bounds__(1024) support_union_kernel(SupArgs g) {
  __shared__ long long red[32];
  const int pool = blockIdx.x, h = blockIdx.y;
  const unsigned char* mk = g.mark + ((long long)h * g.npools + pool) * g.Nk;
  long long c = 0;
  for (int j = threadIdx.x; j < g.Nk; j += blockDim.x) c += mk[j];
  c = block_sum_ll(c, red);
  if (threadIdx.x == 0) g.pooled[(long long)h * g.npools + pool] = (int)c;
}

// ------------------------------------------------------------------------- O3 affine fit
struct AffArgs {
  int H, Nq, d, dtype;
  const float* Osp;       // [H][Nq][d] group-major
  const int* inv;         // [H][Nq] original row -> group-major position
  const void* dense;      // [H][Nq][d] original order, params dtype
  double* mu;             // [H][4][d]: column means of O_sp and of R, |R_c|^2, |R|^2 per column
  double* gram;           // [H][d][2d + 2]: X^T X | X^T R_c (two spare entries per row)
  double* explained;      // [H]
  double* err;            // [H]
};

constexpr int kAffCols = 8;                         // columns of X per Gram block

__device__ __forceinline__ double osp_at(const AffArgs& a, int h, int n, int c) {
  const int pos = a.inv[(long long)h * a.Nq + n];
  return (double)a.Osp[((long long)h * a.Nq + pos) * a.d + c];
}
__device__ __forceinline__ double dense_at(const AffArgs& a, int h, int n, int c) {
  return load_d(a.dense, ((long long)h * a.Nq + n) * a.d + c, a.dtype);
}

// one thread per (column, side): the mean over all rows in row order; for the residual
// side also its centred and plain squared norms (second pass)
__global__ void __launch_bounds__(256) affine_means_kernel(AffArgs a) {
  const int h = blockIdx.y;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;     // t < 2d: side t / d, column t % d
  if (t >= 2 * a.d) return;
  const int side = t / a.d, c = t % a.d;
  double s = 0.0;
  for (int n = 0; n < a.Nq; ++n) {
    const double x = osp_at(a, h, n, c);
    s += side == 0 ? x : dense_at(a, h, n, c) - x;
  }
  const double mean = s / (double)a.Nq;
  double* muh = a.mu + (long long)h * 4 * a.d;
  muh[side * a.d + c] = mean;
  if (side == 1) {
    double rc = 0.0, r2 = 0.0;
    for (int n = 0; n < a.Nq; ++n) {
      const double r = dense_at(a, h, n, c) - osp_at(a, h, n, c);
      rc = fma(r - mean, r - mean, rc);
      r2 = fma(r, r, r2);
    }
    muh[2 * a.d + c] = rc;
    muh[3 * a.d + c] = r2;
  }
}

// block (column tile, head): thread (i, j) sums X_i X_j (j < d) or X_i R_c,j (j >= d)
// over all rows in row order; rows staged through shared memory
__global__ void __launch_bounds__(256) affine_gram_kernel(AffArgs a) {
  constexpr int kRowsStage = 16;
  __shared__ double xs[kRowsStage][kMaxD];
  __shared__ double rs[kRowsStage][kMaxD];
  const int h = blockIdx.y, c0 = blockIdx.x * kAffCols, d = a.d;
  const double* mux = a.mu + (long long)h * 4 * d;
  const double* mur = mux + d;
  const int ncell = kAffCols * 2 * d;                     // at most 8 * 256 = 2048 entries
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int n0 = 0; n0 < a.Nq; n0 += kRowsStage) {
    const int nr = min(kRowsStage, a.Nq - n0);
    __syncthreads();
    for (int e = threadIdx.x; e < nr * d; e += blockDim.x) {
      const int rr_ = e / d, c = e % d, n = n0 + rr_;
      const double x = osp_at(a, h, n, c);
      xs[rr_][c] = x - mux[c];
      rs[rr_][c] = (dense_at(a, h, n, c) - x);
    }
    __syncthreads();
    for (int k = 0; k < 8; ++k) {
      const int cell = threadIdx.x + k * blockDim.x;
      if (cell >= ncell) break;
      const int i = c0 + cell / (2 * d), j = cell % (2 * d);
      if (i >= d) continue;
      double s = acc[k];
      for (int q = 0; q < nr; ++q) s = fma(xs[q][i], j < d ? xs[q][j] : rs[q][j - d] - mur[j - d], s);
      acc[k] = s;
    }
  }
  double* gh = a.gram + (long long)h * d * (2 * d + 2);
  for (int k = 0; k < 8; ++k) {
    const int cell = threadIdx.x + k * blockDim.x;
    if (cell >= ncell) break;
    const int i = c0 + cell / (2 * d), j = cell % (2 * d);
    if (i < d) gh[(long long)i * (2 * d + 2) + j] = acc[k];
  }
}

__global__ void __launch_bounds__(1024) affine_solve_kernel(AffArgs a, double tol) {
  extern __shared__ double S[];                 // [d][d] scaled Gram (column-major), then C
  __shared__ double nrm[kMaxD], lam[kMaxD], red[32], hn[kMaxD];
  __shared__ int flag;
  const int h = blockIdx.x, d = a.d;
  const double* gh = a.gram + (long long)h * d * (2 * d + 2);
  const int ld = 2 * d + 2;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const double g = gh[(long long)c * ld + c];
    nrm[c] = g > 0.0 ? sqrt(g) : 0.0;          // zero columns are left out of the fit
  }
  __syncthreads();
  for (int e = threadIdx.x; e < d * d; e += blockDim.x) {
    const int j = e / d, i = e % d;             // column j, row i
    S[e] = (nrm[i] > 0.0 && nrm[j] > 0.0) ? gh[(long long)i * ld + j] / (nrm[i] * nrm[j]) : 0.0;
  }
  __syncthreads();
  hestenes(S, d, d, &flag, red, hn);
  // columns of S V: lambda_j v_j (S is symmetric PSD)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int j = warp; j < d; j += nw) {
    double s = 0.0;
    for (int i = lane; i < d; i += 32) s += S[j * d + i] * S[j * d + i];
    s = warp_sum(s);
    if (lane == 0) lam[j] = sqrt(s);
  }
  __syncthreads();
  double lmax = 0.0;
  for (int j = 0; j < d; ++j) lmax = fmax(lmax, lam[j]);
  // fitted squared norm: sum over kept j of |C^T v_j|^2 / lambda_j, C_ik = G_i,d+k / nrm_i
  double part = 0.0;
  for (int e = threadIdx.x; e < d * d; e += blockDim.x) {
    const int j = e / d, k = e % d;             // eigenvector j, residual column k
    if (!(lam[j] > tol * tol * lmax) || lam[j] <= 0.0) continue;
    double s = 0.0;
    for (int i = 0; i < d; ++i) {
      if (nrm[i] <= 0.0) continue;
      const double vij = S[j * d + i] / lam[j];
      s = fma(vij, gh[(long long)i * ld + d + k] / nrm[i], s);
    }
    part += s * s / lam[j];
  }
  const double fit = block_sum(part, red);
  const double* muh = a.mu + (long long)h * 4 * d;
  if (threadIdx.x == 0) {
    double rc = 0.0, tot = 0.0;                 // |R_c|^2 and |R|^2 over the columns
    for (int c = 0; c < d; ++c) {
      rc += muh[2 * d + c];
      tot += muh[3 * d + c];
    }
    const double e = fmax(rc - fit, 0.0);
    a.err[h] = e;
    a.explained[h] = tot > 0.0 ? 1.0 - e / tot : 0.0;
  }
}

}  // namespace

size_t support_ws_bytes(int H, int nrows, int npools, int Nk) {
  return align256((size_t)H * nrows * Nk * sizeof(double)) + align256((size_t)H * nrows * sizeof(double)) +
         align256((size_t)H * npools * Nk);
}

}  // namespace spr

using namespace spr;

extern "C" {

sparsepr_status sparsepr_support_workspace_size(const sparsepr_params* params, int32_t nrows,
                                                int32_t npools, size_t* bytes) {
  if (!params || !bytes || nrows < 1 || npools < 1 || npools > nrows) return SPARSEPR_ERR_ARG;
  if (params->H < 1 || params->N_k < 1) return SPARSEPR_ERR_SHAPE;
  *bytes = support_ws_bytes(params->H, nrows, npools, params->N_k);
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_support_densities(const sparsepr_params* params, const void* Q,
                                           const void* K, const int32_t* rows,
                                           const int32_t* pool, int32_t nrows, int32_t npools,
                                           double alpha, void* workspace, size_t workspace_bytes,
                                           int32_t* sizes, int32_t* pooled, void* stream) {
  if (!params || !Q || !K || !rows || !pool || !sizes || !pooled) return SPARSEPR_ERR_ARG;
  if (!(alpha > 0.0 && alpha <= 1.0)) return SPARSEPR_ERR_ARG;
  if (nrows < 1 || npools < 1 || npools > nrows) return SPARSEPR_ERR_ARG;
  if (params->dtype != SPARSEPR_F32 && params->dtype != SPARSEPR_BF16) return SPARSEPR_ERR_DTYPE;
  if (params->H < 1 || params->H > 65535 || params->N_q < 1 || params->N_k < 1) return SPARSEPR_ERR_SHAPE;
  if (params->d < 8 || params->d > kMaxD || params->d % 8) return SPARSEPR_ERR_SHAPE;
  if (nrows > 65535 || npools > 65535) return SPARSEPR_ERR_SHAPE;
  if (params->G < 0 || (params->G > 1 && params->H % params->G != 0)) return SPARSEPR_ERR_SHAPE;
  const size_t need = support_ws_bytes(params->H, nrows, npools, params->N_k);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) || workspace_bytes < need)
    return SPARSEPR_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  SupArgs g{};
  g.H = params->H; g.Nq = params->N_q; g.Nk = params->N_k; g.d = params->d; g.dtype = params->dtype;
  g.G = params->G > 1 ? params->G : 1;
  g.nrows = nrows; g.npools = npools;
  g.Q = Q; g.K = K; g.rows = rows; g.pool = pool; g.alpha = alpha;
  char* c = reinterpret_cast<char*>(workspace);
  g.w = reinterpret_cast<double*>(c);
  c += align256((size_t)g.H * nrows * g.Nk * sizeof(double));
  g.Z = reinterpret_cast<double*>(c);
  c += align256((size_t)g.H * nrows * sizeof(double));
  g.mark = reinterpret_cast<unsigned char*>(c);
  g.sizes = sizes; g.pooled = pooled;
  SPR_CUDA_OK(cudaMemsetAsync(g.mark, 0, (size_t)g.H * npools * g.Nk, st));
  support_weights_kernel<<<dim3(nrows, g.H), kSupThreads, 0, st>>>(g);
  SPR_LAUNCH_OK();
  support_select_kernel<<<dim3(nrows, g.H), kSelThreads, 0, st>>>(g);
  SPR_LAUNCH_OK();
  support_union_kernel<<<dim3(npools, g.H), 1024, 0, st>>>(g);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

}  // extern "C"

namespace spr {
// Launched by sparsepr_affine_fit (api.cu) with the plan's buffers.
sparsepr_status launch_affine_fit(const Plan& p, const void* dense, double* ws, double* explained,
                                  double* err, cudaStream_t st) {
  const Dims& m = p.dm;
  AffArgs a{};
  a.H = m.H; a.Nq = m.Nq; a.d = m.d; a.dtype = m.dtype;
  a.Osp = p.b.Osp; a.inv = p.b.invQ; a.dense = dense;
  a.mu = ws;
  a.gram = ws + (size_t)m.H * 4 * m.d;
  a.explained = explained; a.err = err;
  affine_means_kernel<<<dim3(cdiv(2 * m.d, 256), m.H), 256, 0, st>>>(a);
  SPR_LAUNCH_OK();
  affine_gram_kernel<<<dim3(cdiv(m.d, kAffCols), m.H), 256, 0, st>>>(a);
  SPR_LAUNCH_OK();
  const size_t smem = (size_t)m.d * m.d * sizeof(double);
  SPR_CUDA_OK(cudaFuncSetAttribute(affine_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  affine_solve_kernel<<<m.H, 1024, smem, st>>>(a, 1e-10);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}
size_t affine_ws_doubles(const Dims& m) { return (size_t)m.H * 4 * m.d + (size_t)m.H * m.d * (2 * m.d + 2); }
}  // namespace spr
