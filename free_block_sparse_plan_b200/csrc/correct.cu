// Corrected output (review page step 5; paper S4.2, App. D.2):
//   unprobed rows  O_hat = O_sp + c + O_sp B',  with B' = diag(1/s) B P and
//                  c = mu_R - (mu_x / s) B P folded by the fit (the same affine map as
//                  mu_R + ((O_sp - mu_x) / s) B P);
//   probe rows     the exact dense output;
// written in the original token order (scatter through the group-major permutation).
#include "common.cuh"

namespace spr {
namespace {

constexpr int kCRows = 64;

__global__ void __launch_bounds__(256) correct_kernel(Dims m, Buffers b, void* Out) {
  extern __shared__ float sm[];
  const int d = m.d, h = blockIdx.y;
  float* Bs = sm;                  // [d][d]
  float* X = sm + d * d;           // [kCRows][d+1]
  __shared__ float cs[kMaxD];
  const float* Bh = b.Bp + (long long)h * d * d;
  for (int e = threadIdx.x; e < d * d; e += blockDim.x) Bs[e] = Bh[e];
  for (int j = threadIdx.x; j < d; j += blockDim.x) cs[j] = b.cvec[(long long)h * d + j];
  const long long p0 = (long long)blockIdx.x * kCRows;
  for (int e = threadIdx.x; e < kCRows * d; e += blockDim.x) {
    const int r = e / d, j = e % d;
    const long long pos = p0 + r;
    X[r * (d + 1) + j] = pos < m.Nq ? b.Osp[((long long)h * m.Nq + pos) * d + j] : 0.0f;
  }
  __syncthreads();
  const int r = threadIdx.x >> 2, qq = threadIdx.x & 3;
  const long long pos = p0 + r;
  if (pos >= m.Nq) return;
  const int row = b.permQ[(long long)h * m.Nq + pos];
  const float* x = X + r * (d + 1);
  float acc[kMaxD / 4];
#pragma unroll
  for (int k = 0; k < kMaxD / 4; ++k) acc[k] = 0.0f;
  for (int i = 0; i < d; ++i) {
    const float xi = x[i];
#pragma unroll
    for (int k = 0; k < kMaxD / 4; ++k) {
      const int j = qq + 4 * k;
      if (j < d) acc[k] = fmaf(xi, Bs[i * d + j], acc[k]);
    }
  }
  const long long obase = ((long long)h * m.Nq + row) * d;
#pragma unroll
  for (int k = 0; k < kMaxD / 4; ++k) {
    const int j = qq + 4 * k;
    if (j < d) store_from_float(Out, obase + j, x[j] + cs[j] + acc[k], m.dtype);
  }
}

__global__ void probe_rows_kernel(Dims m, Buffers b, void* Out) {
  const int p = blockIdx.x, h = blockIdx.y, j = threadIdx.x;
  if (j >= m.d) return;
  const int row = b.probes[(long long)h * m.M + p];
  store_from_float(Out, ((long long)h * m.Nq + row) * m.d + j,
                   b.Odense[((long long)h * m.M + p) * m.d + j], m.dtype);
}

}  // namespace

sparsepr_status launch_correct(const Plan& p, void* Out, cudaStream_t st) {
  const Dims& m = p.dm;
  const size_t smem = (size_t)(m.d * m.d + kCRows * (m.d + 1)) * sizeof(float);
  SPR_CUDA_OK(cudaFuncSetAttribute(correct_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  correct_kernel<<<dim3(cdiv(m.Nq, kCRows), m.H), 256, smem, st>>>(m, p.b, Out);
  SPR_LAUNCH_OK();
  probe_rows_kernel<<<dim3(m.M, m.H), kMaxD, 0, st>>>(m, p.b, Out);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

}  // namespace spr
