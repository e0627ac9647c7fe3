// Corrected output (review page step 5; paper S4.2, App. D.2):
//   unprobed rows  O_hat = O_sp + c + O_sp B',  with B' = diag(1/s) B P and
//                  c = mu_R - (mu_x / s) B P folded by the fit (the same affine map as
//                  mu_R + ((O_sp - mu_x) / s) B P);
//   probe rows     the exact dense output;
// written in the original token order (scatter through the group-major permutation).
// A block takes 64 rows: the rows are staged transposed in shared memory so one float4
// read gives four rows, B' rows as float4 segments; each thread owns 4 rows x d/16
// columns (32 fused multiply-adds per three vector reads at d = 128).
#include "common.cuh"

namespace spr {
namespace {

constexpr int kCRows = 64;
constexpr int kCPad = 4;        // keeps the transposed tile's float4 reads aligned

template <int D>
__global__ void __launch_bounds__(256) correct_kernel(Dims m, Buffers b, void* Out) {
  constexpr int CPT = D / 16;   // columns per thread
  extern __shared__ __align__(16) float sm[];
  float* Bs = sm;                          // [D][D]
  float* Xt = sm + D * D;                  // [D][kCRows + kCPad] transposed rows
  __shared__ float cs[kMaxD];
  const int d = m.d, h = blockIdx.y;
  const float* Bh = b.Bp + (long long)h * d * d;
  for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
    const int i = e / D, j = e % D;
    Bs[e] = (i < d && j < d) ? Bh[i * d + j] : 0.0f;
  }
  for (int j = threadIdx.x; j < D; j += blockDim.x) cs[j] = j < d ? b.cvec[(long long)h * d + j] : 0.0f;
  const long long p0 = (long long)blockIdx.x * kCRows;
  for (int e = threadIdx.x; e < kCRows * D; e += blockDim.x) {
    const int r = e / D, j = e % D;
    const long long pos = p0 + r;
    Xt[j * (kCRows + kCPad) + r] = (pos < m.Nq && j < d) ? b.Osp[((long long)h * m.Nq + pos) * d + j] : 0.0f;
  }
  __syncthreads();
  const int tr = threadIdx.x >> 4, tcol = threadIdx.x & 15;
  const int r0 = 4 * tr, c0 = CPT * tcol;
  float acc[4][CPT];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int q = 0; q < CPT; ++q) acc[a][q] = 0.0f;
  for (int i = 0; i < D; ++i) {
    const float4 x = *reinterpret_cast<const float4*>(Xt + i * (kCRows + kCPad) + r0);
    float bv[CPT];
#pragma unroll
    for (int q = 0; q < CPT; q += 4) {
      const float4 t = *reinterpret_cast<const float4*>(Bs + i * D + c0 + q);
      bv[q] = t.x; bv[q + 1] = t.y; bv[q + 2] = t.z; bv[q + 3] = t.w;
    }
#pragma unroll
    for (int q = 0; q < CPT; ++q) {
      acc[0][q] = fmaf(x.x, bv[q], acc[0][q]);
      acc[1][q] = fmaf(x.y, bv[q], acc[1][q]);
      acc[2][q] = fmaf(x.z, bv[q], acc[2][q]);
      acc[3][q] = fmaf(x.w, bv[q], acc[3][q]);
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const long long pos = p0 + r0 + a;
    if (pos >= m.Nq) continue;
    const int row = b.permQ[(long long)h * m.Nq + pos];
    const long long obase = ((long long)h * m.Nq + row) * d;
#pragma unroll
    for (int q = 0; q < CPT; ++q) {
      const int j = c0 + q;
      if (j < d) store_from_float(Out, obase + j, Xt[j * (kCRows + kCPad) + r0 + a] + cs[j] + acc[a][q], m.dtype);
    }
  }
}

__global__ void probe_rows_kernel(Dims m, Buffers b, void* Out) {
  const int p = blockIdx.x, h = blockIdx.y, j = threadIdx.x;
  if (j >= m.d) return;
  const int row = b.probes[(long long)h * m.M + p];
  store_from_float(Out, ((long long)h * m.Nq + row) * m.d + j,
                   b.Odense[((long long)h * m.M + p) * m.d + j], m.dtype);
}

template <int D>
sparsepr_status launch_correct_d(const Plan& p, void* Out, cudaStream_t st) {
  const Dims& m = p.dm;
  const size_t smem = (size_t)(D * D + D * (kCRows + kCPad)) * sizeof(float);
  SPR_CUDA_OK(cudaFuncSetAttribute(correct_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  correct_kernel<D><<<dim3(cdiv(m.Nq, kCRows), m.H), 256, smem, st>>>(m, p.b, Out);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

}  // namespace

sparsepr_status launch_correct(const Plan& p, void* Out, cudaStream_t st) {
  const Dims& m = p.dm;
  sparsepr_status s = correct_tc_applies(m.dtype, m.d, m.engine) ? launch_correct_tc(p, Out, st)
                      : m.d <= 64 ? launch_correct_d<64>(p, Out, st) : launch_correct_d<128>(p, Out, st);
  if (s != SPARSEPR_OK) return s;
  probe_rows_kernel<<<dim3(m.M, m.H), kMaxD, 0, st>>>(m, p.b, Out);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

}  // namespace spr
