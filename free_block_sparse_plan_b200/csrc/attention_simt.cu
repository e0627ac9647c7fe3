// Attention on CUDA cores in fp32 (the reference engine, and the fp32 path).
//
//   sparse:  renormalised hard drop (paper S2): a query row of group a attends, with the
//            softmax renormalised over them, to the keys of the K/V groups selected for
//            a.  One block per query group; the selected groups' key ranges in the
//            group-major K/V copies are walked as one concatenated key sequence.
//   probes:  exact rows (paper S4.2, App. A.2): the M probe rows against all keys, split
//            over key chunks into partial (max, sum, numerator) triples, then combined.
//   dense:   softmax(Q K^T / sqrt(d)) V for every row.
//
// Tile: 64 query rows x 64 keys per step; four threads per query row, each holding a
// quarter of the head dimension; online softmax in fp32 with expf.
#include <cmath>
#include <type_traits>

#include "common.cuh"

namespace spr {
namespace {

constexpr int kRows = 64, kKeys = 64, kThreads = 256;

struct KeyRange {     // keys [k0, k1) of a row-major [*, d] array
  const void* K;
  const void* V;
  long long k0, k1;
};

// Interleaved smem slot of dimension t so the four quarter-threads hit distinct banks.
template <int D>
__device__ __forceinline__ int islot(int t) {
  return (t % (D / 4)) * 4 + t / (D / 4);
}

// Core: 64 query rows (q_rows[r] = element offset of row r, or -1) against a key
// sequence whose physical row offsets come from `key_row(v)`; returns per-thread
// (m, l, o[D/4]) unnormalised.
template <int D, class KeyRow>
__device__ void attend_core(const Dims& m, const void* Qsrc, const long long* q_rows,
                            const void* Ksrc, const void* Vsrc, long long nkeys, KeyRow key_row,
                            float* ks, float* vs, long long* krow, float& mrow, float& lrow,
                            float (&o)[D / 4]) {
  constexpr int Q4 = D / 4;
  const int d = m.d;
  const float tau = 1.0f / sqrtf((float)d);
  const int r = threadIdx.x >> 2, qq = threadIdx.x & 3;
  float q[Q4];
  const long long qoff = q_rows[r];
#pragma unroll
  for (int k = 0; k < Q4; ++k) {
    const int t = qq * Q4 + k;
    q[k] = (qoff >= 0 && t < d) ? load_as_float(Qsrc, qoff + t, m.dtype) * tau : 0.0f;
    o[k] = 0.0f;
  }
  mrow = -INFINITY;
  lrow = 0.0f;
  for (long long v0 = 0; v0 < nkeys; v0 += kKeys) {
    const int nk = (nkeys - v0) < kKeys ? (int)(nkeys - v0) : kKeys;
    __syncthreads();
    if (threadIdx.x < kKeys) krow[threadIdx.x] = threadIdx.x < nk ? key_row(v0 + threadIdx.x) : -1;
    __syncthreads();
    for (int e = threadIdx.x; e < kKeys * D; e += blockDim.x) {
      const int j = e / D, t = e % D;
      const long long kr = krow[j];
      float kv = 0.0f, vv = 0.0f;
      if (kr >= 0 && t < d) {
        kv = load_as_float(Ksrc, kr + t, m.dtype);
        vv = load_as_float(Vsrc, kr + t, m.dtype);
      }
      ks[j * D + islot<D>(t)] = kv;
      vs[j * D + islot<D>(t)] = vv;
    }
    __syncthreads();
    for (int half = 0; half < kKeys; half += 32) {
      float s[32];
      float smax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float* kr = ks + (half + j) * D;
        float a = 0.0f;
#pragma unroll
        for (int k = 0; k < Q4; ++k) a = fmaf(q[k], kr[k * 4 + qq], a);
        a += __shfl_xor_sync(0xffffffffu, a, 1);
        a += __shfl_xor_sync(0xffffffffu, a, 2);
        s[j] = (half + j < nk) ? a : -INFINITY;
        smax = fmaxf(smax, s[j]);
      }
      const float mnew = fmaxf(mrow, smax);
      if (mnew == -INFINITY) continue;   // nothing valid yet
      const float corr = expf(mrow - mnew);
      lrow *= corr;
#pragma unroll
      for (int k = 0; k < Q4; ++k) o[k] *= corr;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float pj = expf(s[j] - mnew);
        lrow += pj;
        const float* vr = vs + (half + j) * D;
#pragma unroll
        for (int k = 0; k < Q4; ++k) o[k] = fmaf(pj, vr[k * 4 + qq], o[k]);
      }
      mrow = mnew;
    }
  }
}

// ---------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kThreads) sparse_simt_kernel(Dims m, Buffers b) {
  extern __shared__ float sm[];
  float* ks = sm;
  float* vs = sm + kKeys * D;
  int* csum = reinterpret_cast<int*>(vs + kKeys * D);      // [C_k + 1]
  int* cbase = csum + (kMaxC + 1);                          // [C_k] physical start rows
  __shared__ long long krow[kKeys];
  __shared__ long long qrow[kRows];
  __shared__ int sh[32];
  const int h = blockIdx.y, a = blockIdx.x, d = m.d;
  if (a >= b.nQ[h]) return;
  const int labq = b.usedQ[(long long)h * m.Cq + a];
  const int q0 = b.offQ[(long long)h * (m.Cq + 1) + labq];
  const int q1 = b.offQ[(long long)h * (m.Cq + 1) + labq + 1];
  const int cnt = b.cellCnt[(long long)h * m.Cq + a];
  const int* ids = b.cellIds + ((long long)h * m.Cq + a) * m.Ck;
  // concatenated key sequence of the selected groups (ascending group id)
  for (int base = 0; base < cnt; base += blockDim.x) {
    const int i = base + threadIdx.x;
    int sz = 0, start = 0;
    if (i < cnt) {
      const int kb = ids[i];
      const int labk = b.usedK[(long long)(h / m.G) * m.Ck + kb];
      start = b.offK[(long long)(h / m.G) * (m.Ck + 1) + labk];
      sz = b.offK[(long long)(h / m.G) * (m.Ck + 1) + labk + 1] - start;
    }
    int tot;
    const int ex = block_exclusive_scan(sz, sh, &tot);
    const int prev = base == 0 ? 0 : csum[base];
    if (i < cnt) {
      csum[i] = prev + ex;
      cbase[i] = start;
    }
    __syncthreads();
    if (threadIdx.x == 0) csum[(base + blockDim.x < cnt ? base + blockDim.x : cnt)] = prev + tot;
    __syncthreads();
  }
  const long long nkeys = cnt > 0 ? csum[cnt] : 0;
  const long long kbase = (long long)(h / m.G) * m.Nk * d;   // K/V head h / G
  auto key_row = [&](long long v) -> long long {
    int lo = 0, hi = cnt - 1;      // last i with csum[i] <= v
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (csum[mid] <= v) lo = mid; else hi = mid - 1;
    }
    return kbase + ((long long)cbase[lo] + (v - csum[lo])) * d;
  };
  for (int t0 = q0; t0 < q1; t0 += kRows) {
    __syncthreads();
    if (threadIdx.x < kRows) {
      const int pos = t0 + threadIdx.x;
      qrow[threadIdx.x] = pos < q1 ? ((long long)h * m.Nq + pos) * d : -1;
    }
    __syncthreads();
    float mrow, lrow, o[D / 4];
    attend_core<D>(m, b.Qp, qrow, b.Kp, b.Vp, nkeys, key_row, ks, vs, krow, mrow, lrow, o);
    const int r = threadIdx.x >> 2, qq = threadIdx.x & 3;
    const int pos = t0 + r;
    if (pos < q1) {
      float* out = b.Osp + ((long long)h * m.Nq + pos) * d;
      const float inv = 1.0f / lrow;
#pragma unroll
      for (int k = 0; k < D / 4; ++k) {
        const int t = qq * (D / 4) + k;
        if (t < d) out[t] = o[k] * inv;
      }
    }
  }
}

// Partial exact attention of probe rows against keys [s*kProbeSplit, ...).
template <int D>
__global__ void __launch_bounds__(kThreads) probe_simt_kernel(Dims m, Buffers b, const void* Q,
                                                              const void* K, const void* V) {
  extern __shared__ float sm[];
  float* ks = sm;
  float* vs = sm + kKeys * D;
  __shared__ long long krow[kKeys];
  __shared__ long long qrow[kRows];
  const int s = blockIdx.x, rt = blockIdx.y, h = blockIdx.z, d = m.d;
  if (threadIdx.x < kRows) {
    const int p = rt * kRows + threadIdx.x;
    qrow[threadIdx.x] = p < m.M ? ((long long)h * m.Nq + b.probes[(long long)h * m.M + p]) * d : -1;
  }
  __syncthreads();
  const long long k0 = (long long)s * kProbeSplit;
  const long long k1 = (k0 + kProbeSplit < m.Nk) ? k0 + kProbeSplit : m.Nk;
  const long long kbase = (long long)(h / m.G) * m.Nk * d;   // K/V head h / G
  auto key_row = [&](long long v) -> long long { return kbase + (k0 + v) * d; };
  float mrow, lrow, o[D / 4];
  attend_core<D>(m, Q, qrow, K, V, k1 - k0, key_row, ks, vs, krow, mrow, lrow, o);
  const int r = threadIdx.x >> 2, qq = threadIdx.x & 3;
  const int p = rt * kRows + r;
  if (p < m.M) {
    const long long slot = ((long long)h * m.M + p) * m.nsplit + s;
    float* out = b.Opart + slot * d;
#pragma unroll
    for (int k = 0; k < D / 4; ++k) {
      const int t = qq * (D / 4) + k;
      if (t < d) out[t] = o[k];
    }
    if (qq == 0) {
      b.MLpart[2 * slot] = mrow;
      b.MLpart[2 * slot + 1] = lrow;
    }
  }
}

__global__ void probe_combine_kernel(Dims m, Buffers b) {
  const int p = blockIdx.x, h = blockIdx.y, j = threadIdx.x;
  const long long slot0 = ((long long)h * m.M + p) * m.nsplit;
  float mx = -INFINITY;
  for (int s = 0; s < m.nsplit; ++s) mx = fmaxf(mx, b.MLpart[2 * (slot0 + s)]);
  float l = 0.0f, acc = 0.0f;
  for (int s = 0; s < m.nsplit; ++s) {
    const float w = expf(b.MLpart[2 * (slot0 + s)] - mx);
    l += w * b.MLpart[2 * (slot0 + s) + 1];
    if (j < m.d) acc += w * b.Opart[(slot0 + s) * m.d + j];
  }
  if (j < m.d) b.Odense[((long long)h * m.M + p) * m.d + j] = acc / l;
}

template <int D>
__global__ void __launch_bounds__(kThreads) dense_simt_kernel(Dims m, const void* Q, const void* K,
                                                              const void* V, void* Out) {
  extern __shared__ float sm[];
  float* ks = sm;
  float* vs = sm + kKeys * D;
  __shared__ long long krow[kKeys];
  __shared__ long long qrow[kRows];
  const int h = blockIdx.y, d = m.d;
  const long long r0 = (long long)blockIdx.x * kRows;
  if (threadIdx.x < kRows) {
    const long long row = r0 + threadIdx.x;
    qrow[threadIdx.x] = row < m.Nq ? ((long long)h * m.Nq + row) * d : -1;
  }
  __syncthreads();
  const long long kbase = (long long)(h / m.G) * m.Nk * d;   // K/V head h / G
  auto key_row = [&](long long v) -> long long { return kbase + v * d; };
  float mrow, lrow, o[D / 4];
  attend_core<D>(m, Q, qrow, K, V, m.Nk, key_row, ks, vs, krow, mrow, lrow, o);
  const int r = threadIdx.x >> 2, qq = threadIdx.x & 3;
  const long long row = r0 + r;
  if (row < m.Nq) {
    const float inv = 1.0f / lrow;
#pragma unroll
    for (int k = 0; k < D / 4; ++k) {
      const int t = qq * (D / 4) + k;
      if (t < d) store_from_float(Out, ((long long)h * m.Nq + row) * d + t, o[k] * inv, m.dtype);
    }
  }
}

template <class F>
sparsepr_status with_d(int d, F f) {
  if (d <= 32) return f(std::integral_constant<int, 32>());
  if (d <= 64) return f(std::integral_constant<int, 64>());
  return f(std::integral_constant<int, 128>());
}

}  // namespace

sparsepr_status launch_sparse_attention_simt(const Plan& p, cudaStream_t st) {
  return with_d(p.dm.d, [&](auto DD) -> sparsepr_status {
    constexpr int D = decltype(DD)::value;
    const size_t smem = 2 * kKeys * D * sizeof(float) + (2 * kMaxC + 2) * sizeof(int);
    SPR_CUDA_OK(cudaFuncSetAttribute(sparse_simt_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    sparse_simt_kernel<D><<<dim3(p.dm.Cq, p.dm.H), kThreads, smem, st>>>(p.dm, p.b);
    SPR_LAUNCH_OK();
    return SPARSEPR_OK;
  });
}

sparsepr_status launch_probe_attention_simt(const Plan& p, cudaStream_t st) {
  const Dims& m = p.dm;
  return with_d(m.d, [&](auto DD) -> sparsepr_status {
    constexpr int D = decltype(DD)::value;
    const size_t smem = 2 * kKeys * D * sizeof(float);
    SPR_CUDA_OK(cudaFuncSetAttribute(probe_simt_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    probe_simt_kernel<D><<<dim3(m.nsplit, cdiv(m.M, kRows), m.H), kThreads, smem, st>>>(m, p.b, p.Q, p.K, p.V);
    SPR_LAUNCH_OK();
    return SPARSEPR_OK;
  });
}

sparsepr_status launch_probe_combine(const Plan& p, cudaStream_t st) {
  probe_combine_kernel<<<dim3(p.dm.M, p.dm.H), kMaxD, 0, st>>>(p.dm, p.b);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

sparsepr_status launch_dense_attention_simt(const Dims& m, const void* Q, const void* K,
                                            const void* V, void* Out, cudaStream_t st) {
  return with_d(m.d, [&](auto DD) -> sparsepr_status {
    constexpr int D = decltype(DD)::value;
    const size_t smem = 2 * kKeys * D * sizeof(float);
    SPR_CUDA_OK(cudaFuncSetAttribute(dense_simt_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    dense_simt_kernel<D><<<dim3(cdiv(m.Nq, kRows), m.H), kThreads, smem, st>>>(m, Q, K, V, Out);
    SPR_LAUNCH_OK();
    return SPARSEPR_OK;
  });
}

// Engine choice: the tensor-core engine for bf16 with d in {64, 128} unless the CUDA-core
// engine is requested; the CUDA-core engine for everything else.
sparsepr_status launch_sparse_attention(const Plan& p, cudaStream_t st) {
  if (tc_engine_applies(p.dm.dtype, p.dm.d, p.dm.engine)) return launch_sparse_attention_tc(p, st);
  return launch_sparse_attention_simt(p, st);
}

sparsepr_status launch_probe_attention(const Plan& p, cudaStream_t st) {
  sparsepr_status s = tc_engine_applies(p.dm.dtype, p.dm.d, p.dm.engine)
                          ? launch_probe_attention_tc(p, st)
                          : launch_probe_attention_simt(p, st);
  if (s != SPARSEPR_OK) return s;
  return launch_probe_combine(p, st);
}

sparsepr_status launch_dense_attention(const Dims& m, const void* Q, const void* K, const void* V,
                                       void* Out, cudaStream_t st) {
  if (tc_engine_applies(m.dtype, m.d, m.engine)) return launch_dense_attention_tc(m, Q, K, V, Out, nullptr, st);
  return launch_dense_attention_simt(m, Q, K, V, Out, st);
}

}  // namespace spr
