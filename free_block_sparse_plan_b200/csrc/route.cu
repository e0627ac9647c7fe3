// Routing, group-major permutation and probe selection.
//   Routing (paper App. B.3, S4.3): a score per (query group, K/V group) cell from the
//   query, key and value centroids; each query group keeps the shortest prefix of K/V
//   groups ranked by decreasing score whose key-token count reaches the common budget
//   beta = (rho* - M/N_q) N_k.  The score is a reading of the SVG-EAR value error score
//   the paper names: the centroid estimate of the hard-drop residual (App. A.1) of
//   omitting group b alone, l_ab = tau qbar_a.kbar_b + ln|G_b|, pi_ab = softmax_b(l_ab),
//   ohat_a^(-b) = sum_{c != b} pi_ac vbar_c / (1 - pi_ab),
//   score_ab = pi_ab ||vbar_b - ohat_a^(-b)||, in fp64.
//   Permutation (review page step 3): Q, K, V copied into group-major order.
//   Probes (App. A.2, Algorithm A.1): stratified radial round robin.
#include <cmath>

#include "common.cuh"

namespace spr {
namespace {

// Routing score of every (query group a, K/V group b) cell, fp64.  For b other than the
// largest-mass group, vbar_b - ohat^(-b) = (vbar_b - ohat) / (1 - pi_b) exactly, with
// 1 - pi_b >= 1/2; for the largest-mass group ohat^(-b) is formed from the others.
// A block scores kScoreQ query groups, so every K/V centroid row it streams through
// shared memory (32 rows at a time, rows padded to d + 1 doubles so the 32 rows read by a
// warp fall in distinct banks) serves all of them: logits, then per query group the two
// softmax weightings, then the value mixtures, then the distances.
constexpr int kScoreQ = 8;          // query groups per block (one warp each in phase 2)
constexpr int kScoreK = 32;         // centroid rows per shared-memory chunk
__global__ void __launch_bounds__(256) score_kernel(Dims m, Buffers b) {
  extern __shared__ double ssm[];
  __shared__ double sZ[kScoreQ], sZr[kScoreQ];
  __shared__ int sTop[kScoreQ];
  const int h = blockIdx.y, a0 = blockIdx.x * kScoreQ, d = m.d, ld = d + 1;
  const int nq = b.nQ[h];
  if (a0 >= nq) return;
  const int na = min(kScoreQ, nq - a0);
  const int hk = h / m.G;                 // the K/V head of this query head
  const int n = b.nK[hk];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  double* out0 = b.scores + ((long long)h * m.Cq + a0) * m.Ck;
  if (n == 1) {
    if (tid < na) out0[(long long)tid * m.Ck] = 0.0;
    return;
  }
  double* qa = ssm;                       // [kScoreQ][ld] qbar, later ohat
  double* orr = qa + kScoreQ * ld;        // [kScoreQ][ld] ohat over the others
  double* kv = orr + kScoreQ * ld;        // [kScoreK][ld] chunk of kbar or vbar rows
  double* zz = kv + kScoreK * ld;         // [kScoreQ][n] logits, then exp(l - max)
  double* zr = zz + kScoreQ * n;          // [kScoreQ][n] exp(l - second max), 0 at the top
  const double tau = 1.0 / sqrt((double)d);
  const double* kb = b.kbar + (long long)hk * m.Ck * d;
  const double* vb = b.vbar + (long long)hk * m.Ck * d;
  const int* sz = b.sizeK + (long long)hk * m.Ck;
  for (int e = tid; e < kScoreQ * d; e += blockDim.x) {
    const int a = e / d, j = e % d;
    qa[a * ld + j] = a < na ? b.qbar[((long long)h * m.Cq + a0 + a) * d + j] : 0.0;
  }
  // chunks of kScoreK centroid rows go through registers into shared memory; the next
  // chunk's loads are issued before the current chunk is used, so their latency overlaps
  // the arithmetic
  constexpr int kStage = kScoreK * kMaxD / 256;      // elements per thread (blockDim 256)
  double pre[kStage];
  auto fetch = [&](const double* src, int k0) {
#pragma unroll
    for (int i = 0; i < kStage; ++i) {
      const int e = tid + 256 * i;
      const int kk = e / d, j = e % d;
      pre[i] = (e < kScoreK * d && k0 + kk < n) ? src[(long long)(k0 + kk) * d + j] : 0.0;
    }
  };
  auto put = [&]() {
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kStage; ++i) {
      const int e = tid + 256 * i;
      if (e < kScoreK * d) kv[(e / d) * ld + e % d] = pre[i];
    }
    __syncthreads();
  };
  const int ta = tid >> 5, tk = tid & 31;   // phases 1 and 4: thread = (query group, row)
  // ---- phase 1: logits l_ab = tau qbar_a . kbar_b + ln |G_b|
  fetch(kb, 0);
  for (int k0 = 0; k0 < n; k0 += kScoreK) {
    put();
    if (k0 + kScoreK < n) fetch(kb, k0 + kScoreK);
    const int k = k0 + tk;
    if (ta < na && k < n) {
      // four independent partial sums (d is a multiple of 8): a quarter of the latency
      double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
      for (int j = 0; j < d; j += 4) {
        s0 = fma(qa[ta * ld + j], kv[tk * ld + j], s0);
        s1 = fma(qa[ta * ld + j + 1], kv[tk * ld + j + 1], s1);
        s2 = fma(qa[ta * ld + j + 2], kv[tk * ld + j + 2], s2);
        s3 = fma(qa[ta * ld + j + 3], kv[tk * ld + j + 3], s3);
      }
      zz[ta * n + k] = tau * ((s0 + s1) + (s2 + s3)) + log((double)sz[k]);
    }
  }
  __syncthreads();
  // ---- phase 2 (warp a): largest logit (first index), largest among the others, weights
  if (warp < na) {
    double* la = zz + warp * n;
    double* ra = zr + warp * n;
    double mx = -INFINITY;
    int top = 0x7fffffff;
    for (int k = lane; k < n; k += 32)
      if (la[k] > mx || (la[k] == mx && k < top)) { mx = la[k]; top = k; }
    for (int o = 16; o > 0; o >>= 1) {
      const double om = __shfl_xor_sync(0xffffffffu, mx, o);
      const int oi = __shfl_xor_sync(0xffffffffu, top, o);
      if (om > mx || (om == mx && oi < top)) { mx = om; top = oi; }
    }
    double m2 = -INFINITY;
    for (int k = lane; k < n; k += 32)
      if (k != top) m2 = fmax(m2, la[k]);
    for (int o = 16; o > 0; o >>= 1) m2 = fmax(m2, __shfl_xor_sync(0xffffffffu, m2, o));
    double pz = 0.0, pr = 0.0;
    for (int k = lane; k < n; k += 32) {
      const double l = la[k];
      const double e1 = exp(l - mx), e2 = (k == top) ? 0.0 : exp(l - m2);
      la[k] = e1;
      ra[k] = e2;
      pz += e1;
      pr += e2;
    }
    pz = warp_sum(pz);
    pr = warp_sum(pr);
    if (lane == 0) {
      sZ[warp] = pz;
      sZr[warp] = pr;
      sTop[warp] = top;
    }
  }
  // ---- phase 3: ohat_a = sum_b zz_ab vbar_b / Z_a, and over b != top with zr
  constexpr int kJ = kMaxD / 32;
  double acc_h[kJ], acc_r[kJ];
#pragma unroll
  for (int i = 0; i < kJ; ++i) acc_h[i] = acc_r[i] = 0.0;
  fetch(vb, 0);
  for (int k0 = 0; k0 < n; k0 += kScoreK) {
    put();
    if (k0 + kScoreK < n) fetch(vb, k0 + kScoreK);
    if (ta < na) {
      const int kn = min(kScoreK, n - k0);
      for (int kk = 0; kk < kn; ++kk) {
        const double w1 = zz[ta * n + k0 + kk], w2 = zr[ta * n + k0 + kk];
#pragma unroll
        for (int i = 0; i < kJ; ++i) {
          const int j = tk + 32 * i;
          if (j < d) {
            const double v = kv[kk * ld + j];
            acc_h[i] = fma(w1, v, acc_h[i]);
            acc_r[i] = fma(w2, v, acc_r[i]);
          }
        }
      }
    }
  }
  __syncthreads();
  if (ta < na) {
#pragma unroll
    for (int i = 0; i < kJ; ++i) {
      const int j = tk + 32 * i;
      if (j < d) {
        qa[ta * ld + j] = acc_h[i] / sZ[ta];
        orr[ta * ld + j] = acc_r[i] / sZr[ta];
      }
    }
  }
  // ---- phase 4: score_ab = pi_ab ||vbar_b - ohat_a^(-b)||
  fetch(vb, 0);
  for (int k0 = 0; k0 < n; k0 += kScoreK) {
    put();
    if (k0 + kScoreK < n) fetch(vb, k0 + kScoreK);
    const int k = k0 + tk;
    if (ta < na && k < n) {
      const bool istop = k == sTop[ta];
      const double* ref = istop ? orr + ta * ld : qa + ta * ld;
      double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
      for (int j = 0; j < d; j += 4) {
        const double t0 = kv[tk * ld + j] - ref[j], t1 = kv[tk * ld + j + 1] - ref[j + 1];
        const double t2 = kv[tk * ld + j + 2] - ref[j + 2], t3 = kv[tk * ld + j + 3] - ref[j + 3];
        s0 = fma(t0, t0, s0);
        s1 = fma(t1, t1, s1);
        s2 = fma(t2, t2, s2);
        s3 = fma(t3, t3, s3);
      }
      const double s = (s0 + s1) + (s2 + s3);
      const double Z = sZ[ta], z = zz[ta * n + k];
      out0[(long long)ta * m.Ck + k] = istop ? (z / Z) * sqrt(s) : z * sqrt(s) / (Z - z);
    }
  }
}

// Prefix budget selection for one query group; selected ids written ascending.
// ranks_only (calibrated budget, first pass): only the key counts of the score-ranked
// prefixes are written (rankPref); the selection pass then reads the head's budget from
// betaH.  With the prefix rule the budget is m.beta, recorded in betaH.
__global__ void __launch_bounds__(1024) select_kernel(Dims m, Buffers b, int ranks_only) {
  __shared__ double key[kMaxC];
  __shared__ int id[kMaxC];
  __shared__ int flag[kMaxC];
  __shared__ int sh[32];
  __shared__ int cut;
  const int h = blockIdx.y, a = blockIdx.x;
  if (a >= b.nQ[h]) {            // no such group: the count is defined as zero
    if (threadIdx.x == 0) b.cellCnt[(long long)h * m.Cq + a] = 0;
    return;
  }
  const int hk = h / m.G;        // the K/V head of this query head
  const int n = b.nK[hk];
  int P2 = 1;
  while (P2 < n) P2 <<= 1;
  const double* S = b.scores + ((long long)h * m.Cq + a) * m.Ck;
  for (int t = threadIdx.x; t < P2; t += blockDim.x) {
    key[t] = t < n ? S[t] : -INFINITY;
    id[t] = t < n ? t : (1 << 30) + t;
  }
  if (threadIdx.x == 0) cut = n;
  __syncthreads();
  // bitonic sort: decreasing score, ties by increasing id
  for (int k = 2; k <= P2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = threadIdx.x; t < P2; t += blockDim.x) {
        const int u = t ^ j;
        if (u > t) {
          const bool up = (t & k) == 0;
          const bool t_first = key[t] > key[u] || (key[t] == key[u] && id[t] < id[u]);
          if (t_first != up) {
            const double kk = key[t]; key[t] = key[u]; key[u] = kk;
            const int ii = id[t]; id[t] = id[u]; id[u] = ii;
          }
        }
      }
      __syncthreads();
    }
  }
  const int* sz = b.sizeK + (long long)hk * m.Ck;
  const int t = threadIdx.x;
  const int mine = t < n ? sz[id[t]] : 0;
  int tot;
  const int excl = block_exclusive_scan(mine, sh, &tot);
  const long long incl = (long long)excl + mine;
  if (ranks_only) {
    if (t < n) b.rankPref[((long long)h * m.Cq + a) * m.Ck + t] = (int)incl;
    return;
  }
  const double beta = m.budget == SPARSEPR_BUDGET_CALIBRATED ? b.betaH[h] : m.beta;
  if (m.budget != SPARSEPR_BUDGET_CALIBRATED && a == 0 && t == 0) b.betaH[h] = m.beta;
  if (t < n && (double)incl >= beta && (t == 0 || (double)excl < beta)) cut = t + 1;
  __syncthreads();
  const int cnt = cut;
  for (int u = threadIdx.x; u < n; u += blockDim.x) flag[u] = 0;
  __syncthreads();
  if (t < cnt) flag[id[t]] = 1;
  __syncthreads();
  const int f = t < n ? flag[t] : 0;
  const int pos = block_exclusive_scan(f, sh, &tot);
  int* ids = b.cellIds + ((long long)h * m.Cq + a) * m.Ck;
  if (f) ids[pos] = t;
  // routed pairs: |G_a| * (selected key tokens)
  long long keys = 0;
  if (t < n && flag[t]) keys = sz[t];
  for (int o = 16; o > 0; o >>= 1) keys += __shfl_xor_sync(0xffffffffu, keys, o);
  if ((t & 31) == 0 && keys)
    atomicAdd(reinterpret_cast<unsigned long long*>(b.pairs + h),
              (unsigned long long)(keys * (long long)b.sizeQ[(long long)h * m.Cq + a]));
  if (t == 0) b.cellCnt[(long long)h * m.Cq + a] = cnt;
}

// Routed pairs of head h under the common integer budget beta: every query group keeps
// the shortest score-ranked prefix whose key count reaches beta (its last prefix holds
// every key, N_k >= beta).  Block-wide sum, returned to every thread.
__device__ long long pairs_at(const Dims& m, const Buffers& b, int h, int beta, long long* red) {
  const int n = b.nK[h / m.G], nq = b.nQ[h];
  long long acc = 0;
  for (int a = threadIdx.x; a < nq; a += blockDim.x) {
    const int* pref = b.rankPref + ((long long)h * m.Cq + a) * m.Ck;
    int lo = 0, hi = n - 1;                       // first prefix with count >= beta
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (pref[mid] >= beta) hi = mid; else lo = mid + 1;
    }
    acc += (long long)b.sizeQ[(long long)h * m.Cq + a] * pref[lo];
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  long long s = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];   // fixed order: deterministic
  return s;
}

// Calibrated budget (App. D.2, calibrated toward the target): routed pairs never
// decrease in beta, so a bisection over integer beta in [1, N_k] finds the smallest beta
// reaching T = rho* N_q N_k - M N_k; of its selection and that of beta - 1 (the last below
// T) the one nearer T is kept, the denser on a tie, and reported by the smallest beta that
// gives it (a second bisection when it is the one below).  One block per head.
__global__ void __launch_bounds__(256) calibrate_kernel(Dims m, Buffers b) {
  __shared__ long long red[8];
  const int h = blockIdx.x;
  const double T = m.rho * (double)m.Nq * (double)m.Nk - (double)m.M * (double)m.Nk;
  int lo = 1, hi = m.Nk;
  long long plo = pairs_at(m, b, h, lo, red), phi = -1;
  int beta = 1;
  if ((double)plo < T) {
    phi = pairs_at(m, b, h, hi, red);             // every key: reaches T since rho* <= 1
    while (hi - lo > 1) {                          // invariant: pairs(lo) < T <= pairs(hi)
      const int mid = lo + (hi - lo) / 2;
      const long long pm = pairs_at(m, b, h, mid, red);
      if ((double)pm >= T) { hi = mid; phi = pm; } else { lo = mid; plo = pm; }
    }
    beta = hi;                                     // the smallest beta of its selection
    if (T - (double)plo < (double)phi - T) {
      // the selection below T: the smallest beta that gives it (pairs(beta) >= pairs(lo))
      int l2 = 0, h2 = lo;                         // pairs(l2) < plo <= pairs(h2); pairs(0) := -1
      while (h2 - l2 > 1) {
        const int mid = l2 + (h2 - l2) / 2;
        if (pairs_at(m, b, h, mid, red) >= plo) h2 = mid; else l2 = mid;
      }
      beta = h2;
    }
  }
  if (threadIdx.x == 0) b.betaH[h] = (double)beta;
}

// Group-major copies of Q, K, V with 16-byte vector loads; inverse query permutation.
__global__ void gather_kernel(const void* src, void* dst, const int* perm, int* inv, int H, int N,
                              int row_chunks) {
  const long long total = (long long)H * N * row_chunks;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const long long row = t / row_chunks;          // h * N + pos
    const int c = (int)(t % row_chunks);
    const long long h = row / N;
    const int srow = perm[row];
    const uint4* s = reinterpret_cast<const uint4*>(src) + (h * N + srow) * row_chunks + c;
    uint4* o = reinterpret_cast<uint4*>(dst) + row * row_chunks + c;
    *o = __ldg(s);
    if (inv && c == 0) inv[h * N + srow] = (int)(row - h * N);
  }
}

// Padded row offsets of the K/V groups in the tensor-core layout: each group's rows rounded
// up to a multiple of 8, in raw-label order; entry C_k is where the 128 zero rows start.
__global__ void __launch_bounds__(1024) kv_pad_offsets_kernel(Dims m, Buffers b) {
  __shared__ int sh[32];
  const long long o = (long long)blockIdx.x * (m.Ck + 1);
  const int lab = threadIdx.x;
  const int sz = lab < m.Ck ? b.offK[o + lab + 1] - b.offK[o + lab] : 0;
  int tot;
  const int ex = block_exclusive_scan((sz + 7) & ~7, sh, &tot);
  if (lab < m.Ck) b.poffK[o + lab] = ex;
  if (lab == 0) b.poffK[o + m.Ck] = tot;
}

// K and V rows into the tensor-core layout (kv_tiled_rows): group-major position `pos` of
// K/V head hk goes to panel row poffK[label] + (pos - offK[label]), each 16-byte chunk at
// its swizzled place.
__global__ void kv_tiled_kernel(Dims m, Buffers b, const uint4* K, const uint4* V, uint4* Kt, uint4* Vt) {
  const int chunks = m.d / 8, np = m.d / 64;
  const long long rp = kv_tiled_rows(m.Nk, m.Ck);
  const long long total = (long long)m.Hk * m.Nk * chunks;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const long long row = t / chunks;                  // hk * N_k + pos
    const int c = (int)(t % chunks);
    const int hk = (int)(row / m.Nk), pos = (int)(row - (long long)hk * m.Nk);
    const int srow = b.permK[row];
    const int lab = b.labK[(long long)hk * m.Nk + srow];
    const long long o = (long long)hk * (m.Ck + 1) + lab;
    const long long prow = b.poffK[o] + (pos - b.offK[o]);
    const long long src = ((long long)hk * m.Nk + srow) * chunks + c;
    const long long dst = (((long long)hk * np + (c >> 3)) * rp + prow) * 8 + ((c & 7) ^ (int)(prow & 7));
    Kt[dst] = __ldg(K + src);
    Vt[dst] = __ldg(V + src);
  }
}

// Zero rows of the tensor-core layout: the padding after each group (block x < C_k) and the
// 128 rows after the last group (block x = C_k), for every panel of K/V head blockIdx.y.
__global__ void kv_tiled_zero_kernel(Dims m, Buffers b, uint4* Kt, uint4* Vt) {
  const int hk = blockIdx.y, lab = blockIdx.x, np = m.d / 64;
  const long long rp = kv_tiled_rows(m.Nk, m.Ck);
  const long long o = (long long)hk * (m.Ck + 1) + lab;
  long long r0, r1;
  if (lab < m.Ck) {
    r0 = b.poffK[o] + (b.offK[o + 1] - b.offK[o]);
    r1 = b.poffK[o + 1];
  } else {
    r0 = b.poffK[o];
    r1 = r0 + 128;
  }
  const int n = (int)(r1 - r0) * np * 8;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int pnl = e / ((int)(r1 - r0) * 8), rem = e % ((int)(r1 - r0) * 8);
    const long long dst = (((long long)hk * np + pnl) * rp + r0) * 8 + rem;
    Kt[dst] = z;
    Vt[dst] = z;
  }
}

// Squared distance of each query's phi_Q to its group centre (fp64, ascending dims).
__global__ void probe_dist_kernel(Dims m, Buffers b) {
  const int h = blockIdx.y;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= m.Nq) return;
  const int lab = b.labQ[(long long)h * m.Nq + i];
  const double* x = b.phiQ + ((long long)h * m.Nq + i) * m.rQ;
  const double* c = b.centQ + ((long long)h * m.Cq + lab) * m.rQ;
  double s = 0.0;
  for (int k = 0; k < m.rQ; ++k) {
    const double t = x[k] - c[k];
    s = fma(t, t, s);
  }
  b.dist[(long long)h * m.Nq + i] = s;
}

// Passes P of the round robin: smallest p with sum_a min(|G_a|, p) >= M.
__device__ int probe_passes(const int* sz, int n, int M) {
  int p = 1;
  for (;; ++p) {
    long long c = 0;
    for (int a = 0; a < n; ++a) c += sz[a] < p ? sz[a] : p;
    if (c >= M || p >= M) return p;
  }
}

// Per query group: its first min(P, |G_a|) rows by (d_i, row) ascending. One warp.
__global__ void __launch_bounds__(32) probe_rank_kernel(Dims m, Buffers b) {
  const int h = blockIdx.y, a = blockIdx.x, lane = threadIdx.x;
  const int n = b.nQ[h];
  if (a >= n) return;
  const int* sz = b.sizeQ + (long long)h * m.Cq;
  const int P = probe_passes(sz, n, m.M);
  const int lab = b.usedQ[(long long)h * m.Cq + a];
  const int m0 = b.offQ[(long long)h * (m.Cq + 1) + lab], m1 = b.offQ[(long long)h * (m.Cq + 1) + lab + 1];
  const int take = (m1 - m0) < P ? (m1 - m0) : P;
  const int* perm = b.permQ + (long long)h * m.Nq;
  const double* dist = b.dist + (long long)h * m.Nq;
  double pd = -INFINITY;
  int pi = -1;
  for (int t = 0; t < take; ++t) {
    double bd = INFINITY;
    int bi = 0x7fffffff;
    for (int mm = m0 + lane; mm < m1; mm += 32) {
      const int row = perm[mm];
      const double dv = dist[row];
      const bool after = dv > pd || (dv == pd && row > pi);
      const bool better = dv < bd || (dv == bd && row < bi);
      if (after && better) {
        bd = dv;
        bi = row;
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      const double od = __shfl_xor_sync(0xffffffffu, bd, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (od < bd || (od == bd && oi < bi)) {
        bd = od;
        bi = oi;
      }
    }
    if (lane == 0) b.probeTop[((long long)h * m.Cq + a) * m.M + t] = bi;
    pd = bd;
    pi = bi;
  }
}

// Round robin over groups by decreasing size (ties by index); weights w_p = |G_a|/m_a.
__global__ void __launch_bounds__(1024) probe_pick_kernel(Dims m, Buffers b) {
  __shared__ int ord[kMaxC];
  __shared__ int ksz[kMaxC];
  __shared__ int cnt[kMaxC];
  const int h = blockIdx.x, n = b.nQ[h];
  const int* sz = b.sizeQ + (long long)h * m.Cq;
  int P2 = 1;
  while (P2 < n) P2 <<= 1;
  for (int t = threadIdx.x; t < P2; t += blockDim.x) {
    ord[t] = t;
    ksz[t] = t < n ? sz[t] : -1;
  }
  for (int t = threadIdx.x; t < m.Cq; t += blockDim.x) cnt[t] = 0;
  __syncthreads();
  for (int k = 2; k <= P2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = threadIdx.x; t < P2; t += blockDim.x) {
        const int u = t ^ j;
        if (u > t) {
          const bool up = (t & k) == 0;
          const bool t_first = ksz[t] > ksz[u] || (ksz[t] == ksz[u] && ord[t] < ord[u]);
          if (t_first != up) {
            int x = ksz[t]; ksz[t] = ksz[u]; ksz[u] = x;
            x = ord[t]; ord[t] = ord[u]; ord[u] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  if (threadIdx.x == 0) {
    const int P = probe_passes(sz, n, m.M);
    int taken = 0;
    for (int t = 0; t < P && taken < m.M; ++t) {
      for (int k = 0; k < n && taken < m.M; ++k) {
        const int a = ord[k];
        if (sz[a] > t) {
          b.probes[(long long)h * m.M + taken] = b.probeTop[((long long)h * m.Cq + a) * m.M + t];
          b.probeA[(long long)h * m.M + taken] = a;
          cnt[a] += 1;
          ++taken;
        }
      }
    }
    if (taken < m.M) atomicOr(b.err, kErrProbe);
  }
  __syncthreads();
  for (int a = threadIdx.x; a < m.Cq; a += blockDim.x) b.mA[(long long)h * m.Cq + a] = cnt[a];
  for (int p = threadIdx.x; p < m.M; p += blockDim.x) {
    const int a = b.probeA[(long long)h * m.M + p];
    b.wP[(long long)h * m.M + p] = (double)sz[a] / (double)cnt[a];
  }
}

}  // namespace

sparsepr_status launch_route(const Plan& p, cudaStream_t st) {
  const Dims& m = p.dm;
  const size_t ssmem = (size_t)((2 * kScoreQ + kScoreK) * (m.d + 1) + 2 * kScoreQ * m.Ck) * sizeof(double);
  SPR_CUDA_OK(cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssmem));
  score_kernel<<<dim3(cdiv(m.Cq, kScoreQ), m.H), 256, ssmem, st>>>(m, p.b);
  SPR_LAUNCH_OK();
  if (m.budget == SPARSEPR_BUDGET_CALIBRATED) {
    select_kernel<<<dim3(m.Cq, m.H), 1024, 0, st>>>(m, p.b, 1);
    SPR_LAUNCH_OK();
    calibrate_kernel<<<m.H, 256, 0, st>>>(m, p.b);
    SPR_LAUNCH_OK();
  }
  select_kernel<<<dim3(m.Cq, m.H), 1024, 0, st>>>(m, p.b, 0);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

sparsepr_status launch_permute(const Plan& p, cudaStream_t st) {
  const Dims& m = p.dm;
  const int es = m.dtype == SPARSEPR_BF16 ? 2 : 4;
  const int chunks = m.d * es / 16;
  const int blocks = 148 * 8;
  gather_kernel<<<blocks, 256, 0, st>>>(p.Q, p.b.Qp, p.b.permQ, p.b.invQ, m.H, m.Nq, chunks);
  SPR_LAUNCH_OK();
  if (tc_engine_applies(m.dtype, m.d, m.engine)) {
    kv_pad_offsets_kernel<<<m.Hk, 1024, 0, st>>>(m, p.b);
    SPR_LAUNCH_OK();
    kv_tiled_kernel<<<blocks, 256, 0, st>>>(m, p.b, static_cast<const uint4*>(p.K), static_cast<const uint4*>(p.V),
                                            static_cast<uint4*>(p.b.Kp), static_cast<uint4*>(p.b.Vp));
    SPR_LAUNCH_OK();
    kv_tiled_zero_kernel<<<dim3(m.Ck + 1, m.Hk), 128, 0, st>>>(m, p.b, static_cast<uint4*>(p.b.Kp),
                                                                static_cast<uint4*>(p.b.Vp));
    SPR_LAUNCH_OK();
    return SPARSEPR_OK;
  }
  gather_kernel<<<blocks, 256, 0, st>>>(p.K, p.b.Kp, p.b.permK, nullptr, m.Hk, m.Nk, chunks);
  SPR_LAUNCH_OK();
  gather_kernel<<<blocks, 256, 0, st>>>(p.V, p.b.Vp, p.b.permK, nullptr, m.Hk, m.Nk, chunks);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

sparsepr_status launch_select_probes(const Plan& p, cudaStream_t st) {
  const Dims& m = p.dm;
  probe_dist_kernel<<<dim3(cdiv(m.Nq, 256), m.H), 256, 0, st>>>(m, p.b);
  SPR_LAUNCH_OK();
  probe_rank_kernel<<<dim3(m.Cq, m.H), 32, 0, st>>>(m, p.b);
  SPR_LAUNCH_OK();
  probe_pick_kernel<<<m.H, 1024, 0, st>>>(m, p.b);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

}  // namespace spr
