// Response-Coupled Partitioning on the GPU (paper S4.1, App. B.1-B.2, App. C):
// key / query response coordinates, batched Lloyd k-means, and the groups it yields.
//
// k-means is batched over heads; every head stops on its own as soon as an assignment
// step changes no label (or after kmeans_max_iter steps), tracked by device flags so
// the host never synchronises.  Centre updates are deterministic: the labels are
// stably counting-sorted (this order is also the group-major order the attention
// uses) and each cluster's members are summed in that fixed order in fp64.
#include "common.cuh"

namespace spr {
namespace {

// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): output n of the generator whose state
// starts at `key` is mix(key + n * gamma).
__device__ __forceinline__ unsigned long long sm64_mix(unsigned long long z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}
constexpr unsigned long long kGamma = 0x9E3779B97F4A7C15ULL;

struct KmView {         // one k-means instance (keys or queries) for all heads
  const double* X;      // [H][N][r] features (fp64)
  double* cent;         // [H][C][r] centres (fp64)
  int* lab;             // [H][N]
  int* hist;            // [H][C][nch]
  int* perm;            // [H][N]
  int* off;             // [H][C+1]
  int* km;              // [H][4]: done, changed[0], changed[1], iterations
  double* obj;          // [H][C]
  double* delta;        // [H][C] centre movement of each update, or null
  unsigned long long* dmax;   // [2][H][G] largest movement per 32-centre group (double bits)
  int N, C, r, nch, stage;
  int H;                // instances: query heads, or K/V heads for the key side
  unsigned long long* fx;     // [H][C][64][3] exact member sums (three 40-bit limbs)
  int* fxcnt;                 // [H][C] member counts
  unsigned long long* chg;    // [H][N] last label change of each point (chg_entry)
};

KmView view(const Plan& p, bool query) {
  const Buffers& b = p.b;
  const Dims& m = p.dm;
  if (query)
    return {b.phiQ, b.centQ, b.labQ, b.histQ, b.permQ, b.offQ, b.kmQ, b.objQ, b.kmDelta, b.kmDmax,
            m.Nq, m.Cq, m.rQ, m.nchQ, 1, m.H, b.kmFx, b.kmFxCnt, b.kmChg};
  return {b.phiK, b.centK, b.labK, b.histK, b.permK, b.offK, b.kmK, b.objK, b.kmDelta, b.kmDmax,
          m.Nk, m.Ck, m.rK, m.nchK, 0, m.Hk, b.kmFx, b.kmFxCnt, b.kmChg};
}

// ---------------------------------------------------------------------------------
// Response coordinates in fp64: phi = X F (keys), phi = z / max(rms(z), 1e-6) with
// z = X F (queries) (paper S4.1, App. B.1-B.2).  X is exact in its dtype; F is the fp64
// factor; each coordinate is one fp64 dot product over d in ascending order.
// A block takes 256 rows in four tiles of 64: F is staged once per block, each X tile
// transposed (column j of the tile contiguous, 16-byte loads, one row per lane); thread
// (tr, tc) forms rows 4tr..4tr+3 x columns tc, tc+16, ... (a register
// tile, so every shared-memory value feeds several fp64 FMAs and the 16 column threads
// of a row group read 16 consecutive F values).  When the tensor-core k-means will
// cluster these coordinates, the block also writes its input: each row split into two
// bf16 pieces (rows padded to 64 columns, zero rows up to Npad) and |phi|.
constexpr int kProjRows = 64;
constexpr int kProjTiles = 4;              // 64-row tiles per block
constexpr int kProjXs = kProjRows + 4;     // transposed tile row stride (floats)
template <int R, bool RMS>
__global__ void __launch_bounds__(256) project_kernel(Dims m, const void* X, int N, const double* Fall, int r,
                                                      double* out, __nv_bfloat16* xhi, __nv_bfloat16* xlo,
                                                      float* xn, int Npad, int fdiv) {
  constexpr int CPT = R / 16;              // columns per thread
  extern __shared__ double smd[];
  const int d = m.d, h = blockIdx.y;
  double* F = smd;                         // [d][R], zero columns k >= r
  float* Xt = reinterpret_cast<float*>(smd + d * R);  // [d][kProjXs]: Xt[j][row]
  const double* Fh = Fall + (long long)(h / fdiv) * d * r;   // queries: their K/V head's F_Q
  for (int e = threadIdx.x; e < d * R; e += blockDim.x) {
    const int j = e / R, k = e % R;
    F[e] = k < r ? Fh[j * r + k] : 0.0;
  }
  const long long base = ((long long)h * N) * d;
  const int tr = threadIdx.x >> 4, tc = threadIdx.x & 15;
  for (int tile = 0; tile < kProjTiles; ++tile) {
  const long long row0 = ((long long)blockIdx.x * kProjTiles + tile) * kProjRows;
  if (row0 >= (xhi ? Npad : N)) break;
  __syncthreads();                         // the previous tile's reads of Xt are done
  // one row per lane, 16 bytes per load: consecutive lanes write consecutive banks
  const int per = m.dtype == SPARSEPR_BF16 ? 8 : 4;        // elements per 16-byte load
  const bool vec = (reinterpret_cast<uintptr_t>(X) & 15) == 0;
  for (int e = threadIdx.x; e < kProjRows * (d / per); e += blockDim.x) {
    const int i = e % kProjRows, c = e / kProjRows;
    const long long row = row0 + i;
    float v[8];
    if (row < N && !vec) {
      for (int q = 0; q < per; ++q) v[q] = load_as_float(X, base + row * d + c * per + q, m.dtype);
    } else if (row < N) {
      if (m.dtype == SPARSEPR_BF16) {
        const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(X) + base + row * d + c * 8);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          v[2 * q] = __uint_as_float(w[q] << 16);
          v[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
        }
      } else {
        const float4 f = *reinterpret_cast<const float4*>(static_cast<const float*>(X) + base + row * d + c * 4);
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = 0.0f;
    }
    for (int q = 0; q < per; ++q) Xt[(c * per + q) * kProjXs + i] = v[q];
  }
  __syncthreads();
  double acc[4][CPT];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[a][c] = 0.0;
  for (int j = 0; j < d; ++j) {
    const float4 x4 = *reinterpret_cast<const float4*>(Xt + j * kProjXs + 4 * tr);
    const double xv[4] = {(double)x4.x, (double)x4.y, (double)x4.z, (double)x4.w};
    double fv[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) fv[c] = F[j * R + tc + 16 * c];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < CPT; ++c) acc[a][c] = fma(xv[a], fv[c], acc[a][c]);
  }
  // the 16 column threads of a row group are one half-warp: row sums by shuffles
  auto row_sum = [](double v) {
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
  };
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const long long row = row0 + 4 * tr + a;
    if (RMS) {
      double ss = 0.0;
#pragma unroll
      for (int c = 0; c < CPT; ++c) ss = fma(acc[a][c], acc[a][c], ss);
      ss = row_sum(ss);
      const double scale = 1.0 / fmax(sqrt(ss / (double)r), 1e-6);
#pragma unroll
      for (int c = 0; c < CPT; ++c) acc[a][c] *= scale;
    }
    if (row < N) {
      double* o = out + ((long long)h * N + row) * r;
#pragma unroll
      for (int c = 0; c < CPT; ++c)
        if (tc + 16 * c < r) o[tc + 16 * c] = acc[a][c];
    }
    if (xhi) {
      double ss = 0.0;
#pragma unroll
      for (int c = 0; c < CPT; ++c) ss = fma(acc[a][c], acc[a][c], ss);
      ss = row_sum(ss);
      if (row < Npad) {
        const long long xb = ((long long)h * Npad + row) * 64;
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
          const double v = row < N ? acc[a][c] : 0.0;
          const __nv_bfloat16 hi = __double2bfloat16(v);
          xhi[xb + tc + 16 * c] = hi;
          xlo[xb + tc + 16 * c] = __double2bfloat16(v - (double)__bfloat162float(hi));
        }
        for (int cz = R + tc; cz < 64; cz += 16) {
          xhi[xb + cz] = __float2bfloat16_rn(0.0f);
          xlo[xb + cz] = __float2bfloat16_rn(0.0f);
        }
        if (tc == 0 && row < N) xn[(long long)h * N + row] = (float)sqrt(ss);
      }
    }
  }
  }
}

// query: one block row per query head, each reading its K/V head's factor (fdiv = G);
// keys: one per K/V head.  RMS: the query coordinates' normalisation (not in the semantic
// partition, whose coordinates are the raw rows).
template <bool RMS>
sparsepr_status launch_project(const Plan& p, bool query, const void* X, int N, const double* F, int r,
                               double* out, __nv_bfloat16* xhi, __nv_bfloat16* xlo, float* xn, int Npad,
                               cudaStream_t st) {
  const int d = p.dm.d;
  const int rows = xhi ? Npad : N;
  const int fdiv = query ? p.dm.G : 1;
  dim3 grid(cdiv(rows, kProjRows * kProjTiles), query ? p.dm.H : p.dm.Hk);
  auto run = [&](auto kern, int R) -> sparsepr_status {
    const size_t smem = (size_t)d * R * sizeof(double) + (size_t)d * kProjXs * sizeof(float);
    SPR_CUDA_OK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    kern<<<grid, 256, smem, st>>>(p.dm, X, N, F, r, out, xhi, xlo, xn, Npad, fdiv);
    SPR_LAUNCH_OK();
    return SPARSEPR_OK;
  };
  if (r <= 16) return run(project_kernel<16, RMS>, 16);
  if (r <= 32) return run(project_kernel<32, RMS>, 32);
  if (r <= 48) return run(project_kernel<48, RMS>, 48);
  return run(project_kernel<64, RMS>, 64);
}

// ---------------------------------------------------------------------------------
// k-means initialisation: C rows drawn with replacement (paper App. C), SplitMix64
// stream (2h + stage + 1) of `seed`, index = (hi32 * N) >> 32.
__global__ void km_init_kernel(KmView v, unsigned long long seed) {
  const int h = blockIdx.x;
  const unsigned long long key = sm64_mix(seed + (unsigned long long)(2 * h + v.stage + 1) * kGamma);
  for (int e = threadIdx.x; e < v.C * v.r; e += blockDim.x) {
    const int c = e / v.r, k = e % v.r;
    const unsigned long long z = sm64_mix(key + (unsigned long long)(c + 1) * kGamma);
    const long long idx = (long long)(((z >> 32) * (unsigned long long)v.N) >> 32);
    v.cent[((long long)h * v.C + c) * v.r + k] = v.X[((long long)h * v.N + idx) * v.r + k];
  }
}

// Warm initialisation (paper App. C: later calls start from the previous centroids in
// the original space, mapped into the current response coordinates): label c starts at
// phi(cbar_c), phi(x) = x F for keys and (x F) / max(rms(x F), 1e-6) for queries, when
// label c was non-empty in the previous call; otherwise at the fresh draw c of the
// init stream.  A state that does not match the plan starts every label fresh.  One
// warp per label, lanes over the coordinates.
__global__ void __launch_bounds__(256) km_warm_init_kernel(KmView v, unsigned long long seed, Dims m,
                                                           const int* hdr, const double* cprev,
                                                           const int* used, const double* F) {
  const int h = blockIdx.y, lane = threadIdx.x & 31;
  const int c = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (c >= v.C) return;
  const int d = m.d, r = v.r;
  double* out = v.cent + ((long long)h * v.C + c) * r;
  if (state_matches(hdr, m) && used[(long long)h * v.C + c]) {
    const double* cb = cprev + ((long long)h * v.C + c) * d;
    const double* Fh = F + (long long)(v.stage == 1 ? h / m.G : h) * d * r;
    double z0 = 0.0, z1 = 0.0;
    for (int j = 0; j < d; ++j) {
      const double x = cb[j];
      if (lane < r) z0 += x * Fh[j * r + lane];
      if (lane + 32 < r) z1 += x * Fh[j * r + lane + 32];
    }
    double sc = 1.0;
    if (v.stage == 1) {
      const double rms = sqrt(warp_sum(z0 * z0 + z1 * z1) / (double)r);
      sc = 1.0 / (rms > 1e-6 ? rms : 1e-6);
    }
    if (lane < r) out[lane] = v.stage == 1 ? z0 * sc : z0;
    if (lane + 32 < r) out[lane + 32] = v.stage == 1 ? z1 * sc : z1;
  } else {
    const unsigned long long key = sm64_mix(seed + (unsigned long long)(2 * h + v.stage + 1) * kGamma);
    const unsigned long long z = sm64_mix(key + (unsigned long long)(c + 1) * kGamma);
    const long long idx = (long long)(((z >> 32) * (unsigned long long)v.N) >> 32);
    for (int k = lane; k < r; k += 32) out[k] = v.X[((long long)h * v.N + idx) * r + k];
  }
}

// The state a finished plan leaves for the next call: header, factors, and per label
// the original-space centroid (zero for an empty label) with its non-empty flag.
__global__ void __launch_bounds__(1024) save_state_kernel(Dims m, Buffers b, char* state) {
  const StateLayout L = state_layout(m);
  const int h = blockIdx.x, d = m.d;
  if (h == 0 && threadIdx.x < 16) {
    const int vals[8] = {kStateMagic, m.H, m.d, m.rK, m.rQ, m.Ck, m.Cq, 1};
    reinterpret_cast<int*>(state)[threadIdx.x] = threadIdx.x < 8 ? vals[threadIdx.x] : 0;
  }
  double* FK = reinterpret_cast<double*>(state + L.FK) + (long long)h * d * m.rK;
  double* FQ = reinterpret_cast<double*>(state + L.FQ) + (long long)h * d * m.rQ;
  for (int e = threadIdx.x; e < d * m.rK; e += blockDim.x) FK[e] = b.FK64[(long long)h * d * m.rK + e];
  for (int e = threadIdx.x; e < d * m.rQ; e += blockDim.x) FQ[e] = b.FQ64[(long long)h * d * m.rQ + e];
  for (int side = 0; side < 2; ++side) {
    const int C = side ? m.Cq : m.Ck;
    const int* comp = (side ? b.compQ : b.compK) + (long long)h * C;
    const double* bar = (side ? b.qbar : b.kbar) + (long long)h * C * d;
    double* cs = reinterpret_cast<double*>(state + (side ? L.QC : L.KC)) + (long long)h * C * d;
    int* us = reinterpret_cast<int*>(state + (side ? L.qu : L.ku)) + (long long)h * C;
    for (int e = threadIdx.x; e < C * d; e += blockDim.x) {
      const int c = e / d, j = e % d;
      const int g = comp[c];
      cs[e] = g >= 0 ? bar[(long long)g * d + j] : 0.0;
      if (j == 0) us[c] = g >= 0 ? 1 : 0;
    }
  }
}

// Assignment: label = argmin_c ||x - c||^2 (direct sum of squared differences in fp64,
// dimensions in ascending order; ties to the lowest index).
template <int R>
__global__ void __launch_bounds__(128) km_assign_kernel(KmView v, int it) {
  constexpr int TILE = 32;
  __shared__ double cs[TILE * R];
  const int h = blockIdx.y;
  int* km = v.km + 4 * h;
  if (km[0]) return;
  const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const bool valid = row < v.N;
  double x[R];
  const double* xp = v.X + ((long long)h * v.N + (valid ? row : 0)) * v.r;
#pragma unroll
  for (int k = 0; k < R; ++k) x[k] = (k < v.r) ? xp[k] : 0.0;
  double best = 1.7976931348623157e308;
  int bi = 0;
  const double* ch = v.cent + (long long)h * v.C * v.r;
  for (int c0 = 0; c0 < v.C; c0 += TILE) {
    const int nc = (v.C - c0) < TILE ? (v.C - c0) : TILE;
    __syncthreads();
    for (int e = threadIdx.x; e < nc * R; e += blockDim.x) {
      const int c = e / R, k = e % R;
      cs[e] = k < v.r ? ch[(long long)(c0 + c) * v.r + k] : 0.0;
    }
    __syncthreads();
    for (int c = 0; c < nc; ++c) {
      double dsum = 0.0;
#pragma unroll
      for (int k = 0; k < R; ++k) {
        if (k < v.r) {
          const double t = x[k] - cs[c * R + k];
          dsum = fma(t, t, dsum);
        }
      }
      if (dsum < best) {
        best = dsum;
        bi = c0 + c;
      }
    }
  }
  if (valid) {
    int* lp = v.lab + (long long)h * v.N + row;
    const int old = *lp;
    if (old != bi) {
      *lp = bi;
      km[1 + (it & 1)] = 1;
      v.chg[(long long)h * v.N + row] = chg_entry(old, bi, it);
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) km[3] += 1;
}

// Should the update of iteration `it` run?  force: always (final pass / given labels).
__device__ __forceinline__ bool km_skip(const KmView& v, int h, int it, bool force) {
  if (force) return false;
  const int* km = v.km + 4 * h;
  return km[0] || !km[1 + (it & 1)];
}

// Stable counting sort, pass 1: per-chunk label histograms hist[h][c][chunk].
__global__ void __launch_bounds__(kSortChunk) cs_hist_kernel(KmView v, int it, bool force) {
  __shared__ int hist[kMaxC];
  const int h = blockIdx.y, ch = blockIdx.x;
  if (km_skip(v, h, it, force)) return;
  for (int c = threadIdx.x; c < v.C; c += blockDim.x) hist[c] = 0;
  __syncthreads();
  const long long row = (long long)ch * kSortChunk + threadIdx.x;
  if (row < v.N) atomicAdd(&hist[v.lab[(long long)h * v.N + row]], 1);
  __syncthreads();
  int* g = v.hist + (long long)h * v.C * v.nch;
  for (int c = threadIdx.x; c < v.C; c += blockDim.x) g[(long long)c * v.nch + ch] = hist[c];
}

// Pass 2: exclusive scan of hist in (label, chunk) order; off[c] = start of label c.
__global__ void __launch_bounds__(1024) cs_scan_kernel(KmView v, int it, bool force) {
  __shared__ int sh[32];
  const int h = blockIdx.x;
  if (km_skip(v, h, it, force)) return;
  int* g = v.hist + (long long)h * v.C * v.nch;
  const long long len = (long long)v.C * v.nch;
  const long long per = (len + blockDim.x - 1) / blockDim.x;
  const long long s0 = threadIdx.x * per, s1 = (s0 + per < len) ? s0 + per : len;
  int local = 0;
  for (long long e = s0; e < s1; ++e) local += g[e];
  int total;
  int run = block_exclusive_scan(local, sh, &total);
  for (long long e = s0; e < s1; ++e) {
    const int c = g[e];
    g[e] = run;
    run += c;
  }
  __syncthreads();
  int* off = v.off + (long long)h * (v.C + 1);
  for (int c = threadIdx.x; c < v.C; c += blockDim.x) off[c] = g[(long long)c * v.nch];
  if (threadIdx.x == 0) off[v.C] = v.N;
}

// Pass 3: stable scatter; rank inside the chunk among equal labels at lower rows.
__global__ void __launch_bounds__(kSortChunk) cs_scatter_kernel(KmView v, int it, bool force) {
  constexpr int W = kSortChunk / 32;
  extern __shared__ int wcs[];            // [W][C] per-warp label counts
  const int h = blockIdx.y, ch = blockIdx.x;
  if (km_skip(v, h, it, force)) return;
  for (int e = threadIdx.x; e < W * v.C; e += blockDim.x) wcs[e] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const long long row = (long long)ch * kSortChunk + threadIdx.x;
  const int lab = row < v.N ? v.lab[(long long)h * v.N + row] : -1;
  const unsigned peers = __match_any_sync(0xffffffffu, lab);
  const int lower = __popc(peers & ((1u << lane) - 1u));
  if (lab >= 0 && lower == 0) wcs[w * v.C + lab] = __popc(peers);
  __syncthreads();
  if (lab < 0) return;
  int before = 0;
  for (int k = 0; k < w; ++k) before += wcs[k * v.C + lab];
  const int* g = v.hist + (long long)h * v.C * v.nch;
  const int pos = g[(long long)lab * v.nch + ch] + before + lower;
  v.perm[(long long)h * v.N + pos] = (int)row;
}

// Pass 4: centre = mean of members (fp64 sums in group-major order); empty clusters keep
// their centre.  The final pass (force) also forms the cluster's share of the objective
// at its new centre.  Member rows are read through the permutation, four at a time per
// thread so that several gathers are in flight.
constexpr int kMeanSub = 4;
constexpr int kMeanIdx = 1024;      // member indices staged in shared memory per round
__global__ void __launch_bounds__(kMeanSub * kMaxR) cs_mean_kernel(KmView v, int it, bool force) {
  __shared__ double part[kMeanSub][kMaxR];
  __shared__ double opart[kMeanSub * kMaxR / 32];
  __shared__ int idx[kMeanIdx];
  const int h = blockIdx.y, c = blockIdx.x;
  int* km = v.km + 4 * h;
  if (!force) {
    if (km[0]) return;
    if (!km[1 + (it & 1)]) {            // converged: this assignment changed nothing
      if (c == 0 && threadIdx.x == 0) km[0] = 1;
      return;
    }
    if (c == 0 && threadIdx.x == 0) km[1 + ((it + 1) & 1)] = 0;  // reset next slot
  }
  const int k = threadIdx.x % kMaxR, sub = threadIdx.x / kMaxR;
  const int* off = v.off + (long long)h * (v.C + 1);
  const int m0 = off[c], m1 = off[c + 1];
  const int* perm = v.perm + (long long)h * v.N;
  const double* X = v.X + (long long)h * v.N * v.r;
  const bool kk = k < v.r;
  // member rows in rounds of kMeanIdx; thread (sub, k) sums members sub, sub + 4, ...
  double acc = 0.0;
  for (int b0 = m0; b0 < m1; b0 += kMeanIdx) {
    const int nb = min(kMeanIdx, m1 - b0);
    __syncthreads();
    for (int i = threadIdx.x; i < nb; i += blockDim.x) idx[i] = perm[b0 + i];
    __syncthreads();
    if (kk) {
      int i = sub;
      for (; i + 3 * kMeanSub < nb; i += 4 * kMeanSub) {
        const double x0 = X[(long long)idx[i] * v.r + k];
        const double x1 = X[(long long)idx[i + kMeanSub] * v.r + k];
        const double x2 = X[(long long)idx[i + 2 * kMeanSub] * v.r + k];
        const double x3 = X[(long long)idx[i + 3 * kMeanSub] * v.r + k];
        acc += x0;
        acc += x1;
        acc += x2;
        acc += x3;
      }
      for (; i < nb; i += kMeanSub) acc += X[(long long)idx[i] * v.r + k];
    }
  }
  part[sub][k] = acc;
  __syncthreads();
  const int cnt = m1 - m0;
  double* cent = v.cent + ((long long)h * v.C + c) * v.r;
  double mean = 0.0;
  if (kk) {
    double s = 0.0;
    for (int q = 0; q < kMeanSub; ++q) s += part[q][k];
    mean = cnt > 0 ? s / (double)cnt : cent[k];
  }
  if (!force) {
    // how far the centre moves (rounded up), for the distance bounds of the next step
    double dd = 0.0;
    if (sub == 0 && kk && cnt > 0) {
      const double t = mean - cent[k];
      dd = t * t;
    }
    dd = warp_sum(dd);
    if ((threadIdx.x & 31) == 0) opart[threadIdx.x >> 5] = dd;
    __syncthreads();
    if (threadIdx.x == 0) {
      double s2 = 0.0;
      for (int q = 0; q < kMeanSub * kMaxR / 32; ++q) s2 += opart[q];
      const double dl = sqrt(s2) * (1.0 + 1e-12);
      v.delta[(long long)h * v.C + c] = dl;
      const int G = (v.C + 31) / 32;              // 32-centre groups of the distance bounds
      atomicMax(v.dmax + ((long long)(it & 1) * gridDim.y + h) * G + c / 32,
                (unsigned long long)__double_as_longlong(dl));
    }
  }
  __syncthreads();
  if (cnt > 0 && sub == 0 && kk) cent[k] = mean;
  if (!force) return;
  // objective share: sum over members of ||x - centre||^2
  double o = 0.0;
  if (kk)
    for (int mm = m0 + sub; mm < m1; mm += kMeanSub) {
      const double t = X[(long long)perm[mm] * v.r + k] - mean;
      o += t * t;
    }
  o = warp_sum(o);
  if ((threadIdx.x & 31) == 0) opart[threadIdx.x >> 5] = o;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int q = 0; q < kMeanSub * kMaxR / 32; ++q) s += opart[q];
    v.obj[(long long)h * v.C + c] = s;
  }
}

// ---------------------------------------------------------------------------------
// Exact incremental means.  Every coordinate is taken as round(x 2^80) = l2 2^80 +
// l1 2^40 + l0, the limbs of |x| with the sign of x, |l1|, |l0| <= 2^40 (exact for
// |x| >= 2^-28, the rounding of smaller ones is below 2^-81), and each limb of a centre's member sum is an int64 of its own, so
// integer atomics in any order give the same sums bit for bit.  A step moves only the
// points whose label changed: their limbs leave the old centre and join the new one.
__device__ __forceinline__ void fx_split(double x, long long* l) {
  const double a = fabs(x);
  const double f2 = floor(a);
  const double y1 = (a - f2) * 1099511627776.0;          // 2^40; a - floor(a) is exact for a >= 0
  const double f1 = floor(y1);
  const long long sg = x < 0.0 ? -1 : 1;                 // limbs of |x|, signed together
  l[2] = sg * (long long)f2;
  l[1] = sg * (long long)f1;
  l[0] = sg * llrint((y1 - f1) * 1099511627776.0);
}

__device__ __forceinline__ double fx_value(const unsigned long long* s) {   // sum 2^-80
  const __int128 t = ((__int128)(long long)s[2] << 80) + ((__int128)(long long)s[1] << 40) +
                     (__int128)(long long)s[0];
  const long long hi = (long long)(t >> 64);
  const unsigned long long lo = (unsigned long long)t;
  return ((double)hi * 18446744073709551616.0 + (double)lo) * 8.271806125530277e-25;
}

// The exact sums of every centre from scratch, one block per (centre, head): its members
// in group-major order (the counting sort of this step), limbs summed in int64 (exact,
// any order).  Used after the first assignment, where every point changed label and the
// change log would cost one atomic per limb of every point.
__global__ void __launch_bounds__(256) km_fx_full_kernel(KmView v, int it) {
  __shared__ long long part[4][kMaxR][3];
  const int h = blockIdx.y, c = blockIdx.x;
  if (km_skip(v, h, it, false)) return;
  const int k = threadIdx.x % kMaxR, sub = threadIdx.x / kMaxR;
  const int* off = v.off + (long long)h * (v.C + 1);
  const int m0 = off[c], m1 = off[c + 1];
  const int* perm = v.perm + (long long)h * v.N;
  const double* X = v.X + (long long)h * v.N * v.r;
  long long acc[3] = {0, 0, 0};
  if (k < v.r)
    for (int mm = m0 + sub; mm < m1; mm += 4) {
      long long l[3];
      fx_split(X[(long long)perm[mm] * v.r + k], l);
      acc[0] += l[0];
      acc[1] += l[1];
      acc[2] += l[2];
    }
  for (int j = 0; j < 3; ++j) part[sub][k][j] = acc[j];
  __syncthreads();
  if (sub == 0 && k < v.r) {
    unsigned long long* dst = v.fx + (((long long)h * v.C + c) * 64 + k) * 3;
    for (int j = 0; j < 3; ++j)
      dst[j] = (unsigned long long)(part[0][k][j] + part[1][k][j] + part[2][k][j] + part[3][k][j]);
  }
  if (threadIdx.x == 0) {
    v.fxcnt[(long long)h * v.C + c] = m1 - m0;
  }
}

// Each warp scans 32 points at a time for changes stamped with this step; for every such
// point the whole warp moves its limbs from the old centre to the new one.
__global__ void __launch_bounds__(256) km_fx_apply_kernel(KmView v, int it) {
  const int lane = threadIdx.x & 31;
  const long long HN = (long long)v.H * v.N;
  const long long w0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long base = w0 * 32; base < HN; base += nw * 32) {
    const long long i = base + lane;
    const unsigned long long e = i < HN ? v.chg[i] : ~0ull;
    unsigned todo = __ballot_sync(0xffffffffu, (int)(e >> 32) == it);
    while (todo) {
      const int src = __ffs(todo) - 1;
      todo &= todo - 1;
      const unsigned long long ee = __shfl_sync(0xffffffffu, e, src);
      const long long pi = base + src;
      const int h = (int)(pi / v.N);
      const int cnew = (int)(ee & 0xFFFF), cold = (int)((ee >> 16) & 0xFFFF);
      const double* x = v.X + pi * v.r;
      unsigned long long* to = v.fx + ((long long)h * v.C + cnew) * 64 * 3;
      unsigned long long* from = cold != 0xFFFF ? v.fx + ((long long)h * v.C + cold) * 64 * 3 : nullptr;
      for (int k = lane; k < v.r; k += 32) {
        long long l[3];
        fx_split(x[k], l);
        for (int j = 0; j < 3; ++j) {
          atomicAdd(to + 3 * k + j, (unsigned long long)l[j]);
          if (from) atomicAdd(from + 3 * k + j, (unsigned long long)(-l[j]));
        }
      }
      if (lane == 0) {
        atomicAdd(v.fxcnt + (long long)h * v.C + cnew, 1);
        if (from) atomicAdd(v.fxcnt + (long long)h * v.C + cold, -1);
      }
    }
  }
}

// Centres from the exact sums (S6: an empty centre stays), with the convergence flags and
// the centre moves of cs_mean_kernel; one block of 64 threads per (centre, head).
__global__ void __launch_bounds__(64) km_fx_mean_kernel(KmView v, int it) {
  __shared__ double dd2[2];
  const int h = blockIdx.y, c = blockIdx.x, k = threadIdx.x;
  int* km = v.km + 4 * h;
  if (km[0]) return;
  if (!km[1 + (it & 1)]) {                  // converged: this assignment changed nothing
    if (c == 0 && k == 0) km[0] = 1;
    return;
  }
  if (c == 0 && k == 0) km[1 + ((it + 1) & 1)] = 0;   // reset the next step's flag
  const int cnt = v.fxcnt[(long long)h * v.C + c];
  double* cent = v.cent + ((long long)h * v.C + c) * v.r;
  double t = 0.0, mean = 0.0;
  if (k < v.r) {
    mean = cnt > 0 ? fx_value(v.fx + (((long long)h * v.C + c) * 64 + k) * 3) / (double)cnt : cent[k];
    t = cnt > 0 ? mean - cent[k] : 0.0;
  }
  double s = warp_sum(t * t);
  if ((k & 31) == 0) dd2[k >> 5] = s;
  __syncthreads();
  if (k == 0) {
    const double dl = sqrt(dd2[0] + dd2[1]) * (1.0 + 1e-12);
    v.delta[(long long)h * v.C + c] = dl;
    const int G = (v.C + 31) / 32;
    atomicMax(v.dmax + ((long long)(it & 1) * gridDim.y + h) * G + c / 32,
              (unsigned long long)__double_as_longlong(dl));
  }
  if (k < v.r && cnt > 0) cent[k] = mean;
}

sparsepr_status run_update(const Plan& p, const KmView& v, int it, bool force, cudaStream_t st) {
  const int H = v.H;
  cs_hist_kernel<<<dim3(v.nch, H), kSortChunk, 0, st>>>(v, it, force);
  SPR_LAUNCH_OK();
  cs_scan_kernel<<<H, 1024, 0, st>>>(v, it, force);
  SPR_LAUNCH_OK();
  const size_t wsm = (size_t)(kSortChunk / 32) * v.C * sizeof(int);
  SPR_CUDA_OK(cudaFuncSetAttribute(cs_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)wsm));
  cs_scatter_kernel<<<dim3(v.nch, H), kSortChunk, wsm, st>>>(v, it, force);
  SPR_LAUNCH_OK();
  cs_mean_kernel<<<dim3(v.C, H), kMeanSub * kMaxR, 0, st>>>(v, it, force);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

template <int R>
void assign(const KmView& v, int H, int it, cudaStream_t st) {
  km_assign_kernel<R><<<dim3(cdiv(v.N, 128), H), 128, 0, st>>>(v, it);
}

// ---------------------------------------------------------------------------------
// Groups of the final labels: compact ids in ascending label order, sizes, counts and
// the final objective (sum of per-cluster shares in label order).
__global__ void __launch_bounds__(1024) groups_kernel(KmView v, int* comp, int* used, int* size,
                                                      int* ngroups, double* objH) {
  __shared__ int sh[32];
  __shared__ double red[32];
  const int h = blockIdx.x;
  const int* off = v.off + (long long)h * (v.C + 1);
  int* comph = comp + (long long)h * v.C;
  int* usedh = used + (long long)h * v.C;
  int* sizeh = size + (long long)h * v.C;
  const int c = threadIdx.x;
  const int cnt = c < v.C ? off[c + 1] - off[c] : 0;
  int total;
  const int idx = block_exclusive_scan(cnt > 0 ? 1 : 0, sh, &total);
  if (c < v.C) {
    comph[c] = cnt > 0 ? idx : -1;
    if (cnt > 0) {
      usedh[idx] = c;
      sizeh[idx] = cnt;
    }
  }
  __syncthreads();
  for (int e = total + threadIdx.x; e < v.C; e += blockDim.x) {
    usedh[e] = -1;
    sizeh[e] = 0;
  }
  if (threadIdx.x == 0) ngroups[h] = total;
  // objective in label order (one thread: C <= 1024 terms, deterministic)
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int q = 0; q < v.C; ++q) s += v.obj[(long long)h * v.C + q];
    objH[2 * h + v.stage] = s;
  }
  (void)red;
}

// Group centroids in the original space (compact ids), fp64 sums in group-major order.
constexpr int kCentSub = 4;
__global__ void __launch_bounds__(kCentSub * kMaxD) centroid_kernel(Dims m, const void* X,
                                                                   const void* X2, int N, int C,
                                                                   const int* perm, const int* off,
                                                                   const int* used, const int* ngroups,
                                                                   double* out, double* out2) {
  __shared__ double part[kCentSub][kMaxD];
  __shared__ double part2[kCentSub][kMaxD];
  const int h = blockIdx.y, a = blockIdx.x, d = m.d;
  if (a >= ngroups[h]) return;
  const int lab = used[(long long)h * C + a];
  const int m0 = off[(long long)h * (C + 1) + lab], m1 = off[(long long)h * (C + 1) + lab + 1];
  const int j = threadIdx.x % kMaxD, sub = threadIdx.x / kMaxD;
  const int* ph = perm + (long long)h * N;
  const long long base = (long long)h * N * d;
  double acc = 0.0, acc2 = 0.0;
  if (j < d) {
    for (int mm = m0 + sub; mm < m1; mm += kCentSub) {
      const long long src = base + (long long)ph[mm] * d + j;
      acc += (double)load_as_float(X, src, m.dtype);
      if (X2) acc2 += (double)load_as_float(X2, src, m.dtype);
    }
  }
  part[sub][j] = acc;
  part2[sub][j] = acc2;
  __syncthreads();
  if (sub == 0 && j < d) {
    double s = 0.0, s2 = 0.0;
    for (int q = 0; q < kCentSub; ++q) {
      s += part[q][j];
      s2 += part2[q][j];
    }
    const double cnt = (double)(m1 - m0);
    out[((long long)h * C + a) * d + j] = s / cnt;
    if (X2) out2[((long long)h * C + a) * d + j] = s2 / cnt;
  }
}

// M_Q = (1/C_k') K~^T K~ with K~ = kbar - mean of the non-empty kbar (paper App. B.2).
__global__ void __launch_bounds__(1024) query_metric_kernel(Dims m, const double* kbar,
                                                            const int* ngroups, double* MQ) {
  constexpr int ROWS = 16;
  __shared__ double mu[kMaxD];
  __shared__ double tile[ROWS * kMaxD];
  const int h = blockIdx.x, d = m.d, n = ngroups[h];
  const double* kb = kbar + (long long)h * m.Ck * d;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    double s = 0.0;
    for (int b = 0; b < n; ++b) s += kb[(long long)b * d + j];
    mu[j] = s / (double)n;
  }
  double acc[16];
  for (int k = 0; k < 16; ++k) acc[k] = 0.0;
  for (int b0 = 0; b0 < n; b0 += ROWS) {
    const int nb = (n - b0) < ROWS ? (n - b0) : ROWS;
    __syncthreads();
    for (int e = threadIdx.x; e < nb * d; e += blockDim.x)
      tile[e] = kb[(long long)b0 * d + e] - mu[e % d];
    __syncthreads();
    for (int k = 0; k < 16; ++k) {
      const int e = threadIdx.x + k * blockDim.x;
      if (e >= d * d) break;
      const int i = e / d, j = e % d;
      double a = acc[k];
      for (int b = 0; b < nb; ++b) a += tile[b * d + i] * tile[b * d + j];
      acc[k] = a;
    }
  }
  for (int k = 0; k < 16; ++k) {
    const int e = threadIdx.x + k * blockDim.x;
    if (e >= d * d) break;
    MQ[(long long)h * d * d + e] = acc[k] / (double)n;
  }
}

// Injected labels outside [0, C) are clamped to 0 and flagged.
__global__ void check_labels_kernel(int* lab, long long n, int C, int* err) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int v = lab[i];
    if (v < 0 || v >= C) {
      lab[i] = 0;
      atomicOr(err, kErrLabels);
    }
  }
}

}  // namespace

sparsepr_status launch_check_labels(const Plan& p, bool query, cudaStream_t st) {
  const KmView v = view(p, query);
  check_labels_kernel<<<148 * 4, 256, 0, st>>>(v.lab, (long long)v.H * v.N, v.C, p.b.err);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

// The tensor-core k-means serves a side when the engine allows it and C fits its tiles.
bool km_uses_tc(const Plan& p, bool query) {
  const KmView v = view(p, query);
  return p.dm.engine == SPARSEPR_ENGINE_AUTO && km_tc_supported(v.C) && (long long)v.H * v.N < (1LL << 31);
}

// fp64 coordinates for either engine; the split coordinates of the tensor-core k-means
// come with them when that k-means will run.
sparsepr_status launch_project_side(const Plan& p, bool query, cudaStream_t st) {
  const Dims& m = p.dm;
  const Buffers& b = p.b;
  const void* X = query ? p.Q : p.K;
  const int N = query ? m.Nq : m.Nk, r = query ? m.rQ : m.rK;
  double* out = query ? b.phiQ : b.phiK;
  const double* F = query ? b.FQ64 : b.FK64;
  const bool fuse = km_uses_tc(p, query);
  __nv_bfloat16* xhi = fuse ? b.kmXhi : nullptr;
  __nv_bfloat16* xlo = fuse ? b.kmXlo : nullptr;
  float* xn = fuse ? b.kmXn : nullptr;
  const int Npad = km_tc_npad(N);
  return query && !m.semantic ? launch_project<true>(p, true, X, N, F, r, out, xhi, xlo, xn, Npad, st)
                              : launch_project<false>(p, query, X, N, F, r, out, xhi, xlo, xn, Npad, st);
}

sparsepr_status launch_project_keys(const Plan& p, cudaStream_t st) { return launch_project_side(p, false, st); }

sparsepr_status launch_project_queries(const Plan& p, cudaStream_t st) { return launch_project_side(p, true, st); }

sparsepr_status launch_kmeans(const Plan& p, bool query, cudaStream_t st) {
  const KmView v = view(p, query);
  const int H = v.H;
  SPR_CUDA_OK(cudaMemsetAsync(v.km, 0, sizeof(int) * 4 * H, st));
  SPR_CUDA_OK(cudaMemsetAsync(v.lab, 0xFF, sizeof(int) * (size_t)H * v.N, st));  // labels = -1
  if (p.warm) {
    const StateLayout L = state_layout(p.dm);
    const char* base = static_cast<const char*>(p.warm);
    km_warm_init_kernel<<<dim3(cdiv(v.C, 8), H), 256, 0, st>>>(
        v, p.dm.seed, p.dm, reinterpret_cast<const int*>(base),
        reinterpret_cast<const double*>(base + (query ? L.QC : L.KC)),
        reinterpret_cast<const int*>(base + (query ? L.qu : L.ku)), query ? p.b.FQ64 : p.b.FK64);
  } else {
    km_init_kernel<<<H, 256, 0, st>>>(v, p.dm.seed);
  }
  SPR_LAUNCH_OK();
  // tensor-core scores with exact rescoring (labels identical to the fp64 full scan) when
  // there are enough centres to fill the tiles; the full scan otherwise or on request
  const bool tc = km_uses_tc(p, query);
  const Buffers& b = p.b;
  const KmTcBuffers kb{b.kmXhi, b.kmXlo, b.kmShi, b.kmSlo, b.kmU, b.kmDelta, b.kmL, b.kmDmax, b.kmAidx,
                       b.kmAcnt, b.kmReassigned + (query ? H : 0), b.kmXn, b.kmChi, b.kmClo, b.kmCn, b.kmCmaxb, b.kmQueue, b.kmQcnt,
                       b.kmChg};
  // exact sums start empty; every label starts at -1, so the first step logs every point
  SPR_CUDA_OK(cudaMemsetAsync(b.kmFx, 0, sizeof(unsigned long long) * (size_t)H * v.C * 64 * 3, st));
  SPR_CUDA_OK(cudaMemsetAsync(b.kmFxCnt, 0, sizeof(int) * (size_t)H * v.C, st));
  // no point has a stamped change yet (stamp -1)
  SPR_CUDA_OK(cudaMemsetAsync(b.kmChg, 0xFF, sizeof(unsigned long long) * (size_t)H * v.N, st));
  if (tc) {
    SPR_CUDA_OK(cudaMemsetAsync(b.kmCmaxb, 0, sizeof(int) * 2 * H, st));
    SPR_CUDA_OK(cudaMemsetAsync(b.kmQcnt, 0, sizeof(int) * 2, st));
    SPR_CUDA_OK(cudaMemsetAsync(b.kmAcnt, 0, sizeof(int) * 2 * H, st));
  }
  for (int it = 0; it < p.dm.max_iter; ++it) {
    if (tc) {
      // the distance bounds pay where few points can move: a warm start begins near a
      // fixed point; from fresh centres about half of the points stay undecided by them
      sparsepr_status s = km_tc_assign(kb, v.X, v.cent, H, v.N, v.C, v.r, it, v.lab, v.km, b.err,
                                       p.warm != nullptr, st);
      if (s != SPARSEPR_OK) return s;
    } else {
      if (v.r <= 8) assign<8>(v, H, it, st);
      else if (v.r <= 16) assign<16>(v, H, it, st);
      else if (v.r <= 32) assign<32>(v, H, it, st);
      else if (v.r <= 48) assign<48>(v, H, it, st);
      else assign<64>(v, H, it, st);
      SPR_LAUNCH_OK();
    }
    if (it == 0) {
      // every label changed: group the points (counting sort) and sum each centre's limbs
      cs_hist_kernel<<<dim3(v.nch, H), kSortChunk, 0, st>>>(v, it, false);
      SPR_LAUNCH_OK();
      cs_scan_kernel<<<H, 1024, 0, st>>>(v, it, false);
      SPR_LAUNCH_OK();
      const size_t wsm = (size_t)(kSortChunk / 32) * v.C * sizeof(int);
      SPR_CUDA_OK(cudaFuncSetAttribute(cs_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)wsm));
      cs_scatter_kernel<<<dim3(v.nch, H), kSortChunk, wsm, st>>>(v, it, false);
      SPR_LAUNCH_OK();
      km_fx_full_kernel<<<dim3(v.C, H), 256, 0, st>>>(v, it);
    } else {
      km_fx_apply_kernel<<<8 * 148, 256, 0, st>>>(v, it);
    }
    SPR_LAUNCH_OK();
    km_fx_mean_kernel<<<dim3(v.C, H), 64, 0, st>>>(v, it);
    SPR_LAUNCH_OK();
  }
  return SPARSEPR_OK;
}

sparsepr_status launch_finalize_groups(const Plan& p, bool query, cudaStream_t st) {
  const KmView v = view(p, query);
  sparsepr_status s = run_update(p, v, 0, true, st);
  if (s != SPARSEPR_OK) return s;
  const Buffers& b = p.b;
  if (query) groups_kernel<<<v.H, 1024, 0, st>>>(v, b.compQ, b.usedQ, b.sizeQ, b.nQ, b.objH);
  else groups_kernel<<<v.H, 1024, 0, st>>>(v, b.compK, b.usedK, b.sizeK, b.nK, b.objH);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

sparsepr_status launch_centroids(const Plan& p, bool query, cudaStream_t st) {
  const Buffers& b = p.b;
  const Dims& m = p.dm;
  if (query)
    centroid_kernel<<<dim3(m.Cq, m.H), kCentSub * kMaxD, 0, st>>>(m, p.Q, nullptr, m.Nq, m.Cq, b.permQ, b.offQ, b.usedQ, b.nQ, b.qbar, nullptr);
  else
    centroid_kernel<<<dim3(m.Ck, m.Hk), kCentSub * kMaxD, 0, st>>>(m, p.K, p.V, m.Nk, m.Ck, b.permK, b.offK, b.usedK, b.nK, b.kbar, b.vbar);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

sparsepr_status launch_save_state(const Plan& p, void* state, cudaStream_t st) {
  save_state_kernel<<<p.dm.H, 1024, 0, st>>>(p.dm, p.b, static_cast<char*>(state));
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

sparsepr_status launch_query_metric(const Plan& p, cudaStream_t st) {
  query_metric_kernel<<<p.dm.Hk, 1024, 0, st>>>(p.dm, p.b.kbar, p.b.nK, p.b.MQ);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

}  // namespace spr
