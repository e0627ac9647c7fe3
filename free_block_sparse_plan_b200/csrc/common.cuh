// Shared definitions of the SparsePR CUDA library: problem description, workspace
// pointers, launch helpers and small device utilities.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sparsepr.h"

namespace spr {

constexpr int kMaxD = 128;      // head dimension limit
constexpr int kMaxC = 1024;     // requested group count limit
constexpr int kMaxR = 64;       // response-coordinate rank limit
constexpr int kMaxM = 128;      // probe count limit
constexpr int kSortChunk = 1024; // rows per block of the stable counting sort
constexpr int kProbeSplit = 4096;  // keys per partial of the exact probe attention

// Device error word bits.
enum : int {
  kErrEigK = 1,        // key metric has no positive eigenvalue among the leading r_K
  kErrEigQ = 2,        // query metric has no positive eigenvalue among the leading r_Q
  kErrNonFinite = 4,   // a non-finite value reached the fit
  kErrProbe = 8,       // probe selection could not find M rows
  kErrLabels = 16,     // an injected label was outside [0, C)
  kErrHang = 32,       // a pipeline wait timed out (the kernel abandoned its work)
  kErrWarmState = 64,  // a warm state did not match the plan's dimensions (started cold)
};

// Problem dimensions, passed by value to kernels.
struct Dims {
  int H, Nq, Nk, d, dtype;
  int Ms, rK, rQ, Cq, Ck, M, r;
  double lambda, rho;
  int max_iter, engine;
  unsigned long long seed;
  int estimator;       // sparsepr_estimator
  int G, Hk;           // query heads per K/V head; K/V heads (H / G)
  int semantic;        // semantic reference partition: coordinates = raw rows (rK = rQ = d)
  int nchK, nchQ;      // counting-sort chunks per head
  int nsplit;          // partial blocks of the exact probe attention
  double beta;         // per-query key budget (rho - M/N_q) * N_k of the prefix rule
  int budget;          // sparsepr_budget
};

// Device buffers carved from the caller's workspace (see carve_workspace).
struct Buffers {
  double *MK, *MQ, *lamK, *lamQ, *FK64, *FQ64;
  float *FK, *FQ;
  double *phiK, *phiQ;      // response coordinates [H][N][r] (fp64)
  double *centK, *centQ;     // k-means centres [H][C][r] (fp64)
  int *labK, *labQ;
  int *histK, *histQ;
  int *permK, *permQ, *invQ;
  int *offK, *offQ;          // raw-label offsets [H][C+1]
  int *poffK;                // tensor-core K/V layout: padded raw-label row offsets [H_k][C_k+1]
  int *kmK, *kmQ;            // per-head k-means state [H][4]: done, changed, iters, -
  double *objK, *objQ;       // per-cluster objective partials [H][C]
  double *objH;              // [H][2] final objectives
  int *compK, *compQ;        // raw label -> compact id (-1 if empty) [H][C]
  int *usedK, *usedQ;        // compact id -> raw label [H][C]
  int *nK, *nQ;              // [H] non-empty group counts
  int *sizeK, *sizeQ;        // compact sizes [H][C]
  double *kbar, *vbar, *qbar;  // compact centroids [H][C][d]
  double *scores;            // [H][Cq][Ck]
  int *cellCnt, *cellIds;    // [H][Cq], [H][Cq][Ck]
  int *rankPref;             // calibrated budget: key counts of each score-ranked prefix [H][Cq][Ck]
  double *betaH;             // budget each head's routing used [H]
  long long *pairs;          // [H]
  void *Qp, *Kp, *Vp;        // group-major copies [H][N][d]; K/V in the tensor-core layout
                             // (kv_tiled_rows) when that engine runs
  double *dist;              // [H][Nq]
  int *probeTop;             // [H][Cq][M]
  int *probes, *probeA, *mA; // [H][M], [H][M], [H][Cq]
  double *wP;                // [H][M]
  float *Osp;                // [H][Nq][d] group-major
  float *Opart, *MLpart;     // [H][M][nsplit][d], [H][M][nsplit][2]
  float *Odense;             // [H][M][d]
  double *fitA, *fitY, *fitZ;  // fit scratch
  double *muX, *muR, *sX;    // [H][d]
  double *Bm, *Pm;           // [H][d][d]
  double *sig;               // [H][kMaxM]
  int *reff;                 // [H]
  float *Bp, *cvec;          // folded correction [H][d][d], [H][d]
  float *BpT;                // B' transposed [H][d][d] (tensor-core correction)
  int *work, *nwork;         // tensor-core attention work list [H][max items], [H]
  __nv_bfloat16 *kmXhi, *kmXlo;  // k-means features split into bf16 pieces [H][Npad][64]
  float *kmXn;               // feature norms [H][Nmax]
  __nv_bfloat16 *kmChi, *kmClo;  // centres split into bf16 pieces [H][Cpad][64]
  float *kmCn;               // squared centre norms [H][Cpad]
  int *kmCmaxb;              // largest squared centre norm as float bits [2][H]
  int4 *kmQueue;             // points whose label needs exact rescoring
  double *kmU;               // distance to the own centre, upper bound [H][Nmax]
  float *kmL;                // distance to the other centres of each 32-centre group, lower bound [H][G][N]
  double *kmDelta;           // centre movement of the last update [H][Cmax]
  unsigned long long *kmDmax;  // largest movement per head and group as double bits [2][H][G]
  int *kmAidx, *kmAcnt;      // points to re-assign, compacted [H][Npad]; their counts [2][H]
  long long *kmReassigned;   // points re-assigned, summed over the steps [2 sides][H]
  __nv_bfloat16 *kmShi, *kmSlo;  // their split coordinates, compacted [H][Npad][64]
  int *kmQcnt;               // queue lengths [2]
  int *warmCold;             // heads whose warm factor update fell back to the eigensolve [2][H]
  unsigned long long *kmFx;  // exact member sums of each centre, three 40-bit limbs [H][Cmax][64][3]
  int *kmFxCnt;              // member counts [H][Cmax]
  unsigned long long *kmChg; // last label change of each point: new | old << 16 | step << 32 [H*Nmax]
  int *err;                  // device error word
};

// Warm state handed from one call of a sequence to the next (paper App. C): a header,
// the fp64 metric factors, and the original-space centroid of every label with a
// non-empty flag.  Offsets in bytes from the state base; every block 256-byte aligned.
constexpr int kStateMagic = 0x57525053;
struct StateLayout {
  size_t FK, FQ, KC, QC, ku, qu, total;
};
__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
__device__ inline bool state_matches(const int* hdr, const Dims& m) {
  return hdr[0] == kStateMagic && hdr[1] == m.H && hdr[2] == m.d && hdr[3] == m.rK &&
         hdr[4] == m.rQ && hdr[5] == m.Ck && hdr[6] == m.Cq && hdr[7] == 1;
}
__host__ __device__ inline StateLayout state_layout(const Dims& m) {
  const size_t H = m.H, d = m.d;
  StateLayout L;
  L.FK = 256;                                          // header: 16 int32
  L.FQ = L.FK + align256(H * d * m.rK * sizeof(double));
  L.KC = L.FQ + align256(H * d * m.rQ * sizeof(double));
  L.QC = L.KC + align256(H * (size_t)m.Ck * d * sizeof(double));
  L.ku = L.QC + align256(H * (size_t)m.Cq * d * sizeof(double));
  L.qu = L.ku + align256(H * (size_t)m.Ck * sizeof(int));
  L.total = L.qu + align256(H * (size_t)m.Cq * sizeof(int));
  return L;
}

// Host-side plan handle.
struct Plan {
  Dims dm;
  Buffers b;
  const void *Q, *K, *V;
  const void* warm;          // previous call's state (warm start), or null
  int stage;                 // 1 planned, 2 attended, 3 fitted
};

// ---------------------------------------------------------------------------------
// Launch helpers (host)
#define SPR_CUDA_OK(expr)                                  \
  do {                                                     \
    cudaError_t e_ = (expr);                               \
    if (e_ != cudaSuccess) return SPARSEPR_ERR_CUDA;       \
  } while (0)

// After every kernel launch: count it (sparsepr_launch_count) and check it.
void count_launch();
#define SPR_LAUNCH_OK()                                    \
  do {                                                     \
    count_launch();                                        \
    cudaError_t e_ = cudaGetLastError();                   \
    if (e_ != cudaSuccess) return SPARSEPR_ERR_CUDA;       \
  } while (0)

inline int cdiv(long long a, long long b) { return (int)((a + b - 1) / b); }

// Rows per K/V head of the tensor-core K/V layout: every group's rows padded to a multiple
// of 8 (at most 7 rows per group), then 128 zero rows.  The layout holds per K/V head the
// 64-column panels one after the other ([panel][row][64] bf16, 128-byte rows), with the
// 16-byte chunks of panel row p stored in the order chunk ^ (p & 7).
__host__ __device__ inline long long kv_tiled_rows(int Nk, int Ck) { return (long long)Nk + 7LL * Ck + 128; }

// ---------------------------------------------------------------------------------
// Device utilities

// A point's label change at k-means step `it`: new | old << 16 | it << 32 (old = 0xFFFF
// for none); the exact-sum update applies the entries stamped with its own step, so the
// array needs no clearing between steps.
__device__ __forceinline__ unsigned long long chg_entry(int old, int now, int it) {
  return (unsigned long long)(now & 0xFFFF) | ((unsigned long long)(old & 0xFFFF) << 16) |
         ((unsigned long long)(unsigned)it << 32);
}
__device__ __forceinline__ float load_as_float(const void* p, long long i, int dtype) {
  if (dtype == SPARSEPR_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  return reinterpret_cast<const float*>(p)[i];
}

__device__ __forceinline__ void store_from_float(void* p, long long i, float v, int dtype) {
  if (dtype == SPARSEPR_BF16) reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else reinterpret_cast<float*>(p)[i] = v;
}

__device__ __forceinline__ float warp_sum(float v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum(double v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum of doubles; `red` holds blockDim.x/32 doubles. All threads get the sum.
__device__ __forceinline__ double block_sum(double v, double* red) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  double t = 0.0;
  for (int i = 0; i < nw; ++i) t += red[i];   // fixed order: deterministic
  return t;
}

__device__ __forceinline__ long long block_sum_ll(long long v, long long* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  long long t = 0;
  for (int i = 0; i < nw; ++i) t += red[i];
  return t;
}

// Exclusive block scan of ints (blockDim.x <= 1024); `sh` holds 32 ints.
__device__ __forceinline__ int block_exclusive_scan(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  int x = v;
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) sh[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = (lane < nw) ? sh[lane] : 0;
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < nw) sh[lane] = s;   // inclusive per-warp totals
  }
  __syncthreads();
  int base = (w > 0) ? sh[w - 1] : 0;
  if (total) *total = sh[nw - 1];
  return base + x - v;
}

// ---------------------------------------------------------------------------------
// Stage launchers (defined in the .cu files; all enqueue on `st`, return a status).
sparsepr_status launch_key_metric(const Plan& p, cudaStream_t st);
sparsepr_status launch_eigen_factor(const Plan& p, bool query, cudaStream_t st);
sparsepr_status launch_warm_factor(const Plan& p, bool query, cudaStream_t st);
sparsepr_status launch_identity_factors(const Plan& p, cudaStream_t st);
sparsepr_status launch_save_state(const Plan& p, void* state, cudaStream_t st);
sparsepr_status launch_project_keys(const Plan& p, cudaStream_t st);
sparsepr_status launch_project_queries(const Plan& p, cudaStream_t st);
sparsepr_status launch_kmeans(const Plan& p, bool query, cudaStream_t st);
sparsepr_status launch_finalize_groups(const Plan& p, bool query, cudaStream_t st);
sparsepr_status launch_check_labels(const Plan& p, bool query, cudaStream_t st);
sparsepr_status launch_centroids(const Plan& p, bool query, cudaStream_t st);
sparsepr_status launch_query_metric(const Plan& p, cudaStream_t st);
sparsepr_status launch_route(const Plan& p, cudaStream_t st);
sparsepr_status launch_permute(const Plan& p, cudaStream_t st);
sparsepr_status launch_select_probes(const Plan& p, cudaStream_t st);
sparsepr_status launch_sparse_attention(const Plan& p, cudaStream_t st);
sparsepr_status launch_probe_attention(const Plan& p, cudaStream_t st);
sparsepr_status launch_fit(const Plan& p, cudaStream_t st);
sparsepr_status launch_correct(const Plan& p, void* Out, cudaStream_t st);
sparsepr_status launch_sparse_attention_simt(const Plan& p, cudaStream_t st);
sparsepr_status launch_dense_attention_simt(const Dims& dm, const void* Q, const void* K,
                                            const void* V, void* Out, cudaStream_t st);
bool tc_engine_applies(int dtype, int d, int engine);
int tc_max_items(const Dims& m);
sparsepr_status launch_sparse_attention_tc(const Plan& p, cudaStream_t st);
sparsepr_status launch_probe_attention_tc(const Plan& p, cudaStream_t st);
sparsepr_status launch_probe_attention_simt(const Plan& p, cudaStream_t st);
sparsepr_status launch_probe_combine(const Plan& p, cudaStream_t st);
sparsepr_status launch_dense_attention_tc(const Dims& m, const void* Q, const void* K, const void* V,
                                          void* Out, int* err, cudaStream_t st);
int km_tc_npad(int N);
int km_tc_cpad(int C);
bool km_tc_supported(int C);
bool correct_tc_applies(int dtype, int d, int engine);
sparsepr_status launch_correct_tc(const Plan& p, void* Out, cudaStream_t st);
long long km_tc_queue_cap(int H, int N);
struct KmTcBuffers {
  const __nv_bfloat16 *xhi, *xlo;
  __nv_bfloat16 *shi, *slo;
  double *U, *delta;
  float* L;
  unsigned long long* dmax;
  int *aidx, *acnt;
  long long* reassigned;     // [H] of this side
  const float* xn;
  __nv_bfloat16 *chi, *clo;
  float* cn;
  int* cmaxb;
  int4* queue;
  int* qcnt;
  unsigned long long* chg;   // label change of each point at this step (exact incremental means)
};
sparsepr_status km_tc_assign(const KmTcBuffers& kb, const double* X, const double* cent, int H, int N, int C,
                             int r, int it, int* lab, int* kmstate, int* err, bool bounds, cudaStream_t st);
sparsepr_status launch_dense_attention(const Dims& dm, const void* Q, const void* K,
                                       const void* V, void* Out, cudaStream_t st);
// Device addresses of the error words of the plan-free entry points on the current
// device: sparsepr_dense_attention's, and the sticky word of sparsepr_dense_rows_noalloc.
sparsepr_status dense_error_address(int** out);
sparsepr_status launch_wait_selftest(cudaStream_t st);
sparsepr_status noalloc_error_address(int** out);
// O3 affine-fit diagnostic over a plan's sparse output (diagnostics.cu).
sparsepr_status launch_affine_fit(const Plan& p, const void* dense, double* ws, double* explained,
                                  double* err, cudaStream_t st);
size_t affine_ws_doubles(const Dims& m);

}  // namespace spr
