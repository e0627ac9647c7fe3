// sparsepr_dense_rows_noalloc: exact attention of selected query rows with no device
// allocation by the caller or by the library.
//
// Some callers cannot allocate device memory around this call: code whose device memory
// is owned by another allocator (a framework's caching pool that has reserved the GPU),
// and latency-critical loops that must not pay the implicit device synchronisation of
// cudaMalloc/cudaFree.  They pass inputs and outputs only; the split-key partial results
// live in a fixed file-scope device array of kNoAllocScratchBytes, which every GPU that
// loads this library holds until the process exits.
//
// The array is shared by all calls: two calls whose work overlaps on the GPU (different
// streams, or different host threads) race on it and must be serialised by the caller.
// Its first 256 bytes hold two error words: the call's own (cleared by every call before
// its first kernel, with a memset that allocates nothing) and a sticky copy that keeps
// every bit until sparsepr_dense_check reads and clears it.  Every other scratch element
// a call reads was written earlier in the same call.  If a pipeline wait of the attention
// kernel timed out, that call's output rows are NaN rather than stale partials.
#include <mutex>

#include "common.cuh"

namespace spr {

constexpr size_t kNoAllocScratchBytes = 16u << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_rows_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The first call on a device
// looks it up (cudaGetSymbolAddress, with that device current); later calls reuse it.
sparsepr_status scratch_address(void** out) {
  int dev = -1;
  SPR_CUDA_OK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return SPARSEPR_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_rows_scratch) != cudaSuccess || !p) return SPARSEPR_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SPARSEPR_OK;
}


// Copies the requested rows into the scratch array once per head (the partial-attention
// kernels read a [H][nrows] row list), clamped to [0, N_q) so that no later kernel can
// read outside Q.
__global__ void copy_rows_kernel(const int32_t* rows, int nrows, int Nq, int* dst) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x, h = blockIdx.y;
  if (i >= nrows) return;
  int r = rows[i];
  r = r < 0 ? 0 : (r >= Nq ? Nq - 1 : r);
  dst[(long long)h * nrows + i] = r;
}

// Merges the split-key partials of each row and writes it in the input dtype:
// out = sum_s e^{m_s - m} O_s / sum_s e^{m_s - m} l_s.  `err` is the call's error word
// (err[0]) and the sticky word (err[1]): if the attention kernel set err[0] the partials
// are incomplete and the row is written as NaN; a non-finite result sets kErrNonFinite.
// Every bit found is also ORed into the sticky word.
__global__ void combine_rows_kernel(Dims m, const float* Opart, const float* MLpart, void* Out, int* err) {
  const int p = blockIdx.x, h = blockIdx.y, j = threadIdx.x;
  const long long slot0 = ((long long)h * m.M + p) * m.nsplit;
  const int call_err = *reinterpret_cast<volatile int*>(err);
  float mx = -INFINITY;
  for (int s = 0; s < m.nsplit; ++s) mx = fmaxf(mx, MLpart[2 * (slot0 + s)]);
  float l = 0.0f, acc = 0.0f;
  for (int s = 0; s < m.nsplit; ++s) {
    const float w = expf(MLpart[2 * (slot0 + s)] - mx);
    l += w * MLpart[2 * (slot0 + s) + 1];
    if (j < m.d) acc += w * Opart[(slot0 + s) * m.d + j];
  }
  if (j < m.d) {
    float v = acc / l;
    int bits = call_err;
    if (!isfinite(v)) bits |= kErrNonFinite;
    if (call_err) v = __int_as_float(0x7fc00000);     // NaN: the partials are incomplete
    if (bits) atomicOr(err + 1, bits);
    store_from_float(Out, ((long long)h * m.M + p) * m.d + j, v, m.dtype);
  }
}

}  // namespace

sparsepr_status noalloc_error_address(int** out) {
  void* base = nullptr;
  const sparsepr_status s = scratch_address(&base);
  if (s != SPARSEPR_OK) return s;
  *out = reinterpret_cast<int*>(base) + 1;             // the sticky word
  return SPARSEPR_OK;
}

size_t noalloc_rows_scratch_bytes(int H, int nrows, int Nk, int d) {
  const size_t nsplit = (size_t)cdiv(Nk, kProbeSplit);
  return align256(256) + align256((size_t)H * nrows * sizeof(int)) +
         align256((size_t)H * nrows * nsplit * d * sizeof(float)) +
         align256((size_t)H * nrows * nsplit * 2 * sizeof(float));
}

}  // namespace spr

using namespace spr;

extern "C" sparsepr_status sparsepr_dense_rows_noalloc(const sparsepr_params* params, const void* Q,
                                                       const void* K, const void* V,
                                                       const int32_t* rows, int32_t nrows,
                                                       void* Out, void* stream) {
  if (!params || !Q || !K || !V || !rows || !Out) return SPARSEPR_ERR_ARG;
  if (((reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V)) & 15) != 0)
    return SPARSEPR_ERR_ARG;              // the kernels read Q, K, V with 16-byte copies
  if (params->dtype != SPARSEPR_F32 && params->dtype != SPARSEPR_BF16) return SPARSEPR_ERR_DTYPE;
  if (params->H < 1 || params->N_q < 1 || params->N_k < 1) return SPARSEPR_ERR_SHAPE;
  if (params->d < 8 || params->d > kMaxD || params->d % 8) return SPARSEPR_ERR_SHAPE;
  if (params->engine != SPARSEPR_ENGINE_AUTO && params->engine != SPARSEPR_ENGINE_SIMT) return SPARSEPR_ERR_ARG;
  if (nrows < 1 || nrows > kMaxM) return SPARSEPR_ERR_ARG;
  if (params->G < 0 || (params->G > 1 && params->H % params->G != 0)) return SPARSEPR_ERR_SHAPE;
  if (params->H > 65535) return SPARSEPR_ERR_SHAPE;      // heads are the grid's y dimension
  if (noalloc_rows_scratch_bytes(params->H, nrows, params->N_k, params->d) > kNoAllocScratchBytes)
    return SPARSEPR_ERR_WORKSPACE;
  void* base = nullptr;
  sparsepr_status s = scratch_address(&base);
  if (s != SPARSEPR_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  Plan p{};
  p.dm.H = params->H; p.dm.Nq = params->N_q; p.dm.Nk = params->N_k; p.dm.d = params->d;
  p.dm.dtype = params->dtype; p.dm.engine = params->engine; p.dm.M = nrows;
  p.dm.G = params->G > 1 ? params->G : 1;
  p.dm.Hk = p.dm.H / p.dm.G;
  p.dm.nsplit = cdiv(params->N_k, kProbeSplit);
  p.Q = Q; p.K = K; p.V = V;
  char* c = reinterpret_cast<char*>(base);
  p.b.err = reinterpret_cast<int*>(c);
  c += align256(256);
  p.b.probes = reinterpret_cast<int*>(c);
  c += align256((size_t)p.dm.H * nrows * sizeof(int));
  p.b.Opart = reinterpret_cast<float*>(c);
  c += align256((size_t)p.dm.H * nrows * p.dm.nsplit * p.dm.d * sizeof(float));
  p.b.MLpart = reinterpret_cast<float*>(c);

  SPR_CUDA_OK(cudaMemsetAsync(p.b.err, 0, sizeof(int), st));   // this call's word only
  copy_rows_kernel<<<dim3(cdiv(nrows, 128), p.dm.H), 128, 0, st>>>(rows, nrows, params->N_q, p.b.probes);
  SPR_LAUNCH_OK();
  s = tc_engine_applies(p.dm.dtype, p.dm.d, p.dm.engine) ? launch_probe_attention_tc(p, st)
                                                         : launch_probe_attention_simt(p, st);
  if (s != SPARSEPR_OK) return s;
  combine_rows_kernel<<<dim3(nrows, p.dm.H), kMaxD, 0, st>>>(p.dm, p.b.Opart, p.b.MLpart, Out, p.b.err);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}
