// Corrected output on the tensor cores, for bf16 outputs (review page step 5; paper S4.2,
// App. D.2):  O_hat = O_sp + c + O_sp B' on every row, in the original token order (the
// probe rows are overwritten with their exact dense rows afterwards).
//
// Persistent CTAs, one per SM, each over a contiguous range of 128-row tiles (group-major
// rows of one head): the fp32 O_sp rows (two stages, the next tile copied while the
// current one is processed) and B'^T (once per head) sit in 128-byte-swizzled K-major
// shared memory, delta = O_sp B' comes from
// tcgen05.mma kind::tf32 (M=128, N=d, K=8 per instruction) into TMEM, and thread r adds
// its row's O_sp (from the same shared-memory tile) and c, rounds to bf16 and stores the
// row at its original position.  tf32 keeps 10 mantissa bits of each operand, so delta
// carries a relative error of about 2^-10 of |O_sp||B'|; delta is the small correction
// term, and the result is rounded to bf16 (2^-9) anyway.
#include "common.cuh"
#include "tc_ptx.cuh"

namespace spr {
namespace {

constexpr int kRowsC = 128;
constexpr long long kCWait = 2000000000LL;

// B'^T per head: BT[h][j][i] = B'[h][i][j].
__global__ void transpose_bp_kernel(const float* Bp, int d, float* BT) {
  __shared__ float t[32][33];
  const int h = blockIdx.z;
  const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  const float* src = Bp + (long long)h * d * d;
  float* dst = BT + (long long)h * d * d;
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int i = i0 + y, j = j0 + threadIdx.x;
    t[y][threadIdx.x] = (i < d && j < d) ? src[i * d + j] : 0.0f;
  }
  __syncthreads();
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int j = j0 + y, i = i0 + threadIdx.x;
    if (i < d && j < d) dst[j * d + i] = t[threadIdx.x][y];
  }
}

// Persistent: one CTA per SM takes a contiguous range of (head, 128-row tile) pairs.  B'^T
// of the current head stays in shared memory; the O_sp tiles go through two stages, and
// the copy of tile t+2 starts as soon as tile t has been written out, so that one copy is
// always in flight while a tile is multiplied and written (about 64 KB per SM, which the
// HBM latency needs to reach the copy bandwidth).
template <int D>
__global__ void __launch_bounds__(128, 1) correct_tc_kernel(Dims m, Buffers b, const float* BT,
                                                            __nv_bfloat16* Out, int tiles_per_head,
                                                            long long total) {
  constexpr int NP = D / 32;                          // 128-byte panels per fp32 row
  constexpr uint32_t kAPanel = kRowsC * 128, kBPanel = D * 128;
  constexpr uint32_t kATile = NP * kAPanel, kBTile = NP * kBPanel;
  constexpr int CPR = D / 4;                          // 16-byte chunks per fp32 row
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;       // B'^T, then stage 0, then stage 1
  uint8_t* gbase = smem_raw + (base - raw);
  unsigned long long* bar = reinterpret_cast<unsigned long long*>(gbase + kBTile + 2 * kATile);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  const int tid = threadIdx.x, warp = tid >> 5;
  const long long t0 = total * blockIdx.x / gridDim.x, t1 = total * (blockIdx.x + 1) / gridDim.x;
  if (t0 >= t1) return;

  if (tid == 0) tc::mbar_init(tc::smem_u32(bar), 1);
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(tslot), D);
    tc::tmem_relinquish();
  }
  // rows of tile t into stage s (rows past N_q read as zeros and are not stored)
  auto load_tile = [&](long long t, int s) {
    const int h = (int)(t / tiles_per_head);
    const long long p0 = (t % tiles_per_head) * kRowsC;
    const float* Oh = b.Osp + (long long)h * m.Nq * D;
    const uint32_t st0 = base + kBTile + (uint32_t)s * kATile;
    for (int e = tid; e < kRowsC * CPR; e += 128) {
      const int row = e / CPR, c = e % CPR;
      const bool ok = p0 + row < m.Nq;
      const uint32_t dst = st0 + (c >> 3) * kAPanel + tc::sw128_offset(row, c & 7);
      tc::cp_async16(dst, ok ? (const void*)(Oh + (p0 + row) * D + c * 4) : (const void*)Oh, ok ? 16u : 0u);
    }
  };
  auto load_bt = [&](int h) {
    const float* Bh = BT + (long long)h * D * D;
    for (int e = tid; e < D * CPR; e += 128) {
      const int row = e / CPR, c = e % CPR;
      tc::cp_async16(base + (c >> 3) * kBPanel + tc::sw128_offset(row, c & 7), Bh + (long long)row * D + c * 4, 16u);
    }
  };
  load_tile(t0, 0);
  tc::cp_async_commit();
  if (t0 + 1 < t1) load_tile(t0 + 1, 1);
  tc::cp_async_commit();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tslot;
  int loaded = -1;
  bool ok = true;
  for (long long t = t0; t < t1; ++t) {
    const int s = (int)((t - t0) & 1);
    const int h = (int)(t / tiles_per_head);
    if (h != loaded) {                                // a new head's B'^T: no multiply is
      load_bt(h);                                     // running (the last one was waited for)
      tc::cp_async_commit();
      tc::cp_async_wait_all();
      loaded = h;
    } else {
      tc::cp_async_wait_group1();                     // tile t arrived (t + 1 may be in flight)
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t st0 = base + kBTile + (uint32_t)s * kATile;
    if (tid == 0) {
      constexpr uint32_t idesc = tc::idesc_tf32_f32(kRowsC, D);
#pragma unroll
      for (int kk = 0; kk < D / 8; ++kk) {
        const uint64_t ad = tc::sw128_desc(st0 + (kk >> 2) * kAPanel + (kk & 3) * 32, 16, 1024);
        const uint64_t bd = tc::sw128_desc(base + (kk >> 2) * kBPanel + (kk & 3) * 32, 16, 1024);
        tc::mma_ss_tf32(tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
      }
      tc::mma_commit(tc::smem_u32(bar));
    }
    __syncwarp();
    const bool done = tc::mbar_wait(tc::smem_u32(bar), (uint32_t)((t - t0) & 1), kCWait);
    if (!__all_sync(0xffffffffu, done)) {
      if ((tid & 31) == 0) atomicOr(b.err, kErrHang);
      ok = false;
    }
    if (!__syncthreads_and(ok)) break;                // every thread stops together
    tc::fence_after_sync();
    const long long pos = (t % tiles_per_head) * kRowsC + tid;
    const bool live = pos < m.Nq;
    const long long orow = live ? b.permQ[(long long)h * m.Nq + pos] : 0;
    uint4* dst = reinterpret_cast<uint4*>(Out + ((long long)h * m.Nq + orow) * D);
    const float* cv = b.cvec + (long long)h * D;
    const uint32_t ta = tmem + ((uint32_t)(32 * warp) << 16);
    const uint8_t* arow = gbase + kBTile + (uint32_t)s * kATile;
#pragma unroll 1
    for (int q = 0; q < NP; ++q) {                    // 32 output columns per step
      float dl[32];
      tc::tmem_ld32(ta + 32 * q, dl);
      tc::tmem_wait_ld();
      if (live) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float4 o = *reinterpret_cast<const float4*>(arow + q * kAPanel + tc::sw128_offset(tid, c));
          const float4 cc = __ldg(reinterpret_cast<const float4*>(cv + 32 * q + 4 * c));
          pk[2 * c] = tc::pack_bf16x2(o.x + cc.x + dl[4 * c], o.y + cc.y + dl[4 * c + 1]);
          pk[2 * c + 1] = tc::pack_bf16x2(o.z + cc.z + dl[4 * c + 2], o.w + cc.w + dl[4 * c + 3]);
        }
#pragma unroll
        for (int v = 0; v < 4; ++v)
          dst[4 * q + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      }
    }
    // the accumulator and stage s are free once every thread has read them: tile t+2's
    // copy goes there at once
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (t + 2 < t1) load_tile(t + 2, s);
    tc::cp_async_commit();
  }
  tc::cp_async_wait_all();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, D);
  }
}

template <int D>
sparsepr_status run_correct_tc(const Plan& p, void* Out, cudaStream_t st) {
  const Dims& m = p.dm;
  transpose_bp_kernel<<<dim3(cdiv(D, 32), cdiv(D, 32), m.H), dim3(32, 8), 0, st>>>(p.b.Bp, D, p.b.BpT);
  SPR_LAUNCH_OK();
  const int tph = cdiv(m.Nq, kRowsC);
  const long long total = (long long)tph * m.H;
  int dev = 0, sms = 148;
  SPR_CUDA_OK(cudaGetDevice(&dev));
  SPR_CUDA_OK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const int grid = (int)(total < sms ? total : sms);
  const size_t smem = (size_t)D * D * 4 + 2 * (size_t)kRowsC * D * 4 + 64 + 1024;
  SPR_CUDA_OK(cudaFuncSetAttribute(correct_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  correct_tc_kernel<D><<<grid, 128, smem, st>>>(m, p.b, p.b.BpT, static_cast<__nv_bfloat16*>(Out), tph, total);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

}  // namespace

bool correct_tc_applies(int dtype, int d, int engine) {
  return engine == SPARSEPR_ENGINE_AUTO && dtype == SPARSEPR_BF16 && (d == 64 || d == 128);
}

sparsepr_status launch_correct_tc(const Plan& p, void* Out, cudaStream_t st) {
  return p.dm.d == 64 ? run_correct_tc<64>(p, Out, st) : run_correct_tc<128>(p, Out, st);
}

}  // namespace spr
