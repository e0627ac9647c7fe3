// Attention on the 5th-generation tensor cores (tcgen05 + TMEM), bf16 in, fp32 accumulate.
//
// One CTA computes a 128-row query tile against a key sequence in 128-key tiles:
//   sparse  rows of one query group (group-major) against the concatenated key ranges of
//           the K/V groups selected for it: renormalised hard drop (paper S2);
//   dense   128 consecutive rows against all keys (the dense baseline, same engine);
//   probe   the M probe rows against one chunk of keys, written as partial
//           (max, sum, numerator) for a later combine (paper S4.2, App. A.2).
//
// Warp roles (288 threads):
//   warps 0-3  softmax: thread r owns query row r = TMEM lane r; reads S rows from TMEM,
//              online softmax in base 2, writes P (bf16) to shared memory, rescales the
//              O accumulator row in TMEM when the running max grows, final epilogue;
//   warps 4-7  producers: 16-byte cp.async gathers of the Q tile and of each K/V tile
//              (arbitrary key rows: the selected groups need not be contiguous) into
//              128-byte-swizzled shared memory, two stages;
//   warp 8     one thread issues tcgen05.mma: S_j = Q K_j^T into one of two TMEM S
//              buffers, O += P_j V_j into the TMEM accumulator (V read MN-major), with
//              tcgen05.commit arriving on mbarriers.  The warp owns the TMEM allocation.
// Issue order S_0, S_1, PV_0, S_2, PV_1, ... keeps the tensor cores busy with S_{j+1}
// while the softmax warps work on tile j.
//
// Every mbarrier wait is bounded: on timeout the CTA records kErrHang, all roles stop,
// the MMA thread drains its outstanding MMAs and the TMEM is freed before returning.
#include <cmath>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace spr {
namespace {

constexpr int kTileRows = 128;
constexpr int kTileKeys = 128;
constexpr int kTcThreads = 288;
constexpr long long kWaitCycles = 2000000000LL;   // about one second: a hung pipeline

enum Mode { kModeSparse = 0, kModeDense = 1, kModeProbe = 2 };

// Error word of the workspace-free dense entry point.
__device__ int g_dense_err;

struct TcArgs {
  int mode;
  Dims m;
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  Buffers b;
  const int* work;     // sparse: [H][max_items] (a << 16 | tile)
  const int* nwork;    // sparse: [H]
  int max_items;
  void* out;           // dense: output in the input dtype
  int* err;
};

template <int D>
struct Layout {
  static constexpr uint32_t kTile = kTileRows * D * 2;         // bytes of a Q/K/V tile
  static constexpr uint32_t kPanel = kTileRows * 128;          // one 64-column panel
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oK0 = kTile, oK1 = 2 * kTile;
  static constexpr uint32_t oV0 = 3 * kTile, oV1 = 4 * kTile;
  static constexpr uint32_t oP = 5 * kTile;                    // 128 x 128 bf16 = 32 KB
  static constexpr uint32_t oMisc = oP + 2 * kPanel;
  static constexpr uint32_t kBytes = oMisc + 12 * 1024;
};

struct Misc {
  unsigned long long bars[16];
  long long qrow[kTileRows];
  long long krow[2][kTileKeys];
  int csum[kMaxC + 1];
  int cbase[kMaxC];
  uint32_t tmem_base;
  int abort_flag;
  int sh[32];
};

enum Bar { bQFull = 0, bFull0 = 1, bEmpty0 = 3, bSFull0 = 5, bSFree0 = 7, bPFull = 9, bPvDone = 10, bDrain = 11 };

__device__ __forceinline__ bool wait_bar(Misc* ms, uint32_t bar, uint32_t parity, int* err) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!tc::mbar_try_wait(bar, parity)) {
    if (*reinterpret_cast<volatile int*>(&ms->abort_flag)) return false;
    if (clock64() - t0 > kWaitCycles) {
      if (atomicExch(&ms->abort_flag, 1) == 0) atomicOr(err, kErrHang);
      return false;
    }
  }
  return true;
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) attention_tc_kernel(TcArgs g) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  Misc* ms = reinterpret_cast<Misc*>(gbase + L::oMisc);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Dims& m = g.m;
  const int h = blockIdx.y, d = m.d;

  // ---------------------------------------------------------------- work item
  int q0 = 0, nrows = 0, split = 0;
  long long nkeys = 0;
  int cnt = 0;
  if (g.mode == kModeSparse) {
    if ((int)blockIdx.x >= g.nwork[h]) return;
    const int item = g.work[(long long)h * g.max_items + blockIdx.x];
    const int a = item >> 16, t = item & 0xFFFF;
    const int labq = g.b.usedQ[(long long)h * m.Cq + a];
    const int gs = g.b.offQ[(long long)h * (m.Cq + 1) + labq];
    const int ge = g.b.offQ[(long long)h * (m.Cq + 1) + labq + 1];
    q0 = gs + t * kTileRows;
    nrows = min(kTileRows, ge - q0);
    cnt = g.b.cellCnt[(long long)h * m.Cq + a];
    const int* ids = g.b.cellIds + ((long long)h * m.Cq + a) * m.Ck;
    for (int base_i = 0; base_i < cnt; base_i += blockDim.x) {
      const int i = base_i + tid;
      int sz = 0, start = 0;
      if (i < cnt) {
        const int labk = g.b.usedK[(long long)h * m.Ck + ids[i]];
        start = g.b.offK[(long long)h * (m.Ck + 1) + labk];
        sz = g.b.offK[(long long)h * (m.Ck + 1) + labk + 1] - start;
      }
      int tot;
      const int ex = block_exclusive_scan(sz, ms->sh, &tot);
      const int prev = base_i == 0 ? 0 : ms->csum[base_i];
      if (i < cnt) {
        ms->csum[i] = prev + ex;
        ms->cbase[i] = start;
      }
      __syncthreads();
      if (tid == 0) ms->csum[min(base_i + (int)blockDim.x, cnt)] = prev + tot;
      __syncthreads();
    }
    nkeys = ms->csum[cnt];
  } else if (g.mode == kModeDense) {
    q0 = blockIdx.x * kTileRows;
    nrows = min(kTileRows, m.Nq - q0);
    nkeys = m.Nk;
  } else {
    split = blockIdx.x;
    const long long k0 = (long long)split * kProbeSplit;
    nkeys = min((long long)kProbeSplit, (long long)m.Nk - k0);
    nrows = m.M;
  }
  const int nt = (int)((nkeys + kTileKeys - 1) / kTileKeys);
  const int last_valid = (int)(nkeys - (long long)(nt - 1) * kTileKeys);

  // ---------------------------------------------------------------- setup
  const uint32_t bars = tc::smem_u32(ms->bars);
  auto BAR = [&](int i) -> uint32_t { return bars + 8u * i; };
  if (tid == 0) {
    tc::mbar_init(BAR(bQFull), 128);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(BAR(bFull0 + s), 128);
      tc::mbar_init(BAR(bEmpty0 + s), 1);
      tc::mbar_init(BAR(bSFull0 + s), 1);
      tc::mbar_init(BAR(bSFree0 + s), 128);
    }
    tc::mbar_init(BAR(bPFull), 128);
    tc::mbar_init(BAR(bPvDone), 1);
    tc::mbar_init(BAR(bDrain), 1);
    ms->abort_flag = 0;
  }
  if (warp == 8) {
    tc::tmem_alloc(tc::smem_u32(&ms->tmem_base), 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = ms->tmem_base;
  const uint32_t tS0 = tmem, tS1 = tmem + 128, tO = tmem + 256;

  const uint32_t sQ = base + L::oQ, sP = base + L::oP;
  const uint32_t sK[2] = {base + L::oK0, base + L::oK1};
  const uint32_t sV[2] = {base + L::oV0, base + L::oV1};

  if (warp >= 4 && warp < 8) {
    // ============================================================ producers
    const int p = tid - 128;
    const long long hq = (long long)h * m.Nq * d, hk = (long long)h * m.Nk * d;
    // query row p
    long long qr = -1;
    if (p < nrows) {
      if (g.mode == kModeProbe) qr = hq + (long long)g.b.probes[(long long)h * m.M + p] * d;
      else qr = hq + (long long)(q0 + p) * d;
    }
    ms->qrow[p] = qr;
    tc::named_sync(1, 128);
    constexpr int CPR = D / 8;                // 16-byte chunks per row
    for (int e = p; e < kTileRows * CPR; e += 128) {
      const int row = e / CPR, c = e % CPR;
      const long long off = ms->qrow[row];
      const uint32_t dst = sQ + (c >> 3) * L::kPanel + tc::sw128_offset(row, c & 7);
      tc::cp_async16(dst, off >= 0 ? (const void*)(g.Q + off + c * 8) : (const void*)g.Q, off >= 0 ? 16u : 0u);
    }
    tc::cp_async_commit();
    tc::cp_async_wait_all();
    tc::fence_proxy_async();
    tc::mbar_arrive(BAR(bQFull));
    for (int j = 0; j < nt; ++j) {
      const int s = j & 1;
      // every producer thread takes the same decision (they meet at named barriers)
      const bool got = j < 2 || wait_bar(ms, BAR(bEmpty0 + s), ((j >> 1) + 1) & 1, g.err);
      if (!tc::named_sync_and(1, 128, got)) break;
      const long long v = (long long)j * kTileKeys + p;
      long long kr = -1;
      if (v < nkeys) {
        if (g.mode == kModeSparse) {
          int lo = 0, hi = cnt - 1;
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (ms->csum[mid] <= v) lo = mid; else hi = mid - 1;
          }
          kr = hk + ((long long)ms->cbase[lo] + (v - ms->csum[lo])) * d;
        } else if (g.mode == kModeDense) {
          kr = hk + v * d;
        } else {
          kr = hk + ((long long)split * kProbeSplit + v) * d;
        }
      }
      ms->krow[s][p] = kr;
      tc::named_sync(1, 128);
      for (int e = p; e < kTileKeys * CPR; e += 128) {
        const int row = e / CPR, c = e % CPR;
        const long long off = ms->krow[s][row];
        const uint32_t o = (c >> 3) * L::kPanel + tc::sw128_offset(row, c & 7);
        const bool ok = off >= 0;
        tc::cp_async16(sK[s] + o, ok ? (const void*)(g.K + off + c * 8) : (const void*)g.K, ok ? 16u : 0u);
        tc::cp_async16(sV[s] + o, ok ? (const void*)(g.V + off + c * 8) : (const void*)g.V, ok ? 16u : 0u);
      }
      tc::cp_async_commit();
      tc::cp_async_wait_all();
      tc::fence_proxy_async();
      tc::mbar_arrive(BAR(bFull0 + s));
    }
    tc::cp_async_wait_all();
  } else if (warp == 8) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idQK = tc::idesc_bf16_f32(kTileRows, kTileKeys, false);
      constexpr uint32_t idPV = tc::idesc_bf16_f32(kTileRows, D, true);
      bool ok = wait_bar(ms, BAR(bQFull), 0, g.err);
      auto issue_pv = [&](int j) -> bool {
        if (!wait_bar(ms, BAR(bPFull), j & 1, g.err)) return false;
        tc::fence_after_sync();
        const int s = j & 1;
#pragma unroll
        for (int kk = 0; kk < kTileKeys / 16; ++kk) {
          const uint64_t ad = tc::sw128_desc(sP + (kk >> 2) * L::kPanel + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = tc::sw128_desc(sV[s] + kk * 2048, L::kPanel, 1024);
          tc::mma_ss(tO, ad, bd, idPV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(BAR(bPvDone));
        tc::mma_commit(BAR(bEmpty0 + s));
        return true;
      };
      for (int j = 0; ok && j < nt; ++j) {
        const int s = j & 1;
        if (!wait_bar(ms, BAR(bFull0 + s), (j >> 1) & 1, g.err)) { ok = false; break; }
        if (j >= 2 && !wait_bar(ms, BAR(bSFree0 + s), ((j >> 1) + 1) & 1, g.err)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t tS = s ? tS1 : tS0;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = tc::sw128_desc(sQ + (kk >> 2) * L::kPanel + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = tc::sw128_desc(sK[s] + (kk >> 2) * L::kPanel + (kk & 3) * 32, 16, 1024);
          tc::mma_ss(tS, ad, bd, idQK, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(BAR(bSFull0 + s));
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(nt - 1);
      tc::mma_commit(BAR(bDrain));
      // bounded: completes when every MMA issued above has finished
      const long long t0 = clock64();
      while (!tc::mbar_try_wait(BAR(bDrain), 0)) {
        if (clock64() - t0 > kWaitCycles) { atomicOr(g.err, kErrHang); break; }
      }
    }
    __syncwarp();
  } else {
    // ============================================================ softmax / epilogue
    const int r = tid;                                  // query row = TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    const float sl2 = 1.4426950408889634f / sqrtf((float)d);
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    // tcgen05.ld/st are warp-collective (.sync.aligned): every branch around them below
    // is uniform across the warp, including the outcome of bounded waits.
    for (int j = 0; j < nt; ++j) {
      const int s = j & 1;
      if (!__all_sync(0xffffffffu, wait_bar(ms, BAR(bSFull0 + s), (j >> 1) & 1, g.err))) { ok = false; break; }
      tc::fence_after_sync();
      const uint32_t tS = (s ? tS1 : tS0) + lane_off;
      const int valid = (j == nt - 1) ? last_valid : kTileKeys;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tc::tmem_ld32(tS + 32 * c, v);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (32 * c + i < valid) mx = fmaxf(mx, v[i]);
      }
      const float m_new = fmaxf(m_run, mx * sl2);
      // PV of the previous tile must be complete: P is reused and O is rescaled below
      if (j >= 1) {
        if (!__all_sync(0xffffffffu, wait_bar(ms, BAR(bPvDone), (j - 1) & 1, g.err))) { ok = false; break; }
        tc::fence_after_sync();
      }
      const float alpha = exp2f(m_run - m_new);         // 0 on the first tile, 1 if unchanged
      if (j >= 1 && __any_sync(0xffffffffu, m_new > m_run)) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tc::tmem_ld32(tO + lane_off + 32 * c, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tc::tmem_st32(tO + lane_off + 32 * c, o);
        }
        tc::tmem_wait_st();
      }
      float rs = 0.0f;
      uint8_t* prow = gbase + L::oP;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tc::tmem_ld32(tS + 32 * c, v);
        tc::tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = (32 * c + 2 * i < valid) ? exp2f(fmaf(v[2 * i], sl2, -m_new)) : 0.0f;
          const float p1 = (32 * c + 2 * i + 1 < valid) ? exp2f(fmaf(v[2 * i + 1], sl2, -m_new)) : 0.0f;
          rs += p0 + p1;
          const __nv_bfloat162 bb = __floats2bfloat162_rn(p0, p1);
          pk[i] = *reinterpret_cast<const uint32_t*>(&bb);
        }
        // columns 32c..32c+31 = four 16-byte chunks of panel (c >> 1)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t chunk = (uint32_t)((c & 1) * 4 + q);
          uint4* dst = reinterpret_cast<uint4*>(prow + (c >> 1) * L::kPanel + tc::sw128_offset(r, chunk));
          *dst = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      tc::fence_before_sync();
      tc::mbar_arrive(BAR(bSFree0 + s));
      l_run = l_run * alpha + rs;
      m_run = m_new;
      tc::fence_proxy_async();
      tc::fence_before_sync();
      tc::mbar_arrive(BAR(bPFull));
    }
    if (ok && __all_sync(0xffffffffu, wait_bar(ms, BAR(bPvDone), (nt - 1) & 1, g.err))) {
      tc::fence_after_sync();
      const float inv = 1.0f / l_run;
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tc::tmem_ld32(tO + lane_off + 32 * c, o);
        tc::tmem_wait_ld();
        if (r < nrows) {
          if (g.mode == kModeSparse) {
            float4* dst = reinterpret_cast<float4*>(g.b.Osp + ((long long)h * m.Nq + q0 + r) * d + 32 * c);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv, o[4 * i + 3] * inv);
          } else if (g.mode == kModeDense) {
            const long long ob = ((long long)h * m.Nq + q0 + r) * d + 32 * c;
            if (m.dtype == SPARSEPR_BF16) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const __nv_bfloat162 bb = __floats2bfloat162_rn(o[2 * i] * inv, o[2 * i + 1] * inv);
                pk[i] = *reinterpret_cast<const uint32_t*>(&bb);
              }
              uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(g.out) + ob);
#pragma unroll
              for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
          } else {
            const long long slot = ((long long)h * m.M + r) * m.nsplit + split;
            float4* dst = reinterpret_cast<float4*>(g.b.Opart + slot * d + 32 * c);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
            if (c == 0) {
              g.b.MLpart[2 * slot] = m_run * 0.6931471805599453f;   // back to natural-log scale
              g.b.MLpart[2 * slot + 1] = l_run;
            }
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 8) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// Work list of the sparse mode: one item per 128-row tile of every non-empty query group.
__global__ void __launch_bounds__(1024) build_work_kernel(Dims m, Buffers b, int* work, int* nwork,
                                                          int max_items) {
  __shared__ int sh[32];
  const int h = blockIdx.x, a = threadIdx.x;
  const int n = b.nQ[h];
  const int tiles = a < n ? (b.sizeQ[(long long)h * m.Cq + a] + kTileRows - 1) / kTileRows : 0;
  int tot;
  const int off = block_exclusive_scan(tiles, sh, &tot);
  for (int t = 0; t < tiles; ++t) work[(long long)h * max_items + off + t] = (a << 16) | t;
  if (threadIdx.x == 0) nwork[h] = tot;
}

template <int D>
sparsepr_status launch_tc(const TcArgs& args, dim3 grid, cudaStream_t st) {
  const size_t smem = Layout<D>::kBytes + 1024;
  SPR_CUDA_OK(cudaFuncSetAttribute(attention_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  attention_tc_kernel<D><<<grid, kTcThreads, smem, st>>>(args);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

template <class F>
sparsepr_status with_tc_d(int d, F f) {
  if (d == 64) return f(std::integral_constant<int, 64>());
  return f(std::integral_constant<int, 128>());
}

}  // namespace

bool tc_engine_applies(int dtype, int d, int engine) {
  return engine == SPARSEPR_ENGINE_AUTO && dtype == SPARSEPR_BF16 && (d == 64 || d == 128);
}

int tc_max_items(const Dims& m) { return m.Cq + cdiv(m.Nq, kTileRows); }

sparsepr_status launch_sparse_attention_tc(const Plan& p, cudaStream_t st) {
  const Dims& m = p.dm;
  const int max_items = tc_max_items(m);
  build_work_kernel<<<m.H, 1024, 0, st>>>(m, p.b, p.b.work, p.b.nwork, max_items);
  SPR_LAUNCH_OK();
  TcArgs a{};
  a.mode = kModeSparse;
  a.m = m;
  a.Q = reinterpret_cast<const __nv_bfloat16*>(p.b.Qp);
  a.K = reinterpret_cast<const __nv_bfloat16*>(p.b.Kp);
  a.V = reinterpret_cast<const __nv_bfloat16*>(p.b.Vp);
  a.b = p.b;
  a.work = p.b.work;
  a.nwork = p.b.nwork;
  a.max_items = max_items;
  a.err = p.b.err;
  return with_tc_d(m.d, [&](auto DD) { return launch_tc<decltype(DD)::value>(a, dim3(max_items, m.H), st); });
}

sparsepr_status launch_probe_attention_tc(const Plan& p, cudaStream_t st) {
  const Dims& m = p.dm;
  TcArgs a{};
  a.mode = kModeProbe;
  a.m = m;
  a.Q = reinterpret_cast<const __nv_bfloat16*>(p.Q);
  a.K = reinterpret_cast<const __nv_bfloat16*>(p.K);
  a.V = reinterpret_cast<const __nv_bfloat16*>(p.V);
  a.b = p.b;
  a.err = p.b.err;
  return with_tc_d(m.d, [&](auto DD) { return launch_tc<decltype(DD)::value>(a, dim3(m.nsplit, m.H), st); });
}

sparsepr_status launch_dense_attention_tc(const Dims& m, const void* Q, const void* K, const void* V,
                                          void* Out, int* err, cudaStream_t st) {
  TcArgs a{};
  a.mode = kModeDense;
  a.m = m;
  a.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  a.K = reinterpret_cast<const __nv_bfloat16*>(K);
  a.V = reinterpret_cast<const __nv_bfloat16*>(V);
  a.out = Out;
  a.err = err;
  if (!a.err) SPR_CUDA_OK(cudaGetSymbolAddress(reinterpret_cast<void**>(&a.err), g_dense_err));
  return with_tc_d(m.d, [&](auto DD) { return launch_tc<decltype(DD)::value>(a, dim3(cdiv(m.Nq, kTileRows), m.H), st); });
}

}  // namespace spr
