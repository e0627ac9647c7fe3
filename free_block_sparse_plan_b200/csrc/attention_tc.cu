// Attention on the 5th-generation tensor cores (tcgen05 + TMEM), bf16 in, fp32 accumulate.
//
// One CTA computes up to two 128-row query tiles (A, B) against one key sequence in
// 128-key tiles:
//   sparse  rows of one query group (group-major) against the concatenated key ranges of
//           the K/V groups selected for it: renormalised hard drop (paper S2);
//   dense   256 consecutive rows against all keys (the dense baseline, same engine);
//   probe   the M probe rows against one chunk of keys, written as partial
//           (max, sum, numerator) for a later combine (paper S4.2, App. A.2).
//
// Warp roles (384 threads; twelve warps so each SM sub-partition holds three):
//   warps 0-3, 4-7  softmax of tile A, of tile B (or, for an item of one query tile and
//              several key tiles, of the even and the odd key tiles of that tile, merged
//              at the end): thread r owns query row r = TMEM lane r; reads its S row from
//              TMEM, online softmax in base 2 with lazy rescaling (O is rescaled only when
//              the row max grows by more than 2^8), writes P as bf16 pairs into the TMEM
//              columns of S already read, epilogue;
//   warps 8-10 producers: 16-byte cp.async gathers of the Q tiles; then one thread copies
//              K tiles and another V tiles into their stages (two at d = 128, four at
//              d = 64).  Dense and probe keys are consecutive rows: TMA boxes of 64 rows
//              from a 3-D tensor map.  Sparse keys are the concatenated runs of the
//              selected K/V groups in the tensor-core K/V layout (each group padded with
//              zero rows to a multiple of 8, panels stored in shared-memory swizzle order),
//              one bulk copy per run and panel; the K thread also publishes each tile's
//              padding columns in a ring of mask slots;
//   warp 11    one thread issues tcgen05.mma: S_t = Q_t K_j^T (both operands in shared
//              memory) and O_t += P_t V_j (P read from TMEM, V MN-major), and commits to
//              mbarriers (K stages are released after the S products, V stages after the
//              PV products).  The warp owns the TMEM allocation: two S buffers and two O
//              accumulators (128 columns each).
// Issue order per key tile with two query tiles: PV_A(j), S_A(j+1), PV_B(j), S_B(j+1): the
// softmax of one tile overlaps the matrix products of the other.  tcgen05.commit arrives
// only when every earlier tcgen05 operation of the thread is complete, so "S_t(j) ready"
// also certifies that PV_t(j-1) has finished reading P_t and updating O_t.
//
// Every mbarrier wait is bounded: on timeout the CTA records kErrHang, all roles stop,
// the MMA thread drains its outstanding MMAs and the TMEM is freed before returning.
// Warp-collective TMEM loads/stores sit only in warp-uniform control flow.
#include <cmath>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace spr {
namespace {

constexpr int kTileRows = 128;
constexpr int kTileKeys = 128;
constexpr int kItemRows = 2 * kTileRows;
constexpr int kTcThreads = 384;
constexpr int kProducers = 96;                   // warps 8-10
constexpr long long kWaitCycles = 2000000000LL;   // about one second: a hung pipeline
constexpr float kRescaleLog2 = 8.0f;              // lazy rescale threshold (factor 256)
constexpr int kPolyPairs = 6;                     // of every 16 column pairs: exp2 on the FMA pipe

enum Mode { kModeSparse = 0, kModeDense = 1, kModeProbe = 2 };

// Error word of sparsepr_dense_attention (no plan, no workspace): sticky until
// sparsepr_dense_check reads and clears it.
__device__ int g_dense_err;

struct TcArgs {
  // dense and probe modes: K and V as [H_k][N_k][d] bf16 in boxes of 64 columns x 64 rows
  // (128-byte swizzle; rows past N_k read as zeros)
  CUtensorMap tm_k, tm_v;
  int mode;
  Dims m;
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  Buffers b;
  const int* work;     // sparse: [H][max_items] (a << 16 | item)
  const int* nwork;    // sparse: [H]
  int max_items;
  void* out;           // dense: output in the input dtype
  int* err;
};

// Shared memory: two Q tiles, then S stages of K tiles and S stages of V tiles (four
// stages at d = 64, where the tiles are small; two at d = 128), then bookkeeping.
template <int D>
struct Layout {
  static constexpr int S = D == 64 ? 4 : 2;
  static constexpr uint32_t kTile = kTileRows * D * 2;         // bytes of a Q/K/V tile
  static constexpr uint32_t kPanel = kTileRows * 128;          // one 64-column panel
  static constexpr uint32_t oQ0 = 0;
  static constexpr uint32_t oK0 = 2 * kTile;
  static constexpr uint32_t oV0 = (2 + S) * kTile;
  static constexpr uint32_t oMisc = (2 + 2 * S) * kTile;
  static constexpr uint32_t kBytes = oMisc + 17 * 1024;
};

struct Misc {
  unsigned long long bars[34];
  long long qrow[kItemRows];
  int csum[kMaxC + 1];        // sparse: key position of each selected range (multiples of 8)
  int cbase[kMaxC];           // its first row in the tensor-core K/V layout of the head
  int clen[kMaxC];            // its true length (the rest up to the next position is padding)
  uint32_t kvmask[8][4];      // sparse: key columns that are padding, tile j in slot j % 2S
  float xm[2][kTileRows];     // alternating mode: running max and sum of each half
  float xl[2][kTileRows];
  uint32_t tmem_base;
  int abort_flag;
  int sh[32];
};

static_assert(sizeof(Misc) <= 17 * 1024, "bookkeeping exceeds its shared-memory slot");

enum Bar {
  bQFull = 0, bKFull0 = 1, bKEmpty0 = 5, bSFull0 = 9, bPFull0 = 11, bPvDone0 = 13, bDrain = 15, bOReady = 16,
  bVFull0 = 17, bVEmpty0 = 21, bMask0 = 25
};

// Bounded wait; the clock and the abort flag are read once every 32 polls so that
// waiting warps take few issue slots from the working ones.
__device__ __forceinline__ bool wait_bar(Misc* ms, uint32_t bar, uint32_t parity, int* err) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (unsigned n = 1;; ++n) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    if ((n & 31) == 0) {
      if (*reinterpret_cast<volatile int*>(&ms->abort_flag)) return false;
      if (clock64() - t0 > kWaitCycles) {
        if (atomicExch(&ms->abort_flag, 1) == 0) atomicOr(err, kErrHang);
        return false;
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) attention_tc_kernel(const __grid_constant__ TcArgs g) {
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
    q0 = gs + t * kItemRows;
    nrows = min(kItemRows, ge - q0);
    cnt = g.b.cellCnt[(long long)h * m.Cq + a];
    const int* ids = g.b.cellIds + ((long long)h * m.Cq + a) * m.Ck;
    for (int base_i = 0; base_i < cnt; base_i += blockDim.x) {
      const int i = base_i + tid;
      int sz = 0, start = 0;
      if (i < cnt) {
        const int labk = g.b.usedK[(long long)(h / m.G) * m.Ck + ids[i]];
        const long long o = (long long)(h / m.G) * (m.Ck + 1) + labk;
        start = g.b.poffK[o];
        sz = g.b.offK[o + 1] - g.b.offK[o];
      }
      int tot;
      const int ex = block_exclusive_scan((sz + 7) & ~7, ms->sh, &tot);   // padded to 8
      const int prev = base_i == 0 ? 0 : ms->csum[base_i];
      if (i < cnt) {
        ms->csum[i] = prev + ex;
        ms->cbase[i] = start;
        ms->clen[i] = sz;
      }
      __syncthreads();
      if (tid == 0) ms->csum[min(base_i + (int)blockDim.x, cnt)] = prev + tot;
      __syncthreads();
    }
    nkeys = ms->csum[cnt];
  } else if (g.mode == kModeDense) {
    q0 = blockIdx.x * kItemRows;
    nrows = min(kItemRows, m.Nq - q0);
    nkeys = m.Nk;
  } else {
    split = blockIdx.x;
    const long long k0 = (long long)split * kProbeSplit;
    nkeys = min((long long)kProbeSplit, (long long)m.Nk - k0);
    nrows = m.M;
  }
  const int nt = (int)((nkeys + kTileKeys - 1) / kTileKeys);
  const int last_valid = (int)(nkeys - (long long)(nt - 1) * kTileKeys);
  const bool hasB = nrows > kTileRows;
  // one query tile and two or more key tiles: the even and the odd key tiles go to two
  // softmax warp groups with their own S buffer, running max and O accumulator, merged at
  // the end, so that one group's softmax overlaps the other's products
  const bool alt = !hasB && nt >= 2;

  // ---------------------------------------------------------------- setup
  const uint32_t bars = tc::smem_u32(ms->bars);
  auto BAR = [&](int i) -> uint32_t { return bars + 8u * i; };
  if (tid == 0) {
    tc::mbar_init(BAR(bQFull), kProducers);
    for (int s = 0; s < L::S; ++s) {
      tc::mbar_init(BAR(bKFull0 + s), 1);             // the copying thread's arrive + bytes
      tc::mbar_init(BAR(bKEmpty0 + s), 1);
      tc::mbar_init(BAR(bVFull0 + s), 1);
      tc::mbar_init(BAR(bVEmpty0 + s), 1);
    }
    for (int q = 0; q < 2 * L::S; ++q) tc::mbar_init(BAR(bMask0 + q), 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(BAR(bSFull0 + s), 1);
      tc::mbar_init(BAR(bPFull0 + s), 128);
      tc::mbar_init(BAR(bPvDone0 + s), 1);
    }
    tc::mbar_init(BAR(bDrain), 1);
    tc::mbar_init(BAR(bOReady), 1);
    ms->abort_flag = 0;
  }
  if (warp == 11) {
    tc::tmem_alloc(tc::smem_u32(&ms->tmem_base), 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = ms->tmem_base;

  // tile addresses: Q tile t, K stage s, V stage s (consecutive tiles of kTile bytes)
  auto sQ = [&](int t) -> uint32_t { return base + L::oQ0 + (uint32_t)t * L::kTile; };
  auto sK = [&](int s) -> uint32_t { return base + L::oK0 + (uint32_t)s * L::kTile; };
  auto sV = [&](int s) -> uint32_t { return base + L::oV0 + (uint32_t)s * L::kTile; };

  if (warp >= 8 && warp < 11) {
    // ============================================================ producers
    const int p = tid - 256;
    const long long hq = (long long)h * m.Nq * d;
    for (int row = p; row < kItemRows; row += kProducers) {
      long long qr = -1;
      if (row < nrows) {
        if (g.mode == kModeProbe) qr = hq + (long long)g.b.probes[(long long)h * m.M + row] * d;
        else qr = hq + (long long)(q0 + row) * d;
      }
      ms->qrow[row] = qr;
    }
    tc::named_sync(1, kProducers);
    constexpr int CPR = D / 8;                // 16-byte chunks per row
    for (int e = p; e < kItemRows * CPR; e += kProducers) {
      const int row = e / CPR, c = e % CPR;
      const long long off = ms->qrow[row];
      const uint32_t dst = sQ(row >> 7) + (c >> 3) * L::kPanel + tc::sw128_offset(row & 127, c & 7);
      tc::cp_async16(dst, off >= 0 ? (const void*)(g.Q + off + c * 8) : (const void*)g.Q, off >= 0 ? 16u : 0u);
    }
    tc::cp_async_commit();
    tc::cp_async_wait_all();
    tc::fence_proxy_async();
    tc::mbar_arrive(BAR(bQFull));
    // K and V tiles: stage j % S, K copied by one thread and V by another, each stage
    // refilled as soon as the products reading it have finished (K after the S products,
    // V after the PV products).  Sparse mode: one bulk copy per panel of every run of rows
    // (the tensor-core layout holds each panel's rows in the order of the shared-memory
    // tile, runs start at multiples of 8 rows on both sides); the rest of the last tile
    // comes from the head's zero rows.  Dense and probe modes: TMA boxes of 64 rows (rows
    // past N_k read as zeros; past the item's keys, the softmax masks them).  Every row of
    // a stage is written, so its byte count is fixed.
    if (p == 0 || p == 32) {
      const bool isK = p == 0;
      const int hk = h / m.G;                             // the K/V head
      constexpr int NP = D / 64;
      const long long rp = kv_tiled_rows(m.Nk, m.Ck);
      const uint8_t* src_base = reinterpret_cast<const uint8_t*>(isK ? g.K : g.V) + (long long)hk * NP * rp * 128;
      const CUtensorMap* tmap = isK ? &g.tm_k : &g.tm_v;
      const int zrow = g.mode == kModeSparse ? g.b.poffK[(long long)hk * (m.Ck + 1) + m.Ck] : 0;
      const int full0 = isK ? bKFull0 : bVFull0, empty0 = isK ? bKEmpty0 : bVEmpty0;
      int c = 0;                                          // sparse: current range
      for (int j = 0; j < nt; ++j) {
        const int s = j % L::S, use = j / L::S;
        if (use > 0 && !wait_bar(ms, BAR(empty0 + s), (use - 1) & 1, g.err)) break;
        const uint32_t bar = BAR(full0 + s);
        const uint32_t tile = isK ? sK(s) : sV(s);
        const int t0 = j * kTileKeys;
        if (g.mode == kModeSparse) {
          // rows [src, src + len) of the layout into tile rows [dst, dst + len)
          auto copy_run = [&](long long src, int dst, int len) {
#pragma unroll
            for (int pnl = 0; pnl < NP; ++pnl)
              tc::bulk_g2s(tile + pnl * L::kPanel + (uint32_t)dst * 128u, src_base + ((long long)pnl * rp + src) * 128,
                           (uint32_t)len * 128u, bar);
          };
          while (c < cnt && ms->csum[c + 1] <= t0) ++c;
          tc::mbar_add_tx(bar, L::kTile);
          int pos = t0;                                   // next tile position to fill
          for (int cc = c; cc < cnt && ms->csum[cc] < t0 + kTileKeys; ++cc) {
            const int lo = max(ms->csum[cc], t0), hi = min(ms->csum[cc + 1], t0 + kTileKeys);
            copy_run(ms->cbase[cc] + (lo - ms->csum[cc]), lo - t0, hi - lo);
            pos = hi;
          }
          if (pos < t0 + kTileKeys) copy_run(zrow, pos - t0, t0 + kTileKeys - pos);
          tc::mbar_arrive(bar);
          if (isK) {
            // the padding columns of this tile into mask slot j % 2S, published by that
            // slot's barrier (an arrive is a release).  The slot's previous tile, j - 2S,
            // was read by its softmax warps before the S products of tile j - S were
            // issued, and this thread has waited for those products to finish
            const int slot = j % (2 * L::S);
            uint32_t* mask = ms->kvmask[slot];
#pragma unroll
            for (int q = 0; q < 4; ++q) mask[q] = 0u;
            for (int cc = c; cc < cnt && ms->csum[cc] < t0 + kTileKeys; ++cc) {
              const int hi = min(ms->csum[cc + 1], t0 + kTileKeys);
              for (int q = max(ms->csum[cc] + ms->clen[cc], t0); q < hi; ++q) mask[(q - t0) >> 5] |= 1u << ((q - t0) & 31);
            }
            tc::mbar_arrive(BAR(bMask0 + slot));
          }
        } else {
          tc::mbar_expect_tx(bar, L::kTile);
          const int first = (g.mode == kModeProbe ? split * kProbeSplit : 0) + t0;
#pragma unroll
          for (int half = 0; half < 2; ++half)
#pragma unroll
            for (int pnl = 0; pnl < NP; ++pnl)
              tc::tma_load_3d(tile + pnl * L::kPanel + (uint32_t)half * 64u * 128u, tmap, 64 * pnl, first + 64 * half, hk, bar);
        }
      }
    }
    tc::cp_async_wait_all();
  } else if (warp == 11) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idQK = tc::idesc_bf16_f32(kTileRows, kTileKeys, false);
      constexpr uint32_t idPV = tc::idesc_bf16_f32(kTileRows, D, true);
      // S of query tile t against key tile j into S buffer `buf` (TMEM columns 128 buf)
      auto issue_s = [&](int t, int j, int buf) {
        const int s = j % L::S;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = tc::sw128_desc(sQ(t) + (kk >> 2) * L::kPanel + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = tc::sw128_desc(sK(s) + (kk >> 2) * L::kPanel + (kk & 3) * 32, 16, 1024);
          tc::mma_ss(tmem + 128 * buf, ad, bd, idQK, kk > 0 ? 1u : 0u);
        }
        tc::mma_commit(BAR(bSFull0 + buf));
      };
      // O_t += P V_j with P in S buffer `buf`
      auto issue_pv = [&](int t, int j, int buf, bool acc) {
        const int s = j % L::S;
#pragma unroll
        for (int kk = 0; kk < kTileKeys / 16; ++kk) {
          const uint64_t bd = tc::sw128_desc(sV(s) + kk * 2048, L::kPanel, 1024);
          tc::mma_ts(tmem + 256 + 128 * t, tmem + 128 * buf + 8 * kk, bd, idPV, (acc || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(BAR(bPvDone0 + t));
      };
      // K or V stage j % S, fill j / S
      auto k_ready = [&](int j) -> bool {
        if (!wait_bar(ms, BAR(bKFull0 + j % L::S), (j / L::S) & 1, g.err)) return false;
        tc::fence_after_sync();
        return true;
      };
      auto v_ready = [&](int j) -> bool {
        if (!wait_bar(ms, BAR(bVFull0 + j % L::S), (j / L::S) & 1, g.err)) return false;
        tc::fence_after_sync();
        return true;
      };
      bool ok = wait_bar(ms, BAR(bQFull), 0, g.err) && k_ready(0);
      if (hasB) {
        // two query tiles: the softmax of one overlaps the products of the other
        if (ok) {
          issue_s(0, 0, 0);
          issue_s(1, 0, 1);
          tc::mma_commit(BAR(bKEmpty0));
        }
        for (int j = 0; ok && j < nt; ++j) {
          if (!wait_bar(ms, BAR(bPFull0), j & 1, g.err) || !v_ready(j)) { ok = false; break; }
          issue_pv(0, j, 0, j > 0);
          const bool more = j + 1 < nt;
          if (more) {
            if (!k_ready(j + 1)) { ok = false; break; }
            issue_s(0, j + 1, 0);
          }
          if (!wait_bar(ms, BAR(bPFull0 + 1), j & 1, g.err)) { ok = false; break; }
          tc::fence_after_sync();
          issue_pv(1, j, 1, j > 0);
          tc::mma_commit(BAR(bVEmpty0 + j % L::S));
          if (more) {
            issue_s(1, j + 1, 1);
            tc::mma_commit(BAR(bKEmpty0 + (j + 1) % L::S));
          }
        }
      } else {
        // one query tile, S alternating between the two S buffers so that S(j+1) is ready
        // while the softmax of tile j runs.  Alternating mode: key tile j also into O
        // accumulator j & 1, with its own softmax warp group; S(j+2) follows PV(j) in the
        // same buffer, so its completion also means that accumulator is updated
        if (ok) {
          issue_s(0, 0, 0);
          tc::mma_commit(BAR(bKEmpty0));
          if (nt > 1) {
            ok = k_ready(1);
            if (ok) {
              issue_s(0, 1, 1);
              tc::mma_commit(BAR(bKEmpty0 + 1 % L::S));
            }
          }
        }
        for (int j = 0; ok && j < nt; ++j) {
          const int buf = j & 1;
          if (!wait_bar(ms, BAR(bPFull0 + buf), (j >> 1) & 1, g.err) || !v_ready(j)) { ok = false; break; }
          if (alt) issue_pv(buf, j, buf, j > 1);
          else issue_pv(0, j, buf, j > 0);
          tc::mma_commit(BAR(bVEmpty0 + j % L::S));
          if (j + 2 < nt) {
            if (!k_ready(j + 2)) { ok = false; break; }
            issue_s(0, j + 2, buf);
            tc::mma_commit(BAR(bKEmpty0 + (j + 2) % L::S));
          }
        }
        if (ok && !alt) tc::mma_commit(BAR(bOReady));
      }
      tc::mma_commit(BAR(bDrain));
      // bounded: completes when every MMA issued above has finished
      const long long t0 = clock64();
      while (!tc::mbar_try_wait(BAR(bDrain), 0)) {
        if (clock64() - t0 > kWaitCycles) { atomicOr(g.err, kErrHang); break; }
      }
    }
    __syncwarp();
  } else if (warp < 8 && (warp < 4 || hasB || alt)) {
    // ============================================================ softmax / epilogue
    const int t = warp >> 2;                            // query tile (alternating mode: half)
    const int r = tid - 128 * t;                        // its row = TMEM lane
    const int row0 = alt ? 0 : kTileRows * t;           // the tile's first row in the item
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tO = tmem + 256 + 128 * t + lane_off;
    const float sl2 = 1.4426950408889634f / sqrtf((float)d);
    // a warp none of whose 32 rows is a query row of the item (a group's tail tile) only
    // keeps the barrier phases: its rows read zero-filled Q, their results are not stored,
    // and the issue slots and special-function throughput go to the warps that have rows
    const bool idle = row0 + 32 * (warp & 3) >= nrows;
    const bool live = row0 + r < nrows;                 // a query row of the item
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int j = alt ? t : 0; j < nt; j += alt ? 2 : 1) {
      // S buffer: the tile's (half's) own with two tiles or halves, alternating with one
      const int buf = (hasB || alt) ? t : (j & 1);
      const uint32_t sfp = hasB ? (j & 1) : ((j >> 1) & 1);
      const uint32_t tS = tmem + 128 * buf + lane_off;
      if (!__all_sync(0xffffffffu, wait_bar(ms, BAR(bSFull0 + buf), sfp, g.err))) { ok = false; break; }
      tc::fence_after_sync();
      if (idle) {
        tc::fence_before_sync();
        tc::mbar_arrive(BAR(bPFull0 + buf));
        continue;
      }
      // sparse: padding columns of the tile (rows of no selected range; their K and V rows
      // are zero, so S = 0 there and they add nothing to O).  Waiting on the mask slot's
      // barrier phase of tile j acquires the producer's words; the slot's next phase
      // (tile j + 2S) needs the S products of tile j + S, which follow this warp's P(j).
      uint32_t pw[4] = {0u, 0u, 0u, 0u};
      if (g.mode == kModeSparse) {
        if (!__all_sync(0xffffffffu, wait_bar(ms, BAR(bMask0 + j % (2 * L::S)), (j / (2 * L::S)) & 1, g.err))) { ok = false; break; }
#pragma unroll
        for (int q = 0; q < 4; ++q) pw[q] = ms->kvmask[j % (2 * L::S)][q];
      }
      const bool padded = (pw[0] | pw[1] | pw[2] | pw[3]) != 0u;     // uniform
      const int valid = (j == nt - 1) ? last_valid : kTileKeys;
      const bool whole = valid == kTileKeys;           // uniform: no key column past the keys
      // The padding columns' S = 0 only decides the max where no key column of a query row
      // exceeds 0.  Then (rare) they are set to -inf and the max taken again; otherwise
      // their exp terms, whose values are known and below the row's largest term, come off
      // the row sum after the tile.
      float mx;
      bool pad_in_sum = padded;
#pragma unroll 1
      for (int pass = 0;; ++pass) {
        mx = -INFINITY;
        if (whole) {
          // two 32-column loads per wait, four independent three-operand max chains
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < 4; c += 2) {
            float v[64];
            tc::tmem_ld32(tS + 32 * c, *reinterpret_cast<float(*)[32]>(v));
            tc::tmem_ld32(tS + 32 * c + 32, *reinterpret_cast<float(*)[32]>(v + 32));
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 64; i += 2) m4[(i >> 1) & 3] = tc::fmax3(m4[(i >> 1) & 3], v[i], v[i + 1]);
          }
          mx = tc::fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
        } else {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float v[32];
            tc::tmem_ld32(tS + 32 * c, v);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (32 * c + i < valid) mx = fmaxf(mx, v[i]);
          }
        }
        if (pass > 0 || !padded || !__any_sync(0xffffffffu, !(mx > 0.0f) && live)) break;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t mw = pw[q];
          while (mw) {                                    // uniform across the warp
            const int col = 32 * q + __ffs(mw) - 1;
            mw &= mw - 1;
            tc::tmem_st1(tS + col, __float_as_uint(-INFINITY));
          }
        }
        tc::tmem_wait_st();
        pad_in_sum = false;
      }
      float rs = 0.0f;
      const float m_tile = mx * sl2;
      // lazy rescale: keep the running max unless it grows by more than 2^8
      if (__any_sync(0xffffffffu, m_tile > m_run + kRescaleLog2)) {
        const float m_new = fmaxf(m_run, m_tile);
        const float alpha = tc::ex2(m_run - m_new);     // 0 on the first tile
        // one tile: S(j) may be ready before PV(j-1) has finished updating O
        if (!hasB && !alt && j > 0 && !__all_sync(0xffffffffu, wait_bar(ms, BAR(bPvDone0), (j - 1) & 1, g.err))) {
          ok = false;
          break;
        }
        if (j > 0) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tc::tmem_ld32(tO + 32 * c, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tc::tmem_st32(tO + 32 * c, o);
          }
        }
        l_run *= alpha;
        m_run = m_new;
      }
      if (whole) {
        // two 32-column loads per wait; the scaling and the row sum two lanes per
        // instruction (paired fp32), two independent pair sums
        uint64_t r2[2] = {0ull, 0ull};                 // (0.0f, 0.0f) pairs
        const uint64_t sc2 = tc::f2pack(sl2, sl2), nm2 = tc::f2pack(-m_run, -m_run);
#pragma unroll
        for (int c = 0; c < 4; c += 2) {
          float v[64];
          tc::tmem_ld32(tS + 32 * c, *reinterpret_cast<float(*)[32]>(v));
          tc::tmem_ld32(tS + 32 * c + 32, *reinterpret_cast<float(*)[32]>(v + 32));
          tc::tmem_wait_ld();
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float x0, x1;
            tc::f2unpack(tc::fma2(tc::f2pack(v[2 * i], v[2 * i + 1]), sc2, nm2), x0, x1);
            // kPolyPairs of every 16 pairs on the FMA pipe, the rest on the SFU
            const bool poly = (i & 15) >= 16 - kPolyPairs;
            float p0, p1;
            if (poly) {
              tc::exp2_poly2(x0, x1, p0, p1);
            } else {
              p0 = tc::ex2(x0);
              p1 = tc::ex2(x1);
            }
            r2[i & 1] = tc::add2(r2[i & 1], tc::f2pack(p0, p1));
            pk[i] = tc::pack_bf16x2(p0, p1);
          }
          // P columns 16c..16c+31 lie inside S columns already read (chunks 0..c+1)
          tc::tmem_st16(tS + 16 * c, *reinterpret_cast<uint32_t(*)[16]>(pk));
          tc::tmem_st16(tS + 16 * c + 16, *reinterpret_cast<uint32_t(*)[16]>(pk + 16));
        }
        float s0, s1, s2, s3;
        tc::f2unpack(r2[0], s0, s1);
        tc::f2unpack(r2[1], s2, s3);
        rs = (s0 + s1) + (s2 + s3);
      } else {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float v[32];
          tc::tmem_ld32(tS + 32 * c, v);
          tc::tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = (32 * c + 2 * i < valid) ? tc::ex2(fmaf(v[2 * i], sl2, -m_run)) : 0.0f;
            const float p1 = (32 * c + 2 * i + 1 < valid) ? tc::ex2(fmaf(v[2 * i + 1], sl2, -m_run)) : 0.0f;
            rs += p0 + p1;
            pk[i] = tc::pack_bf16x2(p0, p1);
          }
          tc::tmem_st16(tS + 16 * c, pk);
        }
      }
      tc::tmem_wait_st();
      if (pad_in_sum) {
        // the padding columns' terms: exp2(0 * scale - m_run), on the special-function
        // unit or the polynomial as their column position decided
        constexpr uint32_t kPolyCols = ~0u << (32 - 2 * kPolyPairs);   // per 32-column word
        int n_all = 0, n_poly = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          n_all += __popc(pw[q]);
          n_poly += __popc(pw[q] & kPolyCols);
        }
        const float e_sfu = tc::ex2(-m_run);
        if (whole) {
          float e_poly, e_unused;
          tc::exp2_poly2(-m_run, -m_run, e_poly, e_unused);
          rs -= (float)(n_all - n_poly) * e_sfu + (float)n_poly * e_poly;
        } else {
          rs -= (float)n_all * e_sfu;
        }
      }
      l_run += rs;
      tc::fence_before_sync();
      tc::mbar_arrive(BAR(bPFull0 + buf));
    }
    // PV commits on this tile's (half's) barrier: one per key tile it took
    const int npv = alt ? (nt - t + 1) >> 1 : nt;
    const bool oready = idle || ((hasB || alt) ? wait_bar(ms, BAR(bPvDone0 + t), (npv - 1) & 1, g.err)
                                               : wait_bar(ms, BAR(bOReady), 0, g.err));
    bool store = ok && !idle && __all_sync(0xffffffffu, oready);
    // alternating mode: the two halves' running max and sum for every row, then each half
    // writes half of the columns of the merged rows
    float wA = 1.0f, wB = 0.0f;
    int c0 = 0, c1 = D / 32;
    if (alt) {
      if (store) {
        ms->xm[t][r] = m_run;
        ms->xl[t][r] = l_run;
      }
      // every softmax thread of both halves arrives here exactly once
      store = tc::named_sync_and(2, 256, store || idle) && store;
      if (store) {
        const float mA = ms->xm[0][r], mB = ms->xm[1][r];
        m_run = fmaxf(mA, mB);
        wA = tc::ex2(mA - m_run);
        wB = tc::ex2(mB - m_run);
        l_run = ms->xl[0][r] * wA + ms->xl[1][r] * wB;
        c0 = t * (D / 64);
        c1 = c0 + D / 64;
      }
    }
    if (store) {
      tc::fence_after_sync();
      const float inv = 1.0f / l_run;
      const int row = row0 + r;
      const uint32_t tO0 = tmem + 256 + lane_off, tO1 = tmem + 384 + lane_off;
      for (int c = c0; c < c1; ++c) {
        float o[32];
        if (alt) {
          float o1[32];
          tc::tmem_ld32(tO0 + 32 * c, o);
          tc::tmem_ld32(tO1 + 32 * c, o1);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = o[i] * wA + o1[i] * wB;
        } else {
          tc::tmem_ld32(tO + 32 * c, o);
          tc::tmem_wait_ld();
        }
        if (row < nrows) {
          if (g.mode == kModeSparse) {
            float4* dst = reinterpret_cast<float4*>(g.b.Osp + ((long long)h * m.Nq + q0 + row) * d + 32 * c);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv, o[4 * i + 3] * inv);
          } else if (g.mode == kModeDense) {
            const long long ob = ((long long)h * m.Nq + q0 + row) * d + 32 * c;
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = tc::pack_bf16x2(o[2 * i] * inv, o[2 * i + 1] * inv);
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(g.out) + ob);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          } else {
            const long long slot = ((long long)h * m.M + row) * m.nsplit + split;
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
  if (warp == 11) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// Work list of the sparse mode: one item per 256 rows (two query tiles) of every
// non-empty query group.
__global__ void __launch_bounds__(1024) build_work_kernel(Dims m, Buffers b, int* work, int* nwork,
                                                          int max_items) {
  __shared__ int sh[32];
  const int h = blockIdx.x, a = threadIdx.x;
  const int n = b.nQ[h];
  const int tiles = a < n ? (b.sizeQ[(long long)h * m.Cq + a] + kItemRows - 1) / kItemRows : 0;
  int tot;
  const int off = block_exclusive_scan(tiles, sh, &tot);
  for (int t = 0; t < tiles; ++t) work[(long long)h * max_items + off + t] = (a << 16) | t;
  if (threadIdx.x == 0) nwork[h] = tot;
}

// K or V of shape [H_k][N_k][d] bf16 (row-major, 16-byte aligned) in boxes of 64 columns
// x box_rows rows; rows past N_k read as zeros.
sparsepr_status make_kv_map(CUtensorMap* map, const void* ptr, const Dims& m, int box_rows) {
  auto fn = tmap_encoder();
  if (!fn) return SPARSEPR_ERR_CUDA;
  const cuuint64_t dims[3] = {(cuuint64_t)m.d, (cuuint64_t)m.Nk, (cuuint64_t)m.Hk};
  const cuuint64_t strides[2] = {(cuuint64_t)m.d * 2, (cuuint64_t)m.Nk * m.d * 2};
  const cuuint32_t box[3] = {64u, (cuuint32_t)box_rows, 1u};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
             ? SPARSEPR_OK
             : SPARSEPR_ERR_ARG;
}

template <int D>
sparsepr_status launch_tc(TcArgs args, dim3 grid, cudaStream_t st) {
  if (args.mode != kModeSparse) {
    sparsepr_status s = make_kv_map(&args.tm_k, args.K, args.m, 64);
    if (s == SPARSEPR_OK) s = make_kv_map(&args.tm_v, args.V, args.m, 64);
    if (s != SPARSEPR_OK) return s;
  }
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

// The failure path of the pipeline waits, on a healthy GPU: one warp waits through
// wait_bar on a fresh barrier that nothing arrives on (no copy or product is in flight),
// gives up after kWaitCycles (about one second) and records kErrHang in the error word of
// the plan-free entry points.
__global__ void __launch_bounds__(32) wait_selftest_kernel() {
  __shared__ Misc ms;
  const uint32_t bar = tc::smem_u32(&ms.bars[0]);
  if (threadIdx.x == 0) {
    tc::mbar_init(bar, 1);
    ms.abort_flag = 0;
  }
  __syncthreads();
  (void)__all_sync(0xffffffffu, wait_bar(&ms, bar, 0, &g_dense_err));
}

}  // namespace

sparsepr_status launch_wait_selftest(cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>();
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

sparsepr_status dense_error_address(int** out) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(out), g_dense_err) == cudaSuccess ? SPARSEPR_OK
                                                                                          : SPARSEPR_ERR_CUDA;
}

bool tc_engine_applies(int dtype, int d, int engine) {
  return engine == SPARSEPR_ENGINE_AUTO && dtype == SPARSEPR_BF16 && (d == 64 || d == 128);
}

int tc_max_items(const Dims& m) { return m.Cq + cdiv(m.Nq, kItemRows); }

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
  if (!a.err) {
    const sparsepr_status s = dense_error_address(&a.err);
    if (s != SPARSEPR_OK) return s;
  }
  return with_tc_d(m.d, [&](auto DD) { return launch_tc<decltype(DD)::value>(a, dim3(cdiv(m.Nq, kItemRows), m.H), st); });
}

}  // namespace spr
