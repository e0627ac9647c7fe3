// k-means assignment on the tensor cores, with labels identical to the fp64 full scan.
//
// Scores a_c = ||c||^2 - 2 x.c (argmin a_c = argmin ||x - c||^2) come from three bf16
// products per k-step, x_hi c_hi + x_hi c_lo + x_lo c_hi, with x = x_hi + x_lo + e,
// |e| <= 2^-16 |x| (two round-to-nearest bf16 pieces), accumulated in fp32 in TMEM.
// Their error against exact arithmetic is below
//   E = 1.8e-4 |x| cmax + 4e-6 cmax^2   (dropped terms 3 * 2^-16, accumulation 192 * 2^-24
//                                         with a factor 4 of margin, ||c||^2 rounding),
// and the fp64 direct distance used by the full scan is within 1e-13 (|x| + cmax)^2 of
// exact.  So the full scan's label lies among the centres whose score is within
// T = 2E + 2e-13 (|x| + cmax)^2 of the smallest score (T below is rounded up well past
// that).  Each point keeps its smallest score, that score's centre and the second
// smallest score, branch-free (six instructions per score).  If the runner-up is more
// than T away, the label is the best score's centre.  Otherwise the point goes to a
// queue with its candidates and a second kernel rescores them with the full scan's own
// fp64 formula (ties to the lowest index).  The candidates are every chunk's best at the
// end of that chunk plus, for the rows still ambiguous after a chunk, that chunk's
// centres within T of the running best (a second pass over the chunk's scores, taken
// only by warps holding such a row): a centre within T of the final best is either its
// chunk's best or was within T of a running best no larger than the final one.  With
// more than four centres found in second passes the point is rescanned against every
// centre.  On the Wan-like data 0.4-1.5% of the points are queued.
//
// Persistent kernel, one CTA per SM, each taking a contiguous range of 128-point tiles of
// the heads that have not converged.  The centres of the current head (hi and lo, up to
// three 256-centre chunks) stay in shared memory; point tiles stream through a ring of
// X slots.  Both arrive by TMA (2-D tiled copies, 128-byte swizzle).
//   warps 0-3 / 4-7  epilogue of the tiles of even / odd local index (thread = TMEM lane):
//                    scores from TMEM, running best, its centre and the runner-up,
//                    decision or queue entry;
//   warp 8           TMA producer (one thread);
//   warp 9           MMA issuer (one thread) and TMEM owner: M=128, N=chunk width, K=16,
//                    both operands K-major, into two 256-column accumulators that
//                    alternate job by job (job = one tile against one centre chunk).
// Every accumulator has one "full" mbarrier per epilogue group, so each waiter sees the
// phases of its barrier one by one (a parity wait cannot tell phase k from k - 2).
// Warm plans also keep distance bounds (km_filter_kernel below): the kernel then runs over
// the compacted rows of the points whose label can still change (template flag B);
// cold plans assign every point of the heads that have not converged.
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace spr {
namespace {

constexpr int kKP = 64;                 // padded feature width (one 128-byte row in bf16)
constexpr int kRows = 128;              // points per tile
constexpr int kChunk = 256;             // centres per chunk (largest MMA N)
constexpr int kMaxChunks = 3;           // centres kept in shared memory: C <= 768
constexpr int kKmThreads = 320;         // 10 warps
constexpr int kMaxSlots = 4;
constexpr long long kKmWait = 2000000000LL;
constexpr uint32_t kXBytes = kRows * kKP * 2;      // 16 KB: one x tile (hi or lo)
constexpr uint32_t kCBytes = kChunk * kKP * 2;     // 32 KB: one centre chunk (hi or lo)
constexpr uint32_t kSmemLimit = 232448;            // opt-in shared memory per block

struct KmArgs {
  CUtensorMap tm_xhi, tm_xlo, tm_chi, tm_clo;   // [H*Npad][64] (compacted points), [H*Cpad][64] bf16
  const int* aidx;            // [H][Npad] point of each compacted row
  const int* acnt;            // [H] compacted rows of this step
  double* U;                  // [H][N] upper bound: distance to the own centre
  float* L;                   // [H][G][N] lower bounds: distance to each 32-centre group but the own centre
  const float* xn;            // [H][N] |x|
  const float* cn;            // [H][Cpad] ||c||^2 (+inf for padding centres)
  const int* cmaxb;           // [2][H] max ||c||^2 as float bits, slot it & 1
  int* lab;                   // [H][N]
  int* km;                    // [H][4]
  int4* queue;                // ambiguous points: h * N + n, candidate slots, flags
  int* qcnt;                  // [2] queue lengths, slot it & 1
  unsigned long long* chg;    // [H][N] last label change of each point (chg_entry)
  int qcap;
  const double* X;            // [H][N][r] fp64 features (fallback when the queue is full)
  const double* cent;         // [H][C][r] fp64 centres
  int* err;
  int H, N, Npad, C, Cpad, Cw, nch, r, it, slots, G;
};

constexpr int kGroup = 32;              // centres per lower-bound group

// fp64 direct squared distance in ascending dimensions: the full scan's formula.
__device__ __forceinline__ double exact_d2(const double* x, const double* c, int r) {
  double s = 0.0;
  for (int k = 0; k < r; ++k) {
    const double t = x[k] - c[k];
    s = fma(t, t, s);
  }
  return s;
}

constexpr int kNoCand = 1023;           // empty candidate slot (C <= 768)

struct KmMisc {
  unsigned long long bars[24];
  uint32_t tmem_base;
  int abort_flag;
};

enum KmBar {
  kbCFull = 0, kbCEmpty = 1,
  kbAccFree0 = 2,                 // [2]
  kbAccFull00 = 4,                // [2 accumulators][2 groups]: 4 + 2s + g
  kbXFull0 = 8, kbXEmpty0 = 12,   // [kMaxSlots] each
  kbDrain = 16
};

// Bounded wait; the clock and the abort flag are read once every 32 polls so that
// waiting warps take few issue slots from the working ones.
__device__ __forceinline__ bool km_wait(KmMisc* ms, uint32_t bar, uint32_t parity, int* err) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (unsigned n = 1;; ++n) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    if ((n & 31) == 0) {
      if (*reinterpret_cast<volatile int*>(&ms->abort_flag)) return false;
      if (clock64() - t0 > kKmWait) {
        if (atomicExch(&ms->abort_flag, 1) == 0) atomicOr(err, kErrHang);
        return false;
      }
    }
  }
}

// A distance no larger than every one whose score is at least `a` (score error below Eb),
// rounded down to fp32 with a margin.
__device__ __forceinline__ float dist_floor(float a, double Eb, double x2) {
  if (!(a < 3.0e38f)) return INFINITY;             // only padding centres in the group
  return __double2float_rd(sqrt(fmax((double)a - Eb + x2, 0.0)) * (1.0 - 1e-9));
}

// Points to assign in head h at this step: the compacted list when the distance bounds
// are in use, else every point of a head that has not converged.
template <bool B>
__device__ __forceinline__ int step_count(const KmArgs& g, int h) {
  return B ? g.acnt[h] : (g.km[4 * h] ? 0 : g.N);
}

// Global tile index -> (head, tile within the head) over the points to assign of every
// head (ceil(count / 128) tiles each); queried with non-decreasing tiles.
template <bool B>
struct TileCursor {
  const KmArgs* g;
  int h, base, nt;
  __device__ int head(long long t, int* lt) {
    while (t >= base + nt) {
      base += nt;
      ++h;
      nt = (step_count<B>(*g, h) + kRows - 1) / kRows;
    }
    *lt = (int)(t - base);
    return h;
  }
};

// B: distance bounds in use (points listed by the filter, their rows compacted, bounds
// written for the next step); without them every point of an unconverged head is
// assigned from its own row and no bound is kept.
template <bool B>
__global__ void __launch_bounds__(kKmThreads, 1) km_assign_tc_kernel(const __grid_constant__ KmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t oChi = 0, oClo = g.nch * kCBytes, oX = 2 * g.nch * kCBytes;
  KmMisc* ms = reinterpret_cast<KmMisc*>(smem_raw + (base - raw) + oX + g.slots * 2 * kXBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // tiles of the points to re-assign (converged heads have none), split evenly over CTAs
  long long T = 0;
  for (int h = 0; h < g.H; ++h) T += (step_count<B>(g, h) + kRows - 1) / kRows;
  const long long t0 = T * blockIdx.x / gridDim.x, t1 = T * (blockIdx.x + 1) / gridDim.x;
  const int ntiles = (int)(t1 - t0);
  if (blockIdx.x == 0 && tid == 0) {
    for (int h = 0; h < g.H; ++h)
      if (!g.km[4 * h]) g.km[4 * h + 3] += 1;
    g.qcnt[(g.it + 1) & 1] = 0;                        // the next iteration's queue
  }
  if (ntiles <= 0) return;

  const uint32_t bars = tc::smem_u32(ms->bars);
  auto BAR = [&](int i) -> uint32_t { return bars + 8u * i; };
  if (tid == 0) {
    tc::mbar_init(BAR(kbCFull), 1);
    tc::mbar_init(BAR(kbCEmpty), 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(BAR(kbAccFree0 + s), kRows);
      tc::mbar_init(BAR(kbAccFull00 + 2 * s), 1);
      tc::mbar_init(BAR(kbAccFull00 + 2 * s + 1), 1);
    }
    for (int s = 0; s < kMaxSlots; ++s) {
      tc::mbar_init(BAR(kbXFull0 + s), 1);
      tc::mbar_init(BAR(kbXEmpty0 + s), 1);
    }
    tc::mbar_init(BAR(kbDrain), 1);
    ms->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 9) {
    tc::tmem_alloc(tc::smem_u32(&ms->tmem_base), 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = ms->tmem_base;
  TileCursor<B> act{&g, -1, 0, 0};

  if (warp == 8) {
    // ============================================================ TMA producer
    if (lane == 0) {
      int loaded = -1, nload = 0;
      for (int li = 0; li < ntiles; ++li) {
        const long long t = t0 + li;
        int lt;
        const int h = act.head(t, &lt);
        if (h != loaded) {
          if (nload > 0 && !km_wait(ms, BAR(kbCEmpty), (nload - 1) & 1, g.err)) break;
          tc::mbar_expect_tx(BAR(kbCFull), 2u * g.nch * g.Cw * kKP * 2);
          for (int c = 0; c < g.nch; ++c) {
            const int row = h * g.Cpad + c * kChunk;
            tc::tma_load_2d(base + oChi + c * kCBytes, &g.tm_chi, 0, row, BAR(kbCFull));
            tc::tma_load_2d(base + oClo + c * kCBytes, &g.tm_clo, 0, row, BAR(kbCFull));
          }
          loaded = h;
          ++nload;
        }
        const int slot = li % g.slots, use = li / g.slots;
        if (use > 0 && !km_wait(ms, BAR(kbXEmpty0 + slot), (use - 1) & 1, g.err)) break;
        tc::mbar_expect_tx(BAR(kbXFull0 + slot), 2u * kXBytes);
        const int row = h * g.Npad + lt * kRows;          // compacted rows of the head
        const uint32_t xs = base + oX + slot * 2 * kXBytes;
        tc::tma_load_2d(xs, &g.tm_xhi, 0, row, BAR(kbXFull0 + slot));
        tc::tma_load_2d(xs + kXBytes, &g.tm_xlo, 0, row, BAR(kbXFull0 + slot));
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(kRows, g.Cw, false);
      int cur = -1, nload = 0, J = 0;
      bool ok = true;
      for (int li = 0; ok && li < ntiles; ++li) {
        const long long t = t0 + li;
        int lt;
        const int h = act.head(t, &lt);
        if (h != cur) {
          if (nload > 0) tc::mma_commit(BAR(kbCEmpty));     // old centres free once done
          if (!km_wait(ms, BAR(kbCFull), nload & 1, g.err)) { ok = false; break; }
          cur = h;
          ++nload;
        }
        const int slot = li % g.slots, use = li / g.slots;
        if (!km_wait(ms, BAR(kbXFull0 + slot), use & 1, g.err)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t xa = base + oX + slot * 2 * kXBytes;
        const int grp = li & 1;
        for (int c = 0; c < g.nch; ++c, ++J) {
          const int s = J & 1, u = J >> 1;
          if (u > 0 && !km_wait(ms, BAR(kbAccFree0 + s), (u - 1) & 1, g.err)) { ok = false; break; }
          tc::fence_after_sync();
          const uint32_t acc = tmem + 256 * s;
          const uint32_t ch = base + oChi + c * kCBytes, cl = base + oClo + c * kCBytes;
          // k-steps of 16 features up to r: the padding columns are zero in both operands
          const int nks = (g.r + 15) >> 4;
#pragma unroll 4
          for (int kk = 0; kk < nks; ++kk) {
            const uint64_t xh = tc::sw128_desc(xa + kk * 32, 16, 1024);
            const uint64_t xl = tc::sw128_desc(xa + kXBytes + kk * 32, 16, 1024);
            const uint64_t chd = tc::sw128_desc(ch + kk * 32, 16, 1024);
            const uint64_t cld = tc::sw128_desc(cl + kk * 32, 16, 1024);
            tc::mma_ss(acc, xh, chd, idesc, kk > 0 ? 1u : 0u);
            tc::mma_ss(acc, xh, cld, idesc, 1u);
            tc::mma_ss(acc, xl, chd, idesc, 1u);
          }
          tc::mma_commit(BAR(kbAccFull00 + 2 * s + grp));
        }
        if (ok) tc::mma_commit(BAR(kbXEmpty0 + slot));
      }
      tc::mma_commit(BAR(kbDrain));
      // bounded: completes when every MMA issued above has finished
      const long long w0 = clock64();
      while (!tc::mbar_try_wait(BAR(kbDrain), 0)) {
        if (clock64() - w0 > kKmWait) { atomicOr(g.err, kErrHang); break; }
      }
    }
    __syncwarp();
  } else {
    // ============================================================ epilogue
    const int grp = warp >> 2, r = 32 * (warp & 3) + lane;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const float BIG = 3.402823466e38f;
    int J = 0;
    int nfull0 = 0, nfull1 = 0;            // waits done on accFull[0][grp], accFull[1][grp]
    // per-point values of this group's next tile, loaded one tile ahead of their use
    TileCursor<B> pre{&g, -1, 0, 0};
    float nxn = 0.0f, ncm = 0.0f;
    int nold = 0, nn = 0;
    auto point_vals = [&](int li2) {
      int lt2;
      const int h2 = pre.head(t0 + li2, &lt2);
      const int j2 = lt2 * kRows + r;
      if (B) nn = j2 < g.acnt[h2] ? g.aidx[(long long)h2 * g.Npad + j2] : -1;
      else nn = j2 < g.N ? j2 : -1;
      const long long pi2 = (long long)h2 * g.N + (nn >= 0 ? nn : 0);
      nxn = g.xn[pi2];
      nold = g.lab[pi2];
      ncm = sqrtf(__int_as_float(g.cmaxb[(g.it & 1) * g.H + h2]));
    };
    if (grp < ntiles) point_vals(grp);
    for (int li = 0; li < ntiles; ++li) {
      const long long t = t0 + li;
      int lt;
      const int h = act.head(t, &lt);
      if ((li & 1) != grp) { J += g.nch; continue; }
      const bool live = nn >= 0;          // this row holds a point to re-assign
      const long long pi = (long long)h * g.N + (live ? nn : 0);
      const float xn = nxn, cm = ncm;
      const int old = nold;
      if (li + 2 < ntiles) point_vals(li + 2);
      // score error bound: a lower bound on a distance from a score is sqrt(a - Eb + |x|^2)
      const double x2 = (double)xn * xn;
      const double Eb = 2e-4 * xn * cm + 5e-6 * (double)cm * cm + 1e-6 * x2;
      const float* cnh = g.cn + (long long)h * g.Cpad;
      float a0 = BIG, a1 = BIG;            // smallest and second smallest score
      int c0 = 0;                           // centre of the smallest (first one on ties)
      int sb[kMaxChunks] = {kNoCand, kNoCand, kNoCand};   // each chunk's best at its end
      int rk0 = kNoCand, rk1 = kNoCand, rk2 = kNoCand, rk3 = kNoCand;
      int nrec = 0;
      bool ok = true;
      for (int c = 0; c < g.nch; ++c, ++J) {
        const int s = J & 1;
        const int nf = s ? nfull1 : nfull0;
        if (!__all_sync(0xffffffffu, km_wait(ms, BAR(kbAccFull00 + 2 * s + grp), nf & 1, g.err))) {
          ok = false;
          break;
        }
        if (s) ++nfull1; else ++nfull0;
        tc::fence_after_sync();
        const uint32_t acc = tmem + 256 * s + lane_off;
        // four independent (smallest, runner-up, centre) chains, chain e over the columns
        // e mod 4, so consecutive scores do not wait on one another; merged below
        float x0[4] = {BIG, BIG, BIG, BIG}, x1[4] = {BIG, BIG, BIG, BIG};
        int xc[4] = {0, 0, 0, 0};
#pragma unroll 1
        for (int q = 0; q < g.Cw; q += 64) {
          const int cb = c * kChunk + q;
          // the centre norms first, so that their loads overlap the TMEM loads
          const float4* cn4 = reinterpret_cast<const float4*>(cnh + cb);
          float4 cq[16];
#pragma unroll
          for (int i4 = 0; i4 < 16; ++i4) cq[i4] = __ldg(cn4 + i4);
          float v[64];
          tc::tmem_ld32(acc + q, *reinterpret_cast<float(*)[32]>(v));
          tc::tmem_ld32(acc + q + 32, *reinterpret_cast<float(*)[32]>(v + 32));
          tc::tmem_wait_ld();
          float gm[2] = {BIG, BIG};         // smallest score of each 32-centre group
#pragma unroll
          for (int i4 = 0; i4 < 16; ++i4) {
            const float cv[4] = {cq[i4].x, cq[i4].y, cq[i4].z, cq[i4].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float a = fmaf(-2.0f, v[4 * i4 + e], cv[e]);
              x1[e] = fminf(x1[e], fmaxf(x0[e], a));
              xc[e] = a < x0[e] ? cb + 4 * i4 + e : xc[e];
              x0[e] = fminf(x0[e], a);
              if (B) gm[i4 >> 3] = fminf(gm[i4 >> 3], a);
            }
          }
          if (B && live) {
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2) {
              const int gi = cb / kGroup + s2;
              if (gi < g.G) g.L[((long long)h * g.G + gi) * g.N + (pi - (long long)h * g.N)] = dist_floor(gm[s2], Eb, x2);
            }
          }
        }
        // merge the chains into the running values: the smallest score with the lowest
        // centre index among equal ones (earlier chunks hold lower indices), and the
        // second smallest of the union, min(max of the two smallests, both runners-up)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          a1 = fminf(fminf(a1, x1[e]), fmaxf(a0, x0[e]));
          const bool take = x0[e] < a0 || (x0[e] == a0 && xc[e] < c0);
          c0 = take ? xc[e] : c0;
          a0 = fminf(a0, x0[e]);
        }
        // the bound, formed here so that the per-point loads above had the pass to land
        const float T = 4e-4f * xn * cm + 1e-5f * (xn + cm) * (xn + cm) + 1e-30f;
        if (c == 0) sb[0] = c0;
        else if (c == 1) sb[1] = c0;
        else sb[2] = c0;
        // rows ambiguous so far: this chunk's centres within T of the running best
        const bool need = live && a1 <= a0 + T;
        if (__any_sync(0xffffffffu, need)) {
          const float lim = need ? a0 + T : -BIG;     // rows that need nothing match nothing
#pragma unroll 1
          for (int q = 0; q < g.Cw; q += 64) {
            const int cb = c * kChunk + q;
            const float4* cn4 = reinterpret_cast<const float4*>(cnh + cb);
            float4 cq[16];
#pragma unroll
            for (int i4 = 0; i4 < 16; ++i4) cq[i4] = __ldg(cn4 + i4);
            float v[64];
            tc::tmem_ld32(acc + q, *reinterpret_cast<float(*)[32]>(v));
            tc::tmem_ld32(acc + q + 32, *reinterpret_cast<float(*)[32]>(v + 32));
            tc::tmem_wait_ld();
            // bit i of (m0, m1): column cb + i lies within the bound (branch-free)
            uint32_t m0 = 0, m1 = 0;
#pragma unroll
            for (int i4 = 0; i4 < 16; ++i4) {
              const float cv[4] = {cq[i4].x, cq[i4].y, cq[i4].z, cq[i4].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int i = 4 * i4 + e;
                const uint32_t hit = fmaf(-2.0f, v[i], cv[e]) <= lim ? 1u : 0u;
                if (i < 32) m0 |= hit << i;
                else m1 |= hit << (i - 32);
              }
            }
            while (m0 | m1) {                   // a few columns, on the ambiguous rows only
              int b;
              if (m0) { b = __ffs(m0) - 1; m0 &= m0 - 1; }
              else { b = 31 + __ffs(m1); m1 &= m1 - 1; }
              const int ci = cb + b;
              if (ci != c0) {
                if (nrec == 0) rk0 = ci;
                else if (nrec == 1) rk1 = ci;
                else if (nrec == 2) rk2 = ci;
                else if (nrec == 3) rk3 = ci;
                ++nrec;
              }
            }
          }
        }
        tc::fence_before_sync();
        tc::mbar_arrive(BAR(kbAccFree0 + s));
      }
      if (!ok) break;
      if (!live) continue;
      const float T = 4e-4f * xn * cm + 1e-5f * (xn + cm) * (xn + cm) + 1e-30f;
      int best = c0;
      if (!(a1 > a0 + T)) {
        if (B) g.U[pi] = INFINITY;                   // near a tie: re-assign at the next step
        const int full = nrec > 4 ? 1 : 0;
        const int slot = atomicAdd(g.qcnt + (g.it & 1), 1);
        if (slot < g.qcap) {
          g.queue[slot] = make_int4((int)pi, c0 | (sb[0] << 10) | (sb[1] << 20),
                                    sb[2] | (rk0 << 10) | (rk1 << 20), rk2 | (rk3 << 10) | (full << 20));
          continue;                                  // the rescoring kernel writes the label
        }
        // queue full: rescan every centre here
        const double* x = g.X + pi * g.r;
        const double* cent = g.cent + (long long)h * g.C * g.r;
        double bd = 1.7976931348623157e308;
        for (int ci = 0; ci < g.C; ++ci) {
          const double d2 = exact_d2(x, cent + (long long)ci * g.r, g.r);
          if (d2 < bd) { bd = d2; best = ci; }
        }
      } else if (B) {
        // the own centre is nearer than u; in its group every other centre scores at
        // least the runner-up a1 (the other groups' bounds were written above)
        g.U[pi] = sqrt(fmax((double)a0 + Eb + x2, 0.0)) * (1.0 + 1e-9);
        g.L[((long long)h * g.G + c0 / kGroup) * g.N + (pi - (long long)h * g.N)] = dist_floor(a1, Eb, x2);
      }
      if (old != best) {
        g.lab[pi] = best;
        g.km[4 * h + 1 + (g.it & 1)] = 1;
        g.chg[pi] = chg_entry(old, best, g.it);
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// Which points can change label at this step (exact; Hamerly's bounds refined per group
// of 32 centres as in Yinyang k-means): u bounds the distance to the point's own centre
// from above, l_g the distance to every centre of group g except the own one from below.
// After an update that moved centre c by delta_c (group g by at most dmax_g),
// u + delta_own and l_g - dmax_g still bound them; if u < min_g l_g the own centre stays
// strictly the nearest and the label cannot change.  Every other point is listed in its
// head's compacted index (warp-aggregated slots; the order inside a head does not affect
// any result).  Step 0 re-assigns every point.
struct KmFilter {
  const int* km;
  const int* lab;
  const double* delta;
  unsigned long long* dmax;
  double* U;
  float* L;
  int *aidx, *acnt;
  long long* reassigned;
  const __nv_bfloat16 *xhi, *xlo;
  __nv_bfloat16 *shi, *slo;
  int H, N, Npad, C, G, it;
};

__global__ void __launch_bounds__(256) km_filter_kernel(const KmFilter f) {
  const int h = blockIdx.y, lane = threadIdx.x & 31;
  if (blockIdx.x == 0) {
    if (threadIdx.x == 0) f.acnt[((f.it + 1) & 1) * f.H + h] = 0;    // the next step's count
    if (threadIdx.x < f.G)                                           // this step's update
      f.dmax[((long long)(f.it & 1) * f.H + h) * f.G + threadIdx.x] = 0ull;
  }
  if (f.km[4 * h]) return;                         // converged head
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  bool act = false;
  if (n < f.N) {
    const long long pi = (long long)h * f.N + n;
    if (f.it == 0) {
      act = true;
    } else {
      const double u = f.U[pi] + f.delta[(long long)h * f.C + f.lab[pi]];
      const unsigned long long* dm = f.dmax + ((long long)((f.it - 1) & 1) * f.H + h) * f.G;
      float* lp = f.L + (long long)h * f.G * f.N + n;          // [g] at lp[g * N]
      // every bound loaded before any is stored back, so the loads are all in flight
      constexpr int kMaxG = kMaxChunks * kChunk / kGroup;
      float lv[kMaxG];
#pragma unroll
      for (int gi = 0; gi < kMaxG; ++gi)
        if (gi < f.G) lv[gi] = lp[(long long)gi * f.N];
      double lmin = INFINITY;
#pragma unroll
      for (int gi = 0; gi < kMaxG; ++gi)
        if (gi < f.G) {
          const double l = (double)lv[gi] - __longlong_as_double((long long)dm[gi]);
          lp[(long long)gi * f.N] = __double2float_rd(l);
          lmin = fmin(lmin, l);
        }
      f.U[pi] = u;
      act = !(u < lmin);
    }
  }
  const unsigned m = __ballot_sync(0xffffffffu, act);
  int base = 0;
  if (lane == 0 && m) {
    base = atomicAdd(f.acnt + (f.it & 1) * f.H + h, __popc(m));
    atomicAdd(reinterpret_cast<unsigned long long*>(f.reassigned + h), (unsigned long long)__popc(m));
  }
  base = __shfl_sync(0xffffffffu, base, 0);
  if (act) f.aidx[(long long)h * f.Npad + base + __popc(m & ((1u << lane) - 1u))] = n;
  // the listed points' split rows into their compacted rows: 16 lanes per point, one
  // 16-byte chunk each (8 of the hi row, 8 of the lo row), two points per pass
  unsigned mm = m;
  while (mm) {
    const int l0 = __ffs(mm) - 1;
    mm &= mm - 1;
    int l1 = -1;
    if (mm) {
      l1 = __ffs(mm) - 1;
      mm &= mm - 1;
    }
    const int src = lane < 16 ? l0 : l1;
    const int sl = src < 0 ? 0 : src;
    const int pn = __shfl_sync(0xffffffffu, n, sl);
    if (src >= 0) {
      const int slot = base + __popc(m & ((1u << sl) - 1u));
      const int c = lane & 7;
      const bool lo = (lane & 8) != 0;
      const uint4* s4 = reinterpret_cast<const uint4*>((lo ? f.xlo : f.xhi) + ((long long)h * f.Npad + pn) * kKP);
      uint4* d4 = reinterpret_cast<uint4*>((lo ? f.slo : f.shi) + ((long long)h * f.Npad + slot) * kKP);
      d4[c] = s4[c];
    }
  }
}

// Exact rescoring of the queued points, one warp per point: lane l < 8 takes candidate
// slot l (or, for a point flagged "all", lanes take centres l, l + 32, ...), fp64 direct
// distance by the full scan's formula, smallest distance with ties to the lowest index.
__global__ void __launch_bounds__(256) km_rescore_kernel(const int4* queue, const int* qcnt, int qcap,
                                                         const double* X, const double* cent, int* lab,
                                                         int* km, int N, int C, int r, int it,
                                                         unsigned long long* chg) {
  const int lane = threadIdx.x & 31;
  const int n = min(qcnt[it & 1], qcap);
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int e = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; e < n; e += nw) {
    const int4 q = queue[e];
    const long long pi = q.x;
    const int h = (int)(pi / N);
    const double* x = X + pi * r;
    const double* ch = cent + (long long)h * C * r;
    double bd = 1.7976931348623157e308;
    int bc = 0x7fffffff;
    if ((q.w >> 20) & 1) {
      for (int c = lane; c < C; c += 32) {
        const double d2 = exact_d2(x, ch + (long long)c * r, r);
        if (d2 < bd) { bd = d2; bc = c; }
      }
    } else if (lane < 8) {
      const int word = lane < 3 ? q.y : lane < 6 ? q.z : q.w;
      const int c = (word >> (10 * (lane % 3))) & 1023;
      if (c != kNoCand) {
        bd = exact_d2(x, ch + (long long)c * r, r);
        bc = c;
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      const double od = __shfl_xor_sync(0xffffffffu, bd, o);
      const int oc = __shfl_xor_sync(0xffffffffu, bc, o);
      if (od < bd || (od == bd && oc < bc)) { bd = od; bc = oc; }
    }
    if (lane == 0 && lab[pi] != bc) {
      const int old = lab[pi];
      lab[pi] = bc;
      km[4 * h + 1 + (it & 1)] = 1;
      chg[pi] = chg_entry(old, bc, it);
    }
  }
}

// centres -> (c_hi, c_lo) bf16 rows padded to 64 and ||c||^2 (+inf for padding rows, so
// they never score), one warp per centre.  The largest ||c||^2 of each head goes to slot
// it & 1 of cmaxb (non-negative floats order like their bit patterns); the other slot is
// cleared for the next iteration.
__global__ void __launch_bounds__(256) km_split_c_kernel(const double* cent, int H, int C, int Cpad, int r,
                                                         int it, const int* kmstate, __nv_bfloat16* chi,
                                                         __nv_bfloat16* clo, float* cn, int* cmaxb) {
  const int h = blockIdx.y, lane = threadIdx.x & 31;
  const int c = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (blockIdx.x == 0 && threadIdx.x == 0) cmaxb[((it + 1) & 1) * H + h] = 0;
  if (kmstate[4 * h] || c >= Cpad) return;
  double ss = 0.0;
  for (int k = lane; k < kKP; k += 32) {
    const double v = (c < C && k < r) ? cent[((long long)h * C + c) * r + k] : 0.0;
    const __nv_bfloat16 hi = __double2bfloat16(v);
    const __nv_bfloat16 lo = __double2bfloat16(v - (double)__bfloat162float(hi));
    chi[((long long)h * Cpad + c) * kKP + k] = hi;
    clo[((long long)h * Cpad + c) * kKP + k] = lo;
    ss = fma(v, v, ss);
  }
  ss = warp_sum(ss);
  if (lane == 0) {
    const float s32 = (float)ss;
    cn[(long long)h * Cpad + c] = c < C ? s32 : INFINITY;
    if (c < C) atomicMax(cmaxb + (it & 1) * H + h, __float_as_int(s32));
  }
}

// ---------------------------------------------------------------- host side
// [rows][64] bf16 with 128-byte rows, copied in boxes of box_rows x 64, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* ptr, long long rows, int box_rows) {
  auto fn = tmap_encoder();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kKP, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kKP * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kKP, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  static int n = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  });
  return n;
}

}  // namespace

int km_tc_npad(int N) { return cdiv(N, 2 * kRows) * 2 * kRows; }
int km_tc_cpad(int C) { return cdiv(C, kChunk) * kChunk; }
bool km_tc_supported(int C) { return C >= 64 && C <= kMaxChunks * kChunk; }
long long km_tc_queue_cap(int H, int N) { return (long long)H * N / 16 + 1024; }

sparsepr_status km_tc_assign(const KmTcBuffers& kb, const double* X, const double* cent, int H, int N, int C,
                             int r, int it, int* lab, int* kmstate, int* err, bool bounds, cudaStream_t st) {
  if (!km_tc_supported(C)) return SPARSEPR_ERR_ARG;
  const int Npad = km_tc_npad(N), Cpad = km_tc_cpad(C);
  const int nch = cdiv(C, kChunk);
  const int Cw = nch > 1 ? kChunk : cdiv(C, 64) * 64;
  const int G = cdiv(C, kGroup);
  if (bounds) {
    const KmFilter f{kmstate, lab, kb.delta, kb.dmax, kb.U, kb.L, kb.aidx, kb.acnt, kb.reassigned, kb.xhi, kb.xlo,
                     kb.shi, kb.slo, H, N, Npad, C, G, it};
    km_filter_kernel<<<dim3(cdiv(N, 256), H), 256, 0, st>>>(f);
    SPR_LAUNCH_OK();
  }
  km_split_c_kernel<<<dim3(Cpad / 8, H), 256, 0, st>>>(cent, H, C, Cpad, r, it, kmstate, kb.chi, kb.clo,
                                                       kb.cn, kb.cmaxb);
  SPR_LAUNCH_OK();
  KmArgs g;
  g.G = G;
  if (!make_map(&g.tm_xhi, bounds ? kb.shi : kb.xhi, (long long)H * Npad, kRows) ||
      !make_map(&g.tm_xlo, bounds ? kb.slo : kb.xlo, (long long)H * Npad, kRows) ||
      !make_map(&g.tm_chi, kb.chi, (long long)H * Cpad, Cw) ||
      !make_map(&g.tm_clo, kb.clo, (long long)H * Cpad, Cw))
    return SPARSEPR_ERR_CUDA;
  const uint32_t fixed = 2u * nch * kCBytes + 1024u + (uint32_t)sizeof(KmMisc);
  int slots = (int)((kSmemLimit - fixed) / (2 * kXBytes));
  slots = slots > kMaxSlots ? kMaxSlots : slots;
  if (slots < 1) return SPARSEPR_ERR_ARG;
  const uint32_t smem = fixed + (uint32_t)slots * 2 * kXBytes;
  g.aidx = kb.aidx; g.acnt = kb.acnt + (it & 1) * H; g.U = kb.U; g.L = kb.L;
  g.xn = kb.xn; g.cn = kb.cn; g.cmaxb = kb.cmaxb; g.lab = lab; g.km = kmstate;
  g.queue = kb.queue; g.qcnt = kb.qcnt; g.qcap = (int)km_tc_queue_cap(H, N);
  g.chg = kb.chg;
  g.X = X; g.cent = cent; g.err = err;
  g.H = H; g.N = N; g.Npad = Npad; g.C = C; g.Cpad = Cpad; g.Cw = Cw; g.nch = nch; g.r = r; g.it = it;
  g.slots = slots;
  auto kern = bounds ? km_assign_tc_kernel<true> : km_assign_tc_kernel<false>;
  SPR_CUDA_OK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  const long long tiles = (long long)H * (Npad / kRows);
  const int grid = (int)(tiles < sm_count() ? tiles : sm_count());
  kern<<<grid, kKmThreads, smem, st>>>(g);
  SPR_LAUNCH_OK();
  km_rescore_kernel<<<4 * sm_count(), 256, 0, st>>>(kb.queue, kb.qcnt, g.qcap, X, cent, lab, kmstate, N, C, r,
                                                    it, kb.chg);
  SPR_LAUNCH_OK();
  return SPARSEPR_OK;
}

}  // namespace spr
