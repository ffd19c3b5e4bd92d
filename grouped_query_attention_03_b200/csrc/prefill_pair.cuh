// prefill_pair.cuh -- tcgen05 prefill for two query heads of one KV group.
//
// What it computes ("Share key/value heads and make context explicit",
// sections "Give each query head an explicit shared KV head" and "Intersect
// the window with the context already permitted"; FlashAttention's running
// max/sum from "GQA, FlashAttention and the KV cache"): for every batch row
// b, query head h and active cell t < n_b, softmax over the permitted keys
// of scale * q.k, mixed with the value rows of the shared lane g(h);
// inactive rows are zero.  It is organised so one CTA owns the same
// 128-row query tile of two heads h0, h0+1 that share KV head g: every K and
// V tile is fetched once and used by both (the GQA sharing applied to
// on-chip traffic), and the two heads' softmax work overlaps the other
// head's tensor-core work.
//
//   warp 0      TMA producer: both Q tiles, then K_0, V_0, K_1, V_1, ... into
//               a ring of NSLOT tile slots (128-byte swizzle, no multicast).
//   warp 1      TMEM allocation (all 512 columns); lane 0 issues tcgen05.mma:
//               S_A(0), S_B(0), then per KV tile j:
//               O_A += P_A(j) V_j, S_A(j+1), O_B += P_B(j) V_j, S_B(j+1)
//               so the tensor pipe runs one head while the other head's
//               softmax warps work.  P V takes P from TMEM (A operand) and
//               V from shared memory, in two halves: keys 0-63 as soon as
//               the softmax has written that half of P, then keys 64-127.
//               S(j+1) overwrites P(j) only after P V(j), since one
//               thread's MMAs execute in issue order; for the same reason
//               S(j+1) being complete means P V(j) is, so the softmax never
//               waits for P V separately.  Every wait of this thread comes
//               before a group of MMAs: an MMA issue blocks while the
//               tensor pipe's short queue is full.
//   warps 2-3   idle (they complete the first warpgroup, which hands most of
//               its registers to the softmax warpgroups with setmaxnreg).
//   warps 4-7   softmax of head A, warps 8-11 softmax of head B: thread = row
//               (TMEM lane); the whole 128-score row is read from TMEM into
//               registers at once, then row max, lazy O rescale, and bf16 P
//               written back to the same TMEM lane over the first 64 S
//               columns (no shared-memory round trip for P), its first half
//               published on its own; O / l epilogue.
// TMEM columns: S_A [0,128) (P_A in [0,64)), S_B [128,256) (P_B in
// [128,192)), O_A [256, 256+d), O_B after it.  Shared memory holds the two
// Q tiles and the K/V ring only.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tma_host.cuh"

namespace gqa {
namespace pf2 {

constexpr int kBM = 128, kBN = 128;
constexpr int kThreads = 384;
// Registers per thread after the split: the first warpgroup (producer, MMA
// issuer, two idle warps) gives registers to the two softmax warpgroups.
// 128 * kRegsLow + 256 * kRegsHigh must not exceed 384 * (launch registers).
constexpr int kRegsLow = 72, kRegsHigh = 216;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxSlots = 12;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// K/V tiles a CTA of a one-wave grid asks L2 for before the dependency
// wait, with its two Q tiles (148 CTAs x 6 tiles x 32 KB at d = 128 is
// 28 MB).
constexpr int kPrefetchTiles = 4;

template <int D>
struct Cfg {
  static constexpr int KB = D / 64;                  // 64-column blocks
  static constexpr int BLK = kBM * 128;              // 128 rows x 128 B
  static constexpr int TILE = KB * BLK;              // a Q, K or V tile
  static constexpr int NSLOT = (D == 128) ? 3 : 6;   // K/V ring slots (deeper measured no faster)
  static constexpr int OFF_QA = 0;
  static constexpr int OFF_QB = TILE;
  static constexpr int OFF_RING = 2 * TILE;
  static constexpr int SMEM = OFF_RING + NSLOT * TILE + 1024;  // + alignment slack
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  static_assert(NSLOT <= kMaxSlots, "ring barriers");
  static constexpr uint32_t TM_O = 256;              // O_A column; O_B = TM_O + D
};

struct Params {
  __nv_bfloat16 *o;
  const int32_t *seq_lens;
  int32_t *status;
  int B, Hq, Hkv, window, num_mt, pairs;  // pairs = (Hq/Hkv) / 2
  int Tq;      // query rows per head (Q and O are [B,Hq,Tq,d])
  int Tk;      // key rows per KV lane (K and V are [B,Hkv,Tk,d])
  int cached;  // 0: prompt, query row t at position t, n_b = active rows;
               // 1: queries after a cache, query row i at position n_b-Tq+i
  const int32_t *seg;  // prompt only: [B,Tq] first key cell of row t's
                       // packed segment, or NULL (segment start 0)
  float scale_log2;
  int prefetch;  // 1: the grid fits in one wave; its tiles are asked of L2
                 // before the dependency wait
};

// First permitted key of query position t ("Intersect the window with the
// context already permitted": the later of the segment start and the
// window start); t + 1 (no key) when the segment start is not in [0, t].
template <bool SEG>
__device__ __forceinline__ int row_lo(const Params &p, int b, int t) {
  int s0 = 0;
  if (SEG) {
    s0 = p.seg[(size_t)b * p.Tq + t];
    if (s0 < 0 || s0 > t) return t + 1;
  }
  return p.window > 0 ? max(s0, t - (p.window - 1)) : s0;
}

struct Bars {
  uint64_t q_full;
  uint64_t full[kMaxSlots], empty[kMaxSlots];
  uint64_t s_full[2], p_half[2], p_full[2], o_done[2];
  uint64_t mma_fin;
  uint64_t v_clean;  // the last V tile's rows past the sequence are zero
  uint32_t tmem_base;
};

// O *= alpha for this thread's TMEM lane (the whole warp takes part).
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t tO, float alpha) {
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    float ov[32];
    tc::tmem_ld32(tO + c * 32, ov);
    tc::tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) ov[i] *= alpha;
    tc::tmem_st32(tO + c * 32, ov);
  }
  tc::tmem_wait_st();
}

// p = 2^(s*scale - m) for this thread's row of kBN scores (special-function
// unit; masked cells give exactly 0), written as bf16 P into this thread's
// TMEM lane over the S columns it came from (column c holds p[2c], p[2c+1]),
// where the P V MMA reads it as its A operand; returns the row sum.
template <int D>
__device__ __forceinline__ float emit_p(const float *s, float sc, float m, uint32_t tP,
                                        uint64_t *half_bar) {
  float2 lsum2 = make_float2(0.f, 0.f);
  const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(-m, -m);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float w[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int i = half * 64 + 2 * e;
      const float2 x = ffma2v(make_float2(s[i], s[i + 1]), sc2, nm2);
      const float2 pv = make_float2(ex2_approx(x.x), ex2_approx(x.y));
      lsum2 = fadd2v(lsum2, pv);
      w[e] = __uint_as_float(pack_bf16(pv.x, pv.y));
    }
    tc::tmem_st32(tP + half * 32, w);
    if (half == 0) {  // keys 0-63 of P: their P V can start
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(half_bar);
    }
  }
  tc::tmem_wait_st();
  return lsum2.x + lsum2.y;
}

// Softmax and epilogue for one head (one 128-thread warpgroup, TMEM lanes
// = query rows).  `hd` selects the head's S/O columns, P buffer, barriers.
template <int D, bool SEG>
__device__ __forceinline__ void softmax_head(const Params &p, Bars &bars, unsigned char *smem,
                                             uint32_t tmem, int hd, int b, int h, int m0,
                                             int a0, int a_end, int lo_max, int j0, int nt,
                                             bool *failed) {
  using K = Cfg<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q4 = warp & 3;
  const int row = q4 * 32 + lane;
  const int t = a0 + row;       // key position of this query row
  const int qr = m0 + row;      // its row in Q and O
  const bool active = t < a_end;
  const int lo_t = active ? row_lo<SEG>(p, b, t) : 0;
  const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
  const uint32_t tS = tmem + lane_base + hd * kBN;
  const uint32_t tO = tmem + lane_base + K::TM_O + hd * D;
  const float sc = p.scale_log2;
  float m_run = -INFINITY, l_run = 0.f;
  bool ok = true;
  for (int j = 0; j < nt; ++j) {
    const int kb = (j0 + j) * kBN;
    if (!__all_sync(0xffffffffu, mbar_wait(&bars.s_full[hd], j & 1, failed))) { ok = false; break; }
    tc::fence_after_sync();
    const bool edge = (kb + kBN - 1 > a0) || (kb < lo_max);
    // the whole row of scores: four TMEM loads, one wait
    float s[kBN];
#pragma unroll
    for (int c = 0; c < kBN / 32; ++c) tc::tmem_ld32(tS + c * 32, s + c * 32);
    tc::tmem_wait_ld();
    // O and P are free here: S(j) was committed after P V(j-1) by the same
    // thread, so S(j) being ready means P V(j-1) has completed.
    if (edge) {
      // key kb + i is permitted for lo_t - kb <= i <= t - kb.  Most rows of an
      // edge tile need only the upper bound (the diagonal), and a warp none of
      // whose rows cuts this tile's keys skips the loop.
      const int hi_i = t - kb, lo_i = lo_t - kb;
      if (__any_sync(0xffffffffu, lo_i > 0)) {
#pragma unroll
        for (int i = 0; i < kBN; ++i)
          if (i > hi_i || i < lo_i) s[i] = -INFINITY;
      } else if (__any_sync(0xffffffffu, hi_i < kBN - 1)) {
#pragma unroll
        for (int i = 0; i < kBN; ++i)
          if (i > hi_i) s[i] = -INFINITY;
      }
    }
    // row maximum of s*scale (sc*max(s) for sc > 0, sc*min(s) otherwise)
    float mx;
    {
      const bool neg = !(sc > 0.f);
      float mc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (!neg) {
#pragma unroll
        for (int i = 0; i < kBN; i += 2) mc[(i >> 1) & 3] = fmax3(mc[(i >> 1) & 3], s[i], s[i + 1]);
      } else {
#pragma unroll
        for (int i = 0; i < kBN; ++i)
          mc[i & 3] = fmaxf(mc[i & 3], s[i] == -INFINITY ? -INFINITY : -s[i]);
      }
      mx = fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3]));
    }
    const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * fabsf(sc);
    if (j == 0) {
      m_run = m_tile;
    } else if (__any_sync(0xffffffffu, m_tile > m_run + kRescaleThreshold)) {
      const float m_new = fmaxf(m_run, m_tile);
      const float alpha = m_new == m_run ? 1.f : exp2f(m_run - m_new);
      rescale_o<D>(tO, alpha);
      l_run *= alpha;
      m_run = m_new;
    }
    const float lsum = emit_p<D>(s, sc, m_run == -INFINITY ? 0.f : m_run, tS, &bars.p_half[hd]);
    l_run += lsum;
    tc::fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.p_full[hd]);
  }

  // epilogue: O / l in bf16, one row per thread; the whole warp reads TMEM
  bool have = false;
  if (nt > 0 && ok) {
    have = __all_sync(0xffffffffu, mbar_wait(&bars.o_done[hd], 0, failed));
    tc::fence_after_sync();
  }
  const float inv = (active && have && l_run > 0.f) ? 1.f / l_run : 0.f;
  __nv_bfloat16 *orow = p.o + (((size_t)b * p.Hq + h) * p.Tq + min(qr, p.Tq - 1)) * D;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    float ov[32];
    if (have) {
      tc::tmem_ld32(tO + c * 32, ov);
      tc::tmem_wait_ld();
    }
    if (!have || !active) {  // inactive rows are exact zeros (their O may be NaN)
#pragma unroll
      for (int i = 0; i < 32; ++i) ov[i] = 0.f;
    }
    if (qr < p.Tq) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t w4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          w4[i] = pack_bf16(ov[e * 8 + 2 * i] * inv, ov[e * 8 + 2 * i + 1] * inv);
        *reinterpret_cast<uint4 *>(orow + c * 32 + e * 8) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
    }
  }
}

// SEG: packed segment starts are given (p.seg); the plain prompt and the
// cached-query forms compile without that code.
template <int D, bool SEG>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const Params p) {
  using K = Cfg<D>;
  extern __shared__ unsigned char smem_raw[];
  __shared__ Bars bars;
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- which tile: longest causal rows first; then (b, g, pair)
  const int per_mt = p.B * p.Hkv * p.pairs;
  const int mt = p.num_mt - 1 - (int)(blockIdx.x / per_mt);
  int rem = (int)(blockIdx.x % per_mt);
  const int pr = rem % p.pairs;
  rem /= p.pairs;
  const int g = rem % p.Hkv, b = rem / p.Hkv;
  const int r = p.Hq / p.Hkv;
  const int h0 = g * r + 2 * pr;
  const int m0 = mt * kBM;
  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < K::NSLOT; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bars.s_full[h], 1);
      mbar_init(&bars.p_half[h], 4);
      mbar_init(&bars.p_full[h], 4);
      mbar_init(&bars.o_done[h], 1);
    }
    mbar_init(&bars.mma_fin, 1);
    mbar_init(&bars.v_clean, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&bars.tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  // Barriers and TMEM are set up.  While the previous kernel on the stream
  // drains, the producer of a grid that fits in one wave asks L2 for both
  // Q tiles and the first K/V tiles of a plain prompt's tile (reads only,
  // planned as if the sequence had all Tk rows: no length is read before
  // the wait; later waves start after the previous kernel anyway).  From
  // the wait on, the CTA reads memory the previous kernel may write: wait
  // for it (a no-op unless launched as a programmatic dependent), then let
  // the next one start.
  if (!SEG && p.prefetch && !p.cached && warp == 0 && lane == 0) {
    const int lo0 = p.window > 0 ? max(0, m0 - (p.window - 1)) : 0;
    const int hi0 = min(m0 + kBM - 1, p.Tk - 1);
    const int jf = lo0 / kBN, nf = m0 < p.Tk ? min(hi0 / kBN - jf + 1, kPrefetchTiles) : 0;
#pragma unroll
    for (int cc = 0; cc < K::KB; ++cc) {
      if (nf > 0) {
        tc::tma_prefetch_3d(&tmQ, cc * 64, m0, b * p.Hq + h0);
        tc::tma_prefetch_3d(&tmQ, cc * 64, m0, b * p.Hq + h0 + 1);
      }
      for (int j = 0; j < nf; ++j) {
        tc::tma_prefetch_3d(&tmK, cc * 64, (jf + j) * kBN, b * p.Hkv + g);
        tc::tma_prefetch_3d(&tmV, cc * 64, (jf + j) * kBN, b * p.Hkv + g);
      }
    }
  }
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();
  // n_b keys of sequence b; `rows` query rows produce output, the query
  // row i sits at key position off + i; a0 = position of this tile's row 0.
  int n_b = p.Tk;
  if (p.seq_lens) {
    n_b = p.seq_lens[b];
    if (n_b < 0 || n_b > p.Tk || (p.cached && n_b < p.Tq)) {
      if (threadIdx.x == 0 && mt == 0 && g == 0 && pr == 0) record_status(p.status, GQA_ERR_CAPACITY);
      n_b = -1;  // the whole sequence is written as zeros
    }
  }
  const int off = (p.cached && n_b >= 0) ? n_b - p.Tq : 0;
  const int rows = n_b < 0 ? 0 : (p.cached ? p.Tq : n_b);
  const int a0 = off + m0;
  // Packed segments: the tile's rows (one per thread of warps 0-3) give the
  // smallest and largest first permitted key; invalid starts are reported.
  __shared__ int s_lo_min[4], s_lo_max[4];
  if (SEG && warp < 4) {
    const int t = a0 + (int)threadIdx.x;
    int lmin = 0x7fffffff, lmax = -1;
    if (t < off + rows) {
      const int lo = row_lo<SEG>(p, b, t);
      if (lo > t) {
        record_status(p.status, GQA_ERR_SEGMENT);
      } else {
        lmin = lo;
        lmax = lo;
      }
    }
    lmin = __reduce_min_sync(0xffffffffu, lmin);
    lmax = __reduce_max_sync(0xffffffffu, lmax);
    if (lane == 0) {
      s_lo_min[warp] = lmin;
      s_lo_max[warp] = lmax;
    }
  }

  if (SEG) __syncthreads();  // s_lo_min / s_lo_max
  // KV tiles [j0, j0 + nt) cover the tile's permitted keys; tiles starting
  // before lo_max need masks (some row's first key lies inside them).
  int lo_min, lo_max;
  if (SEG) {
    lo_min = min(min(s_lo_min[0], s_lo_min[1]), min(s_lo_min[2], s_lo_min[3]));
    lo_max = max(max(s_lo_max[0], s_lo_max[1]), max(s_lo_max[2], s_lo_max[3]));
  } else {
    lo_min = p.window > 0 ? max(0, a0 - (p.window - 1)) : 0;
    lo_max = p.window > 0 ? max(0, a0 + kBM - p.window) : 0;
  }
  int j0 = 0, nt = 0;
  if (rows > m0 && lo_min != 0x7fffffff) {
    const int hi = min(a0 + kBM - 1, off + rows - 1);
    j0 = lo_min / kBN;
    nt = hi / kBN - j0 + 1;
  }
  // Rows [z0, z1) of the last V tile are cells past the sequence that exist
  // in memory (an unwritten cache cell or prompt padding may hold NaN):
  // their p is 0, but 0 * NaN is not, so they are cleared before P V.
  const int kb_last = (j0 + nt - 1) * kBN;
  const int z0 = max(0, max(n_b, 0) - kb_last), z1 = min(kBN, p.Tk - kb_last);
  const bool clear_v = nt > 0 && z0 < z1;
  const uint32_t tmem = bars.tmem_base;
  bool failed = false;
  if (warp >= 4) {
    // ================================================= softmax warpgroups
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    const int hd = (warp - 4) / 4;  // warps 4-7: head A, 8-11: head B
    softmax_head<D, SEG>(p, bars, smem, tmem, hd, b, h0 + hd, m0, a0, off + rows, lo_max, j0,
                         nt, &failed);
  } else {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
  if (warp == 0) {
    // ================================================= TMA producer
    if (lane == 0 && nt > 0) {
      tc::prefetch_tmap(&tmQ);
      tc::prefetch_tmap(&tmK);
      tc::prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(&bars.q_full, 2 * K::TILE);
#pragma unroll
      for (int c = 0; c < K::KB; ++c) {
        tc::tma_load_3d(smem + K::OFF_QA + c * K::BLK, &tmQ, c * 64, m0, b * p.Hq + h0, &bars.q_full);
        tc::tma_load_3d(smem + K::OFF_QB + c * K::BLK, &tmQ, c * 64, m0, b * p.Hq + h0 + 1, &bars.q_full);
      }
      int fills[K::NSLOT];
#pragma unroll
      for (int s = 0; s < K::NSLOT; ++s) fills[s] = 0;
      for (int i = 0; i < 2 * nt; ++i) {  // K_0, V_0, K_1, V_1, ...
        const int s = i % K::NSLOT;
        if (i >= K::NSLOT && !mbar_wait(&bars.empty[s], ((i / K::NSLOT) - 1) & 1, &failed)) break;
        const CUtensorMap *map = (i & 1) ? &tmV : &tmK;
        const int row = (j0 + (i >> 1)) * kBN;
        mbar_arrive_expect_tx(&bars.full[s], K::TILE);
#pragma unroll
        for (int c = 0; c < K::KB; ++c)
          tc::tma_load_3d(smem + K::OFF_RING + s * K::TILE + c * K::BLK, map, c * 64, row,
                          b * p.Hkv + g, &bars.full[s]);
        fills[s]++;
      }
      // Never leave a TMA load in flight into an exiting CTA.
      bool f2 = false;
      mbar_wait(&bars.q_full, 0, &f2);
#pragma unroll
      for (int s = 0; s < K::NSLOT; ++s)
        if (fills[s] > 0) mbar_wait(&bars.full[s], (fills[s] - 1) & 1, &f2);
      failed |= f2;
    }
    if (clear_v) {
      // every copy has landed (lane 0 waited above): clear, then release
      __syncwarp();
      unsigned char *vt = smem + K::OFF_RING + ((2 * nt - 1) % K::NSLOT) * K::TILE;
      for (int idx = lane; idx < (z1 - z0) * K::KB * 8; idx += 32) {
        const int r = z0 + idx / (K::KB * 8), c = (idx / 8) % K::KB, ch = idx % 8;
        *reinterpret_cast<uint4 *>(vt + c * K::BLK + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.v_clean);
    }
  } else if (warp == 1) {
    // ================================================= MMA issuer
    if (lane == 0 && nt > 0) {
      constexpr uint32_t idS = tc::idesc_bf16_f32(kBM, kBN, 0, 0);
      constexpr uint32_t idO = tc::idesc_bf16_f32(kBM, D, 0, 1);
      const uint32_t sQ[2] = {smem_u32(smem + K::OFF_QA), smem_u32(smem + K::OFF_QB)};
      auto slot_addr = [&](int i) { return smem_u32(smem + K::OFF_RING + (i % K::NSLOT) * K::TILE); };
      auto wait_load = [&](int i) {
        return mbar_wait(&bars.full[i % K::NSLOT], (i / K::NSLOT) & 1, &failed);
      };
      auto issue_s = [&](int hd, int j) {
        const uint32_t sK = slot_addr(2 * j);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * K::BLK + (k & 3) * 32;
          tc::mma_bf16_ss(tmem + hd * kBN, tc::sw128_desc(sQ[hd] + off, 16, 1024),
                          tc::sw128_desc(sK + off, 16, 1024), idS, k > 0 ? 1u : 0u);
        }
        tc::mma_commit(&bars.s_full[hd]);
      };
      auto issue_pv = [&](int hd, int j, int k0) {
        // A = P from TMEM (over S of this head: 8 columns per 16 keys);
        // keys [16 k0, 16 k0 + 64)
        const uint32_t sV = slot_addr(2 * j + 1);
#pragma unroll
        for (int k = k0; k < k0 + kBN / 32; ++k) {
          const uint64_t db = tc::sw128_desc(sV + k * 16 * 128, K::BLK, 1024);
          tc::mma_bf16_ts(tmem + K::TM_O + hd * D, tmem + hd * kBN + k * 8, db, idO,
                          (j > 0 || k > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(&bars.q_full, 0, &failed) && wait_load(0);
      if (ok) {
        tc::fence_after_sync();
        issue_s(0, 0);
        issue_s(1, 0);
        tc::mma_commit(&bars.empty[0]);  // K_0
      }
      for (int j = 0; ok && j < nt; ++j) {
        const bool more = j + 1 < nt;
        // head A: first half of P V(j) once its keys 0-63 of P are written,
        // then the second half and S_A(j+1)
        if (!mbar_wait(&bars.p_half[0], j & 1, &failed) || !wait_load(2 * j + 1) ||
            (more && !wait_load(2 * j + 2))) {
          ok = false;
          break;
        }
        if (clear_v && j == nt - 1 && !mbar_wait(&bars.v_clean, 0, &failed)) { ok = false; break; }
        tc::fence_after_sync();
        issue_pv(0, j, 0);
        if (!mbar_wait(&bars.p_full[0], j & 1, &failed)) { ok = false; break; }
        tc::fence_after_sync();
        issue_pv(0, j, 4);
        if (more) issue_s(0, j + 1);
        // head B likewise; then V_j and K_(j+1) are free
        if (!mbar_wait(&bars.p_half[1], j & 1, &failed)) { ok = false; break; }
        tc::fence_after_sync();
        issue_pv(1, j, 0);
        if (!mbar_wait(&bars.p_full[1], j & 1, &failed)) { ok = false; break; }
        tc::fence_after_sync();
        issue_pv(1, j, 4);
        tc::mma_commit(&bars.empty[(2 * j + 1) % K::NSLOT]);
        if (more) {
          issue_s(1, j + 1);
          tc::mma_commit(&bars.empty[(2 * j + 2) % K::NSLOT]);
        }
      }
      tc::mma_commit(&bars.o_done[0]);  // O_A and O_B complete (read by the epilogue)
      tc::mma_commit(&bars.o_done[1]);
      // Drain: every MMA this thread issued has finished before TMEM is freed.
      tc::mma_commit(&bars.mma_fin);
      bool f2 = false;
      mbar_wait(&bars.mma_fin, 0, &f2);
      failed |= f2;
    }
  }
  }

  if (failed) record_status(p.status, kStatusTimeout);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ host
inline bool supported(int d, int Hq, int Hkv) {
  return (d == 64 || d == 128) && (Hq / Hkv) % 2 == 0;
}

template <int D>
gqa_status launch_d(const void *q, const void *k, const void *v, void *o,
                    const int32_t *lens, const int32_t *seg, int B, int Hq, int Hkv,
                    int Tq, int Tk, int cached, int window, float scale_log2,
                    int sms, int32_t *status, cudaStream_t st) {
  using K = Cfg<D>;
  CUtensorMap mq, mk, mv;
  if (!tma::make_bf16_map(&mq, q, D, Tq, B * Hq, 128) ||
      !tma::make_bf16_map(&mk, k, D, Tk, B * Hkv, 128) ||
      !tma::make_bf16_map(&mv, v, D, Tk, B * Hkv, 128))
    return GQA_ERR_CUDA;
  static bool attr_done = false;  // per instantiation; benign race
  if (!attr_done) {
    if (cudaFuncSetAttribute(prefill_pair_kernel<D, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             K::SMEM) != cudaSuccess ||
        cudaFuncSetAttribute(prefill_pair_kernel<D, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             K::SMEM) != cudaSuccess) {
      cudaGetLastError();
      return GQA_ERR_CUDA;
    }
    attr_done = true;
  }
  Params p;
  p.o = (__nv_bfloat16 *)o;
  p.seq_lens = lens;
  p.status = status;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Tq = Tq;
  p.Tk = Tk;
  p.cached = cached;
  p.seg = seg;
  p.window = window;
  p.num_mt = (Tq + kBM - 1) / kBM;
  p.pairs = (Hq / Hkv) / 2;
  p.scale_log2 = scale_log2;
  const long long grid = (long long)B * Hkv * p.pairs * p.num_mt;
  if (grid > 0x7fffffffLL) return GQA_ERR_UNSUPPORTED;
  p.prefetch = grid <= sms ? 1 : 0;
  const cudaError_t e =
      seg ? launch_dependent(prefill_pair_kernel<D, true>, dim3((unsigned)grid), dim3(kThreads),
                             K::SMEM, st, mq, mk, mv, p)
          : launch_dependent(prefill_pair_kernel<D, false>, dim3((unsigned)grid), dim3(kThreads),
                             K::SMEM, st, mq, mk, mv, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_CUDA;
  }
  return GQA_OK;
}

// Prompt (cached = 0: Tq = Tk = T) or queries after a cache (cached = 1:
// Tq new rows against Tk = capacity cells).
inline gqa_status launch(const void *q, const void *k, const void *v, void *o,
                         const int32_t *lens, const int32_t *seg, int B, int Hq, int Hkv,
                         int Tq, int Tk, int cached, int d, int window, float scale_log2,
                         int sms, int32_t *status, cudaStream_t st) {
  if (d == 64)
    return launch_d<64>(q, k, v, o, lens, seg, B, Hq, Hkv, Tq, Tk, cached, window,
                        scale_log2, sms, status, st);
  return launch_d<128>(q, k, v, o, lens, seg, B, Hq, Hkv, Tq, Tk, cached, window,
                       scale_log2, sms, status, st);
}

}  // namespace pf2
}  // namespace gqa
