// prefill_persist.cuh -- persistent tcgen05/TMEM causal-windowed GQA prefill
// for plain prompts, one query head per work item, each 128-key tile's scores
// shared by two softmax warpgroups with their own running maximum, sum and O
// (bf16, sm_100a).
//
// What it computes ("Share key/value heads and make context explicit",
// sections "Give each query head an explicit shared KV head" and "Intersect
// the window with the context already permitted"; FlashAttention's running
// max/sum from "GQA, FlashAttention and the KV cache"): for every batch row
// b, query head h and active cell t < n_b, softmax over the permitted keys
// of scale * q.k, mixed with the value rows of the shared lane g(h);
// inactive rows are zero.
//
// The arithmetic per (query tile, head) is that of prefill_split.cuh (keys
// 0-63 of every tile to one softmax warpgroup, keys 64-127 to the other, each
// with its own online softmax and O, merged once at the end).  What differs
// is the schedule: one CTA per SM walks a list of (query tile, head) items,
// so a CTA's set-up (barriers, TMEM) is paid once, the next item's Q load and
// first QK^T run under the current item's last tiles, and the O / l epilogue
// runs on its own warpgroup while the softmax warps start the next item
// (two O buffers in TMEM at d = 64; at d = 128 the next item's first P V waits
// for the epilogue to have read O).  Items are dealt to CTAs in a snake
// order (round r: CTA c takes item r*G + c for even r, r*G + G-1-c for odd
// r), longest first, so every CTA gets about the same number of KV tiles.
//
//   warp 0      TMA producer: Q of each item (two buffers), K and V tiles
//               into 2-stage rings (128-byte swizzle, no multicast).
//   warp 1      allocates TMEM; lane 0 issues tcgen05.mma: S(j) = Q K_j^T
//               into S[j%2], then O_h += P_h(j-1) V_{j-1}[64h, 64h+64) for
//               key half h once that half's P is written.
//   warps 2-3   idle (the first warpgroup hands registers to the others).
//   warps 4-7   softmax of keys 0-63, warps 8-11 of keys 64-127 (thread =
//               query row = TMEM lane): mask, maximum, lazy rescale of its O,
//               bf16 P over the first half of its own S columns; at the end
//               of an item its (maximum, sum) per row goes to shared memory.
//   warps 12-15 epilogue: O = (O_0 a_0 + O_1 a_1) / (l_0 a_0 + l_1 a_1),
//               a_h = 2^(m_h - max(m_0, m_1)), in bf16, one row per thread.
// TMEM columns: S0 [0,128), S1 [128,256), O buffer ob: half h at
// [256 + 2 d ob + d h, +d).
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tma_host.cuh"

namespace gqa {
namespace pfp {

constexpr int kBM = 128, kBN = 128;
constexpr int kThreads = 512;
// Registers per thread after the split (the launch gives 128 each at 512
// threads): first warpgroup, the two softmax warpgroups, the epilogue one.
constexpr int kRegsLow = 56, kRegsSoft = 168, kRegsEpi = 96;
static_assert(128 * kRegsLow + 256 * kRegsSoft + 128 * kRegsEpi <= 65536, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Query tiles per head from which items are ordered head by head.
constexpr int kHeadMajorTiles = 64;

template <int D>
struct Cfg {
  static constexpr int KB = D / 64;                 // 64-column blocks
  static constexpr int BLK = kBM * 128;             // 128 rows x 128 B = 16 KB
  static constexpr int TILE = KB * BLK;             // a Q, K or V tile
  // K/V stages; equal to the number of S buffers, so that S[s] complete
  // also means K stage s is free and P V[s] complete that V stage s is.
  static constexpr int STAGES = 2;
  static_assert(STAGES == 2, "S buffers and K/V stages share their index");
  static constexpr int NQ = 2;                      // Q buffers
  static constexpr int NOB = (D == 64) ? 2 : 1;     // O buffers in TMEM
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * TILE;
  static constexpr int OFF_V = OFF_K + STAGES * TILE;
  static constexpr int DYN_BYTES = OFF_V + STAGES * TILE;
  static constexpr uint32_t TM_O = 256;
  static_assert(TM_O + NOB * 2 * D <= kTmemCols, "two S buffers and the O buffers must fit in TMEM");
  // At least 120 KB so that only one CTA (which holds all 512 TMEM columns)
  // is resident per SM.
  static constexpr int SMEM = (DYN_BYTES + 1024 > 120 * 1024 ? DYN_BYTES + 1024 : 120 * 1024);
  static_assert(SMEM <= 220 * 1024, "shared memory per CTA");
};

struct Params {
  __nv_bfloat16 *o;
  const int32_t *seq_lens;  // [B] active rows per sequence, or NULL (all T)
  int32_t *status;
  int B, Hq, Hkv, T, window, num_mt, n_items;
  int head_major;  // item order: 1 head by head, 0 query tile by query tile
  float scale_log2;
};

struct Bars {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[2], v_full[2];
  // S[s] written by the MMA; also K stage s read (the stage and the S
  // buffer of a KV tile have the same index, so no separate commit)
  uint64_t s_full[2];
  uint64_t p_full[2][2];  // [s][half]: that half's P written over S[s]
  uint64_t pv_done[2];    // both halves' P V of an S[s] tile complete; V stage s read
  uint64_t o_done[2];     // an item's last P V into O buffer [ob] complete
  uint64_t o_free[2];     // the epilogue has read O buffer [ob]
  uint64_t ml_full[2];    // both halves' (maximum, sum) of the item in [ob] posted
  uint64_t mma_fin;
  uint32_t tmem_base;
};

// One work item: query tile mt of head h of sequence b.
struct Item {
  int b, h, g, m0;
  int rows;          // active query rows of the sequence (n_b), -1 if invalid
  int j0, nt;        // KV tiles [j0, j0 + nt) hold the tile's permitted keys
  int lo_max;        // tiles starting before this key need masks (window)
  bool report;       // this item reports an invalid length (one per sequence)
};

// Item of CTA c in round r of G CTAs (snake order), or -1.
__device__ __forceinline__ int item_of(int c, int r, int G, int n) {
  const long long it = (long long)r * G + ((r & 1) ? (G - 1 - c) : c);
  return it < n ? (int)it : -1;
}

__device__ __forceinline__ Item decode_item(const Params &p, int it) {
  Item x;
  const int BH = p.B * p.Hq;
  int mt, bh;
  if (p.head_major) {
    bh = it / p.num_mt;
    mt = p.num_mt - 1 - it % p.num_mt;
  } else {
    mt = p.num_mt - 1 - it / BH;
    bh = it % BH;
  }
  x.b = bh / p.Hq;
  x.h = bh - x.b * p.Hq;
  x.g = x.h / (p.Hq / p.Hkv);
  x.m0 = mt * kBM;
  int n_b = p.T;
  x.report = false;
  if (p.seq_lens) {
    n_b = p.seq_lens[x.b];
    if (n_b < 0 || n_b > p.T) {
      x.report = (mt == 0 && x.h == 0);
      n_b = -1;  // the whole sequence is written as zeros
    }
  }
  x.rows = n_b;
  const int lo_min = p.window > 0 ? max(0, x.m0 - (p.window - 1)) : 0;
  x.lo_max = p.window > 0 ? max(0, x.m0 + kBM - p.window) : 0;
  x.j0 = 0;
  x.nt = 0;
  if (n_b > x.m0) {
    const int hi = min(x.m0 + kBM - 1, n_b - 1);
    x.j0 = lo_min / kBN;
    x.nt = hi / kBN - x.j0 + 1;
  }
  return x;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_persist_kernel(const __grid_constant__ CUtensorMap tmQ,
                           const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const Params p) {
  using K = Cfg<D>;
  extern __shared__ unsigned char smem_raw[];
  __shared__ Bars bars;
  __shared__ float mlbuf[K::NOB * 2 * 2 * kBM];  // [ob][half][maximum, sum][row]
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.q_full[s], 1);
      mbar_init(&bars.q_empty[s], 1);
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.p_full[s][0], 4);  // the half's four warps
      mbar_init(&bars.p_full[s][1], 4);
      mbar_init(&bars.pv_done[s], 1);
      mbar_init(&bars.o_done[s], 1);
      mbar_init(&bars.o_free[s], 4);     // the four epilogue warps
      mbar_init(&bars.ml_full[s], 8);    // the eight softmax warps
    }
    mbar_init(&bars.mma_fin, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&bars.tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  // Barriers and TMEM are set up; from here on the CTA reads memory the
  // previous kernel on the stream may write: wait for it (a no-op unless
  // launched as a programmatic dependent), then let the next one start.
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();

  const uint32_t tmem = bars.tmem_base;
  const int G = gridDim.x, c = blockIdx.x;
  bool failed = false;

  if (warp >= 4 && warp < 12) {
    // ================================================= softmax warpgroups
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoft));
    const int half = (warp - 4) >> 2;        // keys [64 half, 64 half + 64) of every tile
    const int q4 = warp & 3;                 // TMEM lane quarter of this warp
    const int row = q4 * 32 + lane;          // query row within the tile
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const float sc = p.scale_log2;
    int ai = 0, tcg = 0;  // items with work so far; KV tiles so far
    bool alive = true;    // warp-uniform: every wait below is taken by the whole warp
    for (int r = 0; r * G < p.n_items && alive; ++r) {
      const int it = item_of(c, r, G, p.n_items);
      if (it < 0) continue;
      const Item x = decode_item(p, it);
      if (x.nt == 0) continue;
      const int ob = ai % K::NOB;
      const int t = x.m0 + row;             // key position of this query row
      const int lo_t = p.window > 0 ? max(0, t - (p.window - 1)) : 0;
      const uint32_t tO = tmem + lane_base + K::TM_O + ob * 2 * D + half * D;
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;
      for (int j = 0; j < x.nt; ++j) {
        const int tg = tcg + j, sb = tg & 1;
        const int kt = (x.j0 + j) * kBN;   // key of the tile's first column
        const int kb = kt + half * 64;     // key of this half's first column
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.s_full[sb], (tg >> 1) & 1, &failed))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t tS = tmem + lane_base + sb * kBN + half * 64;
        float s[64];
        tc::tmem_ld32(tS, s);
        tc::tmem_ld32(tS + 32, s + 32);
        tc::tmem_wait_ld();
        const bool edge = (kb + 63 > x.m0) || (kb < x.lo_max);
        if (edge) {
          // key kb + i is permitted for lo_t - kb <= i <= t - kb.  Most rows of an
          // edge tile need only the upper bound (the diagonal), and a warp none of
          // whose rows cuts this half's keys skips the loop.
          const int hi_i = t - kb, lo_i = lo_t - kb;
          if (__any_sync(0xffffffffu, lo_i > 0)) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (i > hi_i || i < lo_i) s[i] = -INFINITY;
          } else if (__any_sync(0xffffffffu, hi_i < 64 - 1)) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (i > hi_i) s[i] = -INFINITY;
          }
        }
        // this half's maximum of s*scale (sc*max(s) for sc > 0, sc*min(s) otherwise)
        float mx;
        {
          const bool neg = !(sc > 0.f);
          float mc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          if (!neg) {
#pragma unroll
            for (int i = 0; i < 64; i += 2) mc[(i >> 1) & 3] = fmax3(mc[(i >> 1) & 3], s[i], s[i + 1]);
          } else {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              mc[i & 3] = fmaxf(mc[i & 3], s[i] == -INFINITY ? -INFINITY : -s[i]);
          }
          mx = fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3]));
        }
        const float m_tile = (mx == -INFINITY) ? -INFINITY : mx * fabsf(sc);
        if (j == 0) {
          m_run = m_tile;
        } else if (__any_sync(0xffffffffu, m_tile > m_run + kRescaleThreshold)) {
          // This half's O must hold P V(j-1) before it is rescaled.  P(j)
          // needs no wait: S(j) was issued after P V(j-2) by the same
          // thread, so S(j) ready means P V(j-2) has read what P(j) overwrites.
          const int pg = tg - 1;
          if (!__all_sync(0xffffffffu,
                          mbar_wait(&bars.pv_done[pg & 1], (pg >> 1) & 1, &failed))) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const float m_new = fmaxf(m_run, m_tile);
          const float alpha = m_new == m_run ? 1.f : exp2f(m_run - m_new);  // 0 from -inf
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            float ov[32];
            tc::tmem_ld32(tO + cc * 32, ov);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] *= alpha;
            tc::tmem_st32(tO + cc * 32, ov);
          }
          tc::tmem_wait_st();
          l_run *= alpha;
          m_run = m_new;
        }
        // bf16 P over the first 32 of this half's S columns (column c holds
        // p[2c], p[2c+1]), where the P V MMA reads it as its A operand.
        {
          const float msub = m_run == -INFINITY ? 0.f : m_run;
          const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(-msub, -msub);
          float2 lsum2 = make_float2(0.f, 0.f);
          float w[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float2 xx = ffma2v(make_float2(s[2 * e], s[2 * e + 1]), sc2, nm2);
            const float2 pv = make_float2(ex2_approx(xx.x), ex2_approx(xx.y));
            lsum2 = fadd2v(lsum2, pv);
            w[e] = __uint_as_float(pack_bf16(pv.x, pv.y));
          }
          tc::tmem_st32(tS, w);
          tc::tmem_wait_st();
          l_run += lsum2.x + lsum2.y;
        }
        if (kt + kBN > x.rows && (row >> 6) == half) {
          // Cells past the sequence in this V tile are not the sequence's
          // (prompt padding may hold NaN): their p is 0, but 0 * NaN is not,
          // so clear those rows before P V is issued.  V row r is cleared by
          // thread r of the half whose keys it holds (rows 0-63: half 0).
          const int vs = tg % K::STAGES;
          const bool vok = mbar_wait(&bars.v_full[vs], (tg / K::STAGES) & 1, &failed);
          if (vok && kt + row >= x.rows) {
            unsigned char *vrow = smem + K::OFF_V + vs * K::TILE + row * 128;
#pragma unroll
            for (int cc = 0; cc < K::KB; ++cc)
#pragma unroll
              for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<uint4 *>(vrow + cc * K::BLK + ch * 16) = make_uint4(0, 0, 0, 0);
          }
          tc::fence_proxy_async_smem();
          if (!__all_sync(0xffffffffu, vok)) {
            ok = false;
            break;
          }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[sb][half]);
      }
      if (!ok) {
        alive = false;
        break;
      }
      // Hand this half's (maximum, sum) of every row to the epilogue.  The
      // buffer's previous item must have been read: its o_free phase.
      if (ai >= K::NOB &&
          !__all_sync(0xffffffffu, mbar_wait(&bars.o_free[ob], ((ai / K::NOB) - 1) & 1, &failed))) {
        alive = false;
        break;
      }
      mlbuf[((ob * 2 + half) * 2 + 0) * kBM + row] = m_run;
      mlbuf[((ob * 2 + half) * 2 + 1) * kBM + row] = l_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.ml_full[ob]);
      tcg += x.nt;
      ai++;
    }
  } else if (warp >= 12) {
    // ================================================= epilogue warpgroup
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    int ai = 0;
    bool alive = true;  // warp-uniform
    for (int r = 0; r * G < p.n_items && alive; ++r) {
      const int it = item_of(c, r, G, p.n_items);
      if (it < 0) continue;
      const Item x = decode_item(p, it);
      if (x.report && warp == 12 && lane == 0) record_status(p.status, GQA_ERR_CAPACITY);
      const int qr = x.m0 + row;
      const bool active = qr < x.rows;
      __nv_bfloat16 *orow = p.o + (((size_t)x.b * p.Hq + x.h) * p.T + min(qr, p.T - 1)) * D;
      bool have = false;
      int ob = 0;
      float a0 = 0.f, a1 = 0.f, inv = 0.f;
      if (x.nt > 0) {
        ob = ai % K::NOB;
        const int ph = (ai / K::NOB) & 1;
        have = __all_sync(0xffffffffu, mbar_wait(&bars.o_done[ob], ph, &failed) &&
                                           mbar_wait(&bars.ml_full[ob], ph, &failed));
        tc::fence_after_sync();
        const float m0v = mlbuf[((ob * 2 + 0) * 2 + 0) * kBM + row];
        const float l0v = mlbuf[((ob * 2 + 0) * 2 + 1) * kBM + row];
        const float m1v = mlbuf[((ob * 2 + 1) * 2 + 0) * kBM + row];
        const float l1v = mlbuf[((ob * 2 + 1) * 2 + 1) * kBM + row];
        const float m_all = fmaxf(m0v, m1v);
        a0 = m_all == -INFINITY ? 0.f : exp2f(m0v - m_all);
        a1 = m_all == -INFINITY ? 0.f : exp2f(m1v - m_all);
        const float l_row = l0v * a0 + l1v * a1;
        inv = (active && have && l_row > 0.f) ? 1.f / l_row : 0.f;
      }
      const uint32_t tO0 = tmem + lane_base + K::TM_O + ob * 2 * D;  // O of key half 0
      const uint32_t tO1 = tO0 + D;                                    // O of key half 1
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        float ov[32], ow[32];
        if (have) {
          tc::tmem_ld32(tO0 + cc * 32, ov);
          tc::tmem_ld32(tO1 + cc * 32, ow);
          tc::tmem_wait_ld();
        }
#pragma unroll
        for (int i = 0; i < 32; ++i)  // inactive rows are exact zeros (their O may be NaN)
          ov[i] = (have && active) ? (ov[i] * a0 + ow[i] * a1) * inv : 0.f;
        if (qr < p.T) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t w4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) w4[i] = pack_bf16(ov[e * 8 + 2 * i], ov[e * 8 + 2 * i + 1]);
            *reinterpret_cast<uint4 *>(orow + cc * 32 + e * 8) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
      if (x.nt > 0) {
        if (!have) {
          alive = false;
          break;
        }
        // O and the (maximum, sum) slots of buffer ob are free again
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.o_free[ob]);
        ai++;
      }
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    if (warp == 0) {
      // ================================================= TMA producer
      if (lane == 0) {
        tc::prefetch_tmap(&tmQ);
        tc::prefetch_tmap(&tmK);
        tc::prefetch_tmap(&tmV);
        int qf[2] = {0, 0}, kf[K::STAGES], vf[K::STAGES];
#pragma unroll
        for (int s = 0; s < K::STAGES; ++s) kf[s] = vf[s] = 0;
        int ai = 0, tcg = 0;
        for (int r = 0; r * G < p.n_items && !failed; ++r) {
          const int it = item_of(c, r, G, p.n_items);
          if (it < 0) continue;
          const Item x = decode_item(p, it);
          if (x.nt == 0) continue;
          const int qb = ai % K::NQ;
          if (ai >= K::NQ && !mbar_wait(&bars.q_empty[qb], ((ai / K::NQ) - 1) & 1, &failed)) break;
          mbar_arrive_expect_tx(&bars.q_full[qb], K::TILE);
#pragma unroll
          for (int cc = 0; cc < K::KB; ++cc)
            tc::tma_load_3d(smem + K::OFF_Q + qb * K::TILE + cc * K::BLK, &tmQ, cc * 64, x.m0,
                            x.b * p.Hq + x.h, &bars.q_full[qb]);
          qf[qb]++;
          for (int j = 0; j < x.nt; ++j) {
            const int tg = tcg + j, s = tg % K::STAGES;
            const int krow = (x.j0 + j) * kBN;
            // stage s is free once S of the tile two back is complete
            if (tg >= K::STAGES && !mbar_wait(&bars.s_full[s], ((tg / K::STAGES) - 1) & 1, &failed)) break;
            mbar_arrive_expect_tx(&bars.k_full[s], K::TILE);
#pragma unroll
            for (int cc = 0; cc < K::KB; ++cc)
              tc::tma_load_3d(smem + K::OFF_K + s * K::TILE + cc * K::BLK, &tmK, cc * 64, krow,
                              x.b * p.Hkv + x.g, &bars.k_full[s]);
            kf[s]++;
            if (tg >= K::STAGES && !mbar_wait(&bars.pv_done[s], ((tg / K::STAGES) - 1) & 1, &failed)) break;
            mbar_arrive_expect_tx(&bars.v_full[s], K::TILE);
#pragma unroll
            for (int cc = 0; cc < K::KB; ++cc)
              tc::tma_load_3d(smem + K::OFF_V + s * K::TILE + cc * K::BLK, &tmV, cc * 64, krow,
                              x.b * p.Hkv + x.g, &bars.v_full[s]);
            vf[s]++;
          }
          tcg += x.nt;
          ai++;
        }
        // Never leave a TMA load in flight into an exiting CTA.
        bool f2 = false;
        for (int s = 0; s < 2; ++s)
          if (qf[s] > 0) mbar_wait(&bars.q_full[s], (qf[s] - 1) & 1, &f2);
#pragma unroll
        for (int s = 0; s < K::STAGES; ++s) {
          if (kf[s] > 0) mbar_wait(&bars.k_full[s], (kf[s] - 1) & 1, &f2);
          if (vf[s] > 0) mbar_wait(&bars.v_full[s], (vf[s] - 1) & 1, &f2);
        }
        failed |= f2;
      }
    } else if (warp == 1) {
      // ================================================= MMA issuer
      if (lane == 0) {
        constexpr uint32_t idS = tc::idesc_bf16_f32(kBM, kBN, 0, 0);
        constexpr uint32_t idO = tc::idesc_bf16_f32(kBM, D, 0, 1);
        int ai = 0, tcg = 0;
        bool issued = false;
        bool s0_ahead = false;  // the current item's first S was issued ahead
        // S of global tile tg from Q buffer qbuf (and Q released after the
        // item's last S).
        auto issue_s = [&](int tg, int qbuf, bool last) -> bool {
          const int sb = tg & 1, ks = tg % K::STAGES;
          if (!mbar_wait(&bars.k_full[ks], (tg / K::STAGES) & 1, &failed)) return false;
          tc::fence_after_sync();
          const uint32_t sQ = smem_u32(smem + K::OFF_Q + qbuf * K::TILE);
          const uint32_t sK = smem_u32(smem + K::OFF_K + ks * K::TILE);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * K::BLK + (k & 3) * 32;
            tc::mma_bf16_ss(tmem + sb * kBN, tc::sw128_desc(sQ + off, 16, 1024),
                            tc::sw128_desc(sK + off, 16, 1024), idS, k > 0 ? 1u : 0u);
          }
          issued = true;
          tc::mma_commit(&bars.s_full[sb]);
          if (last) tc::mma_commit(&bars.q_empty[qbuf]);  // Q read by its last S
          return true;
        };
        for (int r = 0; r * G < p.n_items && !failed; ++r) {
          const int it = item_of(c, r, G, p.n_items);
          if (it < 0) continue;
          const Item x = decode_item(p, it);
          if (x.nt == 0) continue;
          const int qb = ai % K::NQ, ob = ai % K::NOB;
          const uint32_t tO = tmem + K::TM_O + ob * 2 * D;
          // O_h += P_h(jj) V_jj[64h, 64h+64) for key half h, once that half's
          // P is written; the item's first P V starts O afresh, after the
          // epilogue has read this buffer's previous item.
          auto issue_pv = [&](int jj) -> bool {
            const int tg = tcg + jj, s = tg & 1, vs = tg % K::STAGES;
            if (jj == 0 && ai >= K::NOB &&
                !mbar_wait(&bars.o_free[ob], ((ai / K::NOB) - 1) & 1, &failed))
              return false;
            if (!mbar_wait(&bars.v_full[vs], (tg / K::STAGES) & 1, &failed)) return false;
            const uint32_t sV = smem_u32(smem + K::OFF_V + vs * K::TILE);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              if (!mbar_wait(&bars.p_full[s][hh], (tg >> 1) & 1, &failed)) return false;
              tc::fence_after_sync();
#pragma unroll
              for (int k = 4 * hh; k < 4 * hh + 4; ++k) {  // A = P from TMEM, 8 columns per 16 keys
                const uint64_t db = tc::sw128_desc(sV + k * 16 * 128, K::BLK, 1024);
                tc::mma_bf16_ts(tO + hh * D, tmem + s * kBN + hh * 64 + (k - 4 * hh) * 8, db, idO,
                                (jj > 0 || k > 4 * hh) ? 1u : 0u);
              }
            }
            tc::mma_commit(&bars.pv_done[s]);
            return true;
          };
          // (a Q wait of a phase already consumed ahead would be ambiguous)
          if (!s0_ahead && !mbar_wait(&bars.q_full[qb], (ai / K::NQ) & 1, &failed)) break;
          bool ok = true;
          for (int j = 0; j < x.nt; ++j) {
            // S(j) overwrites P of the tile two back, whose P V came first.
            if (!(j == 0 && s0_ahead) && !issue_s(tcg + j, qb, j == x.nt - 1)) { ok = false; break; }
            if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
          }
          // The next item's first S goes ahead of this item's last P V (its
          // S buffer held P of this item's last tile but one, already read),
          // so that the softmax does not wait for both at the item boundary.
          s0_ahead = false;
          for (int r2 = r + 1; ok && r2 * G < p.n_items; ++r2) {
            const int it2 = item_of(c, r2, G, p.n_items);
            if (it2 < 0) continue;
            const Item x2 = decode_item(p, it2);
            if (x2.nt == 0) continue;
            const int qb2 = (ai + 1) % K::NQ;
            ok = mbar_wait(&bars.q_full[qb2], ((ai + 1) / K::NQ) & 1, &failed) &&
                 issue_s(tcg + x.nt, qb2, x2.nt == 1);
            s0_ahead = ok;
            break;
          }
          if (!ok || !issue_pv(x.nt - 1)) break;
          tc::mma_commit(&bars.o_done[ob]);
          tcg += x.nt;
          ai++;
        }
        // Drain: every MMA this thread issued has finished before TMEM is freed.
        if (issued) {
          tc::mma_commit(&bars.mma_fin);
          bool f2 = false;
          mbar_wait(&bars.mma_fin, 0, &f2);
          failed |= f2;
        }
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
inline bool supported(int d) { return d == 64 || d == 128; }

// Prompt of T rows per head (Q, K, V and O [B,H,T,d]); seq_lens optional.
template <int D>
gqa_status launch_d(const void *q, const void *k, const void *v, void *o,
                    const int32_t *lens, int B, int Hq, int Hkv, int T, int window,
                    float scale_log2, int sms, int32_t *status, cudaStream_t st) {
  using K = Cfg<D>;
  CUtensorMap mq, mk, mv;
  if (!tma::make_bf16_map(&mq, q, D, T, B * Hq, 128) ||
      !tma::make_bf16_map(&mk, k, D, T, B * Hkv, 128) ||
      !tma::make_bf16_map(&mv, v, D, T, B * Hkv, 128))
    return GQA_ERR_CUDA;
  static bool attr_done = false;  // per instantiation; benign race
  if (!attr_done) {
    if (cudaFuncSetAttribute(prefill_persist_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  p.T = T;
  p.window = window;
  p.num_mt = (T + kBM - 1) / kBM;
  const long long n_items = (long long)B * Hq * p.num_mt;
  if (n_items > 0x7fffffffLL) return GQA_ERR_UNSUPPORTED;
  p.n_items = (int)n_items;
  p.head_major = p.num_mt >= kHeadMajorTiles;
  p.scale_log2 = scale_log2;
  const int grid = (int)(n_items < sms ? n_items : sms);
  if (launch_dependent(prefill_persist_kernel<D>, dim3((unsigned)grid), dim3(kThreads), K::SMEM, st,
                       mq, mk, mv, p) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_CUDA;
  }
  return GQA_OK;
}

inline gqa_status launch(const void *q, const void *k, const void *v, void *o,
                         const int32_t *lens, int B, int Hq, int Hkv, int T, int d, int window,
                         float scale_log2, int sms, int32_t *status, cudaStream_t st) {
  if (d == 64)
    return launch_d<64>(q, k, v, o, lens, B, Hq, Hkv, T, window, scale_log2, sms, status, st);
  return launch_d<128>(q, k, v, o, lens, B, Hq, Hkv, T, window, scale_log2, sms, status, st);
}

}  // namespace pfp
}  // namespace gqa
