// prefill_split.cuh -- tcgen05/TMEM causal-windowed GQA prefill, one query
// head per CTA, each 128-key tile's scores shared by two softmax warpgroups
// that each keep their own running maximum, sum and O (bf16, sm_100a).
//
// What it computes ("Share key/value heads and make context explicit",
// sections "Give each query head an explicit shared KV head" and "Intersect
// the window with the context already permitted"; FlashAttention's running
// max/sum from "GQA, FlashAttention and the KV cache"): for every batch row
// b, query head h and active cell t < n_b, softmax over the permitted keys
// of scale * q.k, mixed with the value rows of the shared lane g(h);
// inactive rows are zero.  It serves queries after a cache (the multi-token
// decode) and packed prompts of odd group sizes (MHA included), which the
// paired kernel (prefill_pair.cuh) cannot; plain prompts of those shapes run
// the same arithmetic on the persistent kernel (prefill_persist.cuh).
//
// One CTA owns a 128-row query tile of one (b, h) and walks the 128-key
// tiles that intersect its permitted band, skipping tiles wholly outside
// the causal window.  Keys 0-63 of every tile belong to one softmax
// warpgroup and keys 64-127 to the other.  Each runs the online softmax
// over its own keys only (its own running maximum and sum) and accumulates
// its own O_h = sum P_h V_h, so the two never wait for each other inside
// the loop; the epilogue combines them once:
//   O = (O_0 a_0 + O_1 a_1) / (l_0 a_0 + l_1 a_1),  a_h = 2^(m_h - max(m_0, m_1)),
// the same merge as two split-K partials.  S is double-buffered in TMEM, so
// the softmax of tile j runs while the tensor cores compute S(j+1):
//   warp 0      TMA producer: Q once, then K and V tiles into 2-stage rings
//               (128-byte swizzle, no multicast).
//   warp 1      allocates TMEM; lane 0 issues tcgen05.mma: S(j) = Q K_j^T
//               into S[j%2] (M=N=128, K=d), then for each key half h once
//               its P is written, O_h += P_h(j-1) V_{j-1}[64h, 64h+64)
//               (M=128, N=d, K=64, P read from TMEM as the A operand).
//   warps 2-3   idle (they complete the first warpgroup, which hands most of
//               its registers to the softmax warpgroups with setmaxnreg).
//   warps 4-7   softmax of keys 0-63, warps 8-11 of keys 64-127: thread =
//               query row (TMEM lane).  Per tile each half takes its 64
//               scores, masks edge tiles, rescales its O when its maximum
//               grew by more than 2^8 (lazy rescale), and writes 32 columns
//               of bf16 P over the first half of its own S columns.
// TMEM columns: S0 [0,128), S1 [128,256), O_0 [256, 256+d), O_1 [256+d,
// 256+2d); P_h(j) over S[j%2] columns [64h, 64h+32).  S(j) overwrites P(j-2)
// only after P V(j-2), which the same thread issued first.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tma_host.cuh"

namespace gqa {
namespace pfs {

constexpr int kBM = 128, kBN = 128;
constexpr int kThreads = 384;
// Registers per thread after the split: 128 * kRegsLow + 256 * kRegsHigh
// must not exceed 384 * 168 (the launch's registers at one CTA per SM).
constexpr int kRegsLow = 72, kRegsHigh = 216;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * 168, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Query tiles per head from which CTAs are ordered head by head.
constexpr int kHeadMajorTiles = 64;

template <int D>
struct Cfg {
  static constexpr int KB = D / 64;                 // 64-column blocks
  static constexpr int BLK = kBM * 128;             // 128 rows x 128 B = 16 KB
  static constexpr int TILE = KB * BLK;             // a Q, K or V tile
  static constexpr int STAGES = 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE;
  static constexpr int OFF_V = OFF_K + STAGES * TILE;
  static constexpr int DYN_BYTES = OFF_V + STAGES * TILE;
  static constexpr uint32_t TM_O = 256;              // O of key half 0; half 1 at TM_O + D
  static_assert(TM_O + 2 * D <= kTmemCols, "two S buffers and two O halves must fit in TMEM");
  // At least 120 KB so that only one CTA (which holds all 512 TMEM columns)
  // is resident per SM.
  static constexpr int SMEM = (DYN_BYTES + 1024 > 120 * 1024 ? DYN_BYTES + 1024 : 120 * 1024);
};

struct Params {
  __nv_bfloat16 *o;
  const int32_t *seq_lens;
  int32_t *status;
  int B, Hq, Hkv, window, num_mt;
  int Tq;      // query rows per head (Q and O are [B,Hq,Tq,d])
  int Tk;      // key rows per KV lane (K and V are [B,Hkv,Tk,d])
  int cached;  // 0: prompt, query row t at position t, n_b = active rows;
               // 1: queries after a cache, query row i at position n_b-Tq+i
  const int32_t *seg;  // prompt only: [B,Tq] first key cell of row t's
                       // packed segment, or NULL (segment start 0)
  float scale_log2;
  int head_major;  // CTA order: 1 head by head, 0 query tile by query tile
};

// First permitted key of query position t ("Intersect the window with the
// context already permitted": the later of the segment start and the
// window start); t + 1 (no key) when the segment start is not in [0, t].
__device__ __forceinline__ int row_lo(const Params &p, int b, int t) {
  int s0 = 0;
  if (p.seg) {
    s0 = p.seg[(size_t)b * p.Tq + t];
    if (s0 < 0 || s0 > t) return t + 1;
  }
  return p.window > 0 ? max(s0, t - (p.window - 1)) : s0;
}

struct Bars {
  uint64_t q_full;
  uint64_t k_full[2], v_full[2], k_empty[2], v_empty[2];
  uint64_t s_full[2];             // S[s] written by the MMA
  uint64_t p_full[2][2];          // [s][half]: that half's P written over S[s]
  uint64_t o_done[2];             // both halves' P V of an S[s] tile complete
  uint64_t mma_fin;
  uint32_t tmem_base;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_split_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const Params p) {
  using K = Cfg<D>;
  extern __shared__ unsigned char smem_raw[];
  __shared__ Bars bars;
  __shared__ float xbuf[2 * 2 * kBM];  // [m, l][half][row], exchanged once at the end
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- which tile.  Short prompts: longest causal rows first over all
  // heads (the longest CTAs start in the first wave).  Long ones (head_major):
  // head by head, its query tiles from the last, so the CTAs in flight share
  // a few heads' K/V windows in L2 instead of one tile of every head.
  const int BH = p.B * p.Hq;
  int mt, bh;
  if (p.head_major) {
    bh = (int)(blockIdx.x / p.num_mt);
    mt = p.num_mt - 1 - (int)(blockIdx.x % p.num_mt);
  } else {
    mt = p.num_mt - 1 - (int)(blockIdx.x / BH);
    bh = (int)(blockIdx.x % BH);
  }
  const int b = bh / p.Hq, h = bh - b * p.Hq;
  const int g = h / (p.Hq / p.Hkv);
  const int m0 = mt * kBM;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.k_empty[s], 1);
      mbar_init(&bars.v_empty[s], 1);
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.p_full[s][0], 4);  // the half's four warps
      mbar_init(&bars.p_full[s][1], 4);
      mbar_init(&bars.o_done[s], 1);
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

  // n_b keys of sequence b; `rows` query rows produce output, the query
  // row i sits at key position off + i; a0 = position of this tile's row 0.
  int n_b = p.Tk;
  if (p.seq_lens) {
    n_b = p.seq_lens[b];
    if (n_b < 0 || n_b > p.Tk || (p.cached && n_b < p.Tq)) {
      if (threadIdx.x == 0 && mt == 0 && h == 0) record_status(p.status, GQA_ERR_CAPACITY);
      n_b = -1;  // the whole sequence is written as zeros
    }
  }
  const int off = (p.cached && n_b >= 0) ? n_b - p.Tq : 0;
  const int rows = n_b < 0 ? 0 : (p.cached ? p.Tq : n_b);
  const int a0 = off + m0;
  const int n_keys = max(n_b, 0);
  // Packed segments: the tile's rows (one per thread of warps 0-3) give the
  // smallest and largest first permitted key; invalid starts are reported.
  __shared__ int s_lo_min[4], s_lo_max[4];
  if (p.seg && warp < 4) {
    const int t = a0 + (int)threadIdx.x;
    int lmin = 0x7fffffff, lmax = -1;
    if (t < off + rows) {
      const int lo = row_lo(p, b, t);
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
  if (p.seg) __syncthreads();  // s_lo_min / s_lo_max
  // KV tiles [j0, j0 + nt) cover the tile's permitted keys; tiles starting
  // before lo_max need masks (some row's first key lies inside them).
  int lo_min, lo_max;
  if (p.seg) {
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
  const uint32_t tmem = bars.tmem_base;
  bool failed = false;

  if (warp >= 4) {
    // ================================================= softmax warpgroups
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    const int half = (warp - 4) >> 2;        // score columns [64 half, 64 half + 64)
    const int q4 = warp & 3;                 // TMEM lane quarter of this warp
    const int row = q4 * 32 + lane;          // query row within the tile
    const int t = a0 + row;                  // key position of this query row
    const int qr = m0 + row;                 // its row in Q and O
    const bool active = t < off + rows;
    const int lo_t = active ? row_lo(p, b, t) : 0;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const uint32_t tO = tmem + lane_base + K::TM_O + half * D;  // this half's O
    const float sc = p.scale_log2;
    // Each half keeps its own running maximum and sum over its 64 keys of
    // every tile and its own O; the two are combined once, in the epilogue.
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int sb = j & 1;
      const int kt = (j0 + j) * kBN;     // key of the tile's first column
      const int kb = kt + half * 64;     // key of this half's first column
      if (!__all_sync(0xffffffffu, mbar_wait(&bars.s_full[sb], (j >> 1) & 1, &failed))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const uint32_t tS = tmem + lane_base + sb * kBN + half * 64;
      float s[64];
      tc::tmem_ld32(tS, s);
      tc::tmem_ld32(tS + 32, s + 32);
      tc::tmem_wait_ld();
      const bool edge = (kb + 63 > a0) || (kb < lo_max);
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
        // This half's O must hold P V(j-1) before it is rescaled: o_done of
        // S[(j-1)%2] completes its ((j-1)/2)-th phase with it.  P(j) itself
        // needs no wait: S(j) was issued after P V(j-2) by the same thread,
        // so S(j) ready means P V(j-2) has read the P that P(j) overwrites.
        const int pj = j - 1;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&bars.o_done[pj & 1], (pj >> 1) & 1, &failed))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const float m_new = fmaxf(m_run, m_tile);
        const float alpha = m_new == m_run ? 1.f : exp2f(m_run - m_new);  // 0 from -inf
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
          const float2 x = ffma2v(make_float2(s[2 * e], s[2 * e + 1]), sc2, nm2);
          const float2 pv = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          lsum2 = fadd2v(lsum2, pv);
          w[e] = __uint_as_float(pack_bf16(pv.x, pv.y));
        }
        tc::tmem_st32(tS, w);
        tc::tmem_wait_st();
        l_run += lsum2.x + lsum2.y;
      }
      if (kt + kBN > n_keys && (row >> 6) == half) {
        // Cells past the sequence in this V tile are not the sequence's (an
        // unwritten cache cell may hold NaN): their p is 0, but 0 * NaN is
        // not, so clear those rows before P V is issued.  V row r is cleared
        // by thread r of the half whose keys it holds (rows 0-63: half 0).
        bool vok = mbar_wait(&bars.v_full[sb], (j >> 1) & 1, &failed);
        if (vok && kt + row >= n_keys) {
          unsigned char *vrow = smem + K::OFF_V + sb * K::TILE + row * 128;
#pragma unroll
          for (int c = 0; c < K::KB; ++c)
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
              *reinterpret_cast<uint4 *>(vrow + c * K::BLK + ch * 16) = make_uint4(0, 0, 0, 0);
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

    // ---- epilogue.  The last P V of both halves completes the last phase
    // of o_done[(nt-1)%2] (after every earlier MMA of the issuing thread).
    // The halves swap their (maximum, sum) once through shared memory, then
    // each writes d/2 columns of O = (O_0 a_0 + O_1 a_1) / (l_0 a_0 + l_1 a_1),
    // a_h = 2^(m_h - max(m_0, m_1)), one row per thread.
    bool have = false;
    if (nt > 0 && ok) {
      const int lj = nt - 1;
      have = __all_sync(0xffffffffu, mbar_wait(&bars.o_done[lj & 1], (lj >> 1) & 1, &failed));
      tc::fence_after_sync();
    }
    xbuf[half * kBM + row] = m_run;
    xbuf[2 * kBM + half * kBM + row] = l_run;
    asm volatile("bar.sync 1, 256;" ::: "memory");  // the eight softmax warps
    const float m_o = xbuf[(1 - half) * kBM + row];
    const float l_o = xbuf[2 * kBM + (1 - half) * kBM + row];
    const float m_all = fmaxf(m_run, m_o);
    const float a_me = m_all == -INFINITY ? 0.f : exp2f(m_run - m_all);
    const float a_o = m_all == -INFINITY ? 0.f : exp2f(m_o - m_all);
    const float l_row = l_run * a_me + l_o * a_o;
    const float inv = (active && have && l_row > 0.f) ? 1.f / l_row : 0.f;
    // output columns [half * d/2, half * d/2 + d/2): this half's O and the other's
    const uint32_t tOa = tmem + lane_base + K::TM_O + half * (D / 2);        // O_0 columns
    const uint32_t tOb = tmem + lane_base + K::TM_O + D + half * (D / 2);    // O_1 columns
    const float c0 = half == 0 ? a_me : a_o, c1 = half == 0 ? a_o : a_me;
    __nv_bfloat16 *orow =
        p.o + (((size_t)b * p.Hq + h) * p.Tq + min(qr, p.Tq - 1)) * D + half * (D / 2);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      float ov[32], ow[32];
      if (have) {
        tc::tmem_ld32(tOa + c * 32, ov);
        tc::tmem_ld32(tOb + c * 32, ow);
        tc::tmem_wait_ld();
      }
#pragma unroll
      for (int i = 0; i < 32; ++i)  // inactive rows are exact zeros (their O may be NaN)
        ov[i] = (have && active) ? (ov[i] * c0 + ow[i] * c1) * inv : 0.f;
      if (qr < p.Tq) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint32_t w4[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) w4[i] = pack_bf16(ov[e * 8 + 2 * i], ov[e * 8 + 2 * i + 1]);
          *reinterpret_cast<uint4 *>(orow + c * 32 + e * 8) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    if (warp == 0) {
      // ================================================= TMA producer
      if (lane == 0 && nt > 0) {
        tc::prefetch_tmap(&tmQ);
        tc::prefetch_tmap(&tmK);
        tc::prefetch_tmap(&tmV);
        mbar_arrive_expect_tx(&bars.q_full, K::TILE);
#pragma unroll
        for (int c = 0; c < K::KB; ++c)
          tc::tma_load_3d(smem + K::OFF_Q + c * K::BLK, &tmQ, c * 64, m0, b * p.Hq + h,
                          &bars.q_full);
        int kfills[2] = {0, 0}, vfills[2] = {0, 0};
        for (int j = 0; j < nt; ++j) {
          const int s = j & 1;
          const int row = (j0 + j) * kBN;
          if (j >= 2 && !mbar_wait(&bars.k_empty[s], ((j >> 1) - 1) & 1, &failed)) break;
          mbar_arrive_expect_tx(&bars.k_full[s], K::TILE);
#pragma unroll
          for (int c = 0; c < K::KB; ++c)
            tc::tma_load_3d(smem + K::OFF_K + s * K::TILE + c * K::BLK, &tmK, c * 64, row,
                            b * p.Hkv + g, &bars.k_full[s]);
          kfills[s]++;
          if (j >= 2 && !mbar_wait(&bars.v_empty[s], ((j >> 1) - 1) & 1, &failed)) break;
          mbar_arrive_expect_tx(&bars.v_full[s], K::TILE);
#pragma unroll
          for (int c = 0; c < K::KB; ++c)
            tc::tma_load_3d(smem + K::OFF_V + s * K::TILE + c * K::BLK, &tmV, c * 64, row,
                            b * p.Hkv + g, &bars.v_full[s]);
          vfills[s]++;
        }
        // Never leave a TMA load in flight into an exiting CTA.
        bool f2 = false;
        mbar_wait(&bars.q_full, 0, &f2);
        for (int s = 0; s < 2; ++s) {
          if (kfills[s] > 0) mbar_wait(&bars.k_full[s], (kfills[s] - 1) & 1, &f2);
          if (vfills[s] > 0) mbar_wait(&bars.v_full[s], (vfills[s] - 1) & 1, &f2);
        }
        failed |= f2;
      }
    } else if (warp == 1) {
      // ================================================= MMA issuer
      if (lane == 0 && nt > 0) {
        constexpr uint32_t idS = tc::idesc_bf16_f32(kBM, kBN, 0, 0);
        constexpr uint32_t idO = tc::idesc_bf16_f32(kBM, D, 0, 1);
        const uint32_t sQ = smem_u32(smem + K::OFF_Q);
        // O_h += P_h(i) V_i[64h, 64h+64) for key half h: P_h over the first
        // 32 columns of that half of S[i%2], once that half has written it;
        // V from its ring stage.  Commits o_done[i%2] (its (i/2)-th phase)
        // and frees V.
        auto issue_pv = [&](int i) -> bool {
          const int s = i & 1;
          if (!mbar_wait(&bars.v_full[s], (i >> 1) & 1, &failed)) return false;
          const uint32_t sV = smem_u32(smem + K::OFF_V + s * K::TILE);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if (!mbar_wait(&bars.p_full[s][hh], (i >> 1) & 1, &failed)) return false;
            tc::fence_after_sync();
#pragma unroll
            for (int k = 4 * hh; k < 4 * hh + 4; ++k) {  // A = P from TMEM, 8 columns per 16 keys
              const uint64_t db = tc::sw128_desc(sV + k * 16 * 128, K::BLK, 1024);
              tc::mma_bf16_ts(tmem + K::TM_O + hh * D, tmem + s * kBN + hh * 64 + (k - 4 * hh) * 8,
                              db, idO, (i > 0 || k > 4 * hh) ? 1u : 0u);
            }
          }
          tc::mma_commit(&bars.o_done[s]);
          tc::mma_commit(&bars.v_empty[s]);
          return true;
        };
        bool ok = mbar_wait(&bars.q_full, 0, &failed);
        for (int j = 0; ok && j < nt; ++j) {
          const int sb = j & 1;
          // S(j) overwrites P(j-2) in S[sb]: P V(j-2) was issued before it.
          if (!mbar_wait(&bars.k_full[sb], (j >> 1) & 1, &failed)) break;
          tc::fence_after_sync();
          const uint32_t sK = smem_u32(smem + K::OFF_K + sb * K::TILE);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * K::BLK + (k & 3) * 32;
            tc::mma_bf16_ss(tmem + sb * kBN, tc::sw128_desc(sQ + off, 16, 1024),
                            tc::sw128_desc(sK + off, 16, 1024), idS, k > 0 ? 1u : 0u);
          }
          tc::mma_commit(&bars.s_full[sb]);
          tc::mma_commit(&bars.k_empty[sb]);
          if (j >= 1 && !issue_pv(j - 1)) {
            ok = false;
            break;
          }
        }
        if (ok) issue_pv(nt - 1);
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
inline bool supported(int d) { return d == 64 || d == 128; }

template <int D>
gqa_status launch_d(const void *q, const void *k, const void *v, void *o,
                    const int32_t *lens, const int32_t *seg, int B, int Hq, int Hkv,
                    int Tq, int Tk, int cached, int window, float scale_log2,
                    int32_t *status, cudaStream_t st) {
  using K = Cfg<D>;
  CUtensorMap mq, mk, mv;
  if (!tma::make_bf16_map(&mq, q, D, Tq, B * Hq, 128) ||
      !tma::make_bf16_map(&mk, k, D, Tk, B * Hkv, 128) ||
      !tma::make_bf16_map(&mv, v, D, Tk, B * Hkv, 128))
    return GQA_ERR_CUDA;
  static bool attr_done = false;  // per instantiation; benign race
  if (!attr_done) {
    if (cudaFuncSetAttribute(prefill_split_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  p.scale_log2 = scale_log2;
  p.head_major = p.num_mt >= kHeadMajorTiles;
  const long long grid = (long long)B * Hq * p.num_mt;
  if (grid > 0x7fffffffLL) return GQA_ERR_UNSUPPORTED;
  if (launch_dependent(prefill_split_kernel<D>, dim3((unsigned)grid), dim3(kThreads), K::SMEM,
                       st, mq, mk, mv, p) != cudaSuccess) {
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
                         int32_t *status, cudaStream_t st) {
  if (d == 64)
    return launch_d<64>(q, k, v, o, lens, seg, B, Hq, Hkv, Tq, Tk, cached, window, scale_log2,
                        status, st);
  return launch_d<128>(q, k, v, o, lens, seg, B, Hq, Hkv, Tq, Tk, cached, window, scale_log2,
                       status, st);
}

}  // namespace pfs
}  // namespace gqa
