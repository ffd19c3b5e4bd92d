// prefill_tc.cuh -- tcgen05/TMEM causal-windowed GQA prefill (bf16, sm_100a).
//
// What it computes ("Share key/value heads and make context explicit",
// sections "Give each query head an explicit shared KV head" and "Intersect
// the window with the context already permitted"): for every batch row b,
// query head h and active cell t < n_b, softmax over keys
// j in [max(0, t-(w-1)), t] of scale * q_{h,t} . k_{g(h),j}, mixed with the
// value rows of the same shared lane g(h) = floor(h / (Hq/Hkv)); inactive
// rows are zero.  The running-max/running-sum block form is the
// FlashAttention algorithm ("GQA, FlashAttention and the KV cache", section
// "FlashAttention").
//
// One CTA owns a 128-row query tile of one (b, h).  It walks the 128-key
// tiles that intersect the tile's permitted band [lo(m0), min(m0+127,
// n_b-1)], skipping every tile wholly outside the causal window.
//   warp 0      TMA producer: Q once, then K and V tiles into a 2-stage
//               ring (128-byte swizzle, no multicast).
//   warp 1      allocates TMEM; lane 0 issues tcgen05.mma:
//               S[j%2] = Q K_j^T (M=128, N=128, K=d) and O += P_j V_j
//               (M=128, N=d, K=128), committing to mbarriers.
//   warps 2-5   softmax: thread = query row (TMEM lane); tcgen05.ld of the S
//               row, causal/window mask on edge tiles only, online max with
//               lazy O rescaling (only when the max grows by more than 2^8),
//               P in bf16 to TMEM (the PV MMA takes its A operand from
//               there), then the O / l epilogue.
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+d), P [256+d, 320+d).
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tma_host.cuh"

namespace gqa {
namespace pf {

constexpr int kBM = 128, kBN = 128;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale when max grows > 2^8

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
  // TMEM columns: S double buffer [0, 256), O [256, 256 + D), and P (bf16,
  // two keys per 32-bit column) in the 64 columns after O.
  static constexpr uint32_t TM_P = 256 + D;
  static_assert(TM_P + kBN / 2 <= kTmemCols, "S, O and P must fit in 512 TMEM columns");
  // Ask for at least 120 KB so only one CTA (which holds all 512 TMEM
  // columns) is resident per SM.
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
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, o_done, mma_fin;
  uint32_t tmem_base;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const Params p) {
  using K = Cfg<D>;
  extern __shared__ unsigned char smem_raw[];
  __shared__ Bars bars;
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- which tile: longest causal rows first
  const int BH = p.B * p.Hq;
  const int mt = p.num_mt - 1 - (int)(blockIdx.x / BH);
  const int bh = (int)(blockIdx.x % BH);
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
      mbar_init(&bars.s_free[s], 4);
    }
    mbar_init(&bars.p_full, 4);
    mbar_init(&bars.o_done, 1);
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

  if (warp == 0) {
    // ================================================= TMA producer
    if (lane == 0 && nt > 0) {
      tc::prefetch_tmap(&tmQ);
      tc::prefetch_tmap(&tmK);
      tc::prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(&bars.q_full, K::TILE);
#pragma unroll
      for (int c = 0; c < K::KB; ++c)
        tc::tma_load_3d(smem + K::OFF_Q + c * K::BLK, &tmQ, c * 64, m0,
                        b * p.Hq + h, &bars.q_full);
      int kfills[2] = {0, 0}, vfills[2] = {0, 0};
      for (int j = 0; j < nt; ++j) {
        const int s = j & 1;
        const int row = (j0 + j) * kBN;
        if (j >= 2 && !mbar_wait(&bars.k_empty[s], ((j >> 1) - 1) & 1, &failed)) break;
        mbar_arrive_expect_tx(&bars.k_full[s], K::TILE);
#pragma unroll
        for (int c = 0; c < K::KB; ++c)
          tc::tma_load_3d(smem + K::OFF_K + s * K::TILE + c * K::BLK, &tmK,
                          c * 64, row, b * p.Hkv + g, &bars.k_full[s]);
        kfills[s]++;
        if (j >= 2 && !mbar_wait(&bars.v_empty[s], ((j >> 1) - 1) & 1, &failed)) break;
        mbar_arrive_expect_tx(&bars.v_full[s], K::TILE);
#pragma unroll
        for (int c = 0; c < K::KB; ++c)
          tc::tma_load_3d(smem + K::OFF_V + s * K::TILE + c * K::BLK, &tmV,
                          c * 64, row, b * p.Hkv + g, &bars.v_full[s]);
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
      auto issue_pv = [&](int i) -> bool {
        if (!mbar_wait(&bars.p_full, i & 1, &failed)) return false;
        if (!mbar_wait(&bars.v_full[i & 1], (i >> 1) & 1, &failed)) return false;
        tc::fence_after_sync();
        const uint32_t sV = smem_u32(smem + K::OFF_V + (i & 1) * K::TILE);
#pragma unroll
        for (int k = 0; k < kBN / 16; ++k) {  // A = P from TMEM, 8 columns per 16 keys
          const uint64_t db = tc::sw128_desc(sV + k * 16 * 128, K::BLK, 1024);
          tc::mma_bf16_ts(tmem + 256, tmem + K::TM_P + k * 8, db, idO, (i > 0 || k > 0) ? 1u : 0u);
        }
        tc::mma_commit(&bars.o_done);
        tc::mma_commit(&bars.v_empty[i & 1]);
        return true;
      };
      bool ok = mbar_wait(&bars.q_full, 0, &failed);
      for (int j = 0; ok && j < nt; ++j) {
        const int sb = j & 1;
        if (j >= 2 && !mbar_wait(&bars.s_free[sb], ((j >> 1) - 1) & 1, &failed)) break;
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
  } else {
    // ================================================= softmax warps
    const int q4 = warp & 3;                 // TMEM lane quarter of this warp
    const int row = q4 * 32 + lane;          // query row within the tile
    const int t = a0 + row;                  // key position of this query row
    const int qr = m0 + row;                 // its row in Q and O
    const bool active = t < off + rows;
    const int lo_t = active ? row_lo(p, b, t) : 0;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const float sc = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int sb = j & 1;
      const int kb = (j0 + j) * kBN;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars.s_full[sb], (j >> 1) & 1, &failed))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      float s[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c)
        tc::tmem_ld32(tmem + lane_base + sb * kBN + c * 32, s + c * 32);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.s_free[sb]);

      const bool edge = (kb + kBN - 1 > a0) || (kb < lo_max);
      if (edge) {
#pragma unroll
        for (int c = 0; c < kBN; ++c) {
          const int key = kb + c;
          if (key > t || key < lo_t) s[c] = -INFINITY;
        }
      }
      float mx = -INFINITY;
      if (sc > 0.f) {
#pragma unroll
        for (int c = 0; c < kBN; ++c) mx = fmaxf(mx, s[c]);
      } else {
        float mn = INFINITY;
#pragma unroll
        for (int c = 0; c < kBN; ++c) mn = s[c] == -INFINITY ? mn : fminf(mn, s[c]);
        mx = mn == INFINITY ? -INFINITY : mn;
      }
      const float m_tile = mx == -INFINITY ? -INFINITY : mx * sc;

      // O and the P buffer are free once the previous PV has completed.
      if (j >= 1) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.o_done, (j - 1) & 1, &failed))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
      }
      if (j == 0) {
        m_run = m_tile;
      } else if (__any_sync(0xffffffffu, m_tile > m_run + kRescaleThreshold)) {
        // Warp-wide (tcgen05.ld/st are whole-warp): rows whose max did not
        // grow keep their max and scale by 1.
        const float m_new = fmaxf(m_run, m_tile);
        const float alpha = m_new == m_run ? 1.f : exp2f(m_run - m_new);  // 0 from -inf
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float ov[32];
          tc::tmem_ld32(tmem + lane_base + 256 + c * 32, ov);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tc::tmem_st32(tmem + lane_base + 256 + c * 32, ov);
        }
        tc::tmem_wait_st();
        l_run *= alpha;
        m_run = m_new;
      }
      const float msub = m_run == -INFINITY ? 0.f : m_run;
      // bf16 P into this thread's TMEM lane (column c holds p[2c], p[2c+1]),
      // where the P V MMA reads it as its A operand.
      float lsum = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int i = half * 64 + 2 * e;
          const float p0 = ex2_approx(fmaf(s[i], sc, -msub));
          const float p1 = ex2_approx(fmaf(s[i + 1], sc, -msub));
          const __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
          lsum += __low2float(pr) + __high2float(pr);
          w[e] = __uint_as_float(*reinterpret_cast<const uint32_t *>(&pr));
        }
        tc::tmem_st32(tmem + lane_base + K::TM_P + half * 32, w);
      }
      tc::tmem_wait_st();
      l_run += lsum;
      if (kb + kBN > n_keys) {
        // Cells past the sequence in this V tile are not the sequence's (an
        // unwritten cache cell may hold NaN): their p is 0, but 0 * NaN is
        // not, so clear those rows (thread = row) before P V is issued.
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.v_full[sb], (j >> 1) & 1, &failed))) {
          ok = false;
          break;
        }
        if (kb + row >= n_keys) {
          unsigned char *vrow = smem + K::OFF_V + sb * K::TILE + row * 128;
#pragma unroll
          for (int c = 0; c < K::KB; ++c)
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
              *reinterpret_cast<uint4 *>(vrow + c * K::BLK + ch * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full);
    }

    // ---- epilogue: O / l, bf16, one row per thread (the whole warp reads
    // TMEM; only rows inside the tensor are stored)
    bool have = false;
    if (nt > 0 && ok) {
      have = __all_sync(0xffffffffu, mbar_wait(&bars.o_done, (nt - 1) & 1, &failed));
      tc::fence_after_sync();
    }
    const float inv = (active && have && l_run > 0.f) ? 1.f / l_run : 0.f;
    __nv_bfloat16 *orow = p.o + (((size_t)b * p.Hq + h) * p.Tq + min(qr, p.Tq - 1)) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float ov[32];
      if (have) {
        tc::tmem_ld32(tmem + lane_base + 256 + c * 32, ov);
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
          for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 pr =
                __floats2bfloat162_rn(ov[e * 8 + 2 * i] * inv, ov[e * 8 + 2 * i + 1] * inv);
            w4[i] = *reinterpret_cast<const uint32_t *>(&pr);
          }
          *reinterpret_cast<uint4 *>(orow + c * 32 + e * 8) =
              make_uint4(w4[0], w4[1], w4[2], w4[3]);
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
// [rows = T, heads] of d-wide bf16 rows, boxes of 64 columns x 128 rows.
inline bool make_map(CUtensorMap *map, const void *base, int d, int T, int heads) {
  return tma::make_bf16_map(map, base, d, T, heads, 128);
}

inline bool supported(int d) { return d == 64 || d == 128; }

template <int D>
gqa_status launch_d(const void *q, const void *k, const void *v, void *o,
                    const int32_t *lens, const int32_t *seg, int B, int Hq, int Hkv,
                    int Tq, int Tk, int cached, int window, float scale_log2,
                    int32_t *status, cudaStream_t st) {
  using K = Cfg<D>;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, D, Tq, B * Hq) || !make_map(&mk, k, D, Tk, B * Hkv) ||
      !make_map(&mv, v, D, Tk, B * Hkv))
    return GQA_ERR_CUDA;
  static bool attr_done = false;
  if (!attr_done) {
    if (cudaFuncSetAttribute(prefill_kernel<D>,
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
  p.scale_log2 = scale_log2;
  const long long grid = (long long)B * Hq * p.num_mt;
  if (grid > 0x7fffffffLL) return GQA_ERR_UNSUPPORTED;
  if (launch_dependent(prefill_kernel<D>, dim3((unsigned)grid), dim3(kThreads), K::SMEM, st, mq,
                       mk, mv, p) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

// Prompt (cached = 0: Tq = Tk = T) or queries after a cache (cached = 1:
// Tq new rows against Tk = capacity cells).
inline gqa_status launch(const void *q, const void *k, const void *v, void *o,
                         const int32_t *lens, const int32_t *seg, int B, int Hq, int Hkv,
                         int Tq, int Tk, int cached, int d, int window, float scale_log2,
                         int32_t *status, cudaStream_t st) {
  if (d == 64)
    return launch_d<64>(q, k, v, o, lens, seg, B, Hq, Hkv, Tq, Tk, cached, window,
                        scale_log2, status, st);
  return launch_d<128>(q, k, v, o, lens, seg, B, Hq, Hkv, Tq, Tk, cached, window,
                       scale_log2, status, st);
}

}  // namespace pf
}  // namespace gqa
