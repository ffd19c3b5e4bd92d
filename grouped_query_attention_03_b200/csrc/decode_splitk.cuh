// decode_splitk.cuh -- bf16 split-K flash-decode for sm_100a.
//
// One new query token per sequence against a [B,Hkv,C,d] cache
// ("Share key/value heads and make context explicit", section "Extend the
// existing full and cached attention paths": each query head reads its
// shared lane over the eligible suffix [max(0, n_b - w), n_b), scale
// 1/sqrt(d); "GQA, FlashAttention and the KV cache", section "FlashAttention":
// blocks with a running max and sum instead of a materialised score row).
//
// Decomposition ("stream-K" over cache rows): the eligible rows of all
// lanes (b, g) are laid end to end, total = Hkv * sum_b len_b, and CTA c takes
// the contiguous range [c*per, (c+1)*per).  Every CTA gets the same number of
// rows whatever the length mix, every cached byte is read once, and a CTA
// writes one partial (m, l, acc) per lane its range touches, into slot
// lane + c (an injective map: along the staircase of (c, lane) pairs each
// step raises c, lane or both).
//
// Inside a CTA: warp 4 is the producer.  It walks the CTA's row range and
// streams stages of up to ROWS rows of K and V (plus the group's r query rows
// at the start of each lane segment) into a STAGES-deep shared-memory ring
// with non-multicast bulk copies completing on mbarriers.  Warps 0-3 consume
// each stage: warp w takes rows [w*RW, (w+1)*RW); within a warp LPR lanes
// share one row, each lane holding E features (16-byte shared loads), and
// the r query heads of the group are stacked so one K/V read serves all of
// them.  Dot products use packed fp32x2 FMAs, are reduced across the row's
// lanes by a transposed (reduce-scatter) shuffle tree, and the online
// softmax max/sum run on warp shuffles.  At the end of a lane segment the
// four warps' states are combined through shared memory into one partial.
// A second kernel merges the partials of each lane and writes bf16 output.
#pragma once

#include "common.cuh"

namespace gqa {
namespace dec {

constexpr int kFirst = 1, kLast = 2, kEnd = 4;
constexpr int kComputeWarps = 4;
constexpr int kThreads = (kComputeWarps + 1) * 32;

template <int D, int R>
struct Cfg {
  static constexpr int E = (D == 128 && R <= 4) ? 16 : 8;  // features / lane
  static constexpr int LPR = D / E;                        // lanes per row
  static constexpr int RPP = 32 / LPR;                     // rows per pass
  static constexpr int NC = E / 8;                         // 16-B chunks / lane
  static constexpr int ROWS = (D == 128) ? 64 : 128;       // rows per stage
  static constexpr int RW = ROWS / kComputeWarps;          // rows per warp
  static constexpr int NP = RW / RPP;                      // passes per stage
  static constexpr int STAGES = 3;
  static constexpr int KV_BYTES = ROWS * D * 2;
  static constexpr int Q_BYTES = R * D * 2;
  static constexpr int STAGE_BYTES = 2 * KV_BYTES + Q_BYTES;
  static_assert(LPR >= R, "reduce-scatter needs at least R lanes per row");
  static_assert(RW % RPP == 0, "whole passes per warp");
  static_assert(kComputeWarps * R * (D + 2) * 4 <= 2 * KV_BYTES,
                "combine scratch must fit in one stage");
};

struct StageHdr {
  int lane;   // virtual lane b*VL + vl
  int cell0;  // first cache cell of the stage
  int nrows;
  int flags;
  int slot;   // partial slot (lane + CTA index)
  int pad[3];
};

struct WsHdr {
  long long total;
  long long per;
  int valid;
  int pad[11];
};

struct Params {
  const __nv_bfloat16 *q, *kc, *vc;
  __nv_bfloat16 *o;
  const int32_t *seq_lens;
  int B, Hq, Hkv, C, window;
  float scale_log2;
  int r;      // query heads per KV head
  int nsub;   // sub-groups of at most R heads per KV head
  int VL;     // virtual lanes per batch row = Hkv * nsub
  int min_rows;
  WsHdr *hdr;
  long long *lane_start;  // [B*VL]
  float2 *ml;             // [(grid + B*VL) * R]: (m, l)
  float *acc;             // [(grid + B*VL) * R * D]
  int32_t *status;
};

__device__ __forceinline__ int eligible(int n, int window) {
  return window > 0 ? min(n, window) : n;
}

// -------------------------------------------------------------- producer
template <int D, int R>
__device__ void producer(const Params &p, unsigned char *smem, StageHdr *hdrs,
                         uint64_t *full, uint64_t *empty) {
  using K = Cfg<D, R>;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  bool failed = false;
  int fills[K::STAGES];
#pragma unroll
  for (int s = 0; s < K::STAGES; ++s) fills[s] = 0;
  int stage_count = 0;

  // Claim the next ring slot (waits until the consumers released it).
  auto acquire = [&](int &st) -> bool {
    st = stage_count % K::STAGES;
    if (stage_count >= K::STAGES) {
      const uint32_t par = ((stage_count / K::STAGES) - 1) & 1;
      if (!mbar_wait(&empty[st], par, &failed)) return false;
    }
    return true;
  };

  // Pass 1: validity and the total eligible row count.
  bool bad = false;
  long long tot = 0;
  for (int b = lane; b < p.B; b += 32) {
    const int n = p.seq_lens[b];
    bad |= (n < 0 || n > p.C);
    tot += eligible(n, p.window);
  }
  bad = __any_sync(0xffffffffu, bad);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1)
    tot += __shfl_xor_sync(0xffffffffu, tot, off);
  const long long total = tot * p.VL;
  long long per = (total + G - 1) / G;
  if (per < p.min_rows) per = p.min_rows;
  if (c == 0 && lane == 0) {
    p.hdr->valid = bad ? 0 : 1;
    p.hdr->total = total;
    p.hdr->per = per;
    if (bad) record_status(p.status, GQA_ERR_CAPACITY);
  }
  const long long start = (long long)c * per;
  const long long end = min(total, start + per);

  if (!bad && start < end) {
    // Pass 2: find the batch row holding row `start` (warp prefix scan).
    long long cum = 0, cum_b = 0;
    int b = -1;
    for (int b0 = 0; b0 < p.B && b < 0; b0 += 32) {
      const int bb = b0 + lane;
      const long long x =
          bb < p.B ? (long long)eligible(p.seq_lens[bb], p.window) * p.VL : 0;
      long long incl = x;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, cum + incl > start);
      if (hit) {
        const int src = __ffs(hit) - 1;
        b = b0 + src;
        cum_b = cum + __shfl_sync(0xffffffffu, incl - x, src);
      } else {
        cum += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    int n_b = p.seq_lens[b];
    int len = eligible(n_b, p.window);
    int lo = n_b - len;
    long long off0 = start - cum_b;
    int vl = (int)(off0 / len);
    int row = (int)(off0 - (long long)vl * len);
    long long pos = start;
    bool seg_first = true;

    while (pos < end) {
      const int L = b * p.VL + vl;
      const long long SL = cum_b + (long long)vl * len;
      if (row == 0 && seg_first && lane == 0) p.lane_start[L] = SL;
      const int nrows = (int)min((long long)min(K::ROWS, len - row), end - pos);
      const bool last = (row + nrows == len) || (pos + nrows == end);
      int st;
      if (!acquire(st)) break;
      if (lane == 0) {
        StageHdr &h = hdrs[st];
        h.lane = L;
        h.cell0 = lo + row;
        h.nrows = nrows;
        h.flags = (seg_first ? kFirst : 0) | (last ? kLast : 0);
        h.slot = L + c;
        const int g = vl / p.nsub, sub = vl % p.nsub;
        const int h0 = g * p.r + sub * R;
        const int rc = min(R, p.r - sub * R);
        const uint32_t kvb = (uint32_t)nrows * D * 2;
        const uint32_t qb = seg_first ? (uint32_t)rc * D * 2 : 0u;
        unsigned char *base = smem + (size_t)st * K::STAGE_BYTES;
        mbar_arrive_expect_tx(&full[st], 2 * kvb + qb);
        const size_t src = (((size_t)b * p.Hkv + g) * p.C + lo + row) * D;
        bulk_g2s(base, p.kc + src, kvb, &full[st]);
        bulk_g2s(base + K::KV_BYTES, p.vc + src, kvb, &full[st]);
        if (seg_first)
          bulk_g2s(base + 2 * K::KV_BYTES, p.q + ((size_t)b * p.Hq + h0) * D,
                   qb, &full[st]);
      }
      __syncwarp();
      fills[st]++;
      stage_count++;
      pos += nrows;
      row += nrows;
      seg_first = last;
      if (row == len) {
        row = 0;
        if (++vl == p.VL) {
          vl = 0;
          cum_b += (long long)len * p.VL;
          // Next batch row with a non-empty range (warp-parallel search).
          int nb = -1;
          for (int b0 = b + 1; b0 < p.B && nb < 0 && pos < end; b0 += 32) {
            const int bb = b0 + lane;
            const bool ne = bb < p.B && eligible(p.seq_lens[bb], p.window) > 0;
            const unsigned m = __ballot_sync(0xffffffffu, ne);
            if (m) nb = b0 + __ffs(m) - 1;
          }
          if (nb < 0) break;
          b = nb;
          n_b = p.seq_lens[b];
          len = eligible(n_b, p.window);
          lo = n_b - len;
        }
      }
    }
  }
  // End marker.
  int st;
  if (acquire(st)) {
    if (lane == 0) {
      hdrs[st].flags = kEnd;
      mbar_arrive(&full[st]);
    }
    __syncwarp();
    fills[st]++;
  }
  // Never leave a bulk copy in flight into shared memory of an exiting CTA.
  bool f2 = false;
#pragma unroll
  for (int s = 0; s < K::STAGES; ++s)
    if (fills[s] > 0) mbar_wait(&full[s], (fills[s] - 1) & 1, &f2);
  if ((failed || f2) && lane == 0) record_status(p.status, kStatusTimeout);
}

// ------------------------------------------------------------- consumers
template <int D, int R>
__device__ void consumer(const Params &p, unsigned char *smem,
                         const StageHdr *hdrs, uint64_t *full, uint64_t *empty,
                         uint64_t *comb) {
  using K = Cfg<D, R>;
  constexpr int E = K::E, LPR = K::LPR, NC = K::NC, NP = K::NP;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int sub = lane % LPR;          // feature slot within the row
  const int rip = lane / LPR;          // row within a pass
  const int h_lane = sub / (LPR / R);  // head whose score this lane ends with
  bool failed = false;

  float2 q2[R][E / 2];
  float2 acc[R][E / 2];
  float m_run = -INFINITY, l_run = 0.f;
  int stage_count = 0, comb_count = 0;

  while (true) {
    const int st = stage_count % K::STAGES;
    const uint32_t par = (stage_count / K::STAGES) & 1;
    if (!mbar_wait(&full[st], par, &failed)) break;
    const StageHdr hd = hdrs[st];
    if (hd.flags & kEnd) break;
    unsigned char *base = smem + (size_t)st * K::STAGE_BYTES;
    const __nv_bfloat16 *sK = reinterpret_cast<const __nv_bfloat16 *>(base);
    const __nv_bfloat16 *sV =
        reinterpret_cast<const __nv_bfloat16 *>(base + K::KV_BYTES);

    if (hd.flags & kFirst) {
      const __nv_bfloat16 *sQ =
          reinterpret_cast<const __nv_bfloat16 *>(base + 2 * K::KV_BYTES);
      const int vl = hd.lane % p.VL;
      const int rc = min(R, p.r - (vl % p.nsub) * R);
#pragma unroll
      for (int h = 0; h < R; ++h) {
#pragma unroll
        for (int i = 0; i < NC; ++i) {
          uint4 u = make_uint4(0, 0, 0, 0);
          if (h < rc)
            u = *reinterpret_cast<const uint4 *>(sQ + h * D + 8 * (sub + LPR * i));
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            q2[h][i * 4 + j] = make_float2(bf16lo_to_f32(w4[j]) * p.scale_log2,
                                           bf16hi_to_f32(w4[j]) * p.scale_log2);
        }
#pragma unroll
        for (int e = 0; e < E / 2; ++e) acc[h][e] = make_float2(0.f, 0.f);
      }
      m_run = -INFINITY;
      l_run = 0.f;
    }

    // ---- scores for this warp's rows of the stage
    float s[NP];
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
      const int rr = w * K::RW + pp * K::RPP + rip;
      const bool valid = rr < hd.nrows;
      float2 dot[R];
#pragma unroll
      for (int h = 0; h < R; ++h) dot[h] = make_float2(0.f, 0.f);
      if (valid) {
#pragma unroll
        for (int i = 0; i < NC; ++i) {
          const uint4 u = *reinterpret_cast<const uint4 *>(
              sK + rr * D + 8 * (sub + LPR * i));
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 kf = make_float2(bf16lo_to_f32(w4[j]), bf16hi_to_f32(w4[j]));
#pragma unroll
            for (int h = 0; h < R; ++h) ffma2(dot[h], q2[h][i * 4 + j], kf);
          }
        }
      }
      // Transposed reduction over the LPR lanes of the row: each halving
      // step trades half the heads with the partner lane, so the lane ends
      // with the full dot product of head h_lane.
      float v[R];
#pragma unroll
      for (int h = 0; h < R; ++h) v[h] = dot[h].x + dot[h].y;
#pragma unroll
      for (int nv = R, off = LPR / 2; off >= 1; off >>= 1) {
        if (nv > 1) {
          const int half = nv / 2;
          const bool upper = (lane & off) != 0;
#pragma unroll
          for (int i = 0; i < half; ++i) {
            const float send = upper ? v[i] : v[i + half];
            const float keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
          }
          nv = half;
        } else {
          v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
        }
      }
      s[pp] = valid ? v[0] : -INFINITY;
    }

    // ---- online softmax (log2 domain; q carries scale*log2(e))
    float mx = s[0];
#pragma unroll
    for (int pp = 1; pp < NP; ++pp) mx = fmaxf(mx, s[pp]);
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1)
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float m_new = fmaxf(m_run, mx);
    const float msub = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = exp2f(m_run - msub);  // 0 when m_run = -inf
    float lsum = 0.f;
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
      s[pp] = exp2f(s[pp] - msub);
      lsum += s[pp];
    }
    l_run = l_run * alpha + lsum;
    m_run = m_new;
#pragma unroll
    for (int h = 0; h < R; ++h) {
      const float a = __shfl_sync(0xffffffffu, alpha, h * (LPR / R));
#pragma unroll
      for (int e = 0; e < E / 2; ++e) {
        acc[h][e].x *= a;
        acc[h][e].y *= a;
      }
    }

    // ---- value mix
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
      const int rr = w * K::RW + pp * K::RPP + rip;
      float ph[R];
#pragma unroll
      for (int h = 0; h < R; ++h)
        ph[h] = __shfl_sync(0xffffffffu, s[pp], rip * LPR + h * (LPR / R));
      if (rr < hd.nrows) {
#pragma unroll
        for (int i = 0; i < NC; ++i) {
          const uint4 u = *reinterpret_cast<const uint4 *>(
              sV + rr * D + 8 * (sub + LPR * i));
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 vf = make_float2(bf16lo_to_f32(w4[j]), bf16hi_to_f32(w4[j]));
#pragma unroll
            for (int h = 0; h < R; ++h)
              ffma2(acc[h][i * 4 + j], make_float2(ph[h], ph[h]), vf);
          }
        }
      }
    }

    // ---- end of a lane segment: combine the four warps into one partial
    if (hd.flags & kLast) {
      float l_tot = l_run;
#pragma unroll
      for (int off = LPR; off < 32; off <<= 1)
        l_tot += __shfl_xor_sync(0xffffffffu, l_tot, off);
#pragma unroll
      for (int h = 0; h < R; ++h)
#pragma unroll
        for (int e = 0; e < E / 2; ++e)
#pragma unroll
          for (int off = LPR; off < 32; off <<= 1) {
            acc[h][e].x += __shfl_xor_sync(0xffffffffu, acc[h][e].x, off);
            acc[h][e].y += __shfl_xor_sync(0xffffffffu, acc[h][e].y, off);
          }
      // Everyone is done reading this stage's K/V: reuse it as scratch.
      __syncwarp();
      if (lane == 0) mbar_arrive(comb);
      mbar_wait(comb, comb_count & 1, &failed);
      comb_count++;
      float *sm_m = reinterpret_cast<float *>(base);
      float *sm_l = sm_m + kComputeWarps * R;
      float *sm_acc = sm_l + kComputeWarps * R;
      if (rip == 0) {
#pragma unroll
        for (int h = 0; h < R; ++h)
#pragma unroll
          for (int i = 0; i < NC; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              *reinterpret_cast<float2 *>(
                  sm_acc + (w * R + h) * D + 8 * (sub + LPR * i) + 2 * j) =
                  acc[h][i * 4 + j];
        if (sub % (LPR / R) == 0) {
          sm_m[w * R + h_lane] = m_run;
          sm_l[w * R + h_lane] = l_tot;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(comb);
      mbar_wait(comb, comb_count & 1, &failed);
      comb_count++;
      const int tid = threadIdx.x;  // 0..127
      for (int idx = tid; idx < R * D; idx += kComputeWarps * 32) {
        const int h = idx / D, f = idx - (idx / D) * D;
        float mm = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < kComputeWarps; ++ww) mm = fmaxf(mm, sm_m[ww * R + h]);
        float a = 0.f, l = 0.f;
#pragma unroll
        for (int ww = 0; ww < kComputeWarps; ++ww) {
          const float mw = sm_m[ww * R + h];
          const float e = mw == -INFINITY ? 0.f : exp2f(mw - mm);
          a += e * sm_acc[(ww * R + h) * D + f];
          l += e * sm_l[ww * R + h];
        }
        p.acc[((size_t)hd.slot * R + h) * D + f] = a;
        if (f == 0) p.ml[(size_t)hd.slot * R + h] = make_float2(mm, l);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    stage_count++;
  }
  if (failed && lane == 0) record_status(p.status, kStatusTimeout);
}

template <int D, int R>
__global__ void __launch_bounds__(kThreads, 2) split_kernel(const Params p) {
  using K = Cfg<D, R>;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ StageHdr hdrs[K::STAGES];
  __shared__ __align__(8) uint64_t full[K::STAGES], empty[K::STAGES], comb;
  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < K::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kComputeWarps);
    }
    mbar_init(&comb, kComputeWarps);
    fence_mbar_init();
  }
  __syncthreads();
  if ((threadIdx.x >> 5) == kComputeWarps)
    producer<D, R>(p, smem, hdrs, full, empty);
  else
    consumer<D, R>(p, smem, hdrs, full, empty, &comb);
}

// Merge the partials of one virtual lane: grid (VL, B), 128 threads.
template <int D, int R>
__global__ void __launch_bounds__(128) merge_kernel(const Params p) {
  const int vl = blockIdx.x, b = blockIdx.y;
  const int L = b * p.VL + vl;
  const int g = vl / p.nsub, sub = vl % p.nsub;
  const int h0 = g * p.r + sub * R;
  const int rc = min(R, p.r - sub * R);
  __nv_bfloat16 *o = p.o + ((size_t)b * p.Hq + h0) * D;
  const int n = p.seq_lens[b];
  const bool ok = p.hdr->valid != 0 && n > 0;
  if (!ok) {
    for (int idx = threadIdx.x; idx < rc * D; idx += blockDim.x)
      o[idx] = __float2bfloat16_rn(0.f);
    return;
  }
  const long long len = eligible(n, p.window);
  const long long SL = p.lane_start[L];
  const long long per = p.hdr->per;
  const int c0 = (int)(SL / per), c1 = (int)((SL + len - 1) / per);
  for (int idx = threadIdx.x; idx < rc * D; idx += blockDim.x) {
    const int h = idx / D, f = idx - (idx / D) * D;
    float mm = -INFINITY;
    for (int c = c0; c <= c1; ++c) mm = fmaxf(mm, p.ml[(size_t)(L + c) * R + h].x);
    float num = 0.f, den = 0.f;
    for (int c = c0; c <= c1; ++c) {
      const float2 ml = p.ml[(size_t)(L + c) * R + h];
      const float e = ml.x == -INFINITY ? 0.f : exp2f(ml.x - mm);
      num += e * p.acc[((size_t)(L + c) * R + h) * D + f];
      den += e * ml.y;
    }
    o[idx] = __float2bfloat16_rn(num / den);
  }
}

}  // namespace dec
}  // namespace gqa
