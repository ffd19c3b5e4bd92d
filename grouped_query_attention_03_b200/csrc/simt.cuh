// simt.cuh -- CUDA-core GQA kernels: one warp per query row, fp32 FMAs.
//
// Used for fp32 tensors (whose 1e-5 error bound rules out tf32 tensor-core
// arithmetic) and for bf16 head widths the tensor-core kernels do not
// compile for.  The row loop is the flash form of the pages' definition
// ("Share key/value heads and make context explicit", section "Give each
// query head an explicit shared KV head"): scores over the permitted keys
// [lo, hi] of the shared lane, running max/sum softmax, value mix.
#pragma once

#include "common.cuh"

namespace gqa {

// NF = ceil(d/32) features held per lane (d <= 32*NF).
template <typename T, int NF>
__device__ void attend_row_warp(const T *__restrict__ qrow,
                                const T *__restrict__ klane,
                                const T *__restrict__ vlane, int lo, int hi,
                                int d, float scale_log2, T *__restrict__ orow,
                                const T *kcand = nullptr, const T *vcand = nullptr,
                                int jcand = -1) {
  const int lane = threadIdx.x & 31;
  float q[NF], acc[NF];
#pragma unroll
  for (int i = 0; i < NF; ++i) {
    const int f = lane + 32 * i;
    q[i] = f < d ? to_f32(qrow[f]) * scale_log2 : 0.f;
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int j0 = lo; j0 <= hi; j0 += 32) {
    // Scores for up to 32 keys: lane jj ends up holding key j0 + jj.
    float s = -INFINITY;
    const int nk = min(32, hi - j0 + 1);
    for (int jj = 0; jj < nk; ++jj) {
      // Key `jcand` may be a candidate row held outside the lane (fused
      // append).
      const T *kr = (kcand && j0 + jj == jcand) ? kcand : klane + (size_t)(j0 + jj) * d;
      float part = 0.f;
#pragma unroll
      for (int i = 0; i < NF; ++i) {
        const int f = lane + 32 * i;
        if (f < d) part = fmaf(q[i], to_f32(kr[f]), part);
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1)
        part += __shfl_xor_sync(0xffffffffu, part, off);
      if (lane == jj) s = part;
    }
    float mx = s;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float m_new = fmaxf(m, mx);
    const float alpha = exp2f(m - m_new);  // m = -inf on the first block -> 0
    const float p = exp2f(s - m_new);      // masked lanes: s = -inf -> 0
    float psum = p;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
      psum += __shfl_xor_sync(0xffffffffu, psum, off);
    l = l * alpha + psum;
    m = m_new;
#pragma unroll
    for (int i = 0; i < NF; ++i) acc[i] *= alpha;
    for (int jj = 0; jj < nk; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const T *vr = (vcand && j0 + jj == jcand) ? vcand : vlane + (size_t)(j0 + jj) * d;
#pragma unroll
      for (int i = 0; i < NF; ++i) {
        const int f = lane + 32 * i;
        if (f < d) acc[i] = fmaf(pj, to_f32(vr[f]), acc[i]);
      }
    }
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int i = 0; i < NF; ++i) {
    const int f = lane + 32 * i;
    if (f < d) orow[f] = from_f32<T>(acc[i] * inv);
  }
}

template <typename T, int NF>
__device__ void zero_row_warp(T *orow, int d) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < NF; ++i) {
    const int f = lane + 32 * i;
    if (f < d) orow[f] = from_f32<T>(0.f);
  }
}

// Prefill: grid (ceil(Tq/4), Hq, B), 128 threads; warp w owns query row
// i = 4*blockIdx.x + w of head blockIdx.y in batch row blockIdx.z.  Q and O
// are [B,Hq,Tq,d], K and V [B,Hkv,Tk,d].  cached = 0: a prompt (Tq = Tk),
// row i at key position i, rows i >= n_b zero.  cached = 1: Tq new rows
// after a cache of n_b cells (the new ones included), row i at position
// n_b - Tq + i.  seg (prompt only, or NULL): [B,Tq] first key cell of
// row t's packed segment; a start outside [0, t] gives a zero row and
// GQA_ERR_SEGMENT.
template <typename T, int NF>
__global__ void __launch_bounds__(128)
    prefill_simt_kernel(const T *__restrict__ q, const T *__restrict__ k,
                        const T *__restrict__ v, T *__restrict__ o,
                        const int32_t *__restrict__ seq_lens, const int32_t *seg,
                        int Hq, int Hkv, int Tq, int Tk, int cached, int d,
                        int window, float scale_log2, int32_t *status) {
  const int i = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int h = blockIdx.y, b = blockIdx.z;
  if (i >= Tq) return;
  const int r = Hq / Hkv, g = h / r;
  T *orow = o + (((size_t)b * Hq + h) * Tq + i) * d;
  int n = Tk;
  if (seq_lens) {
    n = seq_lens[b];
    if (n < 0 || n > Tk || (cached && n < Tq)) {
      if ((threadIdx.x & 31) == 0 && i == 0 && h == 0)
        record_status(status, GQA_ERR_CAPACITY);
      zero_row_warp<T, NF>(orow, d);
      return;
    }
  }
  const int t = cached ? n - Tq + i : i;
  if (t >= n) {  // inactive padded query: zero output
    zero_row_warp<T, NF>(orow, d);
    return;
  }
  int s0 = 0;
  if (seg) {
    s0 = seg[(size_t)b * Tq + t];
    if (s0 < 0 || s0 > t) {
      if ((threadIdx.x & 31) == 0) record_status(status, GQA_ERR_SEGMENT);
      zero_row_warp<T, NF>(orow, d);
      return;
    }
  }
  const int lo = window > 0 ? max(s0, t - (window - 1)) : s0;
  const size_t lane_off = ((size_t)b * Hkv + g) * Tk * d;
  attend_row_warp<T, NF>(q + (((size_t)b * Hq + h) * Tq + i) * d,
                         k + lane_off, v + lane_off, lo, t, d, scale_log2,
                         orow);
}

// Decode: grid (Hq, B), 32 threads; the query sits at cell n_b - 1 and
// reads cells [max(0, n_b - w), n_b) of the shared cache lane.  An invalid
// length anywhere zeroes the whole output (every warp checks every length).
// With add = 1 (fused append) seq_lens holds the lengths before the step,
// n_b = seq_lens[b] + 1, and cell n_b - 1 is read from kn / vn
// ([B,Hkv,1,d]) instead of the cache, which is written afterwards.
template <typename T, int NF>
__global__ void __launch_bounds__(32)
    decode_simt_kernel(const T *__restrict__ q, const T *__restrict__ kc,
                       const T *__restrict__ vc, T *__restrict__ o,
                       const int32_t *__restrict__ seq_lens, int B, int Hq,
                       int Hkv, int C, int d, int window, float scale_log2,
                       int32_t *status, const T *kn = nullptr,
                       const T *vn = nullptr, int add = 0, int ring = 0) {
  const int h = blockIdx.x, b = blockIdx.y;
  T *orow = o + ((size_t)b * Hq + h) * d;
  bool bad = false;
  for (int i = threadIdx.x; i < B; i += 32) {
    const int n = seq_lens[i] + add;
    bad |= (n < add || (!ring && n > C));
  }
  if (__any_sync(0xffffffffu, bad)) {
    if (threadIdx.x == 0 && b == 0 && h == 0)
      record_status(status, GQA_ERR_CAPACITY);
    zero_row_warp<T, NF>(orow, d);
    return;
  }
  const int n = seq_lens[b] + add;
  if (n == 0) {
    zero_row_warp<T, NF>(orow, d);
    return;
  }
  const int r = Hq / Hkv, g = h / r;
  // Linear: cells [max(0, n-w), n), the newest last.  Ring (rolling buffer
  // of C slots): every occupied slot, the newest at slot (n-1) mod C.
  const int pos = ring ? min(n, C) - 1 : n - 1;
  const int lo = (!ring && window > 0) ? max(0, pos - (window - 1)) : 0;
  const size_t lane_off = ((size_t)b * Hkv + g) * C * d;
  const size_t cand = ((size_t)b * Hkv + g) * d;
  attend_row_warp<T, NF>(q + ((size_t)b * Hq + h) * d, kc + lane_off,
                         vc + lane_off, lo, pos, d, scale_log2, orow,
                         add ? kn + cand : nullptr, add ? vn + cand : nullptr,
                         ring ? (n - 1) % C : pos);
}

}  // namespace gqa
