// append.cuh -- KV-cache append: copy new cells in, then commit the lengths.
//
// "Share key/value heads and make context explicit", sections "Count
// learned weights and retained cache data separately" (fixed-capacity
// [B,Hkv,C,d] storage that keeps every row) and "Extend the existing full
// and cached attention paths" (refuse to exceed capacity; a failed operation
// never partly advances the cache).
//
// Two launches on one stream, with no waiting between CTAs:
//   1. append_copy_kernel: every CTA first checks every length; if any is
//      invalid no CTA writes anything.  Otherwise rows [len_b, len_b+t_new)
//      of each lane are written with 16-byte vector copies (pure bandwidth:
//      2 x new bytes read + written).
//   2. append_commit_kernel (one CTA): repeats the same check on the still
//      unchanged lengths and, only if all are valid, advances them.
//
// ring != 0: a rolling buffer of C slots ("Relate shared heads to local
// context": a rolling buffer that overwrites old KV entries), position p in
// slot p mod C; of t_new new rows only the last C survive, and a length
// only has to stay non-negative and inside int32.
#pragma once

#include "common.cuh"

namespace gqa {

__device__ __forceinline__ bool lengths_fit(const int32_t *seq_lens, int B,
                                            int C, int t_new, int ring) {
  // Block-wide: true iff every 0 <= len_b and len_b + t_new <= C (ring:
  // len_b + t_new fits in int32).
  int bad = 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int n = seq_lens[b];
    bad |= (n < 0 || n > (ring ? 0x7fffffff - t_new : C - t_new));
  }
  return __syncthreads_or(bad) == 0;
}

// VEC = elements of T per vector (16 bytes / sizeof(T)), or 1 for the
// scalar path when rows are not 16-byte multiples.
template <typename V>
__global__ void __launch_bounds__(256)
    append_copy_kernel(V *__restrict__ kc, V *__restrict__ vc,
                       const V *__restrict__ kn, const V *__restrict__ vn,
                       const int32_t *__restrict__ seq_lens, int B, int Hkv,
                       int C, int t_new, int vec_per_row, int ring, int32_t *status) {
  if (!lengths_fit(seq_lens, B, C, t_new, ring)) {
    if (blockIdx.x == 0 && threadIdx.x == 0)
      record_status(status, GQA_ERR_CAPACITY);
    return;
  }
  const size_t total = (size_t)B * Hkv * t_new * vec_per_row;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += stride) {
    const size_t row = idx / vec_per_row;  // row of [B,Hkv,t_new]
    const int e = (int)(idx - row * vec_per_row);
    const int i = (int)(row % t_new);
    const size_t lane = row / t_new;  // b * Hkv + g
    const int b = (int)(lane / Hkv);
    if (ring && t_new - i > C) continue;  // overwritten by a later new row
    const int cell = ring ? (int)(((long long)seq_lens[b] + i) % C) : seq_lens[b] + i;
    const size_t dst = (lane * C + (size_t)cell) * vec_per_row + e;
    kc[dst] = kn[idx];
    vc[dst] = vn[idx];
  }
}

__global__ void __launch_bounds__(256)
    append_commit_kernel(int32_t *seq_lens, int B, int C, int t_new, int ring) {
  if (!lengths_fit(seq_lens, B, C, t_new, ring)) return;
  for (int b = threadIdx.x; b < B; b += blockDim.x) seq_lens[b] += t_new;
}

}  // namespace gqa
