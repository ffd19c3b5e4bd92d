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
// lanes (b, g) are laid end to end, each non-empty lane preceded by `pad`
// virtual rows that carry no work (so a lane segment's fixed cost -- query
// load, combine, partial -- is charged as rows), total = VL * sum_b (len_b +
// pad), and CTA c takes the contiguous range [c*per, (c+1)*per).  Every CTA
// gets the same share whatever the length mix, every cached byte is read
// once, and a CTA
// writes one partial (m, l, acc) per lane its range touches, into slot
// lane + c (an injective map: along the staircase of (c, lane) pairs each
// step raises c, lane or both).
//
// Inside a CTA the last warp is the producer.  It walks the CTA's row range
// and fills a STAGES-deep shared-memory ring: ROWS cache rows of K and of V
// per stage, fetched by TMA tensor copies (no multicast) in 128-byte
// swizzled 64-column boxes, plus the group's query rows (bulk copy) at the
// start of each lane segment.  Each of the NWC compute warps owns 16 rows of
// a stage.  The group's R <= 16 query heads are stacked as the rows of one
// 16-row tile, so the scores of 16 cache rows are one 16x16 tile
// S = Q K^T and the value mix one 16 x d tile O += P V, both on the tensor
// cores (mma.sync m16n8k16, bf16 in, fp32 accumulate; the K and V operands
// come straight from the swizzled stage with ldmatrix).  The online softmax
// works on the accumulator fragments: row max and sum over the four lanes
// that share a head row with warp shuffles, accumulators rescaled lazily
// (only when a running max grows by more than 2^8).  Per cache row that is
// about two tensor instructions and a handful of others, which keeps the SM
// ahead of HBM even when 8 or 16 query heads share each K/V row; the
// CUDA-core formulation cannot do that beyond one or two heads per row.
// At the end of a lane segment the warps' states are combined through the
// just-consumed stage buffer.  A lane covered by one CTA is written out
// directly; otherwise the combined (m, l, acc) goes to the workspace and is
// counted when the CTA's range ends (an atomic counter per split lane, kept
// at the start of the workspace and indexed by the lane's first CTA); the
// last CTA to count a lane resets the counter and merges the lane's partials
// (the exact maximum first, then the terms in ascending order, so the bits
// do not depend on which CTA comes last) and writes bf16 output.  Every
// counter is zero when a call starts and zero again when it ends, so the
// workspace needs no clearing between calls.  No CTA ever waits for another.
//
// Launched as a programmatic dependent of the previous kernel on the stream:
// a CTA sets up its barriers and asks L2 for the first cache rows of its
// range (planned from the lengths as they read then) while that kernel
// drains, then waits for it to complete (griddepcontrol.wait) before it
// reads anything it uses or writes anything.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace gqa {
namespace dec {

constexpr int kFirst = 1, kLast = 2, kEnd = 4;
// Largest grid; the workspace holds kMaxCtas split-lane counters (a split
// lane's first CTA indexes it) and then the count of CTAs that have read
// the lengths (fused append).
constexpr int kMaxCtas = 1024;
constexpr int kCtrFinish = kMaxCtas;
// Lengths of up to this many sequences are cached in shared memory (read
// from global memory once per CTA); a fused append needs that.
constexpr int kLensSmem = 4096;
constexpr float kLazyRescale = 8.0f;  // log2 units
constexpr int kBR = 16;               // rows per compute warp per stage

// Compute warps per CTA, CTAs per SM and ring depth (overridable when
// building, for tuning).
#ifndef GQA_DEC_NWC
#define GQA_DEC_NWC 7
#endif
#ifndef GQA_DEC_MIN_BLOCKS
#define GQA_DEC_MIN_BLOCKS 1
#endif
#ifndef GQA_DEC_STAGES
#define GQA_DEC_STAGES 3
#endif

template <int D, int R>
struct Cfg {
  static constexpr int NWC = GQA_DEC_NWC;              // compute warps
  static constexpr int MIN_BLOCKS = GQA_DEC_MIN_BLOCKS;  // CTAs per SM
  static constexpr int THREADS = (NWC + 1) * 32;
  static constexpr int ROWS = NWC * kBR;               // rows per stage
  static constexpr int KB = D / 64;                    // 64-column boxes
  static constexpr int BOX = ROWS * 128;               // bytes of one box
  static constexpr int KV_BYTES = KB * BOX;            // K (or V) per stage
  // Query rows of the group, then the appended key and value rows (fused
  // append), in one 1024-byte-aligned area after K and V.
  static constexpr int NEWOFF = R * D * 2;
  static constexpr int QRAW = ((R * D * 2 + 4 * D + 1023) / 1024) * 1024;
  static constexpr int STAGE_BYTES = 2 * KV_BYTES + QRAW;
  static constexpr int STAGES = GQA_DEC_STAGES;
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024;  // + alignment slack
  static constexpr int KS = D / 16;                    // k-steps of 16 features
  static constexpr int NT = D / 8;                     // 8-feature output tiles
  static_assert(R <= 16, "one 16-row tile holds the stacked heads");
  static_assert(NWC > 4, "two merges split the compute warps 4 / NWC-4");
  // Row stride (floats) of the combine scratch: padded by 8 when it fits,
  // so the warps' fragment stores hit distinct banks.
  static constexpr int ACC_STRIDE =
      NWC * (2 * 16 + R * (D + 8)) * 4 <= STAGE_BYTES ? D + 8 : D;
  static_assert(NWC * (2 * 16 + R * ACC_STRIDE) * 4 <= STAGE_BYTES,
                "combine scratch must fit in one stage");
  static_assert(STAGE_BYTES % 1024 == 0 && BOX % 1024 == 0, "swizzle alignment");
};

struct StageHdr {
  int lane;   // virtual lane b*VL + vl
  int cell0;  // first cache cell of the stage
  int nrows;
  int flags;
  int slot;   // partial slot (lane + CTA index)
  int c0;     // first CTA whose range touches the lane
  int np;     // number of CTAs whose ranges touch the lane
  int newrow; // stage row of the appended token (fused append), else -1
};

struct Params {
  const __nv_bfloat16 *q;
  __nv_bfloat16 *o;
  const int32_t *seq_lens;
  int B, Hq, Hkv, C, window;
  float scale_log2;
  int r;      // query heads per KV head
  int nsub;   // sub-groups of at most R heads per KV head
  int VL;     // virtual lanes per batch row = Hkv * nsub
  int min_rows;
  int *counters;          // [kMaxCtas + 1], zero at kernel start and left
                          // zero: [c0] counts the partials of the split lane
                          // whose first CTA is c0 (c0 is unique among split
                          // lanes), [kCtrFinish] the CTAs that have read the
                          // lengths (fused append)
  float2 *ml;             // [(grid + B*VL) * R]: (m, l)
  float *acc;             // [(grid + B*VL) * R * D]
  int32_t *status;
  // Fused append: seq_lens holds the lengths before this step (add = 1),
  // the step's key/value rows come from k_new / v_new ([B,Hkv,1,D]) and are
  // written to the cache at cell seq_lens[b]; the last CTA to finish then
  // advances every length by one.  add = 0: plain decode, seq_lens = n_b.
  const __nv_bfloat16 *k_new, *v_new;
  __nv_bfloat16 *k_cache, *v_cache;
  int32_t *lens_out;
  int add;
  int lens_smem;  // 1: B <= kLensSmem, lengths cached in shared memory
  int ring;       // 1: the cache is a rolling buffer of C slots, position p
                  // in slot p mod C; the query reads all min(n_b, C) slots
  int pad;        // virtual rows in front of every non-empty lane (below)
};

// Keys of sequence b for this call (n_b, the appended token included).
__device__ __forceinline__ int nlen(const Params &p, int b) {
  return p.seq_lens[b] + p.add;
}

// a / b for non-negative a and positive b, with the 32-bit divide when
// both fit (the 64-bit one is a long software sequence).
__device__ __forceinline__ long long udiv(long long a, long long b) {
  if (((unsigned long long)a | (unsigned long long)b) < (1ull << 32))
    return (long long)((unsigned)a / (unsigned)b);
  return a / b;
}

// Cells the query of a sequence with n positions reads: the window's last
// cells, or (ring) every occupied slot [0, min(n, C)).
__device__ __forceinline__ int eligible_cells(const Params &p, int n) {
  return p.ring ? min(n, p.C) : (p.window > 0 ? min(n, p.window) : n);
}
__device__ __forceinline__ int first_cell(const Params &p, int n, int len) {
  return p.ring ? 0 : n - len;
}
// A lane's share of the row space the CTAs split: its rows plus `pad`
// virtual rows in front of them that carry no work.  A lane segment costs a
// CTA a fixed amount of work (query load, combine, partial), so a range
// that starts a lane gets that many fewer real rows.
__device__ __forceinline__ int extent(const Params &p, int len) {
  return len > 0 ? len + p.pad : 0;
}


// Byte offset of 16-byte chunk `ch` (0..7) of row `r` inside a 128-byte
// swizzled box (the TMA swizzle XORs the chunk index with r mod 8).
__device__ __forceinline__ int swz(int r, int ch) {
  return r * 128 + ((ch ^ (r & 7)) << 4);
}

// ---------------------------------------------------- prefetch before wait
// Rows of its range a CTA asks L2 for before the previous kernel on the
// stream has completed (a cap, so that the prefetched rows of every CTA fit
// in L2 together with room to spare: 148 CTAs x 512 rows x 512 B at d = 128
// is 39 MB of the 126 MB).
constexpr int kPrefetchRows = 512;

// Runs on the producer warp before griddepcontrol.wait, while the previous
// kernel drains: plans this CTA's range as the producer will (same row
// space, same split) from the lengths as they read now, and asks L2 for
// the first kPrefetchRows cache rows of it (K and V, whole TMA boxes).  The
// lengths may be stale -- a fused append of the previous step may still be
// advancing them -- so this is only a hint: it writes nothing but the
// shared length cache (which the producer fills again after the wait), and
// the producer plans again from the lengths it reads then.  The lengths
// are read through L2 only (ld.global.cg), so no line of them sits in this
// SM's L1 when the producer reads them after the wait.  Invalid lengths,
// or more sequences than the shared cache holds, prefetch nothing.
template <int D, int R>
__device__ void prefetch_range(const Params &p, const CUtensorMap *tmK,
                               const CUtensorMap *tmV, int *s_len) {
  using K = Cfg<D, R>;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  if (!p.lens_smem) return;
  long long tot = 0;
  int bad_local = 0;
  for (int b = lane; b < p.B; b += 32) {
    const int n = __ldcg(p.seq_lens + b) + p.add;
    s_len[b] = n;
    bad_local |= (n < p.add || (!p.ring && n > p.C));
    tot += extent(p, eligible_cells(p, max(n, 0)));
  }
  if (__any_sync(0xffffffffu, bad_local)) return;
  __syncwarp();
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
  const long long total = tot * p.VL;
  long long per = udiv(total + G - 1, G);
  if (per < p.min_rows) per = p.min_rows;
  const long long start = (long long)c * per;
  const long long end = min(min(total, start + per), start + kPrefetchRows);
  if (start >= end) return;
  // the batch row holding row `start` (warp prefix scan, as the producer)
  long long cum = 0, cum_b = 0;
  int b = -1;
  for (int b0 = 0; b0 < p.B && b < 0; b0 += 32) {
    const int bb = b0 + lane;
    const long long x = bb < p.B ? (long long)extent(p, eligible_cells(p, s_len[bb])) * p.VL : 0;
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
  if (b < 0) return;
  int n_b = s_len[b];
  int len = eligible_cells(p, n_b);
  int ext = extent(p, len);
  int lo = first_cell(p, n_b, len);
  const long long off0 = start - cum_b;
  int vl = (int)udiv(off0, ext);
  int row = (int)(off0 - (long long)vl * ext) - p.pad;
  long long pos = start;
  while (pos < end) {
    if (row < 0) {  // the lane's virtual rows
      pos -= row;
      row = 0;
      if (pos >= end) break;
    }
    const int nrows = (int)min((long long)(len - row), end - pos);
    const int y0 = (b * p.Hkv + vl / p.nsub) * p.C + lo + row;
    const int nbox = (nrows + K::ROWS - 1) / K::ROWS;
    for (int i = lane; i < nbox; i += 32) {
#pragma unroll
      for (int kb = 0; kb < K::KB; ++kb) {
        tc::tma_prefetch_2d(tmK, kb * 64, y0 + i * K::ROWS);
        tc::tma_prefetch_2d(tmV, kb * 64, y0 + i * K::ROWS);
      }
    }
    pos += nrows;
    row = -p.pad;
    if (++vl == p.VL) {
      vl = 0;
      // next batch row with cells to read (warp-parallel search)
      int nb = -1;
      for (int b0 = b + 1; b0 < p.B && nb < 0; b0 += 32) {
        const int bb = b0 + lane;
        const unsigned m = __ballot_sync(0xffffffffu, bb < p.B && eligible_cells(p, s_len[bb]) > 0);
        if (m) nb = b0 + __ffs(m) - 1;
      }
      if (nb < 0) return;
      b = nb;
      n_b = s_len[b];
      len = eligible_cells(p, n_b);
      ext = extent(p, len);
      lo = first_cell(p, n_b, len);
    }
  }
}

// Transpose of an 8x8 bf16 tile held as an MMA fragment (thread (g, t) has
// row g, columns 2t and 2t+1 packed): afterwards thread (g, t) has row g of
// the transpose, i.e. rows 2t and 2t+1 of column g.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// -------------------------------------------------------------- producer
template <int D, int R>
__device__ void producer(const Params &p, const CUtensorMap *tmK,
                         const CUtensorMap *tmV, unsigned char *smem,
                         StageHdr *hdrs, uint64_t *full, uint64_t *empty,
                         int *s_len, int *s_bad, uint64_t *lens_ready) {
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
  // Pass 1: validity of every length and the total eligible row count.  The
  // producer checks the lengths itself so that its first copies wait for one
  // round trip to the lengths and no CTA-wide barrier.
  // With lens_smem the lengths are read from global memory here only and
  // cached in shared memory for the rest of the CTA (the compute warps wait
  // for them on lens_ready).
  long long tot = 0;
  int bad_local = 0;
  for (int b = lane; b < p.B; b += 32) {
    const int n = nlen(p, b);
    if (p.lens_smem) s_len[b] = n;
    bad_local |= (n < p.add || (!p.ring && n > p.C));
    tot += extent(p, eligible_cells(p, max(n, 0)));
  }
  const bool bad = __any_sync(0xffffffffu, bad_local) != 0;
  if (lane == 0) *s_bad = bad ? 1 : 0;
  __syncwarp();
  mbar_arrive(lens_ready);
  auto len_of = [&](int bb) { return p.lens_smem ? s_len[bb] : nlen(p, bb); };
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1)
    tot += __shfl_xor_sync(0xffffffffu, tot, off);
  const long long total = tot * p.VL;
  long long per = udiv(total + G - 1, G);
  if (per < p.min_rows) per = p.min_rows;
  const long long start = (long long)c * per;
  const long long end = min(total, start + per);

  if (!bad && start < end) {
    // Pass 2: find the batch row holding row `start` (warp prefix scan).
    long long cum = 0, cum_b = 0;
    int b = -1;
    for (int b0 = 0; b0 < p.B && b < 0; b0 += 32) {
      const int bb = b0 + lane;
      const long long x =
          bb < p.B ? (long long)extent(p, eligible_cells(p, len_of(bb))) * p.VL : 0;
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
    int n_b = len_of(b);
    int len = eligible_cells(p, n_b);
    int ext = extent(p, len);
    int lo = first_cell(p, n_b, len);
    long long off0 = start - cum_b;
    int vl = (int)udiv(off0, ext);
    int row = (int)(off0 - (long long)vl * ext) - p.pad;  // < 0: in the padding
    long long pos = start;
    bool seg_first = true;

    while (pos < end) {
      if (row < 0) {  // skip the lane's virtual rows
        pos -= row;
        row = 0;
        if (pos >= end) break;
      }
      const int L = b * p.VL + vl;
      const long long SR = cum_b + (long long)vl * ext + p.pad;  // first real row
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
        h.c0 = (int)udiv(SR, per);
        h.np = (int)udiv(SR + len - 1, per) - h.c0 + 1;
        // the appended token's cell: the last one, or (ring) its slot
        const int cnew = p.ring ? (n_b - 1) % p.C : n_b - 1;
        h.newrow = (p.add && cnew >= lo + row && cnew < lo + row + nrows) ? cnew - lo - row : -1;
        const int g = vl / p.nsub, sub = vl % p.nsub;
        const int h0 = g * p.r + sub * R;
        const int rc = min(R, p.r - sub * R);
        const uint32_t qb = seg_first ? (uint32_t)rc * D * 2 : 0u;
        const uint32_t nb = h.newrow >= 0 ? 4u * D : 0u;
        unsigned char *base = smem + (size_t)st * K::STAGE_BYTES;
        mbar_arrive_expect_tx(&full[st], 2 * K::KV_BYTES + qb + nb);
        // Whole boxes are fetched; rows past the segment are never used.
        // The cache is streamed once: evict it from L2 first, so that the
        // partials and outputs stay there.
        const int y = (b * p.Hkv + g) * p.C + lo + row;
        const uint64_t pol = tc::l2_policy_evict_first();
#pragma unroll
        for (int kb = 0; kb < K::KB; ++kb) {
          tc::tma_load_2d_hint(base + kb * K::BOX, tmK, kb * 64, y, &full[st], pol);
          tc::tma_load_2d_hint(base + K::KV_BYTES + kb * K::BOX, tmV, kb * 64, y, &full[st],
                               pol);
        }
        if (seg_first)
          bulk_g2s(base + 2 * K::KV_BYTES, p.q + ((size_t)b * p.Hq + h0) * D, qb,
                   &full[st]);
        if (nb) {
          // The appended token's rows (its cache cell is not written yet).
          const size_t src = ((size_t)b * p.Hkv + g) * D;
          bulk_g2s(base + 2 * K::KV_BYTES + K::NEWOFF, p.k_new + src, 2 * D, &full[st]);
          bulk_g2s(base + 2 * K::KV_BYTES + K::NEWOFF + 2 * D, p.v_new + src, 2 * D,
                   &full[st]);
        }
      }
      __syncwarp();
      fills[st]++;
      stage_count++;
      pos += nrows;
      row += nrows;
      seg_first = last;
      if (row == len) {
        row = -p.pad;
        if (++vl == p.VL) {
          vl = 0;
          cum_b += (long long)ext * p.VL;
          // Next batch row with a non-empty range (warp-parallel search).
          int nb = -1;
          for (int b0 = b + 1; b0 < p.B && nb < 0 && pos < end; b0 += 32) {
            const int bb = b0 + lane;
            const bool ne = bb < p.B && eligible_cells(p, len_of(bb)) > 0;
            const unsigned m = __ballot_sync(0xffffffffu, ne);
            if (m) nb = b0 + __ffs(m) - 1;
          }
          if (nb < 0) break;
          b = nb;
          n_b = len_of(b);
          len = eligible_cells(p, n_b);
          ext = extent(p, len);
          lo = first_cell(p, n_b, len);
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
  // Never leave a copy in flight into shared memory of an exiting CTA.
  bool f2 = false;
#pragma unroll
  for (int s = 0; s < K::STAGES; ++s)
    if (fills[s] > 0) mbar_wait(&full[s], (fills[s] - 1) & 1, &f2);
  if ((failed || f2) && lane == 0) record_status(p.status, kStatusTimeout);
}

// Barrier among the compute warps (an mbarrier counting one arrival per
// warp, so a wait can give up instead of hanging).
__device__ __forceinline__ void csync(uint64_t *comb, int &count, bool *failed) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(comb);
  mbar_wait_spin(comb, count & 1, failed);
  count++;
}

// GPU-scope acquire-release fence: taken by one thread after a CTA barrier it
// orders every store of the CTA before the thread's next global operation,
// and (after an atomic that observed other CTAs' releases) their stores
// before every later load of the CTA.
__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// The last CTA to finish lane L merges its np partials (slots L+c0 ..):
// m = max m_i, l = sum e^{m_i - m} l_i, o = sum e^{m_i - m} acc_i / l.
// Each of the NT threads (t = 0 .. NT-1) owns QPT float4 groups of the
// lane's R x D output.  The arithmetic does not depend on NT or on how the
// loads are batched (a lane is merged by 224, 128 or 96 threads depending on
// which CTA finishes it last, which is a matter of timing): m is the exact
// maximum over all partials, then the terms are added in ascending i.  The
// loads of the first NB partials and the maxima of the rest are issued
// together, so a lane of up to NB partials costs one round trip through L2
// (the partials were just written by other CTAs).
template <int D, int R, int NT>
__device__ __noinline__ void merge_lane(const Params &p, int L, int c0, int np,
                                        __nv_bfloat16 *out, int rc, int t) {
  constexpr int G4 = R * D / 4;                 // float4 groups of one partial
  constexpr int QPT = (G4 + NT - 1) / NT;       // groups per thread
  constexpr int NB = QPT == 1 ? 16 : (QPT == 2 ? 8 : (QPT <= 4 ? 4 : 2));  // per batch
  const float2 *ml = p.ml + (size_t)(L + c0) * R;
  const float4 *acc4 = reinterpret_cast<const float4 *>(p.acc + (size_t)(L + c0) * R * D);

  int hq[QPT];
  bool live[QPT];
#pragma unroll
  for (int i = 0; i < QPT; ++i) {
    const int q4 = t + i * NT;
    live[i] = q4 < G4;
    hq[i] = live[i] ? q4 / (D / 4) : 0;
  }
  // the first batch: (m, l) pairs and accumulator groups
  float2 mv[QPT][NB];
  float4 a[QPT][NB];
#pragma unroll
  for (int i = 0; i < QPT; ++i)
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      if (live[i] && j < np) {
        mv[i][j] = __ldcg(ml + (size_t)j * R + hq[i]);
        a[i][j] = __ldcg(acc4 + (size_t)j * G4 + t + i * NT);
      } else {
        mv[i][j] = make_float2(-INFINITY, 0.f);
        a[i][j] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  // m = max over every partial (exact in any order)
  float m[QPT];
#pragma unroll
  for (int i = 0; i < QPT; ++i) {
    m[i] = -INFINITY;
#pragma unroll
    for (int j = 0; j < NB; ++j) m[i] = fmaxf(m[i], mv[i][j].x);
  }
  for (int j0 = NB; j0 < np; j0 += NB) {
#pragma unroll
    for (int i = 0; i < QPT; ++i)
#pragma unroll
      for (int j = 0; j < NB; ++j)
        if (live[i] && j0 + j < np) m[i] = fmaxf(m[i], __ldcg(&ml[(size_t)(j0 + j) * R + hq[i]].x));
  }
  float l[QPT], x[QPT][4];
#pragma unroll
  for (int i = 0; i < QPT; ++i) {
    l[i] = 0.f;
    x[i][0] = x[i][1] = x[i][2] = x[i][3] = 0.f;
  }
  for (int j0 = 0; j0 < np; j0 += NB) {
    if (j0 > 0) {
#pragma unroll
      for (int i = 0; i < QPT; ++i)
#pragma unroll
        for (int j = 0; j < NB; ++j) {
          if (live[i] && j0 + j < np) {
            mv[i][j] = __ldcg(ml + (size_t)(j0 + j) * R + hq[i]);
            a[i][j] = __ldcg(acc4 + (size_t)(j0 + j) * G4 + t + i * NT);
          } else {
            mv[i][j] = make_float2(-INFINITY, 0.f);
            a[i][j] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
    }
#pragma unroll
    for (int i = 0; i < QPT; ++i)
#pragma unroll
      for (int j = 0; j < NB; ++j) {
        const float e = mv[i][j].x == -INFINITY ? 0.f : exp2f(mv[i][j].x - m[i]);
        l[i] += e * mv[i][j].y;
        x[i][0] += e * a[i][j].x;
        x[i][1] += e * a[i][j].y;
        x[i][2] += e * a[i][j].z;
        x[i][3] += e * a[i][j].w;
      }
  }
#pragma unroll
  for (int i = 0; i < QPT; ++i) {
    const int q4 = t + i * NT;
    if (live[i] && hq[i] < rc) {
      const float inv = 1.f / l[i];
      *reinterpret_cast<uint2 *>(out + q4 * 4) =
          make_uint2(pack_bf16(x[i][0] * inv, x[i][1] * inv), pack_bf16(x[i][2] * inv, x[i][3] * inv));
    }
  }
}

// ------------------------------------------------------------- consumers
// Fragment layout of mma.m16n8k16 (g = lane / 4, t = lane % 4):
//   A regs 0..3: (row g, cols 2t..2t+1), (row g+8, same), (row g, cols
//                8+2t..), (row g+8, cols 8+2t..)
//   B regs 0..1: (rows 2t..2t+1, col g), (rows 8+2t.., col g)
//   C regs 0..3: (row g, cols 2t, 2t+1), (row g+8, cols 2t, 2t+1)
// Tile rows are query heads; S columns are cache rows; O columns features.
template <int D, int R>
__device__ void consumer(const Params &p, unsigned char *smem,
                         const StageHdr *hdrs, uint64_t *full, uint64_t *empty,
                         uint64_t *comb, int &merge_flag) {
  using K = Cfg<D, R>;
  constexpr int NWC = K::NWC, KS = K::KS, NT = K::NT;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  bool failed = false;

  // Up to 8 heads (TR) the products are taken transposed, S^T = K Q^T and
  // O^T += V^T P^T: a warp's 16 cache rows fill the MMA's 16-row dimension
  // and the heads its 8 columns, 8 + 8 MMAs per 16 cache rows where the
  // heads as tile rows (up to 16) take 16 + 16.
  constexpr bool TR = R <= 8;
  constexpr int NO = TR ? D / 16 : NT;
  uint32_t qa[KS][TR ? 2 : 4];  // Q per 16-feature k-step: B operand (TR), else A
  float o[NO][4];               // O^T tiles of 16 features (TR), else O tiles of 8
  float m_run[2], l_run[2];     // TR: head columns 2t, 2t + 1; else head rows g, g + 8
  int stage_count = 0, comb_count = 0;
  // Split lanes whose partial this CTA wrote, counted at the end (at most
  // two: the first and the last segment of the range).
  int pend_n = 0, pL0 = 0, pc0 = 0, pn0 = 0, pL1 = 0, pc1 = 0, pn1 = 0;

  while (true) {
    const int st = stage_count % K::STAGES;
    const uint32_t par = (stage_count / K::STAGES) & 1;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[st], par, &failed))) break;
    const StageHdr hd = hdrs[st];
    if (hd.flags & kEnd) break;
    unsigned char *base = smem + (size_t)st * K::STAGE_BYTES;
    const uint32_t sK = smem_u32(base);
    const uint32_t sV = smem_u32(base + K::KV_BYTES);

    if (hd.flags & kFirst) {
      // The group's query rows (bf16, [rc][D]) -> A fragments; rows past the
      // group are zero.
      const __nv_bfloat16 *sQ =
          reinterpret_cast<const __nv_bfloat16 *>(base + 2 * K::KV_BYTES);
      const int vl = hd.lane % p.VL;
      const int rc = min(R, p.r - (vl % p.nsub) * R);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int c0 = ks * 16 + 2 * t;
        if constexpr (TR) {  // B[k][n] = Q[n][k]: features 2t, 2t+1 (+8) of head g
          qa[ks][0] = g < rc ? *reinterpret_cast<const uint32_t *>(sQ + g * D + c0) : 0u;
          qa[ks][1] = g < rc ? *reinterpret_cast<const uint32_t *>(sQ + g * D + c0 + 8) : 0u;
        } else {
          qa[ks][0] = g < rc ? *reinterpret_cast<const uint32_t *>(sQ + g * D + c0) : 0u;
          qa[ks][1] = g + 8 < rc ? *reinterpret_cast<const uint32_t *>(sQ + (g + 8) * D + c0) : 0u;
          qa[ks][2] = g < rc ? *reinterpret_cast<const uint32_t *>(sQ + g * D + c0 + 8) : 0u;
          qa[ks][3] = g + 8 < rc ? *reinterpret_cast<const uint32_t *>(sQ + (g + 8) * D + c0 + 8) : 0u;
        }
      }
#pragma unroll
      for (int n = 0; n < NO; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
      m_run[0] = m_run[1] = -INFINITY;
      l_run[0] = l_run[1] = 0.f;
    }

    const int nv = hd.nrows - w * kBR;  // valid rows of this warp's 16
    // Generic-proxy writes into the stage (below) are fenced against the
    // TMA writes that refill it once it is released.
    bool wrote = (hd.flags & kLast) != 0;
    if (nv < kBR && nv > 0) {
      wrote = true;
      // Rows past the segment hold other data (maybe non-finite): zero this
      // warp's share of them in V so 0 * V stays 0.
      for (int idx = lane; idx < (kBR - nv) * (D / 8); idx += 32) {
        const int row = w * kBR + nv + idx / (D / 8), ch = idx % (D / 8);
        *reinterpret_cast<uint4 *>(base + K::KV_BYTES + (ch >> 3) * K::BOX +
                                   swz(row, ch & 7)) = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }

    if (hd.newrow >= 0 && (hd.newrow >> 4) == w) {
      // This warp's rows hold the appended token, whose cache cell is not
      // written yet: take its key and value from the step's input (staged
      // with the stage), and write them to the cache (the first virtual lane
      // of the KV head does).
      wrote = true;
      const int L = hd.lane, b = L / p.VL, vl = L % p.VL, g = vl / p.nsub;
      const unsigned char *stg = base + 2 * K::KV_BYTES + K::NEWOFF;
      const size_t dst = (((size_t)b * p.Hkv + g) * p.C + hd.cell0 + hd.newrow) * D;
      for (int idx = lane; idx < 2 * (D / 8); idx += 32) {
        const int isv = idx >= D / 8, ch = idx - isv * (D / 8);
        const uint4 x = *reinterpret_cast<const uint4 *>(stg + idx * 16);
        *reinterpret_cast<uint4 *>(base + isv * K::KV_BYTES + (ch >> 3) * K::BOX +
                                   swz(hd.newrow, ch & 7)) = x;
        if (vl % p.nsub == 0)
          *reinterpret_cast<uint4 *>((isv ? p.v_cache : p.k_cache) + dst + ch * 8) = x;
      }
      __syncwarp();
    }

    if constexpr (TR) {
      if (nv > 0) {
        // ---- S^T = K Q^T: the warp's 16 cache rows x 8 head columns (two
        // accumulators over alternate k-steps, so the chains are half as long)
        float s[4] = {0.f, 0.f, 0.f, 0.f}, s2[4] = {0.f, 0.f, 0.f, 0.f};
        const int krow = w * kBR + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const int ch = 2 * ks + (lane >> 4);
          uint32_t a[4];
          ldsm_x4(sK + (ch >> 3) * K::BOX + swz(krow, ch & 7), a[0], a[1], a[2], a[3]);
          mma_16816((ks & 1) ? s2 : s, a, qa[ks][0], qa[ks][1]);
        }
        // ---- online softmax over the rows (log2 domain): this thread has
        // rows g and g + 8 of head columns 2t and 2t + 1
        const bool r0 = g < nv, r1 = g + 8 < nv;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float v = s[e] + s2[e];
          s[e] = (e < 2 ? r0 : r1) ? v * p.scale_log2 : -INFINITY;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float mx = fmaxf(s[j], s[j + 2]);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          if (mx > m_run[j] + kLazyRescale) {
            const float alpha = exp2f(m_run[j] - mx);  // 0 when m_run = -inf
            l_run[j] *= alpha;
            m_run[j] = mx;
#pragma unroll
            for (int n = 0; n < NO; ++n) {
              o[n][j] *= alpha;
              o[n][j + 2] *= alpha;
            }
          }
        }
        float pv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float msub = m_run[e & 1] == -INFINITY ? 0.f : m_run[e & 1];
          pv[e] = exp2f(s[e] - msub);
        }
        const uint32_t p0 = pack_bf16(pv[0], pv[1]);  // row g: heads 2t, 2t + 1
        const uint32_t p1 = pack_bf16(pv[2], pv[3]);  // row g + 8
        // the denominator sums exactly the bf16 weights the MMA uses
        l_run[0] += bf16lo_to_f32(p0) + bf16lo_to_f32(p1);
        l_run[1] += bf16hi_to_f32(p0) + bf16hi_to_f32(p1);
        // P^T as the B operand: rows 2t, 2t + 1 (and + 8) of head column g
        const uint32_t pb0 = movmatrix_t(p0), pb1 = movmatrix_t(p1);
        // ---- O^T += V^T P^T (A = V^T by transposing loads, 16 features a tile)
        const int vrow = w * kBR + (lane & 7) + ((lane >> 4) & 1) * 8;
#pragma unroll
        for (int n = 0; n < NO; ++n) {
          const int ch = 2 * n + ((lane >> 3) & 1);
          uint32_t a[4];
          ldsm_x4_t(sV + (ch >> 3) * K::BOX + swz(vrow, ch & 7), a[0], a[1], a[2], a[3]);
          mma_16816(o[n], a, pb0, pb1);
        }
      }
    } else {
      if (nv > 0) {
        // ---- S = Q K^T for this warp's 16 cache rows (two 8-row tiles)
        float s[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
          const int krow = w * kBR + nt * 8 + (lane & 7);
#pragma unroll
          for (int kk = 0; kk < KS / 2; ++kk) {
            const int ch = 4 * kk + (lane >> 3);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(sK + (ch >> 3) * K::BOX + swz(krow, ch & 7), b0, b1, b2, b3);
            mma_16816(s[nt], qa[2 * kk], b0, b1);
            mma_16816(s[nt], qa[2 * kk + 1], b2, b3);
          }
        }
        // ---- online softmax on the fragments (log2 domain)
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = nt * 8 + 2 * t + (e & 1);
            const float v = col < nv ? s[nt][e] * p.scale_log2 : -INFINITY;
            s[nt][e] = v;
            mx[e >> 1] = fmaxf(mx[e >> 1], v);
          }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
          mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
          if (mx[i] > m_run[i] + kLazyRescale) {
            const float alpha = exp2f(m_run[i] - mx[i]);  // 0 when m_run = -inf
            l_run[i] *= alpha;
            m_run[i] = mx[i];
#pragma unroll
            for (int n = 0; n < NT; ++n) {
              o[n][2 * i] *= alpha;
              o[n][2 * i + 1] *= alpha;
            }
          }
        }
        uint32_t pa[4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          float pv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float msub = m_run[e >> 1] == -INFINITY ? 0.f : m_run[e >> 1];
            pv[e] = exp2f(s[nt][e] - msub);
          }
          pa[2 * nt] = pack_bf16(pv[0], pv[1]);
          pa[2 * nt + 1] = pack_bf16(pv[2], pv[3]);
          // the denominator sums exactly the bf16 weights the MMA uses
          l_run[0] += bf16lo_to_f32(pa[2 * nt]) + bf16hi_to_f32(pa[2 * nt]);
          l_run[1] += bf16lo_to_f32(pa[2 * nt + 1]) + bf16hi_to_f32(pa[2 * nt + 1]);
        }
        // ---- O += P V (A = P over the 16 cache rows, B = V rows from smem)
        const int vrow = w * kBR + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int nn = 0; nn < NT / 2; ++nn) {
          const int ch = 2 * nn + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sV + (ch >> 3) * K::BOX + swz(vrow, ch & 7), b0, b1, b2, b3);
          mma_16816(o[2 * nn], pa, b0, b1);
          mma_16816(o[2 * nn + 1], pa, b2, b3);
        }
      }
    }

    // ---- end of a lane segment: combine the warps, then output or partial
    if (hd.flags & kLast) {
      // the sums over the warp's rows: the four lanes sharing a head row, or
      // (TR) the eight sharing a head column
      float l_tot[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        float l = l_run[i];
        if constexpr (TR) {
          l += __shfl_xor_sync(0xffffffffu, l, 4);
          l += __shfl_xor_sync(0xffffffffu, l, 8);
          l += __shfl_xor_sync(0xffffffffu, l, 16);
        } else {
          l += __shfl_xor_sync(0xffffffffu, l, 1);
          l += __shfl_xor_sync(0xffffffffu, l, 2);
        }
        l_tot[i] = l;
      }
      // Every warp is done with this stage: reuse it as scratch.
      csync(comb, comb_count, &failed);
      float *sm_m = reinterpret_cast<float *>(base);   // [NWC][16]
      float *sm_l = sm_m + NWC * 16;                     // [NWC][16]
      float *sm_acc = sm_l + NWC * 16;                   // [NWC][R][ACC_STRIDE]
      if constexpr (TR) {
        // O^T tile n: features 16n + g (+ 8) of head columns 2t, 2t + 1
        if (g == 0) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            sm_m[w * 16 + 2 * t + j] = m_run[j];
            sm_l[w * 16 + 2 * t + j] = l_tot[j];
          }
        }
#pragma unroll
        for (int n = 0; n < NO; ++n)
#pragma unroll
          for (int j = 0; j < 2; ++j)
            if (2 * t + j < R) {
              float *row = sm_acc + (w * R + 2 * t + j) * K::ACC_STRIDE + n * 16 + g;
              row[0] = o[n][j];
              row[8] = o[n][j + 2];
            }
      } else {
        if (t == 0) {
          sm_m[w * 16 + g] = m_run[0];
          sm_l[w * 16 + g] = l_tot[0];
          sm_m[w * 16 + g + 8] = m_run[1];
          sm_l[w * 16 + g + 8] = l_tot[1];
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          if (g < R)
            *reinterpret_cast<float2 *>(sm_acc + (w * R + g) * K::ACC_STRIDE + n * 8 + 2 * t) =
                make_float2(o[n][0], o[n][1]);
          if (g + 8 < R)
            *reinterpret_cast<float2 *>(sm_acc + (w * R + g + 8) * K::ACC_STRIDE + n * 8 + 2 * t) =
                make_float2(o[n][2], o[n][3]);
        }
      }
      csync(comb, comb_count, &failed);
      const int L = hd.lane, b = L / p.VL, vl = L % p.VL;
      const int h0 = (vl / p.nsub) * p.r + (vl % p.nsub) * R;
      const int rc = min(R, p.r - (vl % p.nsub) * R);
      __nv_bfloat16 *out = p.o + ((size_t)b * p.Hq + h0) * D;
      // Warp w combines head rows w, w + NWC, ...: lane j < NWC weighs warp
      // j's state, the weights reach every lane by shuffles, and each lane
      // sums D/32 features over the warps.
      for (int h = w; h < R; h += NWC) {
        const float mw = lane < NWC ? sm_m[lane * 16 + h] : -INFINITY;
        float mm = mw;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1)
          mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, off));
        const float e = mw == -INFINITY ? 0.f : exp2f(mw - mm);
        float lsum = lane < NWC ? e * sm_l[lane * 16 + h] : 0.f;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1)
          lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
        float a[D / 32];
#pragma unroll
        for (int k = 0; k < D / 32; ++k) a[k] = 0.f;
#pragma unroll
        for (int ww = 0; ww < NWC; ++ww) {
          const float ew = __shfl_sync(0xffffffffu, e, ww);
#pragma unroll
          for (int k = 0; k < D / 32; ++k)
            a[k] += ew * sm_acc[(ww * R + h) * K::ACC_STRIDE + lane + 32 * k];
        }
        if (hd.np == 1) {
          if (h < rc) {
            const float inv = 1.f / lsum;
#pragma unroll
            for (int k = 0; k < D / 32; ++k)
              out[h * D + lane + 32 * k] = __float2bfloat16_rn(a[k] * inv);
          }
        } else {
          // The lane's merge reads this partial at the end of the kernel,
          // after the rest of the cache has streamed through L2: keep it.
          const uint64_t keep = tc::l2_policy_evict_last();
#pragma unroll
          for (int k = 0; k < D / 32; ++k)
            tc::st_global_hint(&p.acc[((size_t)hd.slot * R + h) * D + lane + 32 * k], a[k], keep);
          if (lane == 0)
            tc::st_global_hint(&p.ml[(size_t)hd.slot * R + h], make_float2(mm, lsum), keep);
        }
      }
      // A partial is counted at the end of the CTA's range: nobody needs it
      // sooner (the lane's other pieces end with their CTAs' ranges), and the
      // warps go on to the next segment without waiting for the count.  A
      // range has at most two split lanes, its first and its last.
      if (hd.np > 1 && pend_n < 2) {
        if (pend_n == 0) {
          pL0 = L; pc0 = hd.c0; pn0 = hd.np;
        } else {
          pL1 = L; pc1 = hd.c0; pn1 = hd.np;
        }
        pend_n++;
      }
    }
    if (wrote) tc::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    stage_count++;
  }
  if (pend_n > 0) {
    // Publish and count this CTA's partials; it merges each lane it is the
    // last to finish.  After the barrier one thread's release fence covers
    // the stores of the whole CTA; its acquire fence (when last) covers the
    // loads of the merges, which every thread starts after the second
    // barrier.
    csync(comb, comb_count, &failed);
    if (threadIdx.x == 0) {
      fence_acq_rel_gpu();
      const int o0 = atomicAdd(&p.counters[pc0], 1);
      const int o1 = pend_n > 1 ? atomicAdd(&p.counters[pc1], 1) : 0;
      const int flags = (o0 == pn0 - 1 ? 1 : 0) | (pend_n > 1 && o1 == pn1 - 1 ? 2 : 0);
      // The last count of a lane is its counter's last access in this call:
      // leave it zero for the next call.
      if (flags & 1) p.counters[pc0] = 0;
      if (flags & 2) p.counters[pc1] = 0;
      if (flags) fence_acq_rel_gpu();
      merge_flag = flags;
    }
    csync(comb, comb_count, &failed);
    const int flags = merge_flag;
    // Two merges run side by side (warps 0-3 and the rest), one runs on
    // every compute warp.
    constexpr int NA = 4 * 32, NBT = (NWC - 4) * 32;
    const int i = flags == 3 ? (w < 4 ? 0 : 1) : (flags == 2 ? 1 : 0);
    if (flags) {
      const int L = i ? pL1 : pL0, b = L / p.VL, vl = L % p.VL;
      const int h0 = (vl / p.nsub) * p.r + (vl % p.nsub) * R;
      const int rc = min(R, p.r - (vl % p.nsub) * R);
      __nv_bfloat16 *out = p.o + ((size_t)b * p.Hq + h0) * D;
      if (flags != 3)
        merge_lane<D, R, NWC * 32>(p, L, i ? pc1 : pc0, i ? pn1 : pn0, out, rc, threadIdx.x);
      else if (w < 4)
        merge_lane<D, R, NA>(p, L, pc0, pn0, out, rc, threadIdx.x);
      else
        merge_lane<D, R, NBT>(p, L, pc1, pn1, out, rc, threadIdx.x - NA);
    }
  }
  if (failed && lane == 0) record_status(p.status, kStatusTimeout);
}

template <int D, int R>
__global__ void __launch_bounds__(Cfg<D, R>::THREADS, Cfg<D, R>::MIN_BLOCKS)
    split_kernel(const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const Params p) {
  using K = Cfg<D, R>;
  extern __shared__ unsigned char smem_raw[];
  __shared__ StageHdr hdrs[K::STAGES];
  __shared__ __align__(8) uint64_t full[K::STAGES], empty[K::STAGES], comb;
  __shared__ int merge_flag, s_bad;
  __shared__ __align__(8) uint64_t lens_ready;
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int *s_len = reinterpret_cast<int *>(smem + K::STAGES * K::STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < K::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], K::NWC);
    }
    mbar_init(&comb, K::NWC);
    mbar_init(&lens_ready, 32);
    fence_mbar_init();
  }
  if (warp == K::NWC && lane == 0) {
    tc::prefetch_tmap(&tmK);
    tc::prefetch_tmap(&tmV);
  }
  __syncthreads();
  // Everything above touches only shared memory and the kernel parameters.
  // The producer warp then asks L2 for the first rows of this CTA's range
  // (reads only, planned from lengths that may still change).  From the
  // wait on, the CTA reads and writes global memory that the previous
  // kernel on the stream may use: wait until it has completed (a no-op when
  // the launch is not a programmatic dependent), then let the next kernel
  // start its own set-up.
  if (warp == K::NWC) prefetch_range<D, R>(p, &tmK, &tmV, s_len);
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();
  if (warp == K::NWC) {
    producer<D, R>(p, &tmK, &tmV, smem, hdrs, full, empty, s_len, &s_bad, &lens_ready);
  } else {
    // The producer validates every length (each must give n_b in [0, C];
    // otherwise the call writes only zeros) and caches them.
    bool failed = false;
    const bool ok = mbar_wait(&lens_ready, 0, &failed);
    const bool bad = !ok || s_bad != 0;
    if (!ok && lane == 0) record_status(p.status, kStatusTimeout);
    if (ok && bad && blockIdx.x == 0 && threadIdx.x == 0)
      record_status(p.status, GQA_ERR_CAPACITY);
    if (p.add && warp == 0) {
      // Fused append: this CTA reads no length from global memory any more
      // (the producer has its copy), so the last CTA to get here advances
      // them, unless the call was refused.  This overlaps the first copies.
      int last = 0;
      if (lane == 0) {
        fence_acq_rel_gpu();
        last = atomicAdd(&p.counters[kCtrFinish], 1) == (int)gridDim.x - 1;
        if (last) {
          p.counters[kCtrFinish] = 0;  // every CTA has counted: reset
          fence_acq_rel_gpu();
        }
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      __syncwarp();
      if (last && !bad)
        for (int b = lane; b < p.B; b += 32) p.lens_out[b] += 1;
    }
    // Rows of sequences with nothing to attend to (n_b = 0, or any invalid
    // length) are zeros; CTA c takes batch rows c, c + G, ...
    for (int b = blockIdx.x; b < p.B; b += gridDim.x) {
      if (!bad && (p.lens_smem ? s_len[b] : nlen(p, b)) > 0) continue;
      __nv_bfloat16 *ob = p.o + (size_t)b * p.Hq * D;
      for (int i = threadIdx.x; i < p.Hq * D / 8; i += K::NWC * 32)
        reinterpret_cast<uint4 *>(ob)[i] = make_uint4(0, 0, 0, 0);
    }
    consumer<D, R>(p, smem, hdrs, full, empty, &comb, merge_flag);
  }
}

}  // namespace dec
}  // namespace gqa
