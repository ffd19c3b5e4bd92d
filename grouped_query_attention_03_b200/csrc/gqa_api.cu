// gqa_api.cu -- the C ABI declared in include/gqa.h.
//
// Host-side validation (the checked constructor conditions of "Share
// key/value heads and make context explicit", section "Give each query head
// an explicit shared KV head": positive head counts and width, Hq divisible
// by Hkv; the refused zero window of "Intersect the window ..."; checked size
// products as in its incremental path), then kernel launches on the caller's
// stream.  Nothing here allocates device memory.
#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/gqa.h"
#include "append.cuh"
#include "common.cuh"
#include "decode_splitk.cuh"
#include "prefill_pair.cuh"
#include "prefill_persist.cuh"
#include "prefill_split.cuh"
#include "simt.cuh"

namespace {

using bf16 = __nv_bfloat16;

constexpr int kMaxDecodeCtas = gqa::dec::kMaxCtas;  // workspace is sized for this many
#ifndef GQA_DEC_MIN_ROWS
#define GQA_DEC_MIN_ROWS 320
#endif
// Smallest row range per CTA: small calls use fewer CTAs, so that a lane is
// split into at most about 16 partials, which the merge reads in one batch
// (swept 256-384 on the 16.8 MB sliding-window step: 320 fastest).
constexpr int kDecodeMinRows = GQA_DEC_MIN_ROWS;
#ifndef GQA_DEC_LANE_PAD_BYTES
#define GQA_DEC_LANE_PAD_BYTES 131072
#endif
// A lane segment's fixed cost in a CTA, as cache bytes: the split gives each
// non-empty lane this many bytes of virtual rows (see dec::extent).
constexpr int kDecodeLanePadBytes = GQA_DEC_LANE_PAD_BYTES;


struct DeviceInfo {
  int sms = 0;
  int major = 0;
};

// The paired prefill kernel's grid for a plain prompt leaves SMs idle and
// its longest query tile (the last one) walks more than 4 KV tiles: one
// head per CTA is faster there (see the dispatch in attend_impl).
bool prefill_prefers_split(int B, int Hq, int Hkv, int Tq, int Tk, int cached, bool seg,
                           int window, int sms) {
  if (cached || seg || Tq != Tk || Tq <= 0) return false;
  const long long num_mt = (Tq + 127) / 128;
  const long long pair_grid = (long long)B * Hkv * ((Hq / Hkv) / 2) * num_mt;
  if (pair_grid >= sms) return false;
  const long long a0 = (num_mt - 1) * 128;
  const long long hi = Tq - 1;
  const long long lo = window > 0 ? std::max(0LL, a0 - (window - 1)) : 0;
  return hi / 128 - lo / 128 + 1 > 4;
}

gqa_status device_info(DeviceInfo *out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool have[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return GQA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    DeviceInfo d;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor,
                               dev) != cudaSuccess) {
      cudaGetLastError();
      return GQA_ERR_CUDA;
    }
    cache[dev] = d;
    have[dev] = true;
  }
  *out = cache[dev];
  return out->major == 10 ? GQA_OK : GQA_ERR_DEVICE;
}

// a*b*... in int64 with overflow detection (all factors >= 0).
bool mul_ok(int64_t *acc, int64_t f) {
  if (f < 0) return false;
  if (f != 0 && *acc > INT64_MAX / f) return false;
  *acc *= f;
  return true;
}

bool elems(int64_t *out, std::initializer_list<int64_t> dims) {
  int64_t acc = 1;
  for (int64_t d : dims)
    if (!mul_ok(&acc, d)) return false;
  *out = acc;
  return true;
}

bool aligned16(const void *p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

gqa_status check_heads(int Hq, int Hkv, int d) {
  if (Hq <= 0 || Hkv <= 0 || d <= 0) return GQA_ERR_SHAPE;
  if (Hq % Hkv != 0) return GQA_ERR_GROUPS;
  return GQA_OK;
}

gqa_status check_window(int window) {
  return (window == 0 || window < -1) ? GQA_ERR_WINDOW : GQA_OK;
}

gqa_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}

int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// ------------------------------------------------------------ decode plan
struct DecPlan {
  int R = 1;     // heads stacked per CTA lane (power of two, <= 16)
  int nsub = 1;  // sub-groups per KV head
  int VL = 1;    // virtual lanes per batch row
};

DecPlan decode_plan(int Hq, int Hkv) {
  DecPlan p;
  const int r = Hq / Hkv;
  p.R = r >= 16 ? 16 : next_pow2(r);
  p.nsub = (r + p.R - 1) / p.R;
  p.VL = Hkv * p.nsub;
  return p;
}

struct DecLayout {
  size_t counters = 0, ml = 0, acc = 0, total = 0;
  size_t counter_bytes = 0;
};

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace: the arrival counters (one per possible first CTA of a split
// lane, and one count of CTAs that have read the lengths) at a fixed place
// for every shape, zero between calls; then the (m, l) and acc partials, one
// slot per (lane, CTA) pair touching it.
bool decode_layout(int B, int Hq, int Hkv, int d, DecLayout *L) {
  const DecPlan pl = decode_plan(Hq, Hkv);
  int64_t lanes, slots, ml_elems, acc_elems;
  if (!elems(&lanes, {B, pl.VL})) return false;
  slots = lanes + kMaxDecodeCtas;
  if (!elems(&ml_elems, {slots, pl.R})) return false;
  if (!elems(&acc_elems, {slots, pl.R, d})) return false;
  if (acc_elems > INT64_MAX / 8) return false;
  L->counters = 0;
  L->counter_bytes = (size_t)(gqa::dec::kCtrFinish + 1) * sizeof(int);
  L->ml = round256(L->counter_bytes);
  L->acc = L->ml + round256((size_t)ml_elems * sizeof(float2));
  L->total = L->acc + round256((size_t)acc_elems * sizeof(float));
  return true;
}

bool splitk_supported(gqa_dtype dtype, int d) {
  return dtype == GQA_BF16 && (d == 64 || d == 128);
}

// The split-K kernel addresses cache rows with 32-bit TMA coordinates.
bool splitk_rows_ok(int B, int Hkv, int C) {
  return (long long)B * Hkv * C < (1LL << 31);
}

template <int D, int R>
gqa_status launch_splitk(const gqa::dec::Params &p, const void *k_cache,
                         const void *v_cache, int sms, cudaStream_t st) {
  using K = gqa::dec::Cfg<D, R>;
  CUtensorMap mk, mv;
  const long long rows = (long long)p.B * p.Hkv * p.C;
  if (!gqa::tma::make_bf16_map(&mk, k_cache, D, rows, 0, K::ROWS) ||
      !gqa::tma::make_bf16_map(&mv, v_cache, D, rows, 0, K::ROWS))
    return GQA_ERR_CUDA;
  static bool attr_done = false;  // per instantiation; benign race
  if (!attr_done) {
    if (cudaFuncSetAttribute(gqa::dec::split_kernel<D, R>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             K::SMEM + gqa::dec::kLensSmem * 4) != cudaSuccess) {
      cudaGetLastError();
      return GQA_ERR_CUDA;
    }
    attr_done = true;
  }
  const int grid = std::min(kMaxDecodeCtas, K::MIN_BLOCKS * sms);
  // the lengths' shared-memory copy follows the stages
  const int smem = K::SMEM + (p.lens_smem ? ((p.B * 4 + 15) & ~15) : 0);
  // A programmatic dependent of the previous kernel on the stream: its CTAs
  // set up while that kernel drains and wait for it before touching memory.
  if (gqa::launch_dependent(gqa::dec::split_kernel<D, R>, dim3(grid), dim3(K::THREADS), smem,
                            st, mk, mv, p) != cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_CUDA;
  }
  return launch_status();
}

template <int D>
gqa_status dispatch_splitk_R(int R, const gqa::dec::Params &p, const void *kc,
                             const void *vc, int sms, cudaStream_t st) {
  switch (R) {
    case 1: return launch_splitk<D, 1>(p, kc, vc, sms, st);
    case 2: return launch_splitk<D, 2>(p, kc, vc, sms, st);
    case 4: return launch_splitk<D, 4>(p, kc, vc, sms, st);
    case 8: return launch_splitk<D, 8>(p, kc, vc, sms, st);
    case 16: return launch_splitk<D, 16>(p, kc, vc, sms, st);
  }
  return GQA_ERR_UNSUPPORTED;
}

template <typename T>
gqa_status launch_simt_prefill(const void *q, const void *k, const void *v,
                               void *o, const int32_t *lens, const int32_t *seg,
                               int B, int Hq, int Hkv, int Tq, int Tk, int cached,
                               int d, int window, float scale_log2,
                               int32_t *status, cudaStream_t st) {
  const dim3 grid((Tq + 3) / 4, Hq, B);
  const int nf = (d + 31) / 32;
#define GQA_PF(NF)                                                        \
  gqa::prefill_simt_kernel<T, NF><<<grid, 128, 0, st>>>(                  \
      (const T *)q, (const T *)k, (const T *)v, (T *)o, lens, seg, Hq,    \
      Hkv, Tq, Tk, cached, d, window, scale_log2, status)
  switch (nf) {
    case 1: GQA_PF(1); break;
    case 2: GQA_PF(2); break;
    case 3: GQA_PF(3); break;
    case 4: GQA_PF(4); break;
    case 5: GQA_PF(5); break;
    case 6: GQA_PF(6); break;
    case 7: GQA_PF(7); break;
    case 8: GQA_PF(8); break;
    default: return GQA_ERR_UNSUPPORTED;
  }
#undef GQA_PF
  return launch_status();
}

template <typename T>
gqa_status launch_simt_decode(const void *q, const void *kc, const void *vc,
                              void *o, const int32_t *lens, int B, int Hq,
                              int Hkv, int C, int d, int window,
                              float scale_log2, int32_t *status,
                              cudaStream_t st, const void *kn = nullptr,
                              const void *vn = nullptr, int add = 0, int ring = 0) {
  const dim3 grid(Hq, B);
  const int nf = (d + 31) / 32;
#define GQA_DC(NF)                                                         \
  gqa::decode_simt_kernel<T, NF><<<grid, 32, 0, st>>>(                     \
      (const T *)q, (const T *)kc, (const T *)vc, (T *)o, lens, B, Hq, Hkv, \
      C, d, window, scale_log2, status, (const T *)kn, (const T *)vn, add, ring)
  switch (nf) {
    case 1: GQA_DC(1); break;
    case 2: GQA_DC(2); break;
    case 3: GQA_DC(3); break;
    case 4: GQA_DC(4); break;
    case 5: GQA_DC(5); break;
    case 6: GQA_DC(6); break;
    case 7: GQA_DC(7); break;
    case 8: GQA_DC(8); break;
    default: return GQA_ERR_UNSUPPORTED;
  }
#undef GQA_DC
  return launch_status();
}

}  // namespace

extern "C" {

const char *gqa_version(void) { return "0.1.0"; }

const char *gqa_status_string(gqa_status s) {
  switch (s) {
    case GQA_OK: return "ok";
    case GQA_ERR_NULL: return "a required pointer is NULL";
    case GQA_ERR_SHAPE: return "a size is negative or a head count/width is not positive";
    case GQA_ERR_GROUPS: return "query heads are not a multiple of KV heads";
    case GQA_ERR_WINDOW: return "window must be -1 (none) or positive";
    case GQA_ERR_CAPACITY: return "a sequence length is outside [0, capacity]";
    case GQA_ERR_OVERFLOW: return "an element count overflows";
    case GQA_ERR_UNSUPPORTED: return "head width, dtype, alignment or grid size not supported";
    case GQA_ERR_WORKSPACE: return "workspace missing or too small";
    case GQA_ERR_CUDA: return "CUDA runtime error";
    case GQA_ERR_DEVICE: return "current device is not an sm_100 GPU";
    case GQA_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
    case GQA_ERR_SEGMENT: return "a packed segment start lies outside [0, t]";
  }
  return "unknown status";
}

int gqa_kv_head_for_query(int h, int Hq, int Hkv) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return -1;
  if (h < 0 || h >= Hq) return -1;
  return h / (Hq / Hkv);
}

int gqa_prefill_kernel(int B, int Hq, int Hkv, int T, int d, int window, int sms) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || T <= 0 || d <= 0 || sms <= 0 || Hq % Hkv != 0)
    return -1;
  if (window == 0 || window < -1) return -1;
  if (!gqa::pfs::supported(d)) return 0;
  if (gqa::pf2::supported(d, Hq, Hkv) &&
      !prefill_prefers_split(B, Hq, Hkv, T, T, 0, false, window, sms))
    return 1;
  return 2;
}

int gqa_window_start(int t, int window) {
  if (t < 0 || window == 0 || window < -1) return -1;
  if (window < 0) return 0;
  return t > window - 1 ? t - (window - 1) : 0;
}

uint64_t gqa_cache_bytes(int64_t L, int64_t B, int64_t T, int64_t Hkv,
                         int64_t d, int64_t elem_bytes) {
  const int64_t f[6] = {L, B, T, Hkv, d, elem_bytes};
  uint64_t acc = 2;
  for (int i = 0; i < 6; ++i) {
    if (f[i] < 0) return 0;
    const uint64_t x = (uint64_t)f[i];
    if (x != 0 && acc > UINT64_MAX / x) return 0;
    acc *= x;
  }
  return acc;
}

}  // extern "C"

namespace {

// Attention of Tq query rows per head against Tk key rows per KV lane:
// a prompt (cached = 0, Tq = Tk = T) or new rows after a cache (cached = 1,
// Tk = capacity, query row i at position n_b - Tq + i).
gqa_status attend_impl(gqa_dtype dtype, const void *q, const void *k,
                       const void *v, void *o, const int32_t *seq_lens,
                       const int32_t *seg, int B, int Hq, int Hkv, int Tq,
                       int Tk, int cached, int d, int window, float scale,
                       int32_t *dev_status, gqa_stream_t stream) {
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED;
  if (B < 0 || Tq < 0 || Tk < 0) return GQA_ERR_SHAPE;
  gqa_status s = check_heads(Hq, Hkv, d);
  if (s != GQA_OK) return s;
  if ((s = check_window(window)) != GQA_OK) return s;
  int64_t nq, nk;
  if (!elems(&nq, {B, Hq, Tq, d}) || !elems(&nk, {B, Hkv, Tk, d}) ||
      nq > INT64_MAX / 4 || nk > INT64_MAX / 4)
    return GQA_ERR_OVERFLOW;
  if (B == 0 || Tq == 0) return GQA_OK;
  if (!q || !k || !v || !o) return GQA_ERR_NULL;
  if (cached && (!seq_lens || !dev_status)) return GQA_ERR_NULL;
  if (seg && !dev_status) return GQA_ERR_NULL;
  if (d > GQA_MAX_HEAD_DIM) return GQA_ERR_UNSUPPORTED;
  DeviceInfo di;
  if ((s = device_info(&di)) != GQA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float scale_log2 = scale * gqa::kLog2e;
  if (dtype == GQA_BF16 && gqa::pfs::supported(d) && aligned16(q) &&
      aligned16(k) && aligned16(v) && aligned16(o)) {
    // Heads of a group in pairs (one CTA per pair, each K/V tile fetched
    // once for both) when the group size is even; otherwise one head per
    // CTA, its key tiles split over two softmax warpgroups.  A plain prompt
    // whose paired grid leaves SMs idle and whose longest query tile walks
    // more than 4 KV tiles also takes one head per CTA: there the longest
    // CTA's chain sets the time, and a head's tile costs about half a pair's
    // (measured: B=4, Hq=8, Hkv=2, d=64, T=1024 causal 17.5 against 21.6 us;
    // with a 256-key window, 3 tiles, the pair stays faster, 13.6 against 17.3).
    if (gqa::pf2::supported(d, Hq, Hkv) &&
        !(prefill_prefers_split(B, Hq, Hkv, Tq, Tk, cached, seg != nullptr, window, di.sms)))
      return gqa::pf2::launch(q, k, v, o, seq_lens, seg, B, Hq, Hkv, Tq, Tk, cached,
                              d, window, scale_log2, di.sms, dev_status, st);
    // One head per item: plain prompts on the persistent kernel (one CTA
    // per SM walking its items), queries after a cache and packed segments
    // on one CTA per item.
    if (!cached && !seg)
      return gqa::pfp::launch(q, k, v, o, seq_lens, B, Hq, Hkv, Tq, d, window, scale_log2,
                              di.sms, dev_status, st);
    return gqa::pfs::launch(q, k, v, o, seq_lens, seg, B, Hq, Hkv, Tq, Tk, cached, d,
                            window, scale_log2, dev_status, st);
  }
  if (Hq > 65535 || B > 65535) return GQA_ERR_UNSUPPORTED;
  if (dtype == GQA_F32)
    return launch_simt_prefill<float>(q, k, v, o, seq_lens, seg, B, Hq, Hkv, Tq,
                                      Tk, cached, d, window, scale_log2,
                                      dev_status, st);
  return launch_simt_prefill<bf16>(q, k, v, o, seq_lens, seg, B, Hq, Hkv, Tq, Tk,
                                   cached, d, window, scale_log2, dev_status, st);
}

}  // namespace

extern "C" {

gqa_status gqa_prefill(gqa_dtype dtype, const void *q, const void *k,
                       const void *v, void *o, const int32_t *seq_lens, int B,
                       int Hq, int Hkv, int T, int d, int window, float scale,
                       int32_t *dev_status, gqa_stream_t stream) {
  return attend_impl(dtype, q, k, v, o, seq_lens, nullptr, B, Hq, Hkv, T, T, 0, d,
                     window, scale, dev_status, stream);
}

gqa_status gqa_prefill_packed(gqa_dtype dtype, const void *q, const void *k,
                              const void *v, void *o, const int32_t *seq_lens,
                              const int32_t *seg_start, int B, int Hq, int Hkv,
                              int T, int d, int window, float scale,
                              int32_t *dev_status, gqa_stream_t stream) {
  if (B > 0 && T > 0 && !seg_start) return GQA_ERR_NULL;
  return attend_impl(dtype, q, k, v, o, seq_lens, seg_start, B, Hq, Hkv, T, T, 0, d,
                     window, scale, dev_status, stream);
}

gqa_status gqa_decode_multi(gqa_dtype dtype, const void *q, const void *k_cache,
                            const void *v_cache, void *o, const int32_t *seq_lens,
                            int B, int Hq, int Hkv, int C, int d, int t_new,
                            int window, float scale, int32_t *dev_status,
                            gqa_stream_t stream) {
  if (C < 0 || t_new < 0) return GQA_ERR_SHAPE;
  if (t_new > C) return GQA_ERR_CAPACITY;
  return attend_impl(dtype, q, k_cache, v_cache, o, seq_lens, nullptr, B, Hq, Hkv,
                     t_new, C, 1, d, window, scale, dev_status, stream);
}

size_t gqa_decode_workspace_bytes(gqa_dtype dtype, int B, int Hq, int Hkv,
                                  int C, int d) {
  if (B < 0 || C < 0 || check_heads(Hq, Hkv, d) != GQA_OK) return 0;
  if (!splitk_supported(dtype, d)) return 0;
  DecLayout L;
  if (!decode_layout(B, Hq, Hkv, d, &L)) return 0;
  return L.total;
}

}  // extern "C"

namespace {

gqa_status append_impl(gqa_dtype dtype, void *k_cache, void *v_cache,
                       const void *k_new, const void *v_new, int32_t *seq_lens,
                       int B, int Hkv, int C, int d, int t_new, int ring,
                       int32_t *dev_status, gqa_stream_t stream);

// The fused append's extra operands (null for a plain decode).
struct AppendArgs {
  void *k_cache, *v_cache;
  const void *k_new, *v_new;
  int32_t *seq_lens;
  int ring;  // the cache is a rolling buffer of C slots
};

// clear_counters: zero the workspace's counter region on the stream before
// the split kernel (for a workspace the caller cannot clear itself).
gqa_status decode_impl(gqa_dtype dtype, const void *q, const void *k_cache,
                       const void *v_cache, void *o, const int32_t *seq_lens,
                       int B, int Hq, int Hkv, int C, int d, int window,
                       float scale, void *workspace, size_t workspace_bytes,
                       int32_t *dev_status, gqa_stream_t stream,
                       const AppendArgs *ap, bool clear_counters = false) {
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED;
  if (B < 0 || C < 0) return GQA_ERR_SHAPE;
  gqa_status s = check_heads(Hq, Hkv, d);
  if (s != GQA_OK) return s;
  if ((s = check_window(window)) != GQA_OK) return s;
  int64_t nq, nc;
  if (!elems(&nq, {B, Hq, d}) || !elems(&nc, {B, Hkv, C, d}) ||
      nc > INT64_MAX / 4)
    return GQA_ERR_OVERFLOW;
  if (B == 0) return GQA_OK;
  if (!q || !k_cache || !v_cache || !o || !seq_lens || !dev_status)
    return GQA_ERR_NULL;
  if (ap && (!ap->k_new || !ap->v_new)) return GQA_ERR_NULL;
  if (d > GQA_MAX_HEAD_DIM) return GQA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float scale_log2 = scale * gqa::kLog2e;
  const bool aligned = aligned16(q) && aligned16(k_cache) &&
                       aligned16(v_cache) && aligned16(o) &&
                       (!ap || (aligned16(ap->k_new) && aligned16(ap->v_new)));
  DeviceInfo di;
  // A fused append needs the lengths cached in shared memory.
  const bool lens_fit = !ap || B <= gqa::dec::kLensSmem;
  if (splitk_supported(dtype, d) && aligned && splitk_rows_ok(B, Hkv, C) &&
      lens_fit) {
    DecLayout L;
    if (!decode_layout(B, Hq, Hkv, d, &L)) return GQA_ERR_OVERFLOW;
    if (!workspace || workspace_bytes < L.total ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
      return GQA_ERR_WORKSPACE;
    const DecPlan pl = decode_plan(Hq, Hkv);
    if (pl.VL > 65535 || B > 65535) return GQA_ERR_UNSUPPORTED;
    if ((s = device_info(&di)) != GQA_OK) return s;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    gqa::dec::Params p;
    p.q = (const bf16 *)q;
    p.o = (bf16 *)o;
    p.seq_lens = seq_lens;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.C = C;
    p.window = window;
    p.scale_log2 = scale_log2;
    p.r = Hq / Hkv;
    p.nsub = pl.nsub;
    p.VL = pl.VL;
    p.min_rows = kDecodeMinRows;
    p.counters = reinterpret_cast<int *>(ws + L.counters);
    p.ml = reinterpret_cast<float2 *>(ws + L.ml);
    p.acc = reinterpret_cast<float *>(ws + L.acc);
    p.status = dev_status;
    p.k_new = ap ? (const bf16 *)ap->k_new : nullptr;
    p.v_new = ap ? (const bf16 *)ap->v_new : nullptr;
    p.k_cache = ap ? (bf16 *)ap->k_cache : nullptr;
    p.v_cache = ap ? (bf16 *)ap->v_cache : nullptr;
    p.lens_out = ap ? ap->seq_lens : nullptr;
    p.add = ap ? 1 : 0;
    p.lens_smem = B <= gqa::dec::kLensSmem ? 1 : 0;
    p.ring = (ap && ap->ring) ? 1 : 0;
    p.pad = kDecodeLanePadBytes / (4 * d);  // K and V rows of d bf16
    if (clear_counters &&
        cudaMemsetAsync(p.counters, 0, L.counter_bytes, st) != cudaSuccess) {
      cudaGetLastError();
      return GQA_ERR_CUDA;
    }
    return d == 64 ? dispatch_splitk_R<64>(pl.R, p, k_cache, v_cache, di.sms, st)
                   : dispatch_splitk_R<128>(pl.R, p, k_cache, v_cache, di.sms, st);
  }
  if (Hq > 65535 || B > 65535) return GQA_ERR_UNSUPPORTED;
  if ((s = device_info(&di)) != GQA_OK) return s;
  // CUDA-core path: the decode reads the candidate rows from the input, then
  // the append (same all-or-nothing length rule) writes them and advances
  // the lengths.
  const void *kn = ap ? ap->k_new : nullptr, *vn = ap ? ap->v_new : nullptr;
  const int add = ap ? 1 : 0, ring = (ap && ap->ring) ? 1 : 0;
  s = dtype == GQA_F32
          ? launch_simt_decode<float>(q, k_cache, v_cache, o, seq_lens, B, Hq,
                                      Hkv, C, d, window, scale_log2,
                                      dev_status, st, kn, vn, add, ring)
          : launch_simt_decode<bf16>(q, k_cache, v_cache, o, seq_lens, B, Hq,
                                     Hkv, C, d, window, scale_log2, dev_status,
                                     st, kn, vn, add, ring);
  if (s != GQA_OK || !ap) return s;
  return append_impl(dtype, ap->k_cache, ap->v_cache, ap->k_new, ap->v_new,
                     ap->seq_lens, B, Hkv, C, d, 1, ring, dev_status, stream);
}

}  // namespace

extern "C" {

gqa_status gqa_decode(gqa_dtype dtype, const void *q, const void *k_cache,
                      const void *v_cache, void *o, const int32_t *seq_lens,
                      int B, int Hq, int Hkv, int C, int d, int window,
                      float scale, void *workspace, size_t workspace_bytes,
                      int32_t *dev_status, gqa_stream_t stream) {
  return decode_impl(dtype, q, k_cache, v_cache, o, seq_lens, B, Hq, Hkv, C, d,
                     window, scale, workspace, workspace_bytes, dev_status,
                     stream, nullptr);
}

}  // extern "C"

namespace gqa {
namespace detail {
gqa_status decode_clearing_counters(gqa_dtype dtype, const void *q,
                                    const void *k_cache, const void *v_cache,
                                    void *o, const int32_t *seq_lens, int B,
                                    int Hq, int Hkv, int C, int d, int window,
                                    float scale, void *workspace,
                                    size_t workspace_bytes, int32_t *dev_status,
                                    gqa_stream_t stream) {
  return decode_impl(dtype, q, k_cache, v_cache, o, seq_lens, B, Hq, Hkv, C, d,
                     window, scale, workspace, workspace_bytes, dev_status,
                     stream, nullptr, true);
}
}  // namespace detail
}  // namespace gqa

extern "C" {

gqa_status gqa_decode_append(gqa_dtype dtype, const void *q, void *k_cache,
                             void *v_cache, const void *k_new,
                             const void *v_new, void *o, int32_t *seq_lens,
                             int B, int Hq, int Hkv, int C, int d, int window,
                             float scale, void *workspace,
                             size_t workspace_bytes, int32_t *dev_status,
                             gqa_stream_t stream) {
  const AppendArgs ap{k_cache, v_cache, k_new, v_new, seq_lens, 0};
  return decode_impl(dtype, q, k_cache, v_cache, o, seq_lens, B, Hq, Hkv, C, d,
                     window, scale, workspace, workspace_bytes, dev_status,
                     stream, &ap);
}

gqa_status gqa_ring_decode_append(gqa_dtype dtype, const void *q, void *k_ring,
                                  void *v_ring, const void *k_new,
                                  const void *v_new, void *o, int32_t *seq_lens,
                                  int B, int Hq, int Hkv, int W, int d, float scale,
                                  void *workspace, size_t workspace_bytes,
                                  int32_t *dev_status, gqa_stream_t stream) {
  if (W == 0) return GQA_ERR_SHAPE;
  const AppendArgs ap{k_ring, v_ring, k_new, v_new, seq_lens, 1};
  return decode_impl(dtype, q, k_ring, v_ring, o, seq_lens, B, Hq, Hkv, W, d,
                     GQA_NO_WINDOW, scale, workspace, workspace_bytes, dev_status,
                     stream, &ap);
}

}  // extern "C"

namespace {

// Append t_new rows per sequence into a fixed-capacity cache (ring = 0) or
// a rolling buffer of C slots (ring = 1, position p in slot p mod C).
gqa_status append_impl(gqa_dtype dtype, void *k_cache, void *v_cache,
                       const void *k_new, const void *v_new, int32_t *seq_lens,
                       int B, int Hkv, int C, int d, int t_new, int ring,
                       int32_t *dev_status, gqa_stream_t stream) {
  if (dtype != GQA_F32 && dtype != GQA_BF16) return GQA_ERR_UNSUPPORTED;
  if (B < 0 || C < 0 || t_new < 0) return GQA_ERR_SHAPE;
  if (Hkv <= 0 || d <= 0 || (ring && C == 0)) return GQA_ERR_SHAPE;
  const int esz = dtype == GQA_F32 ? 4 : 2;
  int64_t nc, nn;
  if (!elems(&nc, {B, Hkv, C, d, esz}) || !elems(&nn, {B, Hkv, t_new, d, esz}))
    return GQA_ERR_OVERFLOW;
  if (B == 0 || t_new == 0) return GQA_OK;
  if (!k_cache || !v_cache || !k_new || !v_new || !seq_lens || !dev_status)
    return GQA_ERR_NULL;
  if (!ring && t_new > C) return GQA_ERR_CAPACITY;
  DeviceInfo di;
  gqa_status s = device_info(&di);
  if (s != GQA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t row_bytes = (int64_t)d * esz;
  const bool vec = row_bytes % 16 == 0 && aligned16(k_cache) &&
                   aligned16(v_cache) && aligned16(k_new) && aligned16(v_new);
  const int vpr = vec ? (int)(row_bytes / 16) : d;
  const int64_t total = nn / (vec ? 16 : esz);
  const int64_t want = (total + 255) / 256;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)di.sms * 8));
  if (vec)
    gqa::append_copy_kernel<uint4><<<grid, 256, 0, st>>>(
        (uint4 *)k_cache, (uint4 *)v_cache, (const uint4 *)k_new,
        (const uint4 *)v_new, seq_lens, B, Hkv, C, t_new, vpr, ring, dev_status);
  else if (esz == 4)
    gqa::append_copy_kernel<uint32_t><<<grid, 256, 0, st>>>(
        (uint32_t *)k_cache, (uint32_t *)v_cache, (const uint32_t *)k_new,
        (const uint32_t *)v_new, seq_lens, B, Hkv, C, t_new, vpr, ring, dev_status);
  else
    gqa::append_copy_kernel<uint16_t><<<grid, 256, 0, st>>>(
        (uint16_t *)k_cache, (uint16_t *)v_cache, (const uint16_t *)k_new,
        (const uint16_t *)v_new, seq_lens, B, Hkv, C, t_new, vpr, ring, dev_status);
  if (launch_status() != GQA_OK) return GQA_ERR_CUDA;
  gqa::append_commit_kernel<<<1, 256, 0, st>>>(seq_lens, B, C, t_new, ring);
  return launch_status();
}

}  // namespace

extern "C" {

gqa_status gqa_cache_append(gqa_dtype dtype, void *k_cache, void *v_cache,
                            const void *k_new, const void *v_new,
                            int32_t *seq_lens, int B, int Hkv, int C, int d,
                            int t_new, int32_t *dev_status,
                            gqa_stream_t stream) {
  return append_impl(dtype, k_cache, v_cache, k_new, v_new, seq_lens, B, Hkv, C, d,
                     t_new, 0, dev_status, stream);
}

gqa_status gqa_ring_append(gqa_dtype dtype, void *k_ring, void *v_ring,
                           const void *k_new, const void *v_new, int32_t *seq_lens,
                           int B, int Hkv, int W, int d, int t_new,
                           int32_t *dev_status, gqa_stream_t stream) {
  return append_impl(dtype, k_ring, v_ring, k_new, v_new, seq_lens, B, Hkv, W, d,
                     t_new, 1, dev_status, stream);
}

}  // extern "C"
