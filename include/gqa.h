/*
 * gqa.h -- C ABI of the B200 (sm_100a) grouped-query attention library.
 *
 * Grouped-query attention (GQA): Hq query heads share Hkv key/value heads in
 * groups of r = Hq/Hkv adjacent heads; query head h reads KV head
 * g(h) = floor(h/r) in place (no repeat-interleave copy is made).  Each query
 * row normalises softmax(scale * q.k) over its permitted key cells only and
 * mixes the shared value rows.
 *
 * Sources (page title, section):
 *   [P1] "Share key/value heads and make context explicit" (practical LLM in
 *        Rust, ch. 18): "Give each query head an explicit shared KV head"
 *        (head map, score, normalisation, value mix), "Intersect the window
 *        with the context already permitted" (window w counts the current
 *        cell and at most w-1 earlier cells; zero window refused; inactive
 *        padded queries have zero output), "Extend the existing full and
 *        cached attention paths" (decode reads the shared cache lane over
 *        the eligible suffix; the cache refuses to exceed capacity and a
 *        failed operation never partly advances it), "Count learned weights
 *        and retained cache data separately" (physical cache [B,Hkv,C,d]).
 *   [P3] "GQA, FlashAttention and the KV cache": "Computing the cache
 *        requirement" (M_KV = 2 L B T Hkv d e), "The important mask bug with
 *        a cache" (a single new token sees the whole cached past).
 *   [P4] "How do you implement grouped query attention (GQA)?": Step 1
 *        (shapes [B,H,T,d] and [B,G,T,d]), Step 2 (head map), the
 *        implementation's tril(s - t) mask offset.
 *
 * Conventions for every entry point:
 *   - All tensors are contiguous row-major device buffers owned by the
 *     caller.  The library allocates no device memory and keeps no state.
 *   - Element type: GQA_F32 (float) or GQA_BF16 (bfloat16 storage, fp32
 *     arithmetic).  All tensors of one call share the type.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  Host-detectable errors are returned
 *     before anything is enqueued and leave every buffer untouched.
 *   - `window` is GQA_NO_WINDOW (-1) for plain causal attention, else a
 *     positive cell count that includes the current cell.  0 and values
 *     below -1 return GQA_ERR_WINDOW.
 *   - Device-resident lengths are validated on the device: an invalid
 *     length sets *dev_status (int32, device memory) to a gqa_status code
 *     (the first error wins; the library never clears it, so zero it before
 *     the calls you want to check).  Outputs of a failed call hold zeros
 *     and a failed append writes nothing.  No call traps.
 */
#ifndef GQA_H
#define GQA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *gqa_stream_t; /* same type as cudaStream_t */

typedef enum { GQA_F32 = 0, GQA_BF16 = 1 } gqa_dtype;

typedef enum {
  GQA_OK = 0,
  GQA_ERR_NULL = 1,        /* a required pointer is NULL */
  GQA_ERR_SHAPE = 2,       /* a size is negative, or Hq/Hkv/d is not positive */
  GQA_ERR_GROUPS = 3,      /* Hq is not a multiple of Hkv */
  GQA_ERR_WINDOW = 4,      /* window == 0 or window < -1 */
  GQA_ERR_CAPACITY = 5,    /* a length is negative or exceeds T / C */
  GQA_ERR_OVERFLOW = 6,    /* an element count overflows int64 / size_t */
  GQA_ERR_UNSUPPORTED = 7, /* d, dtype or alignment outside the compiled kernels */
  GQA_ERR_WORKSPACE = 8,   /* workspace NULL or smaller than required */
  GQA_ERR_CUDA = 9,        /* a CUDA runtime call or launch failed */
  GQA_ERR_DEVICE = 10,     /* the current device is not sm_100 */
  GQA_ERR_TIMEOUT = 11,    /* a kernel's bounded internal wait ran out (set
                              in *dev_status only) */
  GQA_ERR_SEGMENT = 12     /* a packed segment start s_{b,t} lies outside
                              [0, t] (set in *dev_status only) */
} gqa_status;

#define GQA_NO_WINDOW (-1)

/* Largest head width the kernels accept (fp32 and the generic bf16 path). */
#define GQA_MAX_HEAD_DIM 256

/*
 * gqa_prefill -- full causal (optionally windowed) pass over a prompt.
 * [P1] "Give each query head an explicit shared KV head" and "Intersect the
 * window ...": for batch row b, query head h and active cell t < n_b, the
 * permitted keys are j in [max(0, t-(w-1)), t] of KV head g(h); rows with
 * t >= n_b are written as zeros.
 *
 *   q        [B,Hq,T,d]   queries (already position-rotated)
 *   k, v     [B,Hkv,T,d]  keys (rotated) and values of the same cells
 *   o        [B,Hq,T,d]   output; the head concatenation [B,T,Hq*d] of the
 *                         pages is its transpose (the output projection W_o
 *                         is not applied)
 *   seq_lens device int32 [B] giving n_b in [0, T], or NULL for n_b = T
 *   scale    score multiplier (1/sqrt(d) in the pages)
 *   dev_status device int32, may be NULL when seq_lens is NULL
 * bf16 with d in {64, 128} runs on the tcgen05 tensor cores; other d up to
 * GQA_MAX_HEAD_DIM and fp32 run on CUDA cores with fp32 FMAs.
 */
gqa_status gqa_prefill(gqa_dtype dtype, const void *q, const void *k,
                       const void *v, void *o, const int32_t *seq_lens,
                       int B, int Hq, int Hkv, int T, int d, int window,
                       float scale, int32_t *dev_status, gqa_stream_t stream);

/*
 * gqa_prefill_packed -- gqa_prefill over packed sequences: several
 * documents share one row of the batch, and a query sees only its own
 * document.  [P1] "Intersect the window with the context already
 * permitted": the first permitted key of cell t is the later of its
 * segment start s_{b,t} and the window start t - (w-1) (saturating), so
 * cell t reads keys [max(s_{b,t}, t-(w-1)), t].
 *
 *   seg_start device int32 [B,T]: s_{b,t}, the first cell of t's segment
 *            (required; only cells t < n_b are read)
 *   everything else as for gqa_prefill.
 * A start outside [0, t] gives that query row no keys: its output is zero
 * and *dev_status is set to GQA_ERR_SEGMENT (dev_status is required).
 */
gqa_status gqa_prefill_packed(gqa_dtype dtype, const void *q, const void *k,
                              const void *v, void *o, const int32_t *seq_lens,
                              const int32_t *seg_start, int B, int Hq, int Hkv,
                              int T, int d, int window, float scale,
                              int32_t *dev_status, gqa_stream_t stream);

/*
 * gqa_decode -- one new query token per sequence against the KV cache.
 * [P1] "Extend the existing full and cached attention paths" and [P3] "The
 * important mask bug with a cache": seq_lens[b] = n_b counts the cached
 * cells INCLUDING the current token (append it first with
 * gqa_cache_append); the query sits at cell n_b - 1 and reads cells
 * [max(0, n_b - w), n_b) of its shared lane.  n_b = 0 gives a zero output.
 *
 *   q        [B,Hq,d]      the new token's queries
 *   k_cache, v_cache [B,Hkv,C,d]  caches of capacity C
 *   o        [B,Hq,d]      output
 *   seq_lens device int32 [B], each in [0, C]
 *   workspace / workspace_bytes  device scratch of at least
 *            gqa_decode_workspace_bytes(...) bytes, 256-byte aligned.  Fill
 *            it with zeros once before its first use; every call that
 *            completes leaves it ready for the next call of any shape, so it
 *            needs no clearing between calls.  After a call that set
 *            GQA_ERR_TIMEOUT, zero it again.  Calls sharing a workspace must
 *            be ordered (one stream, or events).
 *   dev_status device int32 (required)
 * bf16 with d in {64, 128}: split-K flash-decode (TMA-fed shared memory
 * ring, group heads stacked as tensor-core tile rows); the last CTA to
 * finish a lane merges that lane's partials in a fixed order, so the same
 * inputs give the same bits whichever CTA that is.  That kernel is launched
 * as a programmatic dependent of the previous kernel on the stream: its set
 * up overlaps that kernel's tail, and it touches memory only after that
 * kernel has completed.  Other d and fp32 run on CUDA cores.
 */
gqa_status gqa_decode(gqa_dtype dtype, const void *q, const void *k_cache,
                      const void *v_cache, void *o, const int32_t *seq_lens,
                      int B, int Hq, int Hkv, int C, int d, int window,
                      float scale, void *workspace, size_t workspace_bytes,
                      int32_t *dev_status, gqa_stream_t stream);

/* Workspace gqa_decode needs for these sizes (0 means none); 0 is also
 * returned for invalid sizes, which gqa_decode then rejects. */
size_t gqa_decode_workspace_bytes(gqa_dtype dtype, int B, int Hq, int Hkv,
                                  int C, int d);

/*
 * gqa_decode_append -- the decode step with its cache append fused in.
 * [P1] "Extend the existing full and cached attention paths": the step's
 * new key/value row is read from the input as a candidate and takes part in
 * the scores before it is committed to the cache; the append refuses to
 * exceed capacity and never partly advances.
 *
 * Same result as gqa_cache_append(t_new = 1) followed by gqa_decode, in one
 * kernel for bf16 with d in {64, 128} (the candidate row never makes a round
 * trip through the cache):
 *   seq_lens device int32 [B], in/out: len_b = cells cached BEFORE the step,
 *            each in [0, C-1]; the query sits at cell len_b and reads cells
 *            [max(0, len_b + 1 - w), len_b + 1), the last one from k_new /
 *            v_new.  After the call len_b has grown by one.
 *   k_new, v_new [B,Hkv,1,d]  the step's key (rotated) and value rows,
 *            written to cell len_b of k_cache / v_cache
 *   workspace  gqa_decode_workspace_bytes(...) bytes, as for gqa_decode
 *   everything else as for gqa_decode.
 * If any len_b lies outside [0, C-1], *dev_status is set to
 * GQA_ERR_CAPACITY, the output is zero, and neither the caches nor the
 * lengths change.  Other d and fp32 run a CUDA-core decode that reads the
 * candidate rows from k_new / v_new, followed by gqa_cache_append.
 */
gqa_status gqa_decode_append(gqa_dtype dtype, const void *q, void *k_cache,
                             void *v_cache, const void *k_new,
                             const void *v_new, void *o, int32_t *seq_lens,
                             int B, int Hq, int Hkv, int C, int d, int window,
                             float scale, void *workspace,
                             size_t workspace_bytes, int32_t *dev_status,
                             gqa_stream_t stream);

/*
 * gqa_decode_multi -- t_new new query rows per sequence against the cache
 * (multi-token decode, chunked prefill).  [P4] the implementation's
 * tril(s - t) mask offset and [P3] "The important mask bug with a cache":
 * the new rows are the LAST t_new of the n_b cached cells (append them
 * first with gqa_cache_append), so query row i sits at cell
 * p_i = n_b - t_new + i and reads cells [max(0, p_i - (w-1)), p_i] of its
 * shared lane ([P1] "Intersect the window with the context already
 * permitted").  t_new = 1 is gqa_decode; t_new = n_b is a causal prefill of
 * the whole cache.
 *
 *   q        [B,Hq,t_new,d]  the new rows' queries (already rotated)
 *   k_cache, v_cache [B,Hkv,C,d]  caches of capacity C
 *   o        [B,Hq,t_new,d]  output
 *   seq_lens device int32 [B], n_b in [t_new, C] (required)
 *   dev_status device int32 (required)
 * Cells past n_b are never used, whatever they hold.  A length outside
 * [t_new, C] sets *dev_status to GQA_ERR_CAPACITY and writes that
 * sequence's output as zeros.  t_new > C returns GQA_ERR_CAPACITY before
 * anything is enqueued.  bf16 with d in {64, 128} runs the tcgen05 prefill
 * kernels with the query rows offset by n_b - t_new; other d and fp32 run
 * on CUDA cores.
 */
gqa_status gqa_decode_multi(gqa_dtype dtype, const void *q, const void *k_cache,
                            const void *v_cache, void *o, const int32_t *seq_lens,
                            int B, int Hq, int Hkv, int C, int d, int t_new,
                            int window, float scale, int32_t *dev_status,
                            gqa_stream_t stream);

/*
 * Rolling-buffer (ring) cache.  [P1] "Relate shared heads to local context"
 * describes Mistral's rolling buffer that overwrites old KV entries (the
 * chapter itself keeps every row and does not build one).  Here a ring of
 * W slots per KV lane holds position p in slot p mod W, so it always holds
 * the last W positions: attending over it is the window-W decode of
 * [P1] "Intersect the window ..." with W cells of storage instead of the
 * whole prefix.  seq_lens counts positions so far (not capped at W).
 *
 * gqa_ring_append -- write positions [len_b, len_b + t_new) (k_new, v_new
 *   [B,Hkv,t_new,d]; only the last W rows survive) into k_ring/v_ring
 *   [B,Hkv,W,d] and advance seq_lens.  A negative length, or one that would
 *   pass INT32_MAX, sets *dev_status to GQA_ERR_CAPACITY and nothing moves.
 */
gqa_status gqa_ring_append(gqa_dtype dtype, void *k_ring, void *v_ring,
                           const void *k_new, const void *v_new, int32_t *seq_lens,
                           int B, int Hkv, int W, int d, int t_new,
                           int32_t *dev_status, gqa_stream_t stream);

/*
 * gqa_ring_decode_append -- the decode step against a ring, with the step's
 * row appended in the same call (as gqa_decode_append): seq_lens[b] =
 * positions before the step; the query at position len_b reads positions
 * [max(0, len_b + 1 - W), len_b] (every occupied slot, the new one read
 * from k_new / v_new [B,Hkv,1,d] and written to slot len_b mod W); then
 * len_b grows by one.  Workspace: gqa_decode_workspace_bytes(dtype, B, Hq,
 * Hkv, W, d).  A negative length sets GQA_ERR_CAPACITY, zeroes the output
 * and changes nothing.  bf16 with d in {64, 128} runs the split-K kernel;
 * other d and fp32 run on CUDA cores.
 */
gqa_status gqa_ring_decode_append(gqa_dtype dtype, const void *q, void *k_ring,
                                  void *v_ring, const void *k_new,
                                  const void *v_new, void *o, int32_t *seq_lens,
                                  int B, int Hq, int Hkv, int W, int d, float scale,
                                  void *workspace, size_t workspace_bytes,
                                  int32_t *dev_status, gqa_stream_t stream);

/* Size of the fixed device array gqa_decode_noalloc uses as its workspace. */
#define GQA_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

/*
 * gqa_decode_noalloc -- gqa_decode for callers that cannot allocate device
 * memory.  The pages have no counterpart; this is a library convenience.
 *
 * Some callers cannot call cudaMalloc: a host application that passes this
 * library pointers from its own fixed memory pool and forbids any other
 * allocation, a latency-critical loop that cannot accept cudaMalloc's
 * implicit device synchronisation, or a foreign-language caller that only
 * receives device pointers.  This entry point takes the same arguments as
 * gqa_decode minus the workspace and runs the same kernels, using as
 * workspace a fixed GQA_NOALLOC_SCRATCH_BYTES array in device memory that
 * the library defines (every GPU that loads the library holds it until the
 * process exits).  It allocates nothing.
 *
 *   - Sizes whose workspace (gqa_decode_workspace_bytes) exceeds
 *     GQA_NOALLOC_SCRATCH_BYTES return GQA_ERR_WORKSPACE; nothing is
 *     enqueued.  All other arguments and errors are those of gqa_decode.
 *   - All calls on a device share the one array, which keeps the last
 *     call's contents.  Each call first clears the part that must start at
 *     zero (its few-KB counter region, one cudaMemsetAsync, no allocation);
 *     the rest needs no initial value.  Calls whose kernels may overlap on
 *     the GPU (unordered streams) race on it: order them on one stream or
 *     with events.
 *   - The first call on each device looks up the array's address (with that
 *     device current) and caches it for the device's current context; make
 *     that first call before any stream capture begins.  After a
 *     cudaDeviceReset the next call looks it up again (also outside any
 *     capture).  A failed lookup returns GQA_ERR_CUDA.
 */
gqa_status gqa_decode_noalloc(gqa_dtype dtype, const void *q,
                              const void *k_cache, const void *v_cache,
                              void *o, const int32_t *seq_lens, int B, int Hq,
                              int Hkv, int C, int d, int window, float scale,
                              int32_t *dev_status, gqa_stream_t stream);

/*
 * gqa_cache_append -- write t_new new cells per sequence and advance the
 * lengths.  [P1] "Count learned weights and retained cache data separately"
 * and "Extend the existing full and cached attention paths": the cache
 * keeps every row up to its fixed capacity (no eviction), refuses to exceed
 * it, and never partly advances.
 *
 *   k_cache, v_cache [B,Hkv,C,d]  written at cells [len_b, len_b + t_new)
 *   k_new, v_new     [B,Hkv,t_new,d]
 *   seq_lens         device int32 [B], in/out: len_b += t_new on success
 *   dev_status       device int32 (required)
 * All-or-nothing: if any len_b < 0 or len_b + t_new > C, *dev_status is set
 * to GQA_ERR_CAPACITY and neither the caches nor the lengths change.
 */
gqa_status gqa_cache_append(gqa_dtype dtype, void *k_cache, void *v_cache,
                            const void *k_new, const void *v_new,
                            int32_t *seq_lens, int B, int Hkv, int C, int d,
                            int t_new, int32_t *dev_status,
                            gqa_stream_t stream);

/* [P3] "Computing the cache requirement": 2*L*B*T*Hkv*d*e bytes for L
 * layers; 0 if any argument is negative or the product overflows uint64. */
uint64_t gqa_cache_bytes(int64_t L, int64_t B, int64_t T, int64_t Hkv,
                         int64_t d, int64_t elem_bytes);

/* [P1] kv_head_for_query: g(h) = floor(h / (Hq/Hkv)); -1 when Hq or Hkv is
 * not positive, Hq % Hkv != 0, or h is outside [0, Hq). */
int gqa_kv_head_for_query(int h, int Hq, int Hkv);

/* Which tensor-core kernel gqa_prefill runs for a bf16 prompt (no packed
 * segments, 16-byte-aligned tensors) of B x Hq query heads over Hkv KV heads,
 * T cells, head width d and window (GQA_NO_WINDOW or w >= 1) on a device with
 * `sms` SMs:
 *   1  two query heads of one KV group per CTA (even group size), unless:
 *   2  one query head per work item, its keys split over two softmax
 *      warpgroups, on a persistent grid of one CTA per SM (odd group size;
 *      or a prompt whose paired grid has fewer CTAs than `sms` and whose
 *      last query tile walks more than 4 KV tiles);
 *   0  the CUDA-core kernel (d other than 64 or 128);
 *  -1  invalid arguments (non-positive sizes, Hq % Hkv != 0, bad window).
 * Host-only: reads nothing on the device and launches nothing. */
int gqa_prefill_kernel(int B, int Hq, int Hkv, int T, int d, int window, int sms);

/* [P1] causal_window_start with segment start 0: the first permitted key
 * cell of query cell t, max(0, t - (w-1)) (0 for GQA_NO_WINDOW); -1 for an
 * invalid window or t < 0. */
int gqa_window_start(int t, int window);

/*
 * gqa_selftest_wait_timeout -- exercises the kernels' bounded waits, for
 * tests of the failure handling.  [P1] "Extend the existing full and cached
 * attention paths": a failed operation reports an error and leaves nothing
 * half done; here that means a kernel whose internal wait (an mbarrier
 * phase that a copy, an MMA or other warps should complete) runs out of
 * time records GQA_ERR_TIMEOUT and returns instead of hanging the GPU.
 *
 * Launches one CTA of two warps that run the library's two wait routines
 * (suspending and polling) on mbarriers that no thread arrives on, each
 * giving up after limit_us microseconds; no copy or MMA is in flight.
 *   limit_us    1 .. 2,000,000 (else GQA_ERR_SHAPE)
 *   arrive      nonzero: one thread completes both barriers first, so both
 *               waits succeed (the control case)
 *   dev_status  device int32: set to GQA_ERR_TIMEOUT when a wait gave up
 *   gave_up     device int32 [2]: element w is incremented when warp w's
 *               wait gave up (warp 0 suspending, warp 1 polling)
 * Asynchronous on `stream`; the kernel runs for about limit_us when the
 * waits run out.  Returns GQA_ERR_NULL for a NULL pointer and
 * GQA_ERR_DEVICE off sm_100.
 */
gqa_status gqa_selftest_wait_timeout(int64_t limit_us, int arrive,
                                     int32_t *dev_status, int32_t *gave_up,
                                     gqa_stream_t stream);

/* Static English text for a status code (never NULL). */
const char *gqa_status_string(gqa_status status);

/* Library version, e.g. "0.1.0". */
const char *gqa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GQA_H */
