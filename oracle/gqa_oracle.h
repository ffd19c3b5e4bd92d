/*
 * gqa_oracle.h -- plain fp64 CPU oracle for grouped-query attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link
 * or call this code: only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark use it.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * Sources (page title, section):
 *   [P1] "Share key/value heads and make context explicit"
 *        (intale.github.io, Practical LLM in Rust, chapter 18)
 *   [P3] "GQA, FlashAttention and the KV cache" (tokenwerk)
 *   [P4] "How do you implement grouped query attention (GQA)?" (clozo.ai)
 *
 * Layouts are contiguous row-major:
 *   q [B,Hq,T,d]  k,v [B,Hkv,T,d]  o [B,Hq,T,d]        (prefill)
 *   q [B,Hq,d]    k_cache,v_cache [B,Hkv,C,d]  o [B,Hq,d]  (decode)
 * window < 0 means "no local window"; window == 0 is refused.
 * Return codes: 0 ok, 1 bad argument (null, shape, divisibility, window),
 * 2 capacity exceeded / bad length.
 */
#ifndef GQA_ORACLE_H
#define GQA_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* [P1] "Give each query head an explicit shared KV head": g(h) = floor(h/r),
 * r = Hq/Hkv; -1 when the map does not exist. */
long oracle_kv_head_for_query(long h, long Hq, long Hkv);

/* [P1] "Intersect the window with the context already permitted":
 * max(seg_start, t -sat- (w-1)); -1 when w == 0 or seg_start > t.
 * w < 0 means no window (the start is seg_start). */
long oracle_window_start(long t, long seg_start, long w);

/* Full (prefill) pass.  seq_lens may be NULL (every row active); rows t with
 * t >= n_b get zero output.  probs (may be NULL) receives the attention
 * probabilities [B,Hq,T,T], zero outside the permitted set. */
int oracle_prefill(const double *q, const double *k, const double *v,
                   double *o, double *probs, const long *seq_lens, long B,
                   long Hq, long Hkv, long T, long d, long window,
                   double scale);

/* Same, with packed segments: seg_start [B,T] gives s_{b,t}, the first key
 * cell of query t's segment ([P1] "Intersect the window ..."). */
int oracle_prefill_packed(const double *q, const double *k, const double *v,
                          double *o, double *probs, const long *seq_lens,
                          const long *seg_start, long B, long Hq, long Hkv,
                          long T, long d, long window, double scale);

/* Single-token decode: seq_lens[b] = n_b counts the cached cells including
 * the current token (already appended); the query sits at cell n_b - 1. */
int oracle_decode(const double *q, const double *k_cache,
                  const double *v_cache, double *o, const long *seq_lens,
                  long B, long Hq, long Hkv, long C, long d, long window,
                  double scale);

/* Multi-token decode / chunked prefill against the cache: q [B,Hq,t_new,d];
 * query i of sequence b sits at cell n_b - t_new + i ([P4] mask tril(s-t)). */
int oracle_decode_multi(const double *q, const double *k_cache,
                        const double *v_cache, double *o, const long *seq_lens,
                        long B, long Hq, long Hkv, long C, long d, long t_new,
                        long window, double scale);

/* Append k_new/v_new [B,Hkv,t_new,d] at cells [len_b, len_b+t_new) of the
 * [B,Hkv,C,d] caches and advance seq_lens.  All-or-nothing: if any sequence
 * would exceed C (or has a negative length) nothing is written. */
int oracle_cache_append(double *k_cache, double *v_cache, const double *k_new,
                        const double *v_new, long *seq_lens, long B, long Hkv,
                        long C, long d, long t_new);

/* Rolling-buffer (ring) cache of W slots per lane ([P1] "Relate shared heads
 * to local context": a rolling buffer that overwrites old KV entries; the
 * chapter does not implement it).  Reading: position p lives in slot
 * p mod W.  Append writes positions [len_b, len_b + t_new) (only the last W
 * of them survive) and advances seq_lens; refused (nothing written) if a
 * length is negative or would overflow. */
int oracle_ring_append(double *k_ring, double *v_ring, const double *k_new,
                       const double *v_new, long *seq_lens, long B, long Hkv,
                       long W, long d, long t_new);

/* Decode against a ring: n_b = seq_lens[b] positions so far (the current
 * token included); the query at position n_b - 1 reads positions
 * [max(0, n_b - W), n_b) from their slots, in position order (a window of W
 * cells over the positions). */
int oracle_ring_decode(const double *q, const double *k_ring,
                       const double *v_ring, double *o, const long *seq_lens,
                       long B, long Hq, long Hkv, long W, long d, double scale);

/* [P3] "Computing the cache requirement": 2*L*B*T*Hkv*d*e, 0 on overflow. */
uint64_t oracle_cache_bytes(uint64_t L, uint64_t B, uint64_t T, uint64_t Hkv,
                            uint64_t d, uint64_t e);

/* Thread count used by the (b, h) loops; returns the count in effect. */
int oracle_set_threads(int n);

#ifdef __cplusplus
}
#endif
#endif
