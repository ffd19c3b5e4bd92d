/*
 * gqa_oracle.c -- plain, slow, fp64 CPU oracle for grouped-query attention.
 *
 * TEST INFRASTRUCTURE ONLY (see gqa_oracle.h).  Every step is written out as
 * the pages define it: no tiling, no fusion, no online softmax.  Scores are
 * formed in ascending key order, normalised by the max-subtracted two-pass
 * softmax, then mixed with the shared value rows.
 *
 * Sources (page title, section):
 *   [P1] "Share key/value heads and make context explicit":
 *        "Give each query head an explicit shared KV head" (head map, score,
 *        normalisation over the permitted set, value mix),
 *        "Intersect the window with the context already permitted"
 *        (window rule, inactive padded queries),
 *        "Extend the existing full and cached attention paths" (decode loop
 *        over start..prefix with scale 1/sqrt(head width), transactional
 *        cache that refuses to exceed capacity),
 *        "Count learned weights and retained cache data separately" (cache
 *        payload 2*L*B*C*Hkv*d*e).
 *   [P3] "GQA, FlashAttention and the KV cache": "Computing the cache
 *        requirement", "The important mask bug with a cache".
 *   [P4] "How do you implement grouped query attention (GQA)?": Step 2 (head
 *        map by integer division), the implementation's tril(s - t) mask.
 */
#include "gqa_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int g_threads = 1;

int oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n <= 0) n = omp_get_num_procs();
  g_threads = n;
#else
  (void)n;
  g_threads = 1;
#endif
  return g_threads;
}

/* [P1] head map: query head h reads KV head floor(h / (Hq/Hkv)). */
long oracle_kv_head_for_query(long h, long Hq, long Hkv) {
  if (Hkv <= 0 || Hq <= 0 || Hq % Hkv != 0) return -1;
  if (h < 0 || h >= Hq) return -1;
  return h / (Hq / Hkv);
}

/* [P1] window start: the window counts the current cell and at most w-1
 * earlier cells; intersect with the segment start using a saturating
 * subtraction.  w < 0 stands for "no window". */
long oracle_window_start(long t, long seg_start, long w) {
  if (w == 0 || seg_start > t || seg_start < 0 || t < 0) return -1;
  if (w < 0) return seg_start;
  long back = w - 1;
  long sat = t > back ? t - back : 0;
  return seg_start > sat ? seg_start : sat;
}

/* One query row against the permitted keys [lo, hi] of one shared K/V lane.
 * s_j = scale * q . k_j ; m = max s_j ; e_j = exp(s_j - m) ; l = sum e_j ;
 * out = sum_j (e_j / l) v_j.  scratch holds at least hi-lo+1 doubles. */
static void attend_row(const double *qrow, const double *klane,
                       const double *vlane, long lo, long hi, long d,
                       double scale, double *out, double *prow,
                       double *scratch) {
  long n = hi - lo + 1;
  double m = -INFINITY;
  for (long j = lo; j <= hi; ++j) {
    double dot = 0.0;
    for (long f = 0; f < d; ++f) dot += qrow[f] * klane[j * d + f];
    double s = scale * dot;
    scratch[j - lo] = s;
    if (s > m) m = s;
  }
  double l = 0.0;
  for (long i = 0; i < n; ++i) {
    scratch[i] = exp(scratch[i] - m);
    l += scratch[i];
  }
  for (long f = 0; f < d; ++f) out[f] = 0.0;
  for (long j = lo; j <= hi; ++j) {
    double p = scratch[j - lo] / l;
    if (prow) prow[j] = p;
    for (long f = 0; f < d; ++f) out[f] += p * vlane[j * d + f];
  }
}

static int check_heads(long Hq, long Hkv, long d) {
  if (Hq <= 0 || Hkv <= 0 || d <= 0) return 1;
  if (Hq % Hkv != 0) return 1;
  return 0;
}

int oracle_prefill_packed(const double *q, const double *k, const double *v,
                          double *o, double *probs, const long *seq_lens,
                          const long *seg_start, long B, long Hq, long Hkv,
                          long T, long d, long window, double scale) {
  if (B < 0 || T < 0 || check_heads(Hq, Hkv, d)) return 1;
  if (window == 0 || window < -1) return 1;
  if (B == 0 || T == 0) return 0;
  if (!q || !k || !v || !o) return 1;
  for (long b = 0; b < B; ++b) {
    long n = seq_lens ? seq_lens[b] : T;
    if (n < 0 || n > T) return 2;
    if (seg_start)
      for (long t = 0; t < n; ++t) {
        long s0 = seg_start[b * T + t];
        if (s0 < 0 || s0 > t) return 1;
      }
  }
  long r = Hq / Hkv;
  int bad = 0;
#pragma omp parallel num_threads(g_threads) reduction(| : bad)
  {
    double *scratch = (double *)malloc(sizeof(double) * (size_t)T);
    if (!scratch) bad = 1;
#pragma omp for collapse(2) schedule(dynamic)
    for (long b = 0; b < B; ++b) {
      for (long h = 0; h < Hq; ++h) {
        if (!scratch) continue;
        long n = seq_lens ? seq_lens[b] : T;
        long g = h / r;
        const double *klane = k + (b * Hkv + g) * T * d;
        const double *vlane = v + (b * Hkv + g) * T * d;
        for (long t = 0; t < T; ++t) {
          double *orow = o + ((b * Hq + h) * T + t) * d;
          double *prow = probs ? probs + ((b * Hq + h) * T + t) * T : NULL;
          if (prow) memset(prow, 0, sizeof(double) * (size_t)T);
          if (t >= n) { /* inactive padded query: zero output */
            memset(orow, 0, sizeof(double) * (size_t)d);
            continue;
          }
          long s0 = seg_start ? seg_start[b * T + t] : 0;
          long lo = oracle_window_start(t, s0, window);
          attend_row(q + ((b * Hq + h) * T + t) * d, klane, vlane, lo, t, d,
                     scale, orow, prow, scratch);
        }
      }
    }
    free(scratch);
  }
  return bad ? 1 : 0;
}

int oracle_prefill(const double *q, const double *k, const double *v,
                   double *o, double *probs, const long *seq_lens, long B,
                   long Hq, long Hkv, long T, long d, long window,
                   double scale) {
  return oracle_prefill_packed(q, k, v, o, probs, seq_lens, NULL, B, Hq, Hkv,
                               T, d, window, scale);
}

int oracle_decode_multi(const double *q, const double *k_cache,
                        const double *v_cache, double *o, const long *seq_lens,
                        long B, long Hq, long Hkv, long C, long d, long t_new,
                        long window, double scale) {
  if (B < 0 || C < 0 || t_new < 0 || check_heads(Hq, Hkv, d)) return 1;
  if (window == 0 || window < -1) return 1;
  if (B == 0 || t_new == 0) return 0;
  if (!q || !k_cache || !v_cache || !o || !seq_lens) return 1;
  for (long b = 0; b < B; ++b)
    if (seq_lens[b] < 0 || seq_lens[b] > C) return 2;
  long r = Hq / Hkv;
  int bad = 0;
#pragma omp parallel num_threads(g_threads) reduction(| : bad)
  {
    double *scratch = (double *)malloc(sizeof(double) * (size_t)(C + 1));
    if (!scratch) bad = 1;
#pragma omp for collapse(2) schedule(dynamic)
    for (long b = 0; b < B; ++b) {
      for (long h = 0; h < Hq; ++h) {
        if (!scratch) continue;
        long n = seq_lens[b];
        long g = h / r;
        const double *klane = k_cache + (b * Hkv + g) * C * d;
        const double *vlane = v_cache + (b * Hkv + g) * C * d;
        for (long i = 0; i < t_new; ++i) {
          /* [P4] query i sits at absolute cell s - t + i and sees every key
           * up to it; [P3] a single new token sees the whole cache. */
          long pos = n - t_new + i;
          double *orow = o + ((b * Hq + h) * t_new + i) * d;
          if (pos < 0) {
            memset(orow, 0, sizeof(double) * (size_t)d);
            continue;
          }
          long lo = oracle_window_start(pos, 0, window);
          attend_row(q + ((b * Hq + h) * t_new + i) * d, klane, vlane, lo,
                     pos, d, scale, orow, NULL, scratch);
        }
      }
    }
    free(scratch);
  }
  return bad ? 1 : 0;
}

int oracle_decode(const double *q, const double *k_cache,
                  const double *v_cache, double *o, const long *seq_lens,
                  long B, long Hq, long Hkv, long C, long d, long window,
                  double scale) {
  return oracle_decode_multi(q, k_cache, v_cache, o, seq_lens, B, Hq, Hkv, C,
                             d, 1, window, scale);
}

/* [P1] the cache keeps every row up to its fixed capacity, refuses to exceed
 * it, and a failed operation never partly advances it. */
int oracle_cache_append(double *k_cache, double *v_cache, const double *k_new,
                        const double *v_new, long *seq_lens, long B, long Hkv,
                        long C, long d, long t_new) {
  if (B < 0 || C < 0 || t_new < 0 || Hkv <= 0 || d <= 0) return 1;
  if (B == 0 || t_new == 0) return 0;
  if (!k_cache || !v_cache || !k_new || !v_new || !seq_lens) return 1;
  for (long b = 0; b < B; ++b)
    if (seq_lens[b] < 0 || seq_lens[b] + t_new > C) return 2;
  for (long b = 0; b < B; ++b) {
    for (long g = 0; g < Hkv; ++g)
      for (long i = 0; i < t_new; ++i) {
        long dst = ((b * Hkv + g) * C + seq_lens[b] + i) * d;
        long src = ((b * Hkv + g) * t_new + i) * d;
        memcpy(k_cache + dst, k_new + src, sizeof(double) * (size_t)d);
        memcpy(v_cache + dst, v_new + src, sizeof(double) * (size_t)d);
      }
    seq_lens[b] += t_new;
  }
  return 0;
}

/* Rolling buffer: position p in slot p mod W ([P1] "Relate shared heads to
 * local context"). */
int oracle_ring_append(double *k_ring, double *v_ring, const double *k_new,
                       const double *v_new, long *seq_lens, long B, long Hkv,
                       long W, long d, long t_new) {
  if (B < 0 || W <= 0 || t_new < 0 || Hkv <= 0 || d <= 0) return 1;
  if (B == 0 || t_new == 0) return 0;
  if (!k_ring || !v_ring || !k_new || !v_new || !seq_lens) return 1;
  for (long b = 0; b < B; ++b)
    if (seq_lens[b] < 0 || seq_lens[b] > 2147483647L - t_new) return 2;
  for (long b = 0; b < B; ++b) {
    for (long g = 0; g < Hkv; ++g)
      for (long i = 0; i < t_new; ++i) {
        long pos = seq_lens[b] + i;
        if (t_new - i > W) continue; /* overwritten by a later new row */
        long dst = ((b * Hkv + g) * W + pos % W) * d;
        long src = ((b * Hkv + g) * t_new + i) * d;
        memcpy(k_ring + dst, k_new + src, sizeof(double) * (size_t)d);
        memcpy(v_ring + dst, v_new + src, sizeof(double) * (size_t)d);
      }
    seq_lens[b] += t_new;
  }
  return 0;
}

int oracle_ring_decode(const double *q, const double *k_ring,
                       const double *v_ring, double *o, const long *seq_lens,
                       long B, long Hq, long Hkv, long W, long d, double scale) {
  if (B < 0 || W <= 0 || check_heads(Hq, Hkv, d)) return 1;
  if (B == 0) return 0;
  if (!q || !k_ring || !v_ring || !o || !seq_lens) return 1;
  for (long b = 0; b < B; ++b)
    if (seq_lens[b] < 0) return 2;
  long r = Hq / Hkv;
  int bad = 0;
#pragma omp parallel num_threads(g_threads) reduction(| : bad)
  {
    /* the window's keys and values gathered in position order */
    double *kk = (double *)malloc(sizeof(double) * (size_t)(W * d));
    double *vv = (double *)malloc(sizeof(double) * (size_t)(W * d));
    double *scratch = (double *)malloc(sizeof(double) * (size_t)W);
    if (!kk || !vv || !scratch) bad = 1;
#pragma omp for collapse(2) schedule(dynamic)
    for (long b = 0; b < B; ++b) {
      for (long h = 0; h < Hq; ++h) {
        if (!kk || !vv || !scratch) continue;
        long n = seq_lens[b];
        double *orow = o + (b * Hq + h) * d;
        if (n == 0) {
          memset(orow, 0, sizeof(double) * (size_t)d);
          continue;
        }
        long g = h / r;
        long lo = n > W ? n - W : 0;
        for (long pos = lo; pos < n; ++pos) {
          long src = ((b * Hkv + g) * W + pos % W) * d;
          memcpy(kk + (pos - lo) * d, k_ring + src, sizeof(double) * (size_t)d);
          memcpy(vv + (pos - lo) * d, v_ring + src, sizeof(double) * (size_t)d);
        }
        attend_row(q + (b * Hq + h) * d, kk, vv, 0, n - 1 - lo, d, scale, orow,
                   NULL, scratch);
      }
    }
    free(kk);
    free(vv);
    free(scratch);
  }
  return bad ? 1 : 0;
}

/* [P3] M_KV = 2 L B T Hkv d e, checked for uint64 overflow. */
uint64_t oracle_cache_bytes(uint64_t L, uint64_t B, uint64_t T, uint64_t Hkv,
                            uint64_t d, uint64_t e) {
  uint64_t factors[6] = {L, B, T, Hkv, d, e};
  uint64_t acc = 2;
  for (int i = 0; i < 6; ++i) {
    if (factors[i] != 0 && acc > UINT64_MAX / factors[i]) return 0;
    acc *= factors[i];
  }
  return acc;
}
