"""fp64 CPU oracle for grouped-query attention: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never imports, links
or calls it, and it shares no code with the CUDA path.  Inputs are converted
to float64 (bf16 inputs are the already-rounded values), the C loops in
``gqa_oracle.c`` do the arithmetic, and results come back as float64 arrays.

Citations are to the source pages by title and section:
  * "Share key/value heads and make context explicit" (practical LLM in Rust,
    ch. 18): head map, permitted set, score/normalisation/value mix, decode
    loop, cache transaction, worked example.
  * "GQA, FlashAttention and the KV cache": cache-size formula, decode mask.
  * "How do you implement grouped query attention (GQA)?": shapes, tril(s-t).

Functions without a pin of their own are marked "parity unpinned" below;
every function here currently has at least one pin in ``tests/test_oracle_*``.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = _load(path)
    return _lib


def _load(path):
    L = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lp = ctypes.POINTER(ctypes.c_long)
    c_long, c_double = ctypes.c_long, ctypes.c_double
    L.oracle_kv_head_for_query.argtypes = [c_long] * 3
    L.oracle_kv_head_for_query.restype = c_long
    L.oracle_window_start.argtypes = [c_long] * 3
    L.oracle_window_start.restype = c_long
    L.oracle_prefill.argtypes = [dp, dp, dp, dp, dp, lp] + [c_long] * 6 + [c_double]
    L.oracle_prefill.restype = ctypes.c_int
    L.oracle_prefill_packed.argtypes = [dp, dp, dp, dp, dp, lp, lp] + [c_long] * 6 + [c_double]
    L.oracle_prefill_packed.restype = ctypes.c_int
    L.oracle_decode.argtypes = [dp, dp, dp, dp, lp] + [c_long] * 6 + [c_double]
    L.oracle_decode.restype = ctypes.c_int
    L.oracle_decode_multi.argtypes = [dp, dp, dp, dp, lp] + [c_long] * 7 + [c_double]
    L.oracle_decode_multi.restype = ctypes.c_int
    L.oracle_cache_append.argtypes = [dp, dp, dp, dp, lp] + [c_long] * 5
    L.oracle_cache_append.restype = ctypes.c_int
    L.oracle_ring_append.argtypes = [dp, dp, dp, dp, lp] + [c_long] * 5
    L.oracle_ring_append.restype = ctypes.c_int
    L.oracle_ring_decode.argtypes = [dp, dp, dp, dp, lp] + [c_long] * 5 + [c_double]
    L.oracle_ring_decode.restype = ctypes.c_int
    L.oracle_cache_bytes.argtypes = [ctypes.c_uint64] * 6
    L.oracle_cache_bytes.restype = ctypes.c_uint64
    L.oracle_set_threads.argtypes = [ctypes.c_int]
    L.oracle_set_threads.restype = ctypes.c_int
    return L


class OracleError(RuntimeError):
    pass


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _dp(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _lp(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_long))


def _lens(seq_lens):
    if seq_lens is None:
        return None
    return np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int64))


def _window(window):
    return -1 if window is None else int(window)


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what}: oracle status {rc}")


def set_threads(n: int) -> int:
    """Threads for the (batch, head) loops; n <= 0 means every host core."""
    return lib().oracle_set_threads(int(n))


def kv_head_for_query(h, Hq, Hkv):
    """g(h) = floor(h / (Hq/Hkv)); None where the map does not exist."""
    g = lib().oracle_kv_head_for_query(int(h), int(Hq), int(Hkv))
    return None if g < 0 else int(g)


def window_start(t, seg_start, window):
    """max(seg_start, t -sat- (w-1)); None for w == 0 or seg_start > t."""
    s = lib().oracle_window_start(int(t), int(seg_start), _window(window))
    return None if s < 0 else int(s)


def prefill(q, k, v, window=None, scale=None, seq_lens=None, seg_start=None,
            return_probs=False):
    """Full pass.  q [B,Hq,T,d], k/v [B,Hkv,T,d] -> o [B,Hq,T,d] (float64)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.empty((B, Hq, T, d), dtype=np.float64)
    probs = np.empty((B, Hq, T, T), dtype=np.float64) if return_probs else None
    lens = _lens(seq_lens)
    segs = None if seg_start is None else np.ascontiguousarray(np.asarray(seg_start, dtype=np.int64))
    rc = lib().oracle_prefill_packed(_dp(q), _dp(k), _dp(v), _dp(o), _dp(probs),
                                     _lp(lens), _lp(segs), B, Hq, Hkv, T, d,
                                     _window(window), float(scale))
    _check(rc, "prefill")
    return (o, probs) if return_probs else o


def decode(q, k_cache, v_cache, seq_lens, window=None, scale=None):
    """Single-token decode.  q [B,Hq,d], caches [B,Hkv,C,d], n_b includes the
    current token -> o [B,Hq,d]."""
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    B, Hq, d = q.shape
    Hkv, C = kc.shape[1], kc.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.empty((B, Hq, d), dtype=np.float64)
    lens = _lens(seq_lens)
    rc = lib().oracle_decode(_dp(q), _dp(kc), _dp(vc), _dp(o), _lp(lens), B, Hq,
                             Hkv, C, d, _window(window), float(scale))
    _check(rc, "decode")
    return o


def decode_multi(q, k_cache, v_cache, seq_lens, window=None, scale=None):
    """t_new queries per sequence against the cache (bottom-right mask).
    q [B,Hq,t_new,d] -> o [B,Hq,t_new,d]."""
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    B, Hq, t_new, d = q.shape
    Hkv, C = kc.shape[1], kc.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.empty((B, Hq, t_new, d), dtype=np.float64)
    lens = _lens(seq_lens)
    rc = lib().oracle_decode_multi(_dp(q), _dp(kc), _dp(vc), _dp(o), _lp(lens), B,
                                   Hq, Hkv, C, d, t_new, _window(window), float(scale))
    _check(rc, "decode_multi")
    return o


def cache_append(k_cache, v_cache, k_new, v_new, seq_lens):
    """Returns (k_cache', v_cache', seq_lens') as new arrays, or raises
    OracleError (and leaves everything unchanged) if any sequence would
    exceed the capacity."""
    kc, vc = _f64(k_cache).copy(), _f64(v_cache).copy()
    kn, vn = _f64(k_new), _f64(v_new)
    lens = _lens(seq_lens).copy()
    B, Hkv, C, d = kc.shape
    t_new = kn.shape[2]
    rc = lib().oracle_cache_append(_dp(kc), _dp(vc), _dp(kn), _dp(vn), _lp(lens),
                                   B, Hkv, C, d, t_new)
    _check(rc, "cache_append")
    return kc, vc, lens


def ring_append(k_ring, v_ring, k_new, v_new, seq_lens):
    """Rolling buffer of W slots: writes positions [len_b, len_b + t_new) at
    slots p mod W (the last W survive).  Returns (k_ring', v_ring',
    seq_lens') as new arrays, or raises OracleError."""
    kr, vr = _f64(k_ring).copy(), _f64(v_ring).copy()
    kn, vn = _f64(k_new), _f64(v_new)
    lens = _lens(seq_lens).copy()
    B, Hkv, W, d = kr.shape
    t_new = kn.shape[2]
    rc = lib().oracle_ring_append(_dp(kr), _dp(vr), _dp(kn), _dp(vn), _lp(lens),
                                  B, Hkv, W, d, t_new)
    _check(rc, "ring_append")
    return kr, vr, lens


def ring_decode(q, k_ring, v_ring, seq_lens, scale=None):
    """Decode against a rolling buffer: the query at position n_b - 1 reads
    positions [max(0, n_b - W), n_b) from their slots.  q [B,Hq,d]."""
    q, kr, vr = _f64(q), _f64(k_ring), _f64(v_ring)
    B, Hq, d = q.shape
    Hkv, W = kr.shape[1], kr.shape[2]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.empty((B, Hq, d), dtype=np.float64)
    rc = lib().oracle_ring_decode(_dp(q), _dp(kr), _dp(vr), _dp(o), _lp(_lens(seq_lens)),
                                  B, Hq, Hkv, W, d, float(scale))
    _check(rc, "ring_decode")
    return o


def cache_bytes(L, B, T, Hkv, d, e):
    """2*L*B*T*Hkv*d*e bytes; 0 on uint64 overflow."""
    return int(lib().oracle_cache_bytes(L, B, T, Hkv, d, e))


def lib_path():
    return os.path.abspath(_build.LIB)
