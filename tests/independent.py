"""A second, independent fp64 implementation used only to pin the oracle.

It follows the dense formulation of "How do you implement grouped query
attention (GQA)?" (clozo.ai), section 'Worked example' implementation and
'Step 3: Repeat the keys and values, then attend as usual': copy every KV head
Hq/Hkv times with repeat-interleave, form the full score matrix, mask with a
boolean keep-matrix that is lower-triangular with offset s - t (query i of t
sits at absolute cell s - t + i), intersect with the local window, softmax per
row and mix values.  Vectorised numpy, no loops over keys, and no code shared
with the oracle.
"""
import numpy as np


def repeat_kv(x, r, tile=False):
    """[B,Hkv,S,d] -> [B,Hkv*r,S,d]; repeat-interleave (adjacent copies), or
    whole-list tiling when ``tile`` (the mistake the page warns about)."""
    if tile:
        return np.tile(x, (1, r, 1, 1))
    return np.repeat(x, r, axis=1)


def keep_mask(t, s, window=None, seg_start=None):
    """Boolean [t, s]: query i (absolute cell s-t+i) keeps key j iff
    j <= s-t+i, and within the window j > s-t+i-w, and j >= its segment start."""
    i = np.arange(t)[:, None]
    j = np.arange(s)[None, :]
    pos = s - t + i
    keep = j <= pos
    if window is not None:
        keep &= j > pos - window
    if seg_start is not None:
        keep &= j >= np.asarray(seg_start)[:, None]
    return keep


def attention(q, k, v, window=None, scale=None, tile=False, seq_lens=None,
              seg_start=None, return_probs=False):
    """q [B,Hq,t,d], k/v [B,Hkv,s,d] with s >= t; bottom-right aligned mask.
    Rows whose query cell is >= n_b (``seq_lens``) give zero output."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, Hq, t, d = q.shape
    Hkv, s = k.shape[1], k.shape[2]
    r = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    kr, vr = repeat_kv(k, r, tile), repeat_kv(v, r, tile)
    scores = np.einsum("bhtd,bhsd->bhts", q, kr) * scale
    out = np.zeros((B, Hq, t, d))
    probs_all = np.zeros((B, Hq, t, s))
    for b in range(B):
        segs = None if seg_start is None else np.asarray(seg_start)[b]
        keep = keep_mask(t, s, window, segs)
        if seq_lens is not None:
            n = int(seq_lens[b])
            active = (s - t + np.arange(t)) < n
            keep = keep & active[:, None] & (np.arange(s)[None, :] < n)
        sc = np.where(keep[None], scores[b], -np.inf)
        rowmax = sc.max(axis=-1, keepdims=True)
        rowmax = np.where(np.isfinite(rowmax), rowmax, 0.0)
        e = np.where(keep[None], np.exp(sc - rowmax), 0.0)
        den = e.sum(axis=-1, keepdims=True)
        p = np.divide(e, den, out=np.zeros_like(e), where=den > 0)
        probs_all[b] = p
        out[b] = np.einsum("hts,hsd->htd", p, vr[b])
    return (out, probs_all) if return_probs else out
