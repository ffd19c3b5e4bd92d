"""Pins that fix the fp64 oracle to something other than itself.

Each ``pin_*`` takes the oracle module and raises AssertionError when the
oracle disagrees with what the pages print or what the mathematics fixes.
They are run directly by ``test_oracle_pins.py`` and, against deliberately
broken builds of the oracle, by ``test_oracle_mutations.py`` (which checks
that every planted mistake is caught by at least one pin).
"""
import json
import os

import numpy as np

import independent

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rng(seed):
    return np.random.default_rng(seed)


def worked_example_inputs():
    """The fixture of 'Follow four query heads into two shared groups': zero
    Q/K; v_t = x_t W_v with x_t = [t+1, 0, ...] and W_v row 0 = [1,0,0,10]."""
    g = golden("worked_example.json")["fixture"]
    T, Hq, Hkv, d = g["tokens"], g["query_heads"], g["kv_heads"], g["head_width"]
    w0 = np.array(g["value_weight_row0"], dtype=np.float64)
    x0 = np.array(g["first_features"], dtype=np.float64)
    vflat = x0[:, None] * w0[None, :]                    # [T, Hkv*d]
    v = vflat.reshape(T, Hkv, d).transpose(1, 0, 2)[None]  # [1,Hkv,T,d]
    q = np.zeros((1, Hq, T, d))
    k = np.zeros((1, Hkv, T, d))
    return q, k, v


def pin_worked_example(O):
    g = golden("worked_example.json")
    q, k, v = worked_example_inputs()
    Hq, Hkv = q.shape[1], k.shape[1]
    assert [O.kv_head_for_query(h, Hq, Hkv) for h in range(Hq)] == g["head_mapping"]
    assert list(k.shape) == g["key_shape"]
    for case in g["cases"]:
        o, p = O.prefill(q, k, v, window=case["window"], return_probs=True)
        merged = o[0, :, -1, :].reshape(-1)            # concat heads at t=3
        assert merged.tolist() == case["last_merged_output"], (case, merged)
        for h in range(Hq):
            assert p[0, h, -1].tolist() == case["last_query_weights"], (case, h, p[0, h, -1])


def pin_worked_example_earlier_rows(O):
    """Rows t=0..2 of the same fixture: the mean of the permitted first
    coordinates (1, 1.5, 2 causal; 1, 1.5, 2.5 with window 2)."""
    q, k, v = worked_example_inputs()
    full = O.prefill(q, k, v)
    win = O.prefill(q, k, v, window=2)
    assert full[0, 0, :3, 0].tolist() == [1.0, 1.5, 2.0]
    assert win[0, 0, :3, 0].tolist() == [1.0, 1.5, 2.5]
    assert full[0, 2, :3, 1].tolist() == [10.0, 15.0, 20.0]


def pin_head_map(O):
    """Page examples: 8 query heads over 2 KV heads -> heads 0-3 read 0 and
    4-7 read 1 (clozo.ai 'Step 2'); 32 over 8 -> groups of 4 (bibekananda.in
    'It is one dial'); refusals for zero or indivisible counts and an
    out-of-range head (practical LLM ch. 18 kv_head_for_query)."""
    assert [O.kv_head_for_query(h, 8, 2) for h in range(8)] == [0, 0, 0, 0, 1, 1, 1, 1]
    assert [O.kv_head_for_query(h, 32, 8) for h in range(32)] == [h // 4 for h in range(32)]
    assert [O.kv_head_for_query(h, 8, 8) for h in range(8)] == list(range(8))
    assert [O.kv_head_for_query(h, 8, 1) for h in range(8)] == [0] * 8
    assert O.kv_head_for_query(0, 4, 0) is None
    assert O.kv_head_for_query(0, 0, 2) is None
    assert O.kv_head_for_query(0, 6, 4) is None
    assert O.kv_head_for_query(4, 4, 2) is None


def pin_window_start(O):
    """'Intersect the window ...': window 1 -> self; saturating start near
    the beginning; a later segment start wins; zero window refused."""
    assert O.window_start(5, 0, 1) == 5
    assert O.window_start(1, 0, 4) == 0
    assert O.window_start(7, 0, 4) == 4
    assert O.window_start(4, 2, 2) == 3
    assert O.window_start(5, 5, 2) == 5
    assert O.window_start(3, 0, 0) is None
    assert O.window_start(2, 3, 2) is None
    assert O.window_start(9, 0, None) == 0


def pin_packed_window(O):
    """The six-cell packed report: cell 4 keeps keys {3,4}, cell 5 only {5}."""
    g = golden("packed_window.json")
    T = len(g["segment_starts"])
    q = np.zeros((1, 1, T, 1))
    k = np.zeros((1, 1, T, 1))
    v = np.zeros((1, 1, T, 1))
    _, p = O.prefill(q, k, v, window=g["window"], seg_start=[g["segment_starts"]],
                     return_probs=True)
    for cell, want in g["printed"].items():
        t = int(cell)
        assert O.window_start(t, want["segment_start"], g["window"]) == want["window_start"]
        keys = np.nonzero(p[0, 0, t])[0].tolist()
        assert keys == want["keys"], (t, keys)


def pin_zero_qk_mean(O):
    """Zero Q/K: every score is equal, so each output is the arithmetic mean of
    the permitted rows of the shared value lane (generalises the worked
    example).  Checked for several shapes and windows, with ragged lengths."""
    r = _rng(1)
    for (B, Hq, Hkv, T, d, w) in [(2, 4, 2, 7, 3, None), (1, 6, 3, 9, 2, 3),
                                  (2, 8, 1, 5, 4, 1), (1, 4, 4, 6, 2, 10)]:
        v = r.standard_normal((B, Hkv, T, d))
        lens = r.integers(0, T + 1, size=B)
        o = O.prefill(np.zeros((B, Hq, T, d)), np.zeros((B, Hkv, T, d)), v,
                      window=w, seq_lens=lens)
        for b in range(B):
            for h in range(Hq):
                g = h // (Hq // Hkv)
                for t in range(T):
                    if t >= lens[b]:
                        assert np.all(o[b, h, t] == 0.0)
                        continue
                    lo = 0 if w is None else max(0, t - w + 1)
                    want = v[b, g, lo:t + 1].mean(axis=0)
                    np.testing.assert_allclose(o[b, h, t], want, rtol=0, atol=1e-14)


def pin_window_special_cases(O):
    """Window 1 permits only self, so o[b,h,t] = v[b,g(h),t] exactly; a window
    of at least T recovers plain causal attention."""
    r = _rng(2)
    B, Hq, Hkv, T, d = 2, 6, 2, 11, 5
    q = r.standard_normal((B, Hq, T, d))
    k = r.standard_normal((B, Hkv, T, d))
    v = r.standard_normal((B, Hkv, T, d))
    o1 = O.prefill(q, k, v, window=1)
    for h in range(Hq):
        assert np.array_equal(o1[:, h], v[:, h // 3])
    full = O.prefill(q, k, v)
    for w in (T, T + 1, 5 * T):
        assert np.array_equal(O.prefill(q, k, v, window=w), full)


def pin_endpoints_and_brute_force(O):
    """MHA (Hkv=Hq), MQA (Hkv=1) and every divisor in between against the
    independent repeat-interleave implementation, over tiny shapes with
    every window and ragged lengths."""
    r = _rng(3)
    count = 0
    for B in (1, 2):
        for Hq in (1, 2, 4, 8):
            for Hkv in [x for x in (1, 2, 4, 8) if x <= Hq and Hq % x == 0]:
                for T in (1, 2, 5, 9):
                    for d in (1, 2, 3, 4):
                        q = r.standard_normal((B, Hq, T, d))
                        k = r.standard_normal((B, Hkv, T, d))
                        v = r.standard_normal((B, Hkv, T, d))
                        lens = r.integers(0, T + 1, size=B)
                        scale = float(r.uniform(0.2, 1.5))
                        for w in [None] + list(range(1, T + 2)):
                            a = O.prefill(q, k, v, window=w, scale=scale, seq_lens=lens)
                            b = independent.attention(q, k, v, window=w, scale=scale,
                                                      seq_lens=lens)
                            np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
                            count += 1
    assert count > 500


def pin_repeat_is_not_tile(O):
    """Tiling the KV head list (repeat) instead of repeat-interleave pairs
    query heads with the wrong KV heads (clozo.ai 'Trade-offs and edge
    cases'); the oracle must agree with interleave and differ from tile."""
    r = _rng(4)
    q = r.standard_normal((1, 8, 6, 4))
    k = r.standard_normal((1, 2, 6, 4))
    v = r.standard_normal((1, 2, 6, 4))
    o = O.prefill(q, k, v)
    np.testing.assert_allclose(o, independent.attention(q, k, v), rtol=0, atol=1e-12)
    assert np.abs(o - independent.attention(q, k, v, tile=True)).max() > 1e-3


def pin_decode_equals_last_prefill_row(O):
    """Cached decode reproduces the full pass: at every prefix length the
    decode output of the newest token equals that row of the full prefill
    (the chapter's full/cached comparison; with t=1 the query sees the whole
    cache, not only its first key)."""
    r = _rng(5)
    B, Hq, Hkv, T, d = 2, 4, 2, 10, 3
    q = r.standard_normal((B, Hq, T, d))
    k = r.standard_normal((B, Hkv, T, d))
    v = r.standard_normal((B, Hkv, T, d))
    C = T + 3
    for w in (None, 1, 3):
        full = O.prefill(q, k, v, window=w)
        kc = np.zeros((B, Hkv, C, d))
        vc = np.zeros((B, Hkv, C, d))
        lens = np.zeros(B, dtype=np.int64)
        for t in range(T):
            kc, vc, lens = O.cache_append(kc, vc, k[:, :, t:t + 1], v[:, :, t:t + 1], lens)
            o = O.decode(q[:, :, t], kc, vc, lens, window=w)
            np.testing.assert_allclose(o, full[:, :, t], rtol=0, atol=1e-12)


def pin_decode_multi_mask_offset(O):
    """t_new > 1 queries against the cache: query i sits at cell s - t + i
    (clozo.ai implementation's tril(s - t)); equals the independent dense
    implementation and the matching rows of the full pass."""
    r = _rng(6)
    B, Hq, Hkv, d, C = 2, 4, 1, 3, 12
    lens = np.array([9, 5])
    kc = r.standard_normal((B, Hkv, C, d))
    vc = r.standard_normal((B, Hkv, C, d))
    for t_new in (1, 2, 4):
        q = r.standard_normal((B, Hq, t_new, d))
        for w in (None, 2, 4):
            o = O.decode_multi(q, kc, vc, lens, window=w)
            for b in range(B):
                n = int(lens[b])
                want = independent.attention(q[b:b + 1], kc[b:b + 1, :, :n],
                                             vc[b:b + 1, :, :n], window=w)
                np.testing.assert_allclose(o[b:b + 1], want, rtol=0, atol=1e-12)


def pin_softmax_saturation(O):
    """Closed form for extreme scores: when one permitted score exceeds every
    other by far more than the fp64 exponent range, softmax puts all weight on
    it and the output is exactly that value row (needs the max-subtracted
    form; an unshifted exp overflows)."""
    T, d = 4, 2
    q = np.zeros((1, 1, T, d))
    q[0, 0, :, 0] = 1.0
    k = np.zeros((1, 1, T, d))
    k[0, 0, :, 0] = [1000.0, 3000.0, 2000.0, -500.0]
    v = np.arange(T * d, dtype=np.float64).reshape(1, 1, T, d)
    o = O.prefill(q, k, v, scale=1.0)
    assert o[0, 0, 0].tolist() == v[0, 0, 0].tolist()
    assert o[0, 0, 1].tolist() == v[0, 0, 1].tolist()
    assert o[0, 0, 3].tolist() == v[0, 0, 1].tolist()


def pin_two_key_closed_form(O):
    """Two permitted keys with scores a, b: p = 1/(1+e^(b-a)) exactly as the
    logistic function; output is the matching mix of the two value rows."""
    q = np.array([[[[0.0, 0.0], [0.7, -0.2]]]])
    k = np.array([[[[1.0, 2.0], [-0.5, 0.25]]]])
    v = np.array([[[[3.0, -1.0], [0.5, 4.0]]]])
    scale = 0.9
    s0 = scale * (0.7 * 1.0 - 0.2 * 2.0)
    s1 = scale * (0.7 * -0.5 - 0.2 * 0.25)
    p0 = 1.0 / (1.0 + np.exp(s1 - s0))
    want = p0 * v[0, 0, 0] + (1 - p0) * v[0, 0, 1]
    o = O.prefill(q, k, v, scale=scale)
    np.testing.assert_allclose(o[0, 0, 1], want, rtol=0, atol=1e-15)
    assert o[0, 0, 0].tolist() == v[0, 0, 0].tolist()


def pin_inactive_rows(O):
    """Inactive padded queries (t >= n_b) keep zero probabilities and zero
    outputs; active rows ignore the padding."""
    r = _rng(7)
    B, Hq, Hkv, T, d = 3, 4, 2, 8, 3
    q = r.standard_normal((B, Hq, T, d))
    k = r.standard_normal((B, Hkv, T, d))
    v = r.standard_normal((B, Hkv, T, d))
    lens = [0, 3, 8]
    o, p = O.prefill(q, k, v, seq_lens=lens, return_probs=True)
    for b, n in enumerate(lens):
        assert np.all(o[b, :, n:] == 0.0) and np.all(p[b, :, n:] == 0.0)
        if n:
            sub = O.prefill(q[b:b + 1, :, :n], k[b:b + 1, :, :n], v[b:b + 1, :, :n])
            assert np.array_equal(o[b:b + 1, :, :n], sub)
    for b in range(B):
        for t in range(lens[b]):
            np.testing.assert_allclose(p[b, :, t].sum(axis=-1), 1.0, rtol=0, atol=1e-14)


def pin_cache_bytes(O):
    g = golden("cache_sizes.json")
    for c in g["cases"]:
        got = O.cache_bytes(c["L"], c["B"], c["T"], c["Hkv"], c["d"], c["e"])
        assert got == c["bytes"], c
    sm = g["score_macs"]
    assert sm["Hq"] * sm["T"] * sm["d"] == sm["macs"]
    assert O.cache_bytes(2**40, 2**20, 2**10, 1, 1, 1) == 0     # overflow -> 0


def pin_cache_append(O):
    """Append writes rows [len_b, len_b + t_new) and advances the lengths; a
    request that would exceed the capacity for any sequence is refused and
    nothing moves; appending never changes the allocation."""
    r = _rng(8)
    B, Hkv, C, d = 3, 2, 6, 2
    kc = r.standard_normal((B, Hkv, C, d))
    vc = r.standard_normal((B, Hkv, C, d))
    lens = np.array([0, 2, 4])
    kn = r.standard_normal((B, Hkv, 2, d))
    vn = r.standard_normal((B, Hkv, 2, d))
    k2, v2, l2 = O.cache_append(kc, vc, kn, vn, lens)
    assert l2.tolist() == [2, 4, 6] and k2.shape == kc.shape
    for b in range(B):
        n = lens[b]
        assert np.array_equal(k2[b, :, n:n + 2], kn[b]) and np.array_equal(v2[b, :, n:n + 2], vn[b])
        assert np.array_equal(k2[b, :, :n], kc[b, :, :n]) and np.array_equal(k2[b, :, n + 2:], kc[b, :, n + 2:])
    # Refusal: sequence 0 is full, sequence 1 has room.  (Laid out so that
    # even an unguarded write would land inside the buffer, in lane 1.)
    kc1 = r.standard_normal((2, 1, 4, d))
    one = r.standard_normal((2, 1, 1, d))
    try:
        O.cache_append(kc1, kc1, one, one, np.array([4, 0]))
    except O.OracleError:
        pass
    else:
        raise AssertionError("append beyond capacity was accepted")


def pin_ring_equals_windowed_decode(O):
    """A rolling buffer of W slots ("Relate shared heads to local context":
    Mistral's rolling buffer that overwrites old KV entries; the chapter does
    not build it) holds exactly the last W positions, so decoding against it
    equals decoding with window W against the all-prefix cache that the
    chapter keeps -- bit for bit, since both read the same keys in position
    order.  Appends come in random chunk sizes, some longer than W."""
    r = _rng(21)
    B, Hq, Hkv, d = 2, 4, 2, 3
    for W in (1, 2, 3, 5, 8):
        kr = np.zeros((B, Hkv, W, d))
        vr = np.zeros((B, Hkv, W, d))
        C = 40
        kc = np.zeros((B, Hkv, C, d))
        vc = np.zeros((B, Hkv, C, d))
        lr = np.zeros(B, dtype=np.int64)
        lc = np.zeros(B, dtype=np.int64)
        while lc.max() < 30:
            t_new = int(r.integers(1, 2 * W + 2))
            if lc.max() + t_new > C:
                break
            kn = r.standard_normal((B, Hkv, t_new, d))
            vn = r.standard_normal((B, Hkv, t_new, d))
            kr, vr, lr = O.ring_append(kr, vr, kn, vn, lr)
            kc, vc, lc = O.cache_append(kc, vc, kn, vn, lc)
            assert lr.tolist() == lc.tolist()
            # every surviving slot holds the row of its position
            for b in range(B):
                n = lc[b]
                for pos in range(max(0, n - W), n):
                    assert np.array_equal(kr[b, :, pos % W], kc[b, :, pos])
                    assert np.array_equal(vr[b, :, pos % W], vc[b, :, pos])
            q = r.standard_normal((B, Hq, d))
            want = O.decode(q, kc, vc, lc, window=W)
            got = O.ring_decode(q, kr, vr, lr)
            assert np.array_equal(got, want), W


def pin_ring_refusals(O):
    """Negative lengths and an empty ring are refused."""
    kr = np.zeros((1, 1, 4, 2))
    one = np.zeros((1, 1, 1, 2))
    for lens, ring in (([-1], kr), ([0], np.zeros((1, 1, 0, 2)))):
        try:
            O.ring_append(ring, ring, one, one, lens)
        except O.OracleError:
            pass
        else:
            raise AssertionError(f"ring append accepted {lens}, W={ring.shape[2]}")
    try:
        O.ring_decode(np.zeros((1, 2, 2)), kr, kr, [-2])
    except O.OracleError:
        pass
    else:
        raise AssertionError("ring decode accepted a negative length")


def pin_refusals(O):
    """Zero window refused; indivisible heads refused."""
    q = np.zeros((1, 3, 2, 2))
    k = np.zeros((1, 2, 2, 2))
    for bad in (dict(window=0), dict(window=-3)):
        try:
            O.prefill(np.zeros((1, 2, 2, 2)), np.zeros((1, 1, 2, 2)), np.zeros((1, 1, 2, 2)), **bad)
        except O.OracleError:
            pass
        else:
            raise AssertionError(f"accepted {bad}")
    try:
        O.prefill(q, k, k)
    except O.OracleError:
        pass
    else:
        raise AssertionError("accepted Hq % Hkv != 0")


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
