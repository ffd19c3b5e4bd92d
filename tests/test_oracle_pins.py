"""The fp64 oracle against the pages' printed values and the mathematics."""
import numpy as np
import pytest
import torch

import oracle
import oracle_pins
import independent


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle)


def test_library_sdpa_cross_check():
    """The same tiny cases through torch's CPU fp64 scaled_dot_product_attention
    over explicitly repeat-interleaved K/V with a bottom-right boolean mask
    (the tokenwerk page's repeat + SDPA formulation, with the mask fixed as
    'The important mask bug with a cache' requires)."""
    rng = np.random.default_rng(11)
    for (B, Hq, Hkv, T, d, w) in [(2, 4, 2, 9, 8, None), (1, 8, 1, 13, 4, 3), (2, 6, 6, 7, 5, 2)]:
        q = rng.standard_normal((B, Hq, T, d))
        k = rng.standard_normal((B, Hkv, T, d))
        v = rng.standard_normal((B, Hkv, T, d))
        r = Hq // Hkv
        kt = torch.from_numpy(k).repeat_interleave(r, dim=1)
        vt = torch.from_numpy(v).repeat_interleave(r, dim=1)
        keep = torch.from_numpy(independent.keep_mask(T, T, w))
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q), kt, vt, attn_mask=keep).numpy()
        np.testing.assert_allclose(oracle.prefill(q, k, v, window=w), ref, rtol=0, atol=1e-12)


def test_decode_sdpa_single_token_sees_whole_cache():
    """With one new token the bottom-right mask keeps every cached key; the
    top-left causal mask (the page's bug) would keep only the first."""
    rng = np.random.default_rng(12)
    B, Hq, Hkv, C, d = 1, 4, 2, 16, 8
    kc = rng.standard_normal((B, Hkv, C, d))
    vc = rng.standard_normal((B, Hkv, C, d))
    q = rng.standard_normal((B, Hq, d))
    n = 11
    o = oracle.decode(q, kc, vc, [n])
    r = Hq // Hkv
    kt = torch.from_numpy(kc[:, :, :n]).repeat_interleave(r, dim=1)
    vt = torch.from_numpy(vc[:, :, :n]).repeat_interleave(r, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q)[:, :, None], kt, vt)
    np.testing.assert_allclose(o, ref[:, :, 0].numpy(), rtol=0, atol=1e-12)
    bug = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[:, :, None], kt, vt, is_causal=True)
    assert np.abs(o - bug[:, :, 0].numpy()).max() > 1e-3


def test_decode_edges():
    """n_b = 0 gives zero output; n_b beyond capacity is refused."""
    q = np.ones((2, 2, 3))
    kc = np.ones((2, 1, 4, 3))
    o = oracle.decode(q, kc, kc, [0, 4])
    assert np.all(o[0] == 0) and np.allclose(o[1], 1.0)
    with pytest.raises(oracle.OracleError):
        oracle.decode(q, kc, kc, [5, 1])


def test_threads_do_not_change_results():
    rng = np.random.default_rng(13)
    q = rng.standard_normal((2, 8, 33, 16))
    k = rng.standard_normal((2, 2, 33, 16))
    v = rng.standard_normal((2, 2, 33, 16))
    oracle.set_threads(1)
    a = oracle.prefill(q, k, v, window=7)
    oracle.set_threads(4)
    b = oracle.prefill(q, k, v, window=7)
    oracle.set_threads(1)
    assert np.array_equal(a, b)
