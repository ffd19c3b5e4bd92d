"""Multi-token decode (gqa_decode_multi) against the oracle.

t_new query rows per sequence sit at the last t_new of the n_b cached cells
and see the cache with the bottom-right mask ("How do you implement grouped
query attention (GQA)?", the implementation's tril(s - t) offset; "GQA,
FlashAttention and the KV cache", section "The important mask bug with a
cache").  The oracle is oracle_decode_multi.  Cache cells past n_b are
filled with NaN on both sides: they must never reach an output.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, f64
from grouped_query_attention_03_b200 import synthetic

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _threads():
    oracle.set_threads(0)
    yield
    oracle.set_threads(1)


def _inputs(B, Hq, Hkv, C, d, t_new, lens, seed, dtype):
    q = synthetic.normal((B, Hq, t_new, d), seed, 1.0, dtype, offset=31)
    kc = synthetic.normal((B, Hkv, C, d), seed, 1.0, dtype, offset=32)
    vc = synthetic.normal((B, Hkv, C, d), seed, 1.0, dtype, offset=33)
    for b, n in enumerate(lens):
        if 0 <= n < C:
            kc[b, :, n:] = float("nan")
            vc[b, :, n:] = float("nan")
    return q, kc, vc


MULTI_CASES = [
    # (dtype, B, Hq, Hkv, C, d, t_new, lens, window)
    (torch.bfloat16, 2, 8, 2, 700, 128, 7, [700, 300], None),   # paired heads, n_b = C
    (torch.bfloat16, 2, 8, 2, 700, 128, 300, [650, 300], 128),  # n_b = t_new, window
    (torch.bfloat16, 1, 32, 8, 5000, 128, 129, [4000], 1024),   # two query tiles
    (torch.bfloat16, 2, 6, 2, 400, 128, 33, [400, 100], None),  # group of 3: one head per CTA
    (torch.bfloat16, 2, 4, 4, 300, 64, 64, [300, 64], 17),      # MHA, d=64
    (torch.bfloat16, 1, 8, 1, 600, 64, 1, [555], None),         # one row: a decode step
    (torch.bfloat16, 2, 4, 2, 50, 96, 5, [50, 9], None),        # d=96: CUDA cores
    (torch.float32, 2, 8, 2, 300, 64, 20, [300, 20], 7),        # fp32: CUDA cores
]


@pytest.mark.parametrize("case", MULTI_CASES, ids=lambda c: (
    f"{'f32' if c[0] == torch.float32 else 'bf16'}-B{c[1]}Hq{c[2]}Hkv{c[3]}C{c[4]}d{c[5]}"
    f"t{c[6]}w{c[8]}"))
def test_decode_multi_cases(cuda_lib, case):
    dtype, B, Hq, Hkv, C, d, t_new, lens, window = case
    q, kc, vc = _inputs(B, Hq, Hkv, C, d, t_new, lens, C + t_new, dtype)
    want = oracle.decode_multi(f64(q), f64(kc), f64(vc), lens, window=window)
    assert np.isfinite(want).all()
    st = cuda_lib.new_status(DEV)
    lt = torch.tensor(lens, dtype=torch.int32, device=DEV)
    o = cuda_lib.decode_multi(q.to(DEV), kc.to(DEV), vc.to(DEV), lt, window=window, status=st)
    assert int(st.item()) == 0
    assert_close(o, want, dtype, f"decode_multi B{B} Hq{Hq} Hkv{Hkv} t{t_new} w{window}")


def test_decode_multi_whole_cache_equals_prefill(cuda_lib):
    """t_new = n_b = C is a causal prefill of the cache contents."""
    B, Hq, Hkv, T, d = 2, 8, 2, 256, 128
    q, k, v = [t.to(DEV) for t in synthetic.qkv_prefill(B, Hq, Hkv, T, d, seed=41)]
    lt = torch.full((B,), T, dtype=torch.int32, device=DEV)
    for window in (None, 100):
        a = cuda_lib.decode_multi(q, k, v, lt, window=window)
        b = cuda_lib.prefill(q, k, v, window=window)
        assert torch.equal(a, b), window


def test_decode_multi_refuses_short_or_long_lengths(cuda_lib):
    B, Hq, Hkv, C, d, t_new = 2, 8, 2, 64, 128, 10
    q, kc, vc = [t.to(DEV) for t in _inputs(B, Hq, Hkv, C, d, t_new, [C, C], 5, torch.bfloat16)]
    for lens in ([9, 64], [64, 65], [-1, 20]):
        st = cuda_lib.new_status(DEV)
        o = torch.full_like(q, 3.0)
        cuda_lib.decode_multi(q, kc, vc, torch.tensor(lens, dtype=torch.int32, device=DEV),
                              out=o, status=st)
        assert int(st.item()) == 5
        bad = [i for i, n in enumerate(lens) if not (t_new <= n <= C)]
        for i in range(B):
            if i in bad:
                assert torch.all(o[i] == 0)
            else:
                assert torch.isfinite(o[i].float()).all()


def test_prefill_ignores_nan_padding_past_the_length(cuda_lib):
    """Prompt cells past n_b hold NaN: active rows stay exact, the rest zero."""
    B, Hq, Hkv, T, d = 2, 8, 2, 300, 128
    q, k, v = synthetic.qkv_prefill(B, Hq, Hkv, T, d, seed=43)
    lens = [300, 150]
    for t in (q, k, v):
        t[1, :, 150:] = float("nan")
    want = oracle.prefill(f64(q), f64(k), f64(v), seq_lens=lens)
    st = cuda_lib.new_status(DEV)
    o = cuda_lib.prefill(q.to(DEV), k.to(DEV), v.to(DEV),
                         seq_lens=torch.tensor(lens, dtype=torch.int32, device=DEV), status=st)
    assert int(st.item()) == 0
    assert_close(o, want, torch.bfloat16, "prefill with NaN padding")
