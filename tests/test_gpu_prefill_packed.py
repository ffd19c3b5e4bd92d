"""Packed-segment prefill (gqa_prefill_packed) against the oracle.

"Share key/value heads and make context explicit", section "Intersect the
window with the context already permitted": cell t of a packed row reads
keys [max(s_{b,t}, t-(w-1)), t], where s_{b,t} starts t's segment.  The
oracle is oracle_prefill_packed (pinned to the chapter's packed report).

Inputs are N(0, 0.5^2) (the long-context workload's distribution): short
segments leave a row one or two keys, so the output is as large as a value
row, and above |o| = 2 the bf16 rounding of the exact answer alone reaches
the 1e-2 absolute bar.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, f64
from grouped_query_attention_03_b200 import synthetic

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "packed_window.json")


@pytest.fixture(scope="module", autouse=True)
def _threads():
    oracle.set_threads(0)
    yield
    oracle.set_threads(1)


def packed_starts(B, T, max_doc, seed):
    """Segment starts of documents with lengths uniform in [1, max_doc]."""
    rng = np.random.RandomState(seed)
    out = np.zeros((B, T), dtype=np.int32)
    for b in range(B):
        t = 0
        while t < T:
            n = rng.randint(1, max_doc + 1)
            out[b, t:t + n] = t
            t += n
    return out


def test_packed_report_on_gpu(cuda_lib):
    """The chapter's six-cell report: value rows one-hot per cell make each
    output row the mean over exactly the printed key set."""
    g = json.load(open(GOLDEN))
    T, w = len(g["segment_starts"]), g["window"]
    q = torch.zeros((1, 2, T, 64), dtype=torch.bfloat16)
    k = torch.zeros((1, 1, T, 64), dtype=torch.bfloat16)
    v = torch.zeros((1, 1, T, 64), dtype=torch.bfloat16)
    for t in range(T):
        v[0, 0, t, t] = 1.0
    seg = torch.tensor([g["segment_starts"]], dtype=torch.int32, device=DEV)
    st = cuda_lib.new_status(DEV)
    o = cuda_lib.prefill_packed(q.to(DEV), k.to(DEV), v.to(DEV), seg, window=w, status=st)
    assert int(st.item()) == 0
    for cell, want in g["printed"].items():
        row = o[0, 0, int(cell), :T].float().cpu().numpy()
        keys = want["keys"]
        expect = np.zeros(T)
        expect[keys] = 1.0 / len(keys)
        np.testing.assert_array_equal(row, expect)


PACKED_CASES = [
    # (dtype, B, Hq, Hkv, T, d, window, lens, max_doc)
    (torch.bfloat16, 2, 8, 2, 1000, 128, None, [1000, 700], 300),   # paired heads
    (torch.bfloat16, 2, 8, 2, 1000, 128, 64, [1000, 999], 300),     # with a window
    (torch.bfloat16, 1, 8, 2, 520, 64, None, None, 40),             # many short documents
    (torch.bfloat16, 2, 6, 2, 300, 128, 50, [300, 123], 90),        # group of 3
    (torch.bfloat16, 1, 4, 2, 200, 96, None, None, 60),             # d=96: CUDA cores
    (torch.float32, 2, 4, 2, 150, 64, 20, [150, 77], 50),           # fp32: CUDA cores
]


@pytest.mark.parametrize("case", PACKED_CASES, ids=lambda c: (
    f"{'f32' if c[0] == torch.float32 else 'bf16'}-B{c[1]}Hq{c[2]}Hkv{c[3]}T{c[4]}d{c[5]}"
    f"w{c[6]}doc{c[8]}"))
def test_prefill_packed_cases(cuda_lib, case):
    dtype, B, Hq, Hkv, T, d, window, lens, max_doc = case
    q, k, v = synthetic.qkv_prefill(B, Hq, Hkv, T, d, seed=T + d, std=0.5, dtype=dtype)
    seg = packed_starts(B, T, max_doc, seed=T)
    want = oracle.prefill(f64(q), f64(k), f64(v), window=window, seq_lens=lens,
                          seg_start=seg.astype(np.int64))
    st = cuda_lib.new_status(DEV)
    lt = None if lens is None else torch.tensor(lens, dtype=torch.int32, device=DEV)
    o = cuda_lib.prefill_packed(q.to(DEV), k.to(DEV), v.to(DEV),
                                torch.from_numpy(seg).to(DEV), window=window, seq_lens=lt,
                                status=st)
    assert int(st.item()) == 0
    assert_close(o, want, dtype, f"packed B{B} Hq{Hq} T{T} d{d} w{window}")


def test_prefill_packed_one_segment_equals_prefill(cuda_lib):
    B, Hq, Hkv, T, d = 2, 8, 2, 384, 128
    q, k, v = [t.to(DEV) for t in synthetic.qkv_prefill(B, Hq, Hkv, T, d, seed=51)]
    seg = torch.zeros((B, T), dtype=torch.int32, device=DEV)
    for window in (None, 100):
        assert torch.equal(cuda_lib.prefill_packed(q, k, v, seg, window=window),
                           cuda_lib.prefill(q, k, v, window=window))


@pytest.mark.parametrize("d", [128, 96])
def test_prefill_packed_invalid_start_zeroes_that_row(cuda_lib, d):
    B, Hq, Hkv, T = 1, 4, 2, 260
    q, k, v = synthetic.qkv_prefill(B, Hq, Hkv, T, d, seed=53, std=0.5)
    seg = packed_starts(B, T, 70, seed=53)
    good = seg.copy()
    seg[0, 5] = 6        # after the cell itself
    seg[0, 200] = -1     # negative
    want = oracle.prefill(f64(q), f64(k), f64(v), seg_start=good.astype(np.int64))
    want[0, :, [5, 200]] = 0.0
    st = cuda_lib.new_status(DEV)
    o = cuda_lib.prefill_packed(q.to(DEV), k.to(DEV), v.to(DEV),
                                torch.from_numpy(seg).to(DEV), status=st)
    assert int(st.item()) == 12
    assert torch.all(o[0, :, 5] == 0) and torch.all(o[0, :, 200] == 0)
    assert_close(o, want, torch.bfloat16, "packed with two invalid starts")
