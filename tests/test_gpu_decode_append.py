"""Fused append + decode (gqa_decode_append) against the oracle.

The expected result is the oracle's cache append of the step's row followed
by the oracle's decode ("Share key/value heads and make context explicit",
section "Extend the existing full and cached attention paths": the candidate
row takes part in the scores, then is committed; a refused append changes
nothing).  The written cache is compared bit for bit (a copy), the output
within the tolerances of ``parity.py``.
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


def _inputs(B, Hq, Hkv, C, d, seed, dtype):
    q, kc, vc = synthetic.decode_inputs(B, Hq, Hkv, C, d, seed, dtype=dtype)
    kn = synthetic.normal((B, Hkv, 1, d), seed, 1.0, dtype, offset=14)
    vn = synthetic.normal((B, Hkv, 1, d), seed, 1.0, dtype, offset=15)
    return q, kc, vc, kn, vn


def _step(cuda_lib, q, kc, vc, kn, vn, lens, window):
    """One fused step on the GPU; returns (o, status, lens after)."""
    lt = torch.tensor(lens, dtype=torch.int32, device=DEV)
    st = cuda_lib.new_status(DEV)
    o = torch.full_like(q, float("nan"))
    cuda_lib.decode_append(q, kc, vc, kn, vn, lt, window=window, out=o, status=st)
    return o, int(st.item()), lt.tolist()


def _case(cuda_lib, dtype, B, Hq, Hkv, C, d, lens, window, seed):
    q, kc, vc, kn, vn = _inputs(B, Hq, Hkv, C, d, seed, dtype)
    kc2, vc2, lens2 = oracle.cache_append(f64(kc), f64(vc), f64(kn), f64(vn), lens)
    want = oracle.decode(f64(q), kc2, vc2, lens2, window=window)
    qd, kd, vd, knd, vnd = [t.to(DEV) for t in (q, kc, vc, kn, vn)]
    o, status, after = _step(cuda_lib, qd, kd, vd, knd, vnd, lens, window)
    assert status == 0
    assert after == lens2.tolist()
    np.testing.assert_array_equal(f64(kd), kc2)
    np.testing.assert_array_equal(f64(vd), vc2)
    return assert_close(o, want, dtype, f"decode_append B{B} Hq{Hq} Hkv{Hkv} C{C} d{d} w{window}")


FUSED_CASES = [
    # (B, Hq, Hkv, C, d, lens before the step, window)
    (8, 32, 8, 8001, 128, [8000] * 8, None),       # the B=8, n=8001 decode shape
    (3, 4, 2, 10, 128, [0, 1, 9], None),           # empty cache: output = v_new
    (2, 8, 1, 700, 64, [699, 128], None),          # MQA, d=64
    (2, 8, 8, 700, 64, [512, 63], 100),            # MHA, window
    (1, 6, 2, 300, 128, [299], 1),                 # window 1: output = v_new
    (1, 12, 1, 2000, 128, [1998], None),           # r=12 (tile rows padded to 16)
    (2, 16, 1, 999, 128, [998, 2], 500),           # r=16
    (1, 64, 2, 600, 128, [599], None),             # r=32: two virtual lanes per KV head
    (1, 32, 8, 5000, 128, [4999], 4096),           # window inside a long cache
    (64, 4, 1, 40, 128, list(range(0, 39)) + [39] * 25, None),  # many short lanes
    (4100, 2, 1, 4, 128, [b % 4 for b in range(4100)], None),  # lengths not cached: CUDA cores
    (2, 4, 2, 50, 96, [49, 3], None),              # d=96: CUDA-core path
    (2, 3, 1, 50, 32, [16, 49], 5),                # d=32, odd group
    (2, 8, 2, 300, 64, [299, 5], None),            # r=4, d=64 (transposed products)
    (1, 48, 2, 400, 128, [399], 200),              # r=24: sub-lanes of 16 and 8 heads
]


@pytest.mark.parametrize("case", FUSED_CASES,
                         ids=lambda c: f"B{c[0]}Hq{c[1]}Hkv{c[2]}C{c[3]}d{c[4]}w{c[6]}")
def test_decode_append_cases(cuda_lib, case):
    B, Hq, Hkv, C, d, lens, window = case
    _case(cuda_lib, torch.bfloat16, B, Hq, Hkv, C, d, lens, window, seed=C + B + 1)


def test_decode_append_fp32(cuda_lib):
    _case(cuda_lib, torch.float32, 3, 8, 2, 300, 64, [299, 0, 150], None, seed=21)
    _case(cuda_lib, torch.float32, 2, 4, 4, 100, 128, [99, 40], 16, seed=22)


def test_decode_append_matches_unfused_bitwise(cuda_lib):
    """Same kernel decomposition either way, so the fused step equals
    gqa_cache_append followed by gqa_decode bit for bit."""
    B, Hq, Hkv, C, d = 4, 32, 8, 3000, 128
    lens = [2999, 1500, 0, 2048]
    q, kc, vc, kn, vn = [t.to(DEV) for t in _inputs(B, Hq, Hkv, C, d, 5, torch.bfloat16)]
    kc_b, vc_b = kc.clone(), vc.clone()
    o_fused, status, after = _step(cuda_lib, q, kc, vc, kn, vn, lens, None)
    assert status == 0
    lt = torch.tensor(lens, dtype=torch.int32, device=DEV)
    st = cuda_lib.new_status(DEV)
    cuda_lib.cache_append(kc_b, vc_b, kn, vn, lt, status=st)
    o_two = cuda_lib.decode(q, kc_b, vc_b, lt, status=st)
    assert int(st.item()) == 0 and lt.tolist() == after
    assert torch.equal(kc, kc_b) and torch.equal(vc, vc_b)
    assert torch.equal(o_fused, o_two)


@pytest.mark.parametrize("d", [128, 96])
def test_decode_append_refuses_all_or_nothing(cuda_lib, d):
    """A full cache anywhere refuses the whole step: status CAPACITY, zero
    output, caches and lengths unchanged."""
    B, Hq, Hkv, C = 3, 8, 2, 64
    q, kc, vc, kn, vn = [t.to(DEV) for t in _inputs(B, Hq, Hkv, C, d, 7, torch.bfloat16)]
    kc0, vc0 = kc.clone(), vc.clone()
    for lens in ([10, 64, 3], [5, -1, 0]):
        o, status, after = _step(cuda_lib, q, kc, vc, kn, vn, lens, None)
        assert status == 5
        assert after == lens
        assert torch.all(o == 0)
        assert torch.equal(kc, kc0) and torch.equal(vc, vc0)


def test_decode_append_steps_track_oracle(cuda_lib):
    """Twelve fused steps in a row (the window slides past the start of the
    cache), each against the oracle's append + decode."""
    B, Hq, Hkv, C, d, window = 2, 16, 4, 400, 128, 300
    lens = [290, 100]
    _, kc, vc = synthetic.decode_inputs(B, Hq, Hkv, C, d, 31)
    kd, vd = kc.to(DEV), vc.to(DEV)
    k64, v64 = f64(kc), f64(vc)
    lt = torch.tensor(lens, dtype=torch.int32, device=DEV)
    st = cuda_lib.new_status(DEV)
    ws = cuda_lib.decode_workspace(torch.empty((B, Hq, d), dtype=torch.bfloat16, device=DEV), kd)
    for step in range(12):
        q = synthetic.normal((B, Hq, d), 100 + step, 1.0, torch.bfloat16, offset=11)
        kn = synthetic.normal((B, Hkv, 1, d), 100 + step, 1.0, torch.bfloat16, offset=14)
        vn = synthetic.normal((B, Hkv, 1, d), 100 + step, 1.0, torch.bfloat16, offset=15)
        k64, v64, lens64 = oracle.cache_append(k64, v64, f64(kn), f64(vn), lens)
        want = oracle.decode(f64(q), k64, v64, lens64, window=window)
        o = cuda_lib.decode_append(q.to(DEV), kd, vd, kn.to(DEV), vn.to(DEV), lt,
                                   window=window, workspace=ws, status=st)
        assert int(st.item()) == 0
        lens = lens64.tolist()
        assert lt.tolist() == lens
        assert_close(o, want, torch.bfloat16, f"step {step}")
    np.testing.assert_array_equal(f64(kd), k64)
    np.testing.assert_array_equal(f64(vd), v64)


def test_decode_append_is_bitwise_reproducible(cuda_lib):
    """The same calls from the same cache give the same bits.  Which CTA
    finishes a lane last, and so merges it (alone, with 224 threads, or next
    to a second lane, with 128 or 96), is a matter of timing; the merge's
    arithmetic must not depend on it.  Ragged MQA lengths (64 sequences,
    uniform in [1, 8192]) give many lanes split over two to five CTAs."""
    B, Hq, Hkv, d, calls = 64, 8, 1, 128, 100
    lens = (synthetic.lengths_uniform(B, 1, 8192, 3)).tolist()
    C = max(lens) + calls + 1
    _, kc, vc = synthetic.decode_inputs(B, Hq, Hkv, C, d, 3)
    kd0, vd0 = kc.to(DEV), vc.to(DEV)
    qs = synthetic.normal((calls, B, Hq, d), 4, 1.0, torch.bfloat16, offset=11).to(DEV)
    kn = synthetic.normal((calls, B, Hkv, 1, d), 4, 1.0, torch.bfloat16, offset=14).to(DEV)
    vn = synthetic.normal((calls, B, Hkv, 1, d), 4, 1.0, torch.bfloat16, offset=15).to(DEV)
    runs = []
    for _ in range(2):
        kd, vd = kd0.clone(), vd0.clone()
        lt = torch.tensor(lens, dtype=torch.int32, device=DEV)
        st = cuda_lib.new_status(DEV)
        ws = cuda_lib.decode_workspace(qs[0], kd)
        outs = torch.empty_like(qs)
        for i in range(calls):
            cuda_lib.decode_append(qs[i], kd, vd, kn[i], vn[i], lt, out=outs[i], workspace=ws,
                                   status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        runs.append((outs, kd, vd, lt))
    (o1, k1, v1, l1), (o2, k2, v2, l2) = runs
    assert torch.equal(l1, l2) and torch.equal(k1, k2) and torch.equal(v1, v2)
    differ = [i for i in range(calls) if not torch.equal(o1[i], o2[i])]
    assert differ == [], f"calls whose outputs differ between identical runs: {differ}"
