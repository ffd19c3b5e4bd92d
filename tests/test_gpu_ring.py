"""Rolling-buffer (ring) cache on the GPU against the oracle.

"Share key/value heads and make context explicit", section "Relate shared
heads to local context": a rolling buffer overwrites old KV entries.  Here a
ring of W slots holds position p in slot p mod W; gqa_ring_append loads
positions into it and gqa_ring_decode_append runs the decode step (the
step's row appended in the same kernel).  Expected values come from the
oracle's ring_append and ring_decode, which are pinned bit for bit to the
windowed decode over the all-prefix cache.
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


def _run_steps(cuda_lib, dtype, B, Hq, Hkv, W, d, prompt, steps, seed):
    """Load `prompt` positions per sequence into a ring, then run `steps`
    fused decode steps; compare every step and the final ring."""
    kr = torch.zeros((B, Hkv, W, d), dtype=dtype)
    vr = torch.zeros_like(kr)
    krd, vrd = kr.to(DEV), vr.to(DEV)
    k64, v64 = f64(kr), f64(vr)
    lens = np.zeros(B, dtype=np.int64)
    lt = torch.zeros(B, dtype=torch.int32, device=DEV)
    st = cuda_lib.new_status(DEV)
    if prompt:
        kp = synthetic.normal((B, Hkv, prompt, d), seed, 1.0, dtype, offset=61)
        vp = synthetic.normal((B, Hkv, prompt, d), seed, 1.0, dtype, offset=62)
        k64, v64, lens = oracle.ring_append(k64, v64, f64(kp), f64(vp), lens)
        cuda_lib.ring_append(krd, vrd, kp.to(DEV), vp.to(DEV), lt, status=st)
        assert int(st.item()) == 0 and lt.tolist() == lens.tolist()
        np.testing.assert_array_equal(f64(krd), k64)
    ws = cuda_lib.decode_workspace(torch.empty((B, Hq, d), dtype=dtype, device=DEV), krd)
    for i in range(steps):
        q = synthetic.normal((B, Hq, d), seed + 100 + i, 1.0, dtype, offset=63)
        kn = synthetic.normal((B, Hkv, 1, d), seed + 100 + i, 1.0, dtype, offset=64)
        vn = synthetic.normal((B, Hkv, 1, d), seed + 100 + i, 1.0, dtype, offset=65)
        k64, v64, lens = oracle.ring_append(k64, v64, f64(kn), f64(vn), lens)
        want = oracle.ring_decode(f64(q), k64, v64, lens)
        o = cuda_lib.ring_decode_append(q.to(DEV), krd, vrd, kn.to(DEV), vn.to(DEV), lt,
                                        workspace=ws, status=st)
        assert int(st.item()) == 0
        assert lt.tolist() == lens.tolist()
        assert_close(o, want, dtype, f"ring step {i} W{W}")
    np.testing.assert_array_equal(f64(krd), k64)
    np.testing.assert_array_equal(f64(vrd), v64)


RING_CASES = [
    # (dtype, B, Hq, Hkv, W, d, prompt, steps)
    (torch.bfloat16, 2, 32, 8, 300, 128, 700, 6),    # prompt longer than the ring
    (torch.bfloat16, 2, 8, 2, 1000, 128, 100, 4),    # not wrapped yet
    (torch.bfloat16, 3, 8, 1, 64, 64, 60, 9),        # MQA, wraps during the steps
    (torch.bfloat16, 1, 8, 8, 129, 128, 0, 5),       # MHA, empty ring at the start
    (torch.bfloat16, 1, 64, 2, 200, 128, 450, 3),    # group of 32: two virtual lanes
    (torch.bfloat16, 2, 4, 2, 33, 96, 50, 4),        # d=96: CUDA cores
    (torch.float32, 2, 4, 2, 40, 64, 90, 4),         # fp32: CUDA cores
]


@pytest.mark.parametrize("case", RING_CASES, ids=lambda c: (
    f"{'f32' if c[0] == torch.float32 else 'bf16'}-B{c[1]}Hq{c[2]}Hkv{c[3]}W{c[4]}d{c[5]}"
    f"p{c[6]}"))
def test_ring_steps(cuda_lib, case):
    dtype, B, Hq, Hkv, W, d, prompt, steps = case
    _run_steps(cuda_lib, dtype, B, Hq, Hkv, W, d, prompt, steps, seed=W + prompt)


def test_ring_many_sequences_take_the_cuda_core_route(cuda_lib):
    """More sequences than the split kernel caches lengths for."""
    _run_steps(cuda_lib, torch.bfloat16, 4100, 2, 1, 3, 128, 5, 2, seed=7)


def test_ring_matches_windowed_decode_over_the_whole_prefix(cuda_lib):
    """The same tokens through gqa_decode_append with window W over an
    all-prefix cache: the same keys, so the outputs agree to rounding."""
    B, Hq, Hkv, W, d, n = 2, 16, 4, 256, 128, 900
    kp = synthetic.normal((B, Hkv, n, d), 3, 1.0, torch.bfloat16, offset=61).to(DEV)
    vp = synthetic.normal((B, Hkv, n, d), 3, 1.0, torch.bfloat16, offset=62).to(DEV)
    kr = torch.zeros((B, Hkv, W, d), dtype=torch.bfloat16, device=DEV)
    vr = torch.zeros_like(kr)
    kc = torch.zeros((B, Hkv, n + 1, d), dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    lr = torch.zeros(B, dtype=torch.int32, device=DEV)
    lc = torch.zeros(B, dtype=torch.int32, device=DEV)
    cuda_lib.ring_append(kr, vr, kp, vp, lr)
    cuda_lib.cache_append(kc, vc, kp, vp, lc)
    q = synthetic.normal((B, Hq, d), 4, 1.0, torch.bfloat16, offset=63).to(DEV)
    kn = synthetic.normal((B, Hkv, 1, d), 4, 1.0, torch.bfloat16, offset=64).to(DEV)
    vn = synthetic.normal((B, Hkv, 1, d), 4, 1.0, torch.bfloat16, offset=65).to(DEV)
    a = cuda_lib.ring_decode_append(q, kr, vr, kn, vn, lr)
    b = cuda_lib.decode_append(q, kc, vc, kn, vn, lc, window=W)
    assert lr.tolist() == lc.tolist() == [n + 1] * B
    assert float((a.float() - b.float()).abs().max()) <= 1e-2


@pytest.mark.parametrize("d", [128, 96])
def test_ring_refuses_negative_lengths(cuda_lib, d):
    B, Hq, Hkv, W = 2, 8, 2, 16
    kr = synthetic.normal((B, Hkv, W, d), 9, 1.0, torch.bfloat16, offset=61).to(DEV)
    vr = kr.clone()
    k0, v0 = kr.clone(), vr.clone()
    q = synthetic.normal((B, Hq, d), 9, 1.0, torch.bfloat16, offset=63).to(DEV)
    kn = synthetic.normal((B, Hkv, 1, d), 9, 1.0, torch.bfloat16, offset=64).to(DEV)
    lt = torch.tensor([5, -1], dtype=torch.int32, device=DEV)
    st = cuda_lib.new_status(DEV)
    o = torch.full_like(q, 3.0)
    cuda_lib.ring_decode_append(q, kr, vr, kn, kn, lt, out=o, status=st)
    assert int(st.item()) == 5
    assert torch.all(o == 0) and lt.tolist() == [5, -1]
    assert torch.equal(kr, k0) and torch.equal(vr, v0)
    st2 = cuda_lib.new_status(DEV)
    cuda_lib.ring_append(kr, vr, kn, kn, lt, status=st2)
    assert int(st2.item()) == 5 and torch.equal(kr, k0) and lt.tolist() == [5, -1]
