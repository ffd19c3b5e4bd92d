"""The decode workspace contract and back-to-back (programmatically
dependent) launches of the split-K decode.

The workspace holds the arrival counters of the split lanes at a fixed place
for every shape; a call finds them zero and leaves them zero, so one
zero-filled workspace serves any sequence of calls of any shapes without
clearing.  The split kernel is launched as a programmatic dependent of the
previous kernel on the stream: it sets up while that kernel drains and waits
for it before touching memory.  These tests check that:
  - the counter region is zero after calls of several shapes and kinds;
  - a workspace reused across shapes (A, B, A, B) gives bit for bit the
    result of a fresh workspace;
  - calls issued back to back with no host synchronisation, directly and
    replayed from one CUDA graph, give bit for bit the results of the same
    calls issued one at a time, and match the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, f64
from grouped_query_attention_03_b200 import synthetic

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
COUNTER_BYTES = (1024 + 1) * 4   # split-lane counters + the lengths-read count

SHAPES = [
    # (B, Hq, Hkv, C, d, lengths, window)
    (8, 32, 8, 8001, 128, [8001] * 8, None),
    (64, 8, 1, 8193, 128, None, None),            # ragged MQA lengths
    (1, 32, 8, 5000, 128, [5000], 4096),          # windowed long cache
    (3, 16, 2, 3000, 64, [2999, 17, 1500], 700),  # d = 64
]


def _shape_inputs(i):
    B, Hq, Hkv, C, d, lens, window = SHAPES[i]
    if lens is None:
        lens = synthetic.lengths_uniform(B, 1, C, 3).tolist()
    q, kc, vc = synthetic.decode_inputs(B, Hq, Hkv, C, d, 40 + i)
    return q, kc, vc, lens, window


def _big_workspace():
    need = 0
    for i, (B, Hq, Hkv, C, d, _, _) in enumerate(SHAPES):
        from grouped_query_attention_03_b200 import gqa
        need = max(need, gqa.decode_workspace_bytes(torch.bfloat16, B, Hq, Hkv, C, d))
    return torch.zeros(need, dtype=torch.uint8, device=DEV)


def test_counters_are_left_zero(cuda_lib):
    torch.cuda.set_device(DEV)
    ws = _big_workspace()
    st = cuda_lib.new_status(DEV)
    for i in range(len(SHAPES)):
        q, kc, vc, lens, window = _shape_inputs(i)
        qd, kd, vd = q.to(DEV), kc.to(DEV), vc.to(DEV)
        lt = torch.tensor(lens, dtype=torch.int32, device=DEV)
        cuda_lib.decode(qd, kd, vd, lt, window=window, workspace=ws, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert not torch.any(ws[:COUNTER_BYTES]), f"decode shape {i} left counters set"
        # the fused step on the same cache (one cell of room needed)
        B, Hkv, C, d = kd.shape
        lt2 = torch.tensor([min(n, C - 1) for n in lens], dtype=torch.int32, device=DEV)
        kn = synthetic.normal((B, Hkv, 1, d), 50 + i, offset=14).to(DEV)
        vn = synthetic.normal((B, Hkv, 1, d), 50 + i, offset=15).to(DEV)
        cuda_lib.decode_append(qd, kd, vd, kn, vn, lt2, window=window, workspace=ws, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert not torch.any(ws[:COUNTER_BYTES]), f"decode_append shape {i} left counters set"


def test_workspace_reused_across_shapes_without_clearing(cuda_lib):
    torch.cuda.set_device(DEV)
    shared = _big_workspace()
    st = cuda_lib.new_status(DEV)
    inputs = [_shape_inputs(i) for i in range(len(SHAPES))]
    dev_in = [(q.to(DEV), kc.to(DEV), vc.to(DEV),
               torch.tensor(lens, dtype=torch.int32, device=DEV), window)
              for q, kc, vc, lens, window in inputs]
    fresh = []
    for qd, kd, vd, lt, window in dev_in:
        fresh.append(cuda_lib.decode(qd, kd, vd, lt, window=window, status=st))
    for rnd in range(2):
        for i in (0, 1, 2, 3, 1, 0, 3, 2):
            qd, kd, vd, lt, window = dev_in[i]
            o = cuda_lib.decode(qd, kd, vd, lt, window=window, workspace=shared, status=st)
            torch.cuda.synchronize()
            assert int(st.item()) == 0
            assert torch.equal(o, fresh[i]), f"round {rnd} shape {i}"


def test_back_to_back_calls_match_one_at_a_time(cuda_lib):
    """Fused steps of alternating shapes, issued with no host
    synchronisation (each split kernel a programmatic dependent of the one
    before), then the same steps replayed from one CUDA graph: both give the
    bits of the same steps issued one at a time, and match the oracle."""
    torch.cuda.set_device(DEV)
    steps = 6
    cases = []
    for i in (0, 2, 3):
        q, kc, vc, lens, window = _shape_inputs(i)
        B, Hkv, C, d = kc.shape
        C2 = C + steps + 1
        kc2 = torch.cat([kc, synthetic.normal((B, Hkv, steps + 1, d), 60 + i, offset=16)], 2)
        vc2 = torch.cat([vc, synthetic.normal((B, Hkv, steps + 1, d), 60 + i, offset=17)], 2)
        kn = synthetic.normal((steps, B, Hkv, 1, d), 70 + i, offset=14)
        vn = synthetic.normal((steps, B, Hkv, 1, d), 70 + i, offset=15)
        qs = synthetic.normal((steps,) + tuple(q.shape), 80 + i, offset=11)
        lens0 = [min(n, C) for n in lens]
        cases.append(dict(q=qs, kc=kc2, vc=vc2, kn=kn, vn=vn, lens=lens0, window=window, C=C2))

    def run(mode):
        ws = _big_workspace()
        st = cuda_lib.new_status(DEV)
        dev = []
        for c in cases:
            dev.append(dict(q=c["q"].to(DEV), kc=c["kc"].to(DEV), vc=c["vc"].to(DEV),
                            kn=c["kn"].to(DEV), vn=c["vn"].to(DEV),
                            lt=torch.tensor(c["lens"], dtype=torch.int32, device=DEV),
                            o=torch.zeros((steps,) + tuple(c["q"].shape[1:]),
                                          dtype=torch.bfloat16, device=DEV)))
        torch.cuda.synchronize()

        def issue(sync):
            for s in range(steps):
                for c, t in zip(cases, dev):
                    cuda_lib.decode_append(t["q"][s], t["kc"], t["vc"], t["kn"][s], t["vn"][s],
                                           t["lt"], window=c["window"], out=t["o"][s],
                                           workspace=ws, status=st)
                    if sync:
                        torch.cuda.synchronize()
        if mode == "graph":
            g = torch.cuda.CUDAGraph()
            s = torch.cuda.Stream(DEV)
            s.wait_stream(torch.cuda.current_stream(DEV))
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, stream=s):
                    issue(False)
            torch.cuda.current_stream(DEV).wait_stream(s)
            g.replay()
        else:
            issue(mode == "sync")
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert not torch.any(ws[:COUNTER_BYTES])
        return dev

    ref, b2b, graph = run("sync"), run("eager"), run("graph")
    for ci, (c, a, b, g) in enumerate(zip(cases, ref, b2b, graph)):
        for key in ("o", "kc", "vc", "lt"):
            assert torch.equal(a[key], b[key]), f"case {ci}: {key} back to back"
            assert torch.equal(a[key], g[key]), f"case {ci}: {key} graph"
        k64, v64, lens = f64(c["kc"]), f64(c["vc"]), c["lens"]
        for s in range(steps):
            k64, v64, lens64 = oracle.cache_append(k64, v64, f64(c["kn"][s]), f64(c["vn"][s]), lens)
            want = oracle.decode(f64(c["q"][s]), k64, v64, lens64, window=c["window"])
            assert_close(a["o"][s], want, torch.bfloat16, f"case {ci} step {s}")
            lens = lens64.tolist()
