"""gqa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a host that only lends this library pointers from its own
fixed pool, a latency-critical loop that cannot take cudaMalloc's implicit
synchronisation, a foreign-language caller holding only device pointers)
cannot supply gqa_decode's workspace.  gqa_decode_noalloc runs the same
kernels with the library's fixed device array as the workspace.  This test
calls it through the C ABI (ctypes), twice in a row on different inputs so
the second call starts from the first call's leftover scratch contents, and
checks each result bit for bit against gqa_decode with its own workspace
(the decode is reproducible bit for bit, so any stale scratch value that
leaked into a result would show) and against the fp64 oracle within the
bf16 tolerance of the parity tests.  It also checks that sizes whose
workspace exceeds the fixed array are refused before any work is queued.

The file is named so pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, f64
from grouped_query_attention_03_b200 import synthetic

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
GQA_BF16, GQA_ERR_WORKSPACE = 1, 8


def _noalloc(L, q, kc, vc, o, lens, window, status):
    B, Hq, d = q.shape
    Hkv, C = kc.shape[1], kc.shape[2]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.gqa_decode_noalloc(
        GQA_BF16, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()),
        ctypes.c_void_p(vc.data_ptr()), ctypes.c_void_p(o.data_ptr()),
        ctypes.c_void_p(lens.data_ptr()), B, Hq, Hkv, C, d,
        -1 if window is None else window, d ** -0.5,
        ctypes.c_void_p(status.data_ptr()), stream)


def test_noalloc_decode_matches_workspace_decode_and_oracle(cuda_lib):
    L = cuda_lib.lib()
    cases = [
        # 8 sequences x 32 query heads over 8 KV heads, 8001 keys each
        dict(B=8, Hq=32, Hkv=8, C=8001, d=128, lens=[8001] * 8, window=None, seed=1),
        # MQA endpoint with ragged lengths and a window
        dict(B=16, Hq=8, Hkv=1, C=3000, d=128,
             lens=synthetic.lengths_uniform(16, 0, 3000, 5).tolist(), window=700, seed=2),
    ]
    torch.cuda.set_device(DEV)
    for c in cases:
        q, kc, vc = synthetic.decode_inputs(c["B"], c["Hq"], c["Hkv"], c["C"], c["d"], c["seed"])
        qd, kd, vd = (t.to(DEV) for t in (q, kc, vc))
        lens = torch.tensor(c["lens"], dtype=torch.int32, device=DEV)
        want = cuda_lib.decode(qd, kd, vd, lens, window=c["window"])
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        got = torch.full_like(qd, float("nan"))
        rc = _noalloc(L, qd, kd, vd, got, lens, c["window"], status)
        torch.cuda.synchronize()
        assert rc == 0 and int(status.item()) == 0
        assert torch.equal(got, want), f"noalloc differs from gqa_decode: {c}"
        ref = oracle.decode(f64(q), f64(kc), f64(vc), np.array(c["lens"]), window=c["window"])
        assert_close(got, ref, torch.bfloat16, f"noalloc vs oracle {c}")


def test_noalloc_refuses_sizes_beyond_the_fixed_scratch(cuda_lib):
    L = cuda_lib.lib()
    B, Hq, Hkv, C, d = 4096, 64, 8, 1, 128
    need = L.gqa_decode_workspace_bytes(GQA_BF16, B, Hq, Hkv, C, d)
    assert need > cuda_lib.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, Hq, d), dtype=torch.bfloat16, device=DEV)
    kc = torch.zeros((B, Hkv, C, d), dtype=torch.bfloat16, device=DEV)
    lens = torch.ones(B, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = torch.full_like(q, 7.0)
    assert _noalloc(L, q, kc, kc, o, lens, None, status) == GQA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and torch.all(o == 7.0)
