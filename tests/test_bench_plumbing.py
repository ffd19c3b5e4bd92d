"""Host-side pieces of bench.py that need no GPU.

The bench reports ncu's DRAM traffic for a kernel only while the kernel's
code is the code that was captured; the check hashes the sources without
their comments, so a comment edit keeps the figure and a code edit drops it.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_strip_comments_keeps_code_and_literals():
    src = ('int a = 1;  // trailing\n'
           '/* block\n   comment */ float b = 2.f;\n'
           '\n'
           'const char *s = "x // not a comment /* nor this */";\n'
           "char c = '/';  /* c */\n"
           'asm volatile("fence.acq_rel.gpu;" ::: "memory");\n')
    assert bench.strip_comments(src) == (
        'int a = 1;\n'
        ' float b = 2.f;\n'
        'const char *s = "x // not a comment /* nor this */";\n'
        "char c = '/';\n"
        'asm volatile("fence.acq_rel.gpu;" ::: "memory");')


def test_digest_ignores_comments_but_not_code():
    base = ["int f(int x) {\n  return x + 1;  // add one\n}\n"]
    reworded = ["// helper\nint f(int x) {\n  return x + 1;  /* one more */\n}\n\n"]
    changed = ["int f(int x) {\n  return x + 2;  // add one\n}\n"]
    assert bench.source_digest(base) == bench.source_digest(reworded)
    assert bench.source_digest(base) != bench.source_digest(changed)


def test_traffic_only_for_the_captured_configuration():
    # another window or KV-head count than the captured run: no figure
    assert bench.captured_traffic("decode_b8_n8000", "decode", 512, None) is None
    assert bench.captured_traffic("decode_b8_n8000", "decode", None, 1) is None
    assert bench.captured_traffic("no_such_workload", "decode", None, None) is None
    # the GQA and MHA prefills are captured separately (different kernels)
    gqa_pf = bench.captured_traffic("swa_t32768", "prefill", 4096, None)
    mha_pf = bench.captured_traffic("swa_t32768", "prefill", 4096, 32)
    assert gqa_pf is not None and mha_pf is not None and mha_pf > gqa_pf
    assert bench.captured_traffic("swa_t32768", "prefill", 4096, 16) is None
    # the ragged endpoints are captured separately
    mqa = bench.captured_traffic("decode_ragged", "decode", None, 1)
    mha = bench.captured_traffic("decode_ragged", "decode", None, 8)
    assert mqa is not None and mha is not None and mha > 5 * mqa


def test_captured_traffic_describes_the_current_kernels():
    """Every recorded capture matches the kernels' current code (so the bench
    reports it), and each is within 8 % above the launch's algorithmic bytes
    (no wasted re-reads) -- the algorithmic bytes computed here from the
    workload shapes."""
    for e in bench.CAPTURED_TRAFFIC:
        assert bench.captured_traffic(e["workload"], e["phase"], e["window"], e["hkv"]) == e["bytes"]
    alg = {("decode_b8_n8000", None): 2 * 8 * 8 * 8001 * 128 * 2,
           ("swa_t32768", None): 2 * 8 * 4096 * 128 * 2}
    for (wl, hkv), b in alg.items():
        got = bench.captured_traffic(wl, "decode", None, hkv)
        assert b <= got <= 1.08 * b, (wl, got, b)
    # prefill: q, k and v are read once (o may still sit in L2 at the end)
    MB = 1 << 20
    pf_in = {("prefill_b4_t1024", None, None): 4 * (8 + 2 + 2) * 1024 * 64 * 2,
             ("prefill_b4_t1024", 256, None): 4 * (8 + 2 + 2) * 1024 * 64 * 2,
             ("swa_t32768", 4096, None): (32 + 8 + 8) * 32768 * 128 * 2,
             ("swa_t32768", 4096, 32): (32 + 32 + 32) * 32768 * 128 * 2}
    for (wl, win, hkv), b in pf_in.items():
        got = bench.captured_traffic(wl, "prefill", win, hkv)
        assert b <= got <= 1.08 * (b + (32 * 32768 * 128 * 2 if wl == "swa_t32768" else 0)) + MB, (wl, got, b)


def test_prefill_cpu_sample_rows_are_prefill_rows():
    """The prefill CPU baseline times the oracle's multi-token decode of the
    last rows of one KV group over the whole prompt; those are the same rows
    of the oracle's prefill, and the sample's FLOPs count their keys."""
    import types

    import numpy as np
    import torch

    import oracle
    from grouped_query_attention_03_b200 import synthetic

    B, Hq, Hkv, T, d, window = 1, 4, 2, 64, 8, 16
    q, k, v = synthetic.qkv_prefill(B, Hq, Hkv, T, d, 7)
    r, t_new = Hq // Hkv, 24
    f64 = lambda t: t.float().double().numpy()
    full = oracle.prefill(f64(q), f64(k), f64(v), window=window)
    tail = oracle.decode_multi(f64(q[:1, :r, T - t_new:]), f64(k[:1, :1]), f64(v[:1, :1]),
                               np.array([T]), window=window)
    assert np.array_equal(tail, full[:1, :r, T - t_new:])
    w = types.SimpleNamespace(Hq=Hq, T=T, d=d)
    step = types.SimpleNamespace(w=w, Hkv=Hkv, window=window, q=q, k=k, v=v)
    try:
        res = bench.oracle_prefill_sample(step, 0.05)
    finally:
        oracle.set_threads(1)
    assert res["kind"] == "oracle" and res["unit"] == "TFLOP/s" and res["value"] > 0
    assert res["cores"] >= 1 and "query rows of one KV group" in res["sample"]


def test_pass_stats_median_and_spread():
    st = bench.pass_stats([5.0, 1.0, 3.0, 2.0, 4.0])
    assert st["passes"] == 5 and st["median_ms"] == 3.0
    assert st["min_ms"] == 1.0 and st["max_ms"] == 5.0
    assert st["p10_ms"] == 1.0 and st["p90_ms"] == 5.0


def test_pass_count_covers_minimum_passes_and_time():
    import torch
    cpu = torch.device("cpu")
    # a 1 ms pass: 30 passes are 30 ms, so half a second needs 500
    assert bench.n_passes(1.0, cpu, min_passes=30, min_seconds=0.5) == 500
    # a 100 ms pass: the 30-pass minimum decides
    assert bench.n_passes(100.0, cpu, min_passes=30, min_seconds=0.5) == 30
    # never more than the cap
    assert bench.n_passes(1e-6, cpu, min_passes=30, min_seconds=10.0) == 3000


def test_copy_count_keeps_steps_out_of_l2():
    """Inputs above the 126 MB L2 need no copies; smaller ones get enough
    copies that the copies together hold more than twice the L2."""
    assert bench.n_copies(262_000_000) == 1
    assert bench.n_copies(127_000_000) == 1
    for b in (16_777_216, 10_485_760, 1_000_000):
        n = bench.n_copies(b)
        assert n * b > 2 * bench.L2_BYTES or n == 64
        assert (n - 2) * b <= 2 * bench.L2_BYTES  # not more than one copy beyond that


def test_loop_bytes_count_each_copy_growth():
    """Call i of the successive-calls loop runs on copy i mod NL, which has
    grown by i // NL cells; with a window the bytes stop growing."""
    import numpy as np
    from grouped_query_attention_03_b200 import workloads
    s = bench.DecodeStep.__new__(bench.DecodeStep)
    s.w, s.Hkv, s.window, s.cached = workloads.DECODE_B8_N8000, 8, None, [8000] * 8
    s.qo_bytes, s.write_bytes, s.NL = 1000, 100, 1
    per_cell = 2 * 8 * 8 * 128 * 2       # K+V bytes of one more cell in every sequence
    base = s.step_bytes_at(0)
    assert s.loop_bytes(3) == 3 * base + (0 + 1 + 2) * per_cell
    s.NL = 2                             # calls 0,1 at +0 cells, 2,3 at +1, 4 at +2
    assert s.loop_bytes(5) == 5 * base + (0 + 0 + 1 + 1 + 2) * per_cell
    s.window, s.cached = 4096, [32768]   # window-capped: every call reads 4096 cells
    s.w = workloads.SWA_T32768
    assert s.kv_bytes_at(0) == s.kv_bytes_at(63) == 2 * 8 * 4096 * 128 * 2
    assert np.isclose(s.loop_bytes(64), 64 * s.step_bytes_at(0))
