"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Inputs come from the seeded generators in ``synthetic``; the same rounded
tensors go to both sides.  Tolerances live in ``parity.py``.
"""
import numpy as np
import pytest
import torch

import oracle
import oracle_pins
from parity import assert_close, f64
from grouped_query_attention_03_b200 import synthetic, workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _threads():
    oracle.set_threads(0)
    yield
    oracle.set_threads(1)


def _cuda(*ts):
    return [t.to(DEV) for t in ts]


# ------------------------------------------------------------------ prefill
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_prefill_worked_example(cuda_lib, dtype):
    g = oracle_pins.golden("worked_example.json")
    q, k, v = oracle_pins.worked_example_inputs()
    qt, kt, vt = _cuda(*(torch.from_numpy(np.ascontiguousarray(x)).to(dtype) for x in (q, k, v)))
    for case in g["cases"]:
        o = cuda_lib.prefill(qt, kt, vt, window=case["window"])
        merged = f64(o)[0, :, -1, :].reshape(-1).tolist()
        assert merged == case["last_merged_output"], (dtype, case, merged)


@pytest.mark.parametrize("window", [None, 32])
def test_prefill_fp32_small(cuda_lib, window):
    w = workloads.FP32_SMALL
    q, k, v = synthetic.qkv_prefill(w.B, w.Hq, w.Hkv, w.T, w.d, w.seed, dtype=torch.float32)
    want = oracle.prefill(f64(q), f64(k), f64(v), window=window)
    o = cuda_lib.prefill(*_cuda(q, k, v), window=window)
    assert_close(o, want, torch.float32, f"fp32 prefill w={window}")


@pytest.mark.parametrize("window", [None, 256])
def test_prefill_bf16_b4_t1024(cuda_lib, window):
    w = workloads.PREFILL_B4_T1024
    q, k, v = synthetic.qkv_prefill(w.B, w.Hq, w.Hkv, w.T, w.d, w.seed)
    want = oracle.prefill(f64(q), f64(k), f64(v), window=window)
    o = cuda_lib.prefill(*_cuda(q, k, v), window=window)
    assert_close(o, want, torch.bfloat16, f"bf16 prefill w={window}")


PREFILL_EDGES = [
    # (dtype, B, Hq, Hkv, T, d, window, lens)
    (torch.bfloat16, 1, 4, 1, 1, 64, None, None),
    (torch.bfloat16, 2, 4, 2, 200, 64, None, [200, 77]),
    (torch.bfloat16, 2, 8, 2, 333, 128, 100, [0, 333]),
    (torch.bfloat16, 1, 6, 3, 130, 128, 1, None),
    (torch.bfloat16, 1, 4, 4, 257, 64, 1000, None),
    (torch.bfloat16, 1, 16, 1, 129, 64, 128, [129]),
    (torch.bfloat16, 1, 2, 2, 96, 96, None, None),
    (torch.bfloat16, 2, 6, 2, 300, 128, None, [300, 150]),   # group of 3: one head per CTA
    (torch.bfloat16, 1, 3, 3, 513, 128, 200, None),          # MHA with a window
    (torch.bfloat16, 2, 6, 2, 50, 32, 7, [50, 1]),
    (torch.float32, 1, 3, 1, 65, 40, None, [64]),
    (torch.float32, 2, 8, 4, 31, 256, 5, None),
]


@pytest.mark.parametrize("case", PREFILL_EDGES, ids=lambda c: f"{c[0]}-B{c[1]}Hq{c[2]}Hkv{c[3]}T{c[4]}d{c[5]}w{c[6]}")
def test_prefill_edge_cases(cuda_lib, case):
    dtype, B, Hq, Hkv, T, d, window, lens = case
    q, k, v = synthetic.qkv_prefill(B, Hq, Hkv, T, d, seed=100 + T, dtype=dtype)
    want = oracle.prefill(f64(q), f64(k), f64(v), window=window, seq_lens=lens)
    lens_t = None if lens is None else torch.tensor(lens, dtype=torch.int32, device=DEV)
    status = cuda_lib.new_status(DEV)
    o = torch.full((B, Hq, T, d), float("nan"), dtype=dtype, device=DEV)
    cuda_lib.prefill(*_cuda(q, k, v), window=window, seq_lens=lens_t, out=o, status=status)
    assert int(status.item()) == 0
    assert_close(o, want, dtype, str(case))
    if lens is not None:
        for b, n in enumerate(lens):
            assert torch.all(o[b, :, n:] == 0)


LONG_ONE_HEAD = [
    # (B, Hq, Hkv, T, d, window, lens): odd group sizes run one head per CTA;
    # 65 query tiles per head orders the CTAs head by head
    (2, 4, 4, 8229, 64, None, [8229, 6000]),
    (1, 6, 2, 8229, 128, 1000, None),
]


@pytest.mark.parametrize("case", LONG_ONE_HEAD, ids=lambda c: f"B{c[0]}Hq{c[1]}Hkv{c[2]}T{c[3]}d{c[4]}w{c[5]}")
def test_prefill_long_one_head_sampled_rows(cuda_lib, case):
    """Long prompts on the one-head kernel in its head-by-head CTA order:
    the first 256 rows of every head against the oracle's prefill, 48 seeded
    random rows of every head against the oracle's row-by-row decode, and
    rows past a sequence's length exact zeros."""
    B, Hq, Hkv, T, d, window, lens = case
    q, k, v = synthetic.qkv_prefill(B, Hq, Hkv, T, d, seed=300 + d, std=0.5)
    lens_t = None if lens is None else torch.tensor(lens, dtype=torch.int32, device=DEV)
    status = cuda_lib.new_status(DEV)
    o = torch.full((B, Hq, T, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    cuda_lib.prefill(*_cuda(q, k, v), window=window, seq_lens=lens_t, out=o, status=status)
    assert int(status.item()) == 0
    T0 = 256
    want = oracle.prefill(f64(q[:, :, :T0]), f64(k[:, :, :T0]), f64(v[:, :, :T0]), window=window)
    assert_close(o[:, :, :T0], want, torch.bfloat16, f"first rows {case}")
    n = lens or [T] * B
    rng = np.random.default_rng(T)
    cells = sorted(rng.choice(np.arange(T0, min(n)), size=48, replace=False).tolist())
    k64, v64 = f64(k), f64(v)
    got, want = [], []
    for t in cells:
        want.append(oracle.decode(f64(q[:, :, t]), k64, v64, [t + 1] * B, window=window))
        got.append(f64(o[:, :, t]))
    assert_close(np.stack(got), np.stack(want), torch.bfloat16, f"random rows {case}")
    for b, nb in enumerate(n):
        assert torch.all(o[b, :, nb:] == 0)


def test_prefill_invalid_length_sets_status_and_zeroes(cuda_lib):
    q, k, v = _cuda(*synthetic.qkv_prefill(2, 4, 2, 64, 64, seed=5))
    status = cuda_lib.new_status(DEV)
    lens = torch.tensor([64, 65], dtype=torch.int32, device=DEV)
    o = torch.full_like(q, 3.0)
    cuda_lib.prefill(q, k, v, seq_lens=lens, out=o, status=status)
    assert int(status.item()) == 5
    assert torch.all(o[1] == 0)


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (6, 2)], ids=["mha", "group3"])
def test_prefill_one_head_invalid_and_empty_lengths(cuda_lib, Hq, Hkv):
    """The persistent one-head kernel: a sequence with an invalid length is
    written as zeros and reported, an empty one as zeros, the others exact."""
    B, T, d = 3, 300, 64
    q, k, v = synthetic.qkv_prefill(B, Hq, Hkv, T, d, seed=9)
    lens = [T, T + 1, 0]
    status = cuda_lib.new_status(DEV)
    o = torch.full((B, Hq, T, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    cuda_lib.prefill(*_cuda(q, k, v), seq_lens=torch.tensor(lens, dtype=torch.int32, device=DEV),
                     out=o, status=status)
    assert int(status.item()) == 5
    want = oracle.prefill(f64(q[:1]), f64(k[:1]), f64(v[:1]))
    assert_close(o[:1], want, torch.bfloat16, "valid sequence")
    assert torch.all(o[1:] == 0)


def test_prefill_empty(cuda_lib):
    q = torch.empty((0, 4, 8, 64), dtype=torch.bfloat16, device=DEV)
    k = torch.empty((0, 2, 8, 64), dtype=torch.bfloat16, device=DEV)
    assert cuda_lib.prefill(q, k, k).shape == q.shape
    q = torch.empty((2, 4, 0, 64), dtype=torch.bfloat16, device=DEV)
    k = torch.empty((2, 2, 0, 64), dtype=torch.bfloat16, device=DEV)
    assert cuda_lib.prefill(q, k, k).shape == q.shape


# ------------------------------------------------------------------- decode
def _decode_case(cuda_lib, dtype, B, Hq, Hkv, C, d, lens, window, seed, std=1.0):
    q, kc, vc = synthetic.decode_inputs(B, Hq, Hkv, C, d, seed, std=std, dtype=dtype)
    want = oracle.decode(f64(q), f64(kc), f64(vc), lens, window=window)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=DEV)
    status = cuda_lib.new_status(DEV)
    qd, kd, vd = _cuda(q, kc, vc)
    o = torch.full_like(qd, float("nan"))
    cuda_lib.decode(qd, kd, vd, lens_t, window=window, out=o, status=status)
    assert int(status.item()) == 0
    return assert_close(o, want, dtype, f"decode B{B} Hq{Hq} Hkv{Hkv} C{C} d{d} w{window}")


def test_decode_fp32_small_equals_prefill_row(cuda_lib):
    """127 cached cells, append the 128th token, decode: equals row 127 of the
    full pass (and the oracle's decode)."""
    w = workloads.FP32_SMALL
    q, k, v = synthetic.qkv_prefill(w.B, w.Hq, w.Hkv, w.T, w.d, w.seed, dtype=torch.float32)
    qd, kd, vd = _cuda(q, k, v)
    C = w.T
    kc = torch.zeros((w.B, w.Hkv, C, w.d), dtype=torch.float32, device=DEV)
    vc = torch.zeros_like(kc)
    lens = torch.zeros(w.B, dtype=torch.int32, device=DEV)
    st = cuda_lib.new_status(DEV)
    cuda_lib.cache_append(kc, vc, kd[:, :, :w.cached].contiguous(), vd[:, :, :w.cached].contiguous(), lens, status=st)
    cuda_lib.cache_append(kc, vc, kd[:, :, w.cached:].contiguous(), vd[:, :, w.cached:].contiguous(), lens, status=st)
    assert lens.tolist() == [w.T] * w.B and int(st.item()) == 0
    for window in w.windows:
        o = cuda_lib.decode(qd[:, :, -1].contiguous(), kc, vc, lens, window=window)
        full = oracle.prefill(f64(q), f64(k), f64(v), window=window)
        assert_close(o, full[:, :, -1], torch.float32, f"fp32 decode w={window}")
        want = oracle.decode(f64(q[:, :, -1]), f64(kc), f64(vc), [w.T] * w.B, window=window)
        np.testing.assert_allclose(want, full[:, :, -1], rtol=0, atol=1e-12)


def test_decode_bf16_b8_n8000(cuda_lib):
    w = workloads.DECODE_B8_N8000
    n = w.cached + 1
    _decode_case(cuda_lib, torch.bfloat16, w.B, w.Hq, w.Hkv, n, w.d, [n] * w.B, None, w.seed)


@pytest.mark.parametrize("Hkv", [1, 8], ids=["mqa", "mha"])
def test_decode_bf16_ragged_endpoints(cuda_lib, Hkv):
    w = workloads.DECODE_RAGGED
    lo, hi = w.ragged
    L = synthetic.lengths_uniform(w.B, lo, hi, w.seed)
    lens = (L + 1).tolist()
    _decode_case(cuda_lib, torch.bfloat16, w.B, w.Hq, Hkv, hi + 1, w.d, lens, None, w.seed)


DECODE_EDGES = [
    # (B, Hq, Hkv, C, d, lens, window)
    (3, 4, 2, 10, 128, [0, 1, 10], None),
    (2, 8, 1, 700, 64, [700, 129], None),
    (2, 8, 8, 700, 64, [513, 64], 100),
    (1, 6, 2, 300, 128, [300], 1),
    (1, 12, 1, 2000, 128, [1999], None),
    (2, 16, 1, 999, 128, [999, 3], 500),
    (4, 2, 2, 4096, 128, [4096, 1, 2048, 77], 4096),
    (1, 32, 8, 5000, 128, [5000], 4096),
    (64, 4, 1, 40, 128, list(range(0, 40, 1)) + [40] * 24, None),
    (2, 4, 2, 50, 96, [50, 3], None),
    (2, 3, 1, 50, 32, [17, 50], 5),
    (4200, 2, 1, 3, 128, [b % 4 for b in range(4200)], None),  # lengths read from global memory
    # groups of up to 8 heads take the transposed products (cache rows as the
    # MMA's rows): padded head columns, d = 64, windows, partial stages
    (2, 6, 1, 333, 64, [333, 17], None),          # r=6: 8 columns, 6 heads
    (3, 10, 2, 257, 128, [257, 113, 0], 100),     # r=5, window, an empty row
    (2, 4, 2, 500, 64, [500, 250], 64),           # r=2, d=64, window
    (2, 12, 4, 200, 64, [200, 199], None),        # r=3: 4 columns, 3 heads
    (1, 14, 2, 1000, 128, [1000], None),          # r=7
]


@pytest.mark.parametrize("case", DECODE_EDGES, ids=lambda c: f"B{c[0]}Hq{c[1]}Hkv{c[2]}C{c[3]}d{c[4]}w{c[6]}")
def test_decode_edge_cases(cuda_lib, case):
    B, Hq, Hkv, C, d, lens, window = case
    _decode_case(cuda_lib, torch.bfloat16, B, Hq, Hkv, C, d, lens, window, seed=C + B)


def test_decode_fp32_edges(cuda_lib):
    _decode_case(cuda_lib, torch.float32, 3, 8, 2, 300, 64, [300, 1, 0], None, seed=9)
    _decode_case(cuda_lib, torch.float32, 2, 4, 4, 100, 128, [100, 40], 16, seed=10)


def test_decode_invalid_length_sets_status_and_zeroes(cuda_lib):
    q, kc, vc = _cuda(*synthetic.decode_inputs(2, 8, 2, 64, 128, seed=3))
    for lens in ([64, 65], [-1, 3]):
        status = cuda_lib.new_status(DEV)
        o = torch.full_like(q, 3.0)
        cuda_lib.decode(q, kc, vc, torch.tensor(lens, dtype=torch.int32, device=DEV),
                        out=o, status=status)
        assert int(status.item()) == 5
        assert torch.all(o == 0)


def test_decode_equals_last_prefill_row_bf16(cuda_lib):
    """GPU decode of the newest token against the cache equals the GPU full
    pass's last row (both against the oracle row)."""
    B, Hq, Hkv, T, d = 2, 8, 2, 300, 128
    q, k, v = synthetic.qkv_prefill(B, Hq, Hkv, T, d, seed=21)
    qd, kd, vd = _cuda(q, k, v)
    for window in (None, 64):
        full = cuda_lib.prefill(qd, kd, vd, window=window)
        lens = torch.full((B,), T, dtype=torch.int32, device=DEV)
        dec = cuda_lib.decode(qd[:, :, -1].contiguous(), kd, vd, lens, window=window)
        want = oracle.prefill(f64(q), f64(k), f64(v), window=window)[:, :, -1]
        assert_close(dec, want, torch.bfloat16, "decode")
        assert_close(full[:, :, -1], want, torch.bfloat16, "prefill row")


# ------------------------------------------------------------------- append
@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64), (torch.bfloat16, 3)])
def test_append_writes_rows_and_advances(cuda_lib, dtype, d):
    B, Hkv, C, t_new = 3, 2, 20, 4
    kc = synthetic.normal((B, Hkv, C, d), 1, dtype=dtype).to(DEV)
    vc = synthetic.normal((B, Hkv, C, d), 2, dtype=dtype).to(DEV)
    kn = synthetic.normal((B, Hkv, t_new, d), 3, dtype=dtype).to(DEV)
    vn = synthetic.normal((B, Hkv, t_new, d), 4, dtype=dtype).to(DEV)
    lens0 = [0, 7, 16]
    lens = torch.tensor(lens0, dtype=torch.int32, device=DEV)
    want_k, want_v, want_l = oracle.cache_append(f64(kc), f64(vc), f64(kn), f64(vn), lens0)
    st = cuda_lib.cache_append(kc, vc, kn, vn, lens)
    assert int(st.item()) == 0
    assert lens.tolist() == want_l.tolist()
    assert np.array_equal(f64(kc), want_k) and np.array_equal(f64(vc), want_v)


def test_append_refuses_beyond_capacity_all_or_nothing(cuda_lib):
    B, Hkv, C, d = 3, 2, 8, 64
    kc = torch.randn((B, Hkv, C, d), device=DEV).to(torch.bfloat16)
    vc = torch.randn((B, Hkv, C, d), device=DEV).to(torch.bfloat16)
    k0, v0 = kc.clone(), vc.clone()
    kn = torch.ones((B, Hkv, 2, d), dtype=torch.bfloat16, device=DEV)
    lens = torch.tensor([0, 7, 3], dtype=torch.int32, device=DEV)
    st = cuda_lib.cache_append(kc, vc, kn, kn, lens)
    assert int(st.item()) == 5
    assert lens.tolist() == [0, 7, 3]
    assert torch.equal(kc, k0) and torch.equal(vc, v0)
    lens = torch.tensor([0, -1, 3], dtype=torch.int32, device=DEV)
    st = cuda_lib.cache_append(kc, vc, kn, kn, lens)
    assert int(st.item()) == 5 and torch.equal(kc, k0)


def test_six_layer_cache_size_and_append(cuda_lib):
    """Append a whole prompt's K/V into a 6-layer cache: the allocation is
    2*L*B*T*Hkv*d*e = 4 x 3 MiB (the tokenwerk page's 3,145,728 B per
    sequence), and every layer's rows land where the oracle puts them."""
    w = workloads.PREFILL_B4_T1024
    caches, total = [], 0
    for layer in range(w.layers):
        kc = torch.zeros((w.B, w.Hkv, w.T, w.d), dtype=torch.bfloat16, device=DEV)
        vc = torch.zeros_like(kc)
        caches.append((kc, vc))
        total += kc.numel() * kc.element_size() + vc.numel() * vc.element_size()
    assert total == cuda_lib.cache_bytes(w.layers, w.B, w.T, w.Hkv, w.d, 2) == 4 * 3145728
    for layer, (kc, vc) in enumerate(caches):
        _, k, v = synthetic.qkv_prefill(w.B, w.Hq, w.Hkv, w.T, w.d, w.seed + 10 * layer)
        lens = torch.zeros(w.B, dtype=torch.int32, device=DEV)
        st = cuda_lib.cache_append(kc, vc, k.to(DEV), v.to(DEV), lens)
        assert int(st.item()) == 0 and lens.tolist() == [w.T] * w.B
        assert torch.equal(kc.cpu(), k) and torch.equal(vc.cpu(), v)


def test_swa_t32768_decode_steps(cuda_lib):
    """Sliding-window GQA (B=1, Hq=32, Hkv=8, d=128, w=4096): a 32768-cell
    prompt in the cache, then 64 steps of append-one-token + decode, each
    step against the oracle."""
    w = workloads.SWA_T32768
    C = w.T + w.decode_steps
    _, k, v = synthetic.qkv_prefill(w.B, w.Hq, w.Hkv, w.T, w.d, w.seed, std=w.std)
    kc = torch.zeros((w.B, w.Hkv, C, w.d), dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    lens = torch.zeros(w.B, dtype=torch.int32, device=DEV)
    st = cuda_lib.cache_append(kc, vc, k.to(DEV), v.to(DEV), lens)
    k64 = np.zeros((w.B, w.Hkv, C, w.d))
    v64 = np.zeros_like(k64)
    k64[:, :, :w.T] = f64(k)
    v64[:, :, :w.T] = f64(v)
    ws = None
    worst = 0.0
    for step in range(w.decode_steps):
        qn = synthetic.normal((w.B, w.Hq, w.d), w.seed, w.std, offset=1000 + step)
        kn = synthetic.normal((w.B, w.Hkv, 1, w.d), w.seed, w.std, offset=2000 + step)
        vn = synthetic.normal((w.B, w.Hkv, 1, w.d), w.seed, w.std, offset=3000 + step)
        cuda_lib.cache_append(kc, vc, kn.to(DEV), vn.to(DEV), lens, status=st)
        n = w.T + step + 1
        k64[:, :, n - 1] = f64(kn)[:, :, 0]
        v64[:, :, n - 1] = f64(vn)[:, :, 0]
        qd = qn.to(DEV)
        if ws is None:
            ws = cuda_lib.decode_workspace(qd, kc)
        o = cuda_lib.decode(qd, kc, vc, lens, window=w.windows[0], workspace=ws, status=st)
        want = oracle.decode(f64(qn), k64, v64, [n], window=w.windows[0])
        worst = max(worst, assert_close(o, want, torch.bfloat16, f"step {step}")[0])
    assert int(st.item()) == 0 and lens.tolist() == [C]


@pytest.mark.parametrize("Hkv", [8, 32], ids=["gqa", "mha"])
def test_prefill_swa_t32768_sampled_rows(cuda_lib, Hkv):
    """Sliding-window prefill at full size (B=1, Hq=32, d=128, T=32768,
    w=4096; Hkv=8 runs the paired kernel, the MHA endpoint Hkv=32 the
    split-row kernel), checked on a stratified sample the oracle computes row
    by row: every row t < 4096 of heads 0 and 31 (the window's ramp), and all
    32 heads at 64 seeded random cells."""
    w = workloads.SWA_T32768
    window = w.windows[0]
    w = workloads.Workload(w.name, w.dtype, B=w.B, Hq=w.Hq, Hkv=Hkv, d=w.d, T=w.T,
                           windows=w.windows, std=w.std, seed=w.seed)
    q, k, v = synthetic.qkv_prefill(w.B, w.Hq, w.Hkv, w.T, w.d, w.seed, std=w.std)
    o = cuda_lib.prefill(*_cuda(q, k, v), window=window)
    torch.cuda.synchronize()
    r = w.Hq // w.Hkv
    for h in (0, w.Hq - 1):
        g = h // r
        T0 = window
        want = oracle.prefill(f64(q[:, h:h + 1, :T0]), f64(k[:, g:g + 1, :T0]),
                              f64(v[:, g:g + 1, :T0]), window=window)
        assert_close(o[:, h:h + 1, :T0], want, torch.bfloat16, f"ramp rows head {h}")
    k64, v64 = f64(k), f64(v)
    rng = np.random.default_rng(w.seed)
    cells = sorted(rng.choice(np.arange(window, w.T), size=64, replace=False).tolist())
    got, want = [], []
    for t in cells:
        want.append(oracle.decode(f64(q[:, :, t]), k64, v64, [t + 1], window=window))
        got.append(f64(o[:, :, t]))
    assert_close(np.stack(got), np.stack(want), torch.bfloat16, "random rows")
