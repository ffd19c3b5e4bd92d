"""The C ABI on the CPU: the library loads, exports every declared symbol,
and refuses bad arguments on the host before any CUDA call is made."""
import ctypes
import os
import re

import pytest

import oracle
import oracle_pins
from grouped_query_attention_03_b200 import build as gbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa.h")

OK, NULL, SHAPE, GROUPS, WINDOW, CAPACITY, OVERFLOW = 0, 1, 2, 3, 4, 5, 6


@pytest.fixture(scope="module")
def L():
    gbuild.build()
    from grouped_query_attention_03_b200 import gqa
    return gqa.lib()


def declared_functions():
    with open(HEADER) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    return sorted(set(re.findall(r"\b(gqa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("gqa_prefill", "gqa_decode", "gqa_cache_append"):
        assert must in names


def test_every_declared_symbol_is_exported(L):
    from grouped_query_attention_03_b200 import gqa
    names = declared_functions()
    assert set(names) == set(gqa.EXPORTS)
    for name in names:
        assert hasattr(L, name), name


def test_version_and_strings(L):
    assert L.gqa_version().decode().count(".") == 2
    for code in range(13):
        assert L.gqa_status_string(code)
        assert L.gqa_status_string(code) != b"unknown status"
    assert L.gqa_status_string(999) == b"unknown status"


def test_cache_bytes_matches_pages(L):
    for c in oracle_pins.golden("cache_sizes.json")["cases"]:
        assert L.gqa_cache_bytes(c["L"], c["B"], c["T"], c["Hkv"], c["d"], c["e"]) == c["bytes"]
    assert L.gqa_cache_bytes(2**40, 2**20, 2**10, 1, 1, 1) == 0
    assert L.gqa_cache_bytes(-1, 1, 1, 1, 1, 1) == 0


def test_head_map_and_window_start_match_oracle(L):
    for Hq, Hkv in [(4, 2), (8, 2), (32, 8), (8, 1), (8, 8), (6, 4), (4, 0), (0, 2)]:
        for h in range(-1, max(Hq, 1) + 1):
            want = oracle.kv_head_for_query(h, Hq, Hkv) if h >= 0 else None
            got = L.gqa_kv_head_for_query(h, Hq, Hkv)
            assert (None if got < 0 else got) == want, (h, Hq, Hkv)
    for t in range(0, 12):
        for w in [None, 1, 2, 3, 5, 20]:
            got = L.gqa_window_start(t, -1 if w is None else w)
            assert got == oracle.window_start(t, 0, w)
    assert L.gqa_window_start(3, 0) == -1
    assert L.gqa_window_start(3, -2) == -1


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: every case fails first


def _prefill(L, **kw):
    a = dict(dtype=1, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lens=None, B=1, Hq=4, Hkv=2,
             T=8, d=64, window=-1, scale=0.125, status=None)
    a.update(kw)
    return L.gqa_prefill(a["dtype"], a["q"], a["k"], a["v"], a["o"], a["lens"], a["B"],
                         a["Hq"], a["Hkv"], a["T"], a["d"], a["window"], a["scale"],
                         a["status"], None)


def _decode(L, **kw):
    a = dict(dtype=1, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lens=FAKE, B=1, Hq=4, Hkv=2,
             C=8, d=64, window=-1, scale=0.125, ws=FAKE, wsb=1 << 30, status=FAKE)
    a.update(kw)
    return L.gqa_decode(a["dtype"], a["q"], a["k"], a["v"], a["o"], a["lens"], a["B"],
                        a["Hq"], a["Hkv"], a["C"], a["d"], a["window"], a["scale"],
                        a["ws"], a["wsb"], a["status"], None)


def _append(L, **kw):
    a = dict(dtype=1, kc=FAKE, vc=FAKE, kn=FAKE, vn=FAKE, lens=FAKE, B=1, Hkv=2, C=8,
             d=64, t_new=1, status=FAKE)
    a.update(kw)
    return L.gqa_cache_append(a["dtype"], a["kc"], a["vc"], a["kn"], a["vn"], a["lens"],
                              a["B"], a["Hkv"], a["C"], a["d"], a["t_new"], a["status"], None)


def _decode_append(L, **kw):
    a = dict(dtype=1, q=FAKE, kc=FAKE, vc=FAKE, kn=FAKE, vn=FAKE, o=FAKE, lens=FAKE, B=1,
             Hq=4, Hkv=2, C=8, d=64, window=-1, scale=0.125, ws=FAKE, wsb=1 << 30,
             status=FAKE)
    a.update(kw)
    return L.gqa_decode_append(a["dtype"], a["q"], a["kc"], a["vc"], a["kn"], a["vn"], a["o"],
                               a["lens"], a["B"], a["Hq"], a["Hkv"], a["C"], a["d"],
                               a["window"], a["scale"], a["ws"], a["wsb"], a["status"], None)


def _decode_multi(L, **kw):
    a = dict(dtype=1, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lens=FAKE, B=1, Hq=4, Hkv=2, C=8, d=64,
             t_new=2, window=-1, scale=0.125, status=FAKE)
    a.update(kw)
    return L.gqa_decode_multi(a["dtype"], a["q"], a["k"], a["v"], a["o"], a["lens"], a["B"],
                              a["Hq"], a["Hkv"], a["C"], a["d"], a["t_new"], a["window"],
                              a["scale"], a["status"], None)


def test_decode_multi_host_refusals(L):
    assert _decode_multi(L, Hq=3, Hkv=2) == GROUPS
    assert _decode_multi(L, window=0) == WINDOW
    assert _decode_multi(L, t_new=9) == CAPACITY
    assert _decode_multi(L, t_new=-1) == SHAPE
    assert _decode_multi(L, C=-1) == SHAPE
    assert _decode_multi(L, lens=None) == NULL
    assert _decode_multi(L, status=None) == NULL
    assert _decode_multi(L, q=None) == NULL
    assert _decode_multi(L, t_new=0, q=None) == OK
    assert _decode_multi(L, B=0, q=None) == OK


def test_prefill_packed_host_refusals(L):
    f = L.gqa_prefill_packed
    args = [1, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1, 4, 2, 8, 64, -1, 0.125, FAKE, None]
    bad_seg = list(args)
    bad_seg[6] = None
    assert f(*bad_seg) == NULL
    no_status = list(args)
    no_status[14] = None
    assert f(*no_status) == NULL
    groups = list(args)
    groups[8] = 3
    assert f(*groups) == GROUPS
    empty = list(args)
    empty[7] = 0
    empty[6] = None
    assert f(*empty) == OK


def test_ring_host_refusals(L):
    # gqa_ring_append(dtype, k, v, kn, vn, lens, B, Hkv, W, d, t_new, status, stream)
    ra = [1, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 4, 64, 9, FAKE, None]
    w0 = list(ra)
    w0[8] = 0
    assert L.gqa_ring_append(*w0) == SHAPE
    neg = list(ra)
    neg[10] = -1
    assert L.gqa_ring_append(*neg) == SHAPE
    nolens = list(ra)
    nolens[5] = None
    assert L.gqa_ring_append(*nolens) == NULL
    empty = list(ra)
    empty[10] = 0
    assert L.gqa_ring_append(*empty) == OK
    # gqa_ring_decode_append(dtype, q, kr, vr, kn, vn, o, lens, B, Hq, Hkv, W, d, scale,
    #                        ws, wsb, status, stream)
    rd = [1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, 2, 8, 64, 0.125, FAKE, 1 << 30,
          FAKE, None]
    w0 = list(rd)
    w0[11] = 0
    assert L.gqa_ring_decode_append(*w0) == SHAPE
    groups = list(rd)
    groups[9] = 3
    assert L.gqa_ring_decode_append(*groups) == GROUPS
    nokn = list(rd)
    nokn[4] = None
    assert L.gqa_ring_decode_append(*nokn) == NULL
    nows = list(rd)
    nows[14] = None
    assert L.gqa_ring_decode_append(*nows) == 8


def test_prefill_host_refusals(L):
    assert _prefill(L, Hq=6, Hkv=4) == GROUPS
    assert _prefill(L, Hkv=0) == SHAPE
    assert _prefill(L, d=0) == SHAPE
    assert _prefill(L, B=-1) == SHAPE
    assert _prefill(L, window=0) == WINDOW
    assert _prefill(L, window=-2) == WINDOW
    assert _prefill(L, q=None) == NULL
    assert _prefill(L, dtype=7) == 7
    assert _prefill(L, B=2**30, Hq=2**30, Hkv=2**30, T=2**30) == OVERFLOW
    assert _prefill(L, d=300) == 7
    # empty inputs are a successful no-op, with no pointer needed
    assert _prefill(L, B=0, q=None, k=None, v=None, o=None) == OK
    assert _prefill(L, T=0, q=None, k=None, v=None, o=None) == OK


def test_decode_host_refusals(L):
    assert _decode(L, Hq=3, Hkv=2) == GROUPS
    assert _decode(L, window=0) == WINDOW
    assert _decode(L, lens=None) == NULL
    assert _decode(L, status=None) == NULL
    assert _decode(L, C=-1) == SHAPE
    assert _decode(L, B=0, q=None) == OK


def test_decode_append_host_refusals(L):
    assert _decode_append(L, Hq=3, Hkv=2) == GROUPS
    assert _decode_append(L, window=0) == WINDOW
    assert _decode_append(L, kn=None) == NULL
    assert _decode_append(L, vn=None) == NULL
    assert _decode_append(L, lens=None) == NULL
    assert _decode_append(L, status=None) == NULL
    assert _decode_append(L, C=-1) == SHAPE
    assert _decode_append(L, ws=None) == 8
    assert _decode_append(L, B=0, q=None, kn=None) == OK


def test_append_host_refusals(L):
    assert _append(L, t_new=-1) == SHAPE
    assert _append(L, Hkv=0) == SHAPE
    assert _append(L, lens=None) == NULL
    assert _append(L, t_new=9) == CAPACITY
    assert _append(L, t_new=0, kc=None) == OK


def test_workspace_size(L):
    # bf16 split-K path needs a workspace; fp32 and other widths need none.
    n = L.gqa_decode_workspace_bytes(1, 8, 32, 8, 8001, 128)
    assert n > 0 and n % 256 == 0
    assert L.gqa_decode_workspace_bytes(0, 8, 32, 8, 8001, 128) == 0
    assert L.gqa_decode_workspace_bytes(1, 8, 32, 8, 8001, 96) == 0
    assert L.gqa_decode_workspace_bytes(1, 8, 30, 8, 8001, 128) == 0
    assert _decode(L, ws=None) == 8
    assert _decode(L, wsb=16) == 8


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from grouped_query_attention_03_b200 import gqa
    monkeypatch.setattr(gqa, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(gqa, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        gqa.lib()


def test_selftest_wait_host_refusals(L):
    """The wait self-test refuses a limit outside [1 us, 2 s] and NULL
    pointers before any CUDA call (no GPU needed)."""
    fake = ctypes.c_void_p(0x1000)
    assert L.gqa_selftest_wait_timeout(0, 0, fake, fake, None) == SHAPE
    assert L.gqa_selftest_wait_timeout(-5, 0, fake, fake, None) == SHAPE
    assert L.gqa_selftest_wait_timeout(2000001, 0, fake, fake, None) == SHAPE
    assert L.gqa_selftest_wait_timeout(1000, 0, None, fake, None) == NULL
    assert L.gqa_selftest_wait_timeout(1000, 0, fake, None, None) == NULL


def test_prefill_kernel_choice(L):
    """gqa_prefill_kernel names the kernel gqa_prefill runs (host-only)."""
    pick = lambda B, Hq, Hkv, T, d, w, sms=148: L.gqa_prefill_kernel(B, Hq, Hkv, T, d, w, sms)
    assert pick(1, 32, 8, 32768, 128, 4096) == 1   # even group, many CTAs: paired heads
    assert pick(1, 32, 32, 32768, 128, 4096) == 2  # MHA (group of 1): one head per CTA
    assert pick(1, 12, 4, 4096, 64, -1) == 2       # group of 3
    assert pick(4, 8, 2, 1024, 64, -1) == 2        # 128 paired CTAs, last tile walks 8 KV tiles
    assert pick(4, 8, 2, 1024, 64, 256) == 1       # ... with a 256 window only 3
    assert pick(4, 8, 2, 1024, 64, -1, sms=64) == 1  # the paired grid fills the device
    assert pick(4, 8, 2, 512, 64, -1) == 1         # 4 query tiles: the last walks 4 KV tiles
    assert pick(4, 8, 2, 513, 64, -1) == 2         # 5 query tiles, the last walks 5
    assert pick(1, 8, 2, 1024, 96, -1) == 0        # head width without a tensor-core kernel
    for bad in ((0, 8, 2, 64, 64, -1), (1, 8, 3, 64, 64, -1), (1, 8, 2, 64, 64, 0),
                (1, 8, 2, 64, 64, -2), (1, 8, 2, 0, 64, -1), (1, 8, 2, 64, 64, -1, 0)):
        assert pick(*bad) == -1, bad
