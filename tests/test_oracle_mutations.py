"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check
that the pins catch every one of them.  This is what makes the pins worth
trusting: a dropped term, a wrong sign or index, a transposed operand, an
off-by-one in the window or the decode position each fails at least one pin.
"""
import contextlib
import os
import shutil
import subprocess
import tempfile

import pytest

import oracle
import oracle_pins
from oracle import build as oracle_build

SRC = os.path.join(os.path.dirname(oracle_build.SRC), "gqa_oracle.c")
HDR = os.path.join(os.path.dirname(oracle_build.SRC), "gqa_oracle.h")

# (name, text in gqa_oracle.c, replacement)
MUTATIONS = [
    ("head_map_tiled", "long g = h / r;", "long g = h % Hkv;"),
    ("window_off_by_one", "long back = w - 1;", "long back = w;"),
    ("scale_dropped", "double s = scale * dot;", "double s = dot;"),
    ("scale_sign", "double s = scale * dot;", "double s = -scale * dot;"),
    ("values_from_keys", "out[f] += p * vlane[j * d + f];", "out[f] += p * klane[j * d + f];"),
    ("no_normalisation", "double p = scratch[j - lo] / l;", "double p = scratch[j - lo];"),
    ("no_max_shift", "scratch[i] = exp(scratch[i] - m);", "scratch[i] = exp(scratch[i]);"),
    ("self_key_dropped", "for (long j = lo; j <= hi; ++j) {\n    double dot", "for (long j = lo; j < hi; ++j) {\n    double dot"),
    ("inactive_not_zeroed", "if (t >= n) {", "if (t > n) {"),
    ("decode_position", "long pos = n - t_new + i;", "long pos = n - t_new + i - 1;"),
    ("append_offset", "long dst = ((b * Hkv + g) * C + seq_lens[b] + i) * d;",
     "long dst = ((b * Hkv + g) * C + i) * d;"),
    ("append_not_transactional", "if (seq_lens[b] < 0 || seq_lens[b] + t_new > C) return 2;",
     "if (seq_lens[b] < 0) return 2;"),
    ("bytes_factor", "uint64_t acc = 2;", "uint64_t acc = 1;"),
    ("segment_ignored", "long s0 = seg_start ? seg_start[b * T + t] : 0;", "long s0 = 0;"),
    ("query_row_index", "attend_row(q + ((b * Hq + h) * T + t) * d,", "attend_row(q + ((b * Hq + h) * T) * d,"),
    ("ring_slot", "long dst = ((b * Hkv + g) * W + pos % W) * d;",
     "long dst = ((b * Hkv + g) * W + (pos + 1) % W) * d;"),
    ("ring_window_short", "long lo = n > W ? n - W : 0;", "long lo = n > W ? n - W + 1 : 0;"),
    ("ring_overwrite_order", "if (t_new - i > W) continue;", "if (i >= W) continue;"),
    ("segment_window_min", "return seg_start > sat ? seg_start : sat;",
     "return seg_start < sat ? seg_start : sat;"),
    ("no_window_is_self_only", "if (w < 0) return seg_start;", "if (w < 0) return t;"),
]


@contextlib.contextmanager
def _mutated(text, repl, tmp):
    with open(SRC) as f:
        src = f.read()
    assert src.count(text) >= 1, text
    src = src.replace(text, repl)
    path = os.path.join(tmp, "gqa_oracle.c")
    with open(path, "w") as f:
        f.write(src)
    shutil.copy(HDR, tmp)
    lib = os.path.join(tmp, "libmut.so")
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-I", tmp,
                    path, "-o", lib, "-lm"], check=True)
    saved = oracle._lib
    oracle._lib = oracle._load(lib)
    try:
        yield
    finally:
        oracle._lib = saved


@pytest.mark.parametrize("name,text,repl", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(name, text, repl):
    with tempfile.TemporaryDirectory() as tmp, _mutated(text, repl, tmp):
        failed = []
        for pin in oracle_pins.ALL_PINS:
            try:
                pin(oracle)
            except (AssertionError, oracle.OracleError, FloatingPointError, ValueError):
                failed.append(pin.__name__)
        assert failed, f"planted mistake '{name}' was not caught by any pin"
