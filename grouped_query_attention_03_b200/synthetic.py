"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no attention arithmetic: it only draws numbers.  Values are
drawn in float32 from a CPU ``torch.Generator`` with a fixed seed, scaled by
the workload's standard deviation, and rounded to the storage dtype
(round-to-nearest-even for bf16).  The same rounded tensors are handed to the
CUDA library and, converted exactly to float64, to the CPU oracle.
"""
import torch


def normal(shape, seed, std=1.0, dtype=torch.bfloat16, offset=0):
    """i.i.d. N(0, std^2) drawn in float32, then rounded to ``dtype``.

    ``offset`` selects an independent stream under the same seed (one per
    tensor of a workload), so tensors do not share draws.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 1000003 + int(offset))
    x = torch.randn(tuple(shape), generator=g, dtype=torch.float32)
    if std != 1.0:
        x = x * float(std)
    return x.to(dtype)


def lengths_uniform(B, lo, hi, seed, offset=77):
    """Integer lengths drawn uniformly from [lo, hi] inclusive (int32)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 1000003 + int(offset))
    return torch.randint(int(lo), int(hi) + 1, (int(B),), generator=g, dtype=torch.int32)


def qkv_prefill(B, Hq, Hkv, T, d, seed, std=1.0, dtype=torch.bfloat16):
    """Q [B,Hq,T,d], K and V [B,Hkv,T,d]."""
    q = normal((B, Hq, T, d), seed, std, dtype, offset=1)
    k = normal((B, Hkv, T, d), seed, std, dtype, offset=2)
    v = normal((B, Hkv, T, d), seed, std, dtype, offset=3)
    return q, k, v


def decode_inputs(B, Hq, Hkv, C, d, seed, std=1.0, dtype=torch.bfloat16):
    """Q [B,Hq,d], K/V caches [B,Hkv,C,d] (every cell filled with draws)."""
    q = normal((B, Hq, d), seed, std, dtype, offset=11)
    kc = normal((B, Hkv, C, d), seed, std, dtype, offset=12)
    vc = normal((B, Hkv, C, d), seed, std, dtype, offset=13)
    return q, kc, vc
