"""The five synthetic workloads the library is measured and checked on.

Each entry names a workload by what it is.  Shapes, windows, value
distributions and seeds only; no attention arithmetic lives here.

  fp32_small        fp32 GQA B=2 Hq=4 Hkv=2 d=64 T=128, prefill full and
                    window 32, plus one decode step on 127 cached cells.
  decode_b8_n8000   bf16 decode B=8 Hq=32 Hkv=8 d=128, 8000 cached cells
                    per sequence plus the current token.
  prefill_b4_t1024  bf16 causal prefill B=4 Hq=8 Hkv=2 d=64 T=1024, no
                    window and window 256, then a 6-layer cache append.
  decode_ragged     bf16 decode B=64 Hq=8 d=128, cached lengths uniform in
                    [1, 8192]; MQA (Hkv=1) and MHA (Hkv=8) endpoints.
  swa_t32768        bf16 sliding-window GQA B=1 Hq=32 Hkv=8 d=128 T=32768
                    w=4096, N(0, 0.5^2): prefill, then 64 decode steps.
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str                 # "f32" or "bf16"
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int = 0                 # prefill length (0: no prefill leg)
    cached: int = 0            # cells already cached before a decode step
    windows: Tuple[Optional[int], ...] = (None,)
    std: float = 1.0
    seed: int = 0
    ragged: Optional[Tuple[int, int]] = None   # cached length range [lo, hi]
    kv_variants: Tuple[int, ...] = ()          # extra Hkv endpoints
    decode_steps: int = 0
    layers: int = 1
    extra: dict = field(default_factory=dict)


FP32_SMALL = Workload("fp32_small", "f32", B=2, Hq=4, Hkv=2, d=64, T=128,
                      cached=127, windows=(None, 32), seed=0)
DECODE_B8_N8000 = Workload("decode_b8_n8000", "bf16", B=8, Hq=32, Hkv=8, d=128,
                           cached=8000, seed=1)
PREFILL_B4_T1024 = Workload("prefill_b4_t1024", "bf16", B=4, Hq=8, Hkv=2, d=64,
                            T=1024, windows=(None, 256), seed=2, layers=6)
DECODE_RAGGED = Workload("decode_ragged", "bf16", B=64, Hq=8, Hkv=1, d=128,
                         ragged=(1, 8192), kv_variants=(1, 8), seed=3)
SWA_T32768 = Workload("swa_t32768", "bf16", B=1, Hq=32, Hkv=8, d=128, T=32768,
                      windows=(4096,), std=0.5, seed=4, decode_steps=64)

ALL = (FP32_SMALL, DECODE_B8_N8000, PREFILL_B4_T1024, DECODE_RAGGED, SWA_T32768)
BY_NAME = {w.name: w for w in ALL}
