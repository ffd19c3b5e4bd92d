"""Benchmark of the GQA hot path on B200 (one JSON line on rank 0).

A step is one pass of the decode hot path over one batch: one
gqa_decode_append call, which appends the new token's K/V row to the cache
and decodes it against the cache in the same kernel (head map, permitted
window, scores, online softmax, value mix, split-K merge).  Every step reads
the same cells: each step has its own copy of the cached lengths, set before
the timed pass.  The same step unfused (gqa_cache_append, then gqa_decode)
is reported beside it.  The default workload is bf16 decode with B=8,
Hq=32, Hkv=8, d=128 and 8000 cached cells per sequence (8001 keys read with
the new token).

value  = algorithmic bytes per step x steps x ranks / max-over-ranks time,
         algorithmic bytes = K+V of every permitted cell + Q + O + the
         appended rows (read and written); the K-step timed pass is repeated
         (at least 30 times and half a second) and the median pass reported
e2e    = the same through the public API with host buffers: the pinned
         host->device copy of the step's q and new K/V (one packed buffer)
         and the device->host read of o inside the timed region; the step is
         captured in a CUDA graph and replayed (the eager figure is beside it)
roofline = the fused split-K decode kernel alone (back-to-back calls) against
         the measured HBM copy bandwidth
decode = the same measurements on the other decode workloads: the ragged
         MQA and MHA endpoints (B=64, Hq=8, Hkv 1 / 8) and the long-context
         sliding-window step (64 successive steps after a 32768-cell prompt)
prefill = prefill TFLOP/s on the long-context and the T=1024 workloads
cpu_baseline = the fp64 oracle on this host's cores on a bounded sample

Usage: python bench.py [--gpus N --steps K --warmup W] [--impl reference]
                       [--workload NAME] [--phase decode|prefill]
Multi-GPU (torchrun): every rank runs its own independent batch (replicas,
weak scaling; the path has no exchange step), timing is max over ranks.
"""
import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from grouped_query_attention_03_b200 import synthetic, workloads  # noqa: E402

METRIC = "decode KV-cache HBM GB/s (% of 8 TB/s); prefill TFLOP/s (% bf16 peak)"
SPEC_HBM_GBS = 8000.0
SPEC_BF16_TFLOPS = 2250.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126e6  # a step whose inputs fit in it rotates over copies of them
MIN_PASSES = 30          # timed passes per measurement (median reported)
MIN_PASS_SECONDS = 0.5   # ... and at least this much timed time (headline)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": 1590.0}, "fallback"


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons sampled every ~1 ms by NVML
    on a background thread while the timed region runs."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown",
               0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap", 0x80: "hw_power_brake"}

    def __init__(self, gpu_index, period_s=0.001):
        self.gpu = gpu_index
        self.period = period_s
        self.sm, self.smax, self.mask = [], None, 0
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.smax = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.ok = True
        except Exception:  # no NVML: report no samples rather than guess
            return self
        self.stop = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        return self

    def _run(self):
        while not self.stop.is_set():
            try:
                self.sm.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.mask |= int(self.get_reasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        if self.ok:
            self.stop.set()
            self.thread.join(timeout=2)
        return False

    def summary(self):
        reasons = sorted(n for bit, n in self.REASONS.items() if self.mask & bit)
        return {"sm_mhz": statistics.median(self.sm) if self.sm else None,
                "sm_max_mhz": self.smax, "reasons": reasons, "samples": len(self.sm),
                "source": "nvml" if self.ok else "unavailable"}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def dist_max(x, device):
    import torch.distributed as dist
    if not dist.is_initialized():
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_max_list(xs, device):
    """Element-wise maximum over ranks of equally long lists (each rank's
    per-pass times: pass i of the job took as long as its slowest rank)."""
    import torch.distributed as dist
    if not dist.is_initialized():
        return list(xs)
    t = torch.tensor(list(xs), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def pass_stats(ms):
    """Median, spread and count of per-pass times (ms)."""
    s = sorted(ms)
    q = lambda f: s[min(len(s) - 1, int(f * (len(s) - 1) + 0.5))]
    return {"passes": len(s), "median_ms": statistics.median(s), "min_ms": s[0],
            "p10_ms": q(0.1), "p90_ms": q(0.9), "max_ms": s[-1]}


# DRAM bytes (read + write) per launch of the dominant kernel, from the ncu
# captures (the committed summaries name the workload and the kernel), per
# (workload, phase, window, Hkv) as the bench is invoked.  Each holds the
# SHA-256 of the kernel's source files at capture time, comments and blank
# lines stripped: once the code changes the figure no longer describes the
# kernel and is reported as null (a comment edit does not count).
DECODE_SOURCES = ["decode_splitk.cuh", "common.cuh", "tc_ptx.cuh"]
DECODE_SHA = "f5815f28d2eec9e95b0d4534fc3a003f3b7bcf1c684160196fa61561e521d95b"
PAIR_SOURCES = ["prefill_pair.cuh", "common.cuh", "tc_ptx.cuh"]
PAIR_SHA = "b55fbb607750b596aa7e864859eb103b7cdf4955fb5bdd52daec85227937995e"
PERSIST_SOURCES = ["prefill_persist.cuh", "common.cuh", "tc_ptx.cuh"]
PERSIST_SHA = "914d32926d329e3c21c2ce75b7f79d52bc53e403126ff2afbf4fb0ab7a1907b0"
CAPTURED_TRAFFIC = [
    {"workload": "decode_b8_n8000", "phase": "decode", "window": None, "hkv": None,
     "bytes": 268_040_448, "sources": DECODE_SOURCES, "sha256": DECODE_SHA},
    {"workload": "decode_ragged", "phase": "decode", "window": None, "hkv": 1,
     "bytes": 148_212_992, "sources": DECODE_SOURCES, "sha256": DECODE_SHA},
    {"workload": "decode_ragged", "phase": "decode", "window": None, "hkv": 8,
     "bytes": 1_125_684_880, "sources": DECODE_SOURCES, "sha256": DECODE_SHA},
    {"workload": "swa_t32768", "phase": "decode", "window": None, "hkv": None,
     "bytes": 17_117_952, "sources": DECODE_SOURCES, "sha256": DECODE_SHA},
    {"workload": "prefill_b4_t1024", "phase": "prefill", "window": None, "hkv": None,
     "bytes": 6_359_808, "sources": PERSIST_SOURCES, "sha256": PERSIST_SHA},
    {"workload": "prefill_b4_t1024", "phase": "prefill", "window": 256, "hkv": None,
     "bytes": 6_356_480, "sources": PAIR_SOURCES, "sha256": PAIR_SHA},
    {"workload": "swa_t32768", "phase": "prefill", "window": 4096, "hkv": None,
     "bytes": 688_172_544, "sources": PAIR_SOURCES, "sha256": PAIR_SHA},
    {"workload": "swa_t32768", "phase": "prefill", "window": 4096, "hkv": 32,
     "bytes": 1_057_996_800, "sources": PERSIST_SOURCES, "sha256": PERSIST_SHA},
]


def strip_comments(src):
    """C++/CUDA source without comments and blank lines (string and character
    literals kept): what the compiler turns into the kernel."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (ln.rstrip() for ln in "".join(out).split("\n"))
    return "\n".join(ln for ln in lines if ln)


def source_digest(texts):
    """SHA-256 over the comment-stripped sources, in order."""
    import hashlib
    h = hashlib.sha256()
    for t in texts:
        h.update(strip_comments(t).encode())
    return h.hexdigest()


def captured_traffic(workload, phase, window, hkv):
    """ncu DRAM bytes per launch for this workload if the kernel's code (its
    sources without comments) is the captured code, else None."""
    c = next((e for e in CAPTURED_TRAFFIC if (e["workload"], e["phase"], e["window"], e["hkv"])
              == (workload, phase, window, hkv)), None)
    if c is None:
        return None
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "grouped_query_attention_03_b200", "csrc")
    texts = []
    for f in c["sources"]:
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            texts.append(fh.read())
    return c["bytes"] if source_digest(texts) == c["sha256"] else None


def aggregate_rate(units_per_step, steps, world, max_ms):
    """Whole-job throughput: the units every rank processed (each rank runs
    the same per-rank step, weak scaling) over the slowest rank's time."""
    return units_per_step * steps * world / (max_ms / 1e3)


def barrier():
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()


def n_passes(one_pass_ms, device, min_passes=MIN_PASSES, min_seconds=0.0, max_passes=3000):
    """How many timed passes to run: at least `min_passes` and at least
    `min_seconds` of timed work, the same number on every rank."""
    n = max(min_passes, int(math.ceil(min_seconds * 1e3 / max(one_pass_ms, 1e-3))))
    return int(dist_max(float(min(n, max_passes)), device))


# --------------------------------------------------------------- workloads
def decode_shape(w, window):
    """(window, cached cells per sequence, capacity) of a decode step.  The
    sliding-window workload decodes after its whole prompt is cached."""
    if window is None and w.decode_steps and w.windows[0] is not None:
        window = w.windows[0]
    if w.ragged:
        cached = synthetic.lengths_uniform(w.B, w.ragged[0], w.ragged[1], w.seed).tolist()
        return window, cached, w.ragged[1] + 1
    n = w.cached or w.T
    return window, [n] * w.B, n + 1


def n_copies(bytes_per_step):
    """Independent copies of a step's inputs to use in turn so that no step
    finds lines left in the 126 MB L2 by the step before: 1 when one step's
    inputs already exceed the L2, else enough to hold twice the L2 (like the
    layers of a model, each with its own cache)."""
    if bytes_per_step > L2_BYTES:
        return 1
    return int(min(64, math.ceil(2 * L2_BYTES / max(bytes_per_step, 1)) + 1))


class DecodeStep:
    """Append one token per sequence and decode it.

    The step is one gqa_decode_append call (the append fused into the decode
    kernel).  When one step's cache fits in L2, `NL` independent copies of
    the cache (layers) are used in turn, step i on layer i mod NL, so every
    step streams its cache from HBM and the steps still run back to back.
    In the timed steps each step has its own lengths buffer holding the
    cached count (set before the pass), so every step reads the same cells;
    the loop of successive calls advances each layer's lengths instead.
    run_separate() is the same step as gqa_cache_append followed by
    gqa_decode, reported beside it."""

    def __init__(self, w, device, Hkv=None, window=None, calls=0, nbufs=1):
        from grouped_query_attention_03_b200 import gqa
        self.gqa = gqa
        self.w = w
        self.Hkv = Hkv or w.Hkv
        self.window, self.cached, C = decode_shape(w, window)
        B, Hq, d = w.B, w.Hq, w.d
        self.kv_bytes = self.kv_bytes_at(0)
        self.NL = n_copies(self.kv_bytes)
        # spare cells let `calls` successive calls append to the layers
        self.extra = -(-calls // self.NL) + 2
        self.C = C + self.extra
        C = self.C
        q, kc, vc = synthetic.decode_inputs(B, Hq, self.Hkv, C, d, w.seed, std=w.std)
        kc, vc = kc.to(device), vc.to(device)
        self.kcs = [kc] + [kc.clone() for _ in range(self.NL - 1)]
        self.vcs = [vc] + [vc.clone() for _ in range(self.NL - 1)]
        self.kc, self.vc = kc, vc
        kn = synthetic.normal((B, self.Hkv, 1, d), w.seed, w.std, offset=21)
        vn = synthetic.normal((B, self.Hkv, 1, d), w.seed, w.std, offset=22)
        # The step's inputs (q, k_new, v_new) are views of one buffer, so a
        # single host->device copy brings a step's inputs in.
        nq, nk = q.numel(), kn.numel()
        self.inbuf = torch.empty(nq + 2 * nk, dtype=q.dtype, device=device)
        self.q = self.inbuf[:nq].view(q.shape)
        self.kn = self.inbuf[nq:nq + nk].view(kn.shape)
        self.vn = self.inbuf[nq + nk:].view(vn.shape)
        for dst, src in ((self.q, q), (self.kn, kn), (self.vn, vn)):
            dst.copy_(src)
        self.lens0 = torch.tensor(self.cached, dtype=torch.int32, device=device)
        self.lens_bufs = self.lens0.repeat(max(1, nbufs), 1).contiguous()
        self.layer_lens = self.lens0.repeat(self.NL, 1).contiguous()
        self.o = torch.empty_like(self.q)
        self.ws = gqa.decode_workspace(self.q, self.kc)
        self.status = gqa.new_status(device)
        e = 2  # bf16
        self.qo_bytes = int(2 * B * Hq * d * e)
        # the new K/V rows are read once (counted in kv_bytes) and written once
        self.write_bytes = int(2 * B * self.Hkv * d * e)
        self.decode_bytes = self.kv_bytes + self.qo_bytes
        self.step_bytes = self.decode_bytes + self.write_bytes
        self.launches_per_step = 1  # the fused kernel
        self.launches_separate = 3  # append copy + commit, split kernel

    def kv_bytes_at(self, grown):
        """K+V bytes one step reads when `grown` cells were appended since the
        lengths were set (the window caps the cells read)."""
        n = np.array(self.cached) + 1 + grown
        eff = np.minimum(n, self.window) if self.window else n
        return int(2 * self.Hkv * eff.sum() * self.w.d * 2)

    def step_bytes_at(self, grown):
        return self.kv_bytes_at(grown) + self.qo_bytes + self.write_bytes

    def loop_bytes(self, calls):
        """Bytes of `calls` successive calls from the cached lengths, call i
        on layer i mod NL (that layer has grown by i // NL cells)."""
        return sum(self.step_bytes_at(i // self.NL) for i in range(calls))

    def reset(self):
        self.lens_bufs.copy_(self.lens0.expand_as(self.lens_bufs), non_blocking=True)
        self.layer_lens.copy_(self.lens0.expand_as(self.layer_lens), non_blocking=True)

    def call(self, i, lens):
        """One gqa_decode_append call on layer i mod NL with lengths `lens`."""
        l = i % self.NL
        self.gqa.decode_append(self.q, self.kcs[l], self.vcs[l], self.kn, self.vn, lens,
                               window=self.window, out=self.o, workspace=self.ws,
                               status=self.status)

    def step(self, i):
        """Timed step i: layer i mod NL, its own lengths buffer."""
        self.call(i, self.lens_bufs[i])

    def loop_call(self, i):
        """Call i of the successive-calls loop: layer i mod NL, whose lengths
        advance with each of its calls."""
        self.call(i, self.layer_lens[i % self.NL])

    def run_separate(self, i):
        l, lens = i % self.NL, self.lens_bufs[i]
        self.gqa.cache_append(self.kcs[l], self.vcs[l], self.kn, self.vn, lens,
                              status=self.status)
        self.gqa.decode(self.q, self.kcs[l], self.vcs[l], lens, window=self.window, out=self.o,
                        workspace=self.ws, status=self.status)

    def run_host(self, hin, ho, i):
        """Step i through the public API: the step's inputs from a pinned
        host buffer (q, k_new, v_new packed), the output back to pinned host
        memory."""
        self.inbuf.copy_(hin, non_blocking=True)
        self.step(i)
        ho.copy_(self.o, non_blocking=True)

    def describe(self):
        w = self.w
        d = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": self.Hkv, "d": w.d,
             "window": self.window, "capacity": self.C - self.extra,
             "keys_read_per_seq": "cached+1 (the appended token)",
             "l2": "inputs exceed the 126 MB L2; steps back to back" if self.NL == 1 else
                   f"{self.NL} copies of the cache ({self.NL * self.kv_bytes / 1e6:.0f} MB read "
                   f"in turn, above twice the 126 MB L2), step i on copy i mod {self.NL}; "
                   f"steps back to back, no flush"}
        if w.ragged:
            d["cached_lengths"] = f"uniform [{w.ragged[0]}, {w.ragged[1]}], seed {w.seed}"
        else:
            d["cached"] = self.cached[0]
        return d


def capture(fn, device):
    """Capture fn() into a CUDA graph (on a side stream, as torch requires)."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(device)
    s.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(s):
        fn()
        torch.cuda.synchronize(device)
        with torch.cuda.graph(g, stream=s):
            fn()
    torch.cuda.current_stream(device).wait_stream(s)
    torch.cuda.synchronize(device)
    return g


def timed(fn, device):
    """Device time (ms) of fn() (CUDA events on the launching stream, with a
    barrier and a synchronize on both sides)."""
    stream = torch.cuda.current_stream(device)
    barrier()
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    fn()
    b.record(stream)
    torch.cuda.synchronize(device)
    return a.elapsed_time(b)


def repeat_passes(one_pass, device, min_passes=MIN_PASSES, min_seconds=0.0):
    """Per-pass times (ms, max over ranks pass by pass) of `one_pass`."""
    first = one_pass()
    n = n_passes(first, device, min_passes, min_seconds)
    ms = [first] + [one_pass() for _ in range(n - 1)]
    return dist_max_list(ms, device)


def measure_decode(w, device, args, world, Hkv=None, window=None, loop=None,
                   separate=False, min_seconds=0.0, cpu_seconds=None, gpu_index=0):
    """Time the fused decode step on one workload; returns (step, result).

    steps   K steps back to back (one CUDA graph), each gqa_decode_append on
            its own lengths buffer holding the cached count (all set before
            the pass), so every step reads the same cells.  Repeated passes;
            median reported.
    kernel  gqa_decode_append alone, K2 successive calls (one CUDA graph)
            from the cached lengths (call i reads i // NL more cells, its
            bytes counted so) -- with `loop` = K2 this is the workload's own
            loop of successive decode steps.
    e2e     the step through the public API with pinned host buffers.
    """
    K = args.steps
    K2 = loop or min(K, 100)
    step = DecodeStep(w, device, Hkv=Hkv, window=window, calls=K2 + 2, nbufs=K)
    for i in range(args.warmup):
        step.reset()
        step.step(i % K)
    torch.cuda.synchronize(device)
    if int(step.status.item()) != 0:
        raise RuntimeError(f"device status {int(step.status.item())} after warm-up")

    # The passes are captured as CUDA graphs and replayed, so the timed
    # regions hold only device work (no per-call host overhead), the way a
    # serving loop replays its captured steps: each split kernel is a
    # programmatic dependent of the one before.
    g_steps = capture(lambda: [step.step(i) for i in range(K)], device)
    step.reset()
    g_kern = capture(lambda: [step.loop_call(i) for i in range(K2)], device)
    step.reset()

    def steps_pass():
        step.reset()
        return timed(g_steps.replay, device)

    def kernel_pass():
        step.reset()
        return timed(g_kern.replay, device)

    # clocks sampled while the timed passes run
    with ClockSampler(gpu_index) as clocks:
        step_ms = repeat_passes(steps_pass, device, MIN_PASSES, min_seconds)
        kern_ms = repeat_passes(kernel_pass, device, MIN_PASSES, min_seconds)
    sep = None
    if separate:
        g_sep = capture(lambda: [step.run_separate(i) for i in range(K)], device)

        def sep_pass():
            step.reset()
            return timed(g_sep.replay, device)
        sep_ms = repeat_passes(sep_pass, device)
        sep = {"what": "gqa_cache_append then gqa_decode (same step, not fused)",
               "value": round(aggregate_rate(step.step_bytes, K, world,
                                             statistics.median(sep_ms)) / 1e9, 2),
               "ms_per_step": round(statistics.median(sep_ms) / K, 5),
               "gpu_launches_per_step": step.launches_separate}
        del g_sep
    step.reset()
    torch.cuda.synchronize(device)

    # End to end through the public API with pinned host buffers: the step
    # (host->device copy of the inputs, the fused call, device->host copy of
    # the output) captured once in a CUDA graph per step and replayed, as a
    # serving loop runs it; and the same step issued eagerly.
    hin = step.inbuf.cpu().pin_memory()
    ho = torch.empty(step.o.shape, dtype=step.o.dtype).pin_memory()
    step.run_host(hin, ho, 0)
    torch.cuda.synchronize(device)
    g_host = [capture(lambda i=i: step.run_host(hin, ho, i), device) for i in range(K)]
    step.reset()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream(device)
    barrier()
    e2e_ms = e2e_eager_ms = 0.0
    for i in range(K):
        e0.record(stream)
        g_host[i].replay()
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_ms += e0.elapsed_time(e1)
    step.reset()
    for i in range(K):
        e0.record(stream)
        step.run_host(hin, ho, i)
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_eager_ms += e0.elapsed_time(e1)
    e2e_ms = dist_max(e2e_ms, device)
    e2e_eager_ms = dist_max(e2e_eager_ms, device)
    if not torch.equal(ho.to(device), step.o):
        raise RuntimeError("the output read back to the host differs from the device output")
    if int(step.status.item()) != 0:
        raise RuntimeError(f"device status {int(step.status.item())} after timing")
    del g_steps, g_kern, g_host
    step.reset()

    peaks, peak_kind = measured_peaks()
    st = pass_stats(step_ms)
    kt = pass_stats(kern_ms)
    kern_bytes = step.loop_bytes(K2)
    achieved = kern_bytes / (kt["median_ms"] / 1e3) / 1e9
    value = aggregate_rate(step.step_bytes, K, world, st["median_ms"]) / 1e9
    h2d = hin.numel() * hin.element_size()
    d2h = ho.numel() * ho.element_size()
    res = {
        **step.describe(),
        "value": round(value, 2), "unit": "GB/s",
        "ms_per_step": round(st["median_ms"] / K, 5),
        "frac_of_spec_8TBs": round(value / SPEC_HBM_GBS, 4),
        "bytes_per_step": step.step_bytes,
        "timing": {"steps_per_pass": K, **{k: (round(v, 5) if isinstance(v, float) else v)
                                           for k, v in st.items()},
                   "what": "K steps per pass, each on its own lengths buffer, replayed from "
                           "one CUDA graph; CUDA events on the launching stream; median pass"},
        "roofline": {"bound": "hbm",
                     "kernel": "gqa_decode_append (dec::split_kernel: fused append, "
                               "in-kernel merge)",
                     "achieved": round(achieved, 2), "peak": peaks["hbm_gbs"],
                     "peak_kind": f"{peak_kind} copy bandwidth", "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "frac_of_spec_8TBs": round(achieved / SPEC_HBM_GBS, 4),
                     "bytes_per_launch": round(kern_bytes / K2),
                     "launches_per_pass": K2,
                     "avg_launch_us": round(kt["median_ms"] / K2 * 1e3, 3),
                     "passes": kt["passes"],
                     "pass_ms": {k: round(v, 5) for k, v in kt.items() if k != "passes"},
                     "calls": ("successive decode steps from the cached length (the "
                               "workload's loop)" if loop else
                               "successive calls from the cached length"),
                     "traffic": captured_traffic(w.name, "decode", window, Hkv)},
        "e2e": {"value": round(aggregate_rate(step.step_bytes, K, world, e2e_ms) / 1e9, 2),
                "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "mode": "CUDA graph of the public-API step (pinned host->device copy of "
                        "q/k_new/v_new, gqa_decode_append, device->host copy of o), "
                        "replayed once per step",
                "eager": round(aggregate_rate(step.step_bytes, K, world, e2e_eager_ms) / 1e9, 2),
                "eager_mode": "the same step issued from Python each step"},
        "gpu_launches_per_step": step.launches_per_step,
        "clocks": clocks.summary(),
    }
    if sep is not None:
        res["separate_step"] = sep
    if cpu_seconds:
        res["cpu_baseline"] = oracle_decode_sample(step, cpu_seconds, single=True)
    return step, res


class PrefillStep:
    """One gqa_prefill over a whole prompt batch.  When a launch's inputs and
    output fit in L2, NL independent copies are used in turn (launch i on
    copy i mod NL), so no launch finds its data in L2 and launches can run
    back to back."""

    def __init__(self, w, device, window, Hkv=None):
        from grouped_query_attention_03_b200 import gqa
        self.gqa, self.w, self.window = gqa, w, window
        self.Hkv = Hkv or w.Hkv
        q, k, v = [t.to(device) for t in synthetic.qkv_prefill(
            w.B, w.Hq, self.Hkv, w.T, w.d, w.seed, std=w.std)]
        self.q, self.k, self.v = q, k, v
        self.o = torch.empty_like(q)
        t = np.arange(w.T)
        lo = np.maximum(0, t - (window - 1)) if window else np.zeros_like(t)
        self.pairs = int((t - lo + 1).sum())          # permitted pairs per (b, h)
        self.flops = 4 * w.d * self.pairs * w.B * w.Hq  # QK^T + PV, 2 flops per MAC
        self.in_bytes = sum(x.numel() * x.element_size() for x in (q, k, v))
        self.io_bytes = self.in_bytes + self.o.numel() * self.o.element_size()
        self.NL = n_copies(self.io_bytes)
        self.sets = [(q, k, v, self.o)] + [
            (q.clone(), k.clone(), v.clone(), torch.empty_like(self.o)) for _ in range(self.NL - 1)]

    def run(self, i=0):
        q, k, v, o = self.sets[i % self.NL]
        self.gqa.prefill(q, k, v, window=self.window, out=o)

    def describe(self):
        w = self.w
        return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": self.Hkv, "d": w.d, "T": w.T,
                "window": self.window, "permitted_pairs_per_head": self.pairs}

    def kernel(self):
        """The tensor-core kernel gqa_prefill dispatches to for this shape."""
        w = self.w
        return self.gqa.prefill_kernel(w.B, w.Hq, self.Hkv, w.T, w.d, self.window)


KERNEL_NAMES = {
    "simt": "prefill_simt_kernel (CUDA cores)",
    "pair": "pf2::prefill_pair_kernel (two query heads of one KV group per CTA)",
    "split": "pfp::prefill_persist_kernel (one query head per work item, one persistent CTA per "
             "SM; two softmax warpgroups over keys 0-63 and 64-127 of each tile, each with its own "
             "running maximum, sum and O; epilogue on its own warpgroup)",
}


def measure_prefill(w, window, device, reps, warmup, Hkv=None, min_passes=MIN_PASSES):
    """Per-launch prefill time: `reps` launches back to back from one CUDA
    graph (CUDA events around the pass), on NL copies of the inputs in turn
    when they fit in L2; repeated passes, median pass / reps reported."""
    step = PrefillStep(w, device, window, Hkv)
    for i in range(warmup):
        step.run(i)
    torch.cuda.synchronize(device)
    alone = None
    if step.NL == 1:
        # The same launch timed alone, before the long back-to-back leg and
        # with the GPU idle for a few ms before each launch (clocks as for a
        # single call, the burst matmul figure's condition).
        g1 = capture(lambda: step.run(0), device)
        time.sleep(0.2)
        one = []
        for _ in range(max(5, min(reps, 20))):
            time.sleep(0.005)
            one.append(timed(g1.replay, device))
        del g1
        one = dist_max_list(one, device)
        ms1 = statistics.median(one)
        tf1 = step.flops / (ms1 / 1e3) / 1e12
        alone = {"tflops": round(tf1, 2), "us": round(ms1 * 1e3, 2), "launches": len(one),
                 "frac_of_burst": round(tf1 / measured_peaks()[0]["bf16_tflops"], 4),
                 "what": "single launches before the back-to-back leg, the GPU idle 5 ms "
                         "before each; median"}
    graph = capture(lambda: [step.run(i) for i in range(reps)], device)
    ms_pass = repeat_passes(lambda: timed(graph.replay, device), device, min_passes)
    del graph
    st = pass_stats(ms_pass)
    ms = st["median_ms"] / reps
    peaks, kind = measured_peaks()
    tflops = step.flops / (ms / 1e3) / 1e12
    # The burst matmul figure is the peak for a kernel timed alone; launches
    # back to back for a quarter of a second or more run under the power cap,
    # which the sustained figure was measured under.
    sustained = sum(ms_pass) > 250.0 and "bf16_tflops_sustained" in peaks
    peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    res = {
        **step.describe(), "kernel": KERNEL_NAMES[step.kernel()], "tflops": round(tflops, 2), "ms": round(ms, 5),
        "launches_per_pass": reps, "passes": st["passes"],
        "pass_ms": {k: round(v, 5) for k, v in st.items() if k != "passes"},
        "timed_ms": round(sum(ms_pass), 2),
        "flops": step.flops, "peak": peak, "frac_of_measured": round(tflops / peak, 4),
        "peak_kind": f"{kind} bf16 matmul ({'sustained' if sustained else 'burst'})",
        "frac_of_burst": round(tflops / peaks["bf16_tflops"], 4),
        "frac_of_spec_2250": round(tflops / SPEC_BF16_TFLOPS, 4),
        "alone": alone,
        "traffic": captured_traffic(w.name, "prefill", window, Hkv),
        "l2": "inputs exceed the 126 MB L2; launches back to back" if step.NL == 1 else
              f"{step.NL} copies of q, k, v and o ({step.NL * step.io_bytes / 1e6:.0f} MB in "
              f"all, above twice the 126 MB L2), launch i on copy i mod {step.NL}; launches "
              f"back to back, no flush"}
    return step, res


def oracle_decode_sample(step, max_seconds, single=True):
    """Time the fp64 oracle on a bounded sample of the same decode step (on
    all host cores, and with `single` also on one thread).  Only the sampled
    sequences are copied to the host."""
    import oracle
    cores = oracle.set_threads(0)
    B = step.w.B
    lens = np.array(step.cached) + 1

    def host(nb):
        return tuple(t[:nb].float().cpu().double().numpy() for t in (step.q, step.kc, step.vc))

    # one calibration call on a single sequence, then size the sample
    q, kc, vc = host(1)
    t0 = time.perf_counter()
    oracle.decode(q, kc, vc, lens[:1], window=step.window)
    per_seq = max(time.perf_counter() - t0, 1e-4)
    nb = int(max(1, min(B, max_seconds / per_seq)))
    reps = max(1, int(max_seconds / (per_seq * nb)))
    if nb > 1:
        q, kc, vc = host(nb)
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.decode(q[:nb], kc[:nb], vc[:nb], lens[:nb], window=step.window)
    dt = time.perf_counter() - t0
    n = lens[:nb]
    eff = np.minimum(n, step.window) if step.window else n
    bytes_ = reps * (2 * step.Hkv * eff.sum() * step.w.d * 2 + 2 * nb * step.w.Hq * step.w.d * 2)
    res = {"value": bytes_ / dt / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
           "sample": f"{reps} x decode of {nb}/{B} sequences (fp64, all permitted cells)",
           "seconds": dt}
    if not single:
        return res
    # the same on one thread: sequence 0 repeated for a third of the budget
    oracle.set_threads(1)
    try:
        t0 = time.perf_counter()
        oracle.decode(q[:1], kc[:1], vc[:1], lens[:1], window=step.window)
        one = max(time.perf_counter() - t0, 1e-4)
        reps1 = max(1, int(max_seconds / 3 / one))
        t0 = time.perf_counter()
        for _ in range(reps1):
            oracle.decode(q[:1], kc[:1], vc[:1], lens[:1], window=step.window)
        dt1 = time.perf_counter() - t0
    finally:
        oracle.set_threads(0)
    bytes1 = reps1 * (2 * step.Hkv * eff[0] * step.w.d * 2 + 2 * step.w.Hq * step.w.d * 2)
    res["single_thread"] = {"value": bytes1 / dt1 / 1e9, "unit": "GB/s", "cores": 1,
                            "sample": f"{reps1} x decode of sequence 0", "seconds": dt1}
    return res


def oracle_prefill_sample(step, max_seconds):
    """Time the fp64 oracle on a bounded sample of the same prefill: the last
    query rows of one KV group of sequence 0.  The oracle's multi-token
    decode over the whole prompt computes exactly those rows of the prefill
    (with a window they are its steady-state rows)."""
    import oracle
    cores = oracle.set_threads(0)
    w = step.w
    r, T, d = w.Hq // step.Hkv, w.T, w.d
    q = step.q[:1, :r].float().cpu().double().numpy()
    k = step.k[:1, :1].float().cpu().double().numpy()
    v = step.v[:1, :1].float().cpu().double().numpy()
    lens = np.array([T])

    def rows(t_new):
        oracle.decode_multi(q[:, :, T - t_new:], k, v, lens, window=step.window)

    t0 = time.perf_counter()
    rows(8)
    per_row = max((time.perf_counter() - t0) / 8, 1e-6)
    t_new = int(max(1, min(T, max_seconds / per_row)))
    t0 = time.perf_counter()
    rows(t_new)
    dt = time.perf_counter() - t0
    pos = np.arange(T - t_new, T)
    keys = np.minimum(pos + 1, step.window) if step.window else pos + 1
    flops = 4 * d * int(keys.sum()) * r
    # the same on one thread, for a third of the budget
    oracle.set_threads(1)
    try:
        t1 = int(max(1, min(T, max_seconds / 3 / (per_row * cores))))
        t0 = time.perf_counter()
        rows(t1)
        dt1 = time.perf_counter() - t0
    finally:
        oracle.set_threads(0)
    pos1 = np.arange(T - t1, T)
    keys1 = np.minimum(pos1 + 1, step.window) if step.window else pos1 + 1
    flops1 = 4 * d * int(keys1.sum()) * r
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"the last {t_new} of {T} query rows of one KV group ({r} heads) of "
                      f"sequence 0 (fp64)", "seconds": dt,
            "single_thread": {"value": flops1 / dt1 / 1e12, "unit": "TFLOP/s", "cores": 1,
                              "sample": f"the last {t1} rows, same group", "seconds": dt1}}


# The other decode workloads on the default line: (workload, Hkv, loop).
DECODE_ENTRIES = (
    (workloads.DECODE_RAGGED, 1, None),     # MQA endpoint
    (workloads.DECODE_RAGGED, 8, None),     # MHA endpoint
    (workloads.SWA_T32768, None, 64),       # 64 successive steps after the prompt
)


def run_gpu(args, world, rank, local):
    from grouped_query_attention_03_b200 import build as gbuild
    gbuild.build()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = workloads.BY_NAME[args.workload]
    step, head = measure_decode(
        w, device, args, world, Hkv=args.hkv, window=args.window,
        loop=w.decode_steps or None, separate=True, min_seconds=MIN_PASS_SECONDS,
        gpu_index=local)
    if args.traffic is not None:
        head["roofline"]["traffic"] = args.traffic
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_decode_sample(step, args.cpu_seconds)
    del step
    torch.cuda.empty_cache()

    decode_extra = None
    if not args.no_extra:
        decode_extra = []
        for ew, hkv, loop in DECODE_ENTRIES:
            if ew.name == w.name and hkv == args.hkv:
                continue
            s2, r2 = measure_decode(
                ew, device, args, world, Hkv=hkv, loop=loop, gpu_index=local,
                cpu_seconds=(args.cpu_seconds / 3 if rank == 0 and world == 1
                             and not args.no_cpu_baseline else None))
            decode_extra.append(r2)
            del s2
            torch.cuda.empty_cache()

    prefill_extra = None
    if not args.no_prefill:
        prefill_extra = []
        for pw, pwin, reps in ((workloads.SWA_T32768, 4096, 10),
                               (workloads.PREFILL_B4_T1024, None, 50),
                               (workloads.PREFILL_B4_T1024, 256, 50)):
            prefill_extra.append(measure_prefill(pw, pwin, device, reps, 3)[1])
            torch.cuda.empty_cache()

    if rank != 0:
        return None
    timing = head.pop("timing")
    line = {
        "metric": METRIC, "value": head.pop("value"), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head.pop("ms_per_step"),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1) rounded to bf16)",
        "config": {**{k: head.pop(k) for k in ("workload", "B", "Hq", "Hkv", "d", "window",
                                               "capacity", "keys_read_per_seq", "l2")},
                   **({"cached": head.pop("cached")} if "cached" in head else {}),
                   **({"cached_lengths": head.pop("cached_lengths")}
                      if "cached_lengths" in head else {}),
                   "timing": timing, "parallelism": f"replicas x{world}"},
        "frac_of_spec_8TBs": head.pop("frac_of_spec_8TBs"),
        "separate_step": head.pop("separate_step"),
        "roofline": head.pop("roofline"),
        "e2e": head.pop("e2e"),
        "gpu_launches": head["gpu_launches_per_step"] * args.steps,
        "clocks": head.pop("clocks"),
        "cpu_baseline": cpu,
        "decode": decode_extra,
        "prefill": prefill_extra,
    }
    return line


def run_gpu_prefill(args, world, rank, local):
    """--phase prefill: the main line is prefill TFLOP/s on one workload."""
    from grouped_query_attention_03_b200 import build as gbuild
    gbuild.build()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = workloads.BY_NAME[args.workload]
    window = args.window if args.window is not None else w.windows[0]
    barrier()
    with ClockSampler(local) as clocks:
        step, res = measure_prefill(w, window, device, args.steps, args.warmup, args.hkv)
    ms = dist_max(res["ms"], device)
    peaks, kind = measured_peaks()
    value = aggregate_rate(step.flops, 1, world, ms) / 1e12

    # End to end through the public API: q, k, v copied in from pinned host
    # memory and o copied back, inside the timed region; the step captured
    # as a CUDA graph and replayed, and the same step issued eagerly.
    hq, hk, hv = (t.cpu().pin_memory() for t in (step.q, step.k, step.v))
    ho = torch.empty(step.o.shape, dtype=step.o.dtype).pin_memory()

    def run_host():
        step.q.copy_(hq, non_blocking=True)
        step.k.copy_(hk, non_blocking=True)
        step.v.copy_(hv, non_blocking=True)
        step.run()
        ho.copy_(step.o, non_blocking=True)

    stream = torch.cuda.current_stream(device)
    for _ in range(2):
        run_host()
    torch.cuda.synchronize(device)
    g_host = capture(run_host, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = e2e_eager_ms = 0.0
    K_e2e = min(args.steps, 20)  # each step moves the whole prompt over PCIe
    for i in range(K_e2e):
        e0.record(stream)
        g_host.replay()
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_ms += e0.elapsed_time(e1)
    for i in range(K_e2e):
        e0.record(stream)
        run_host()
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_eager_ms += e0.elapsed_time(e1)
    e2e_ms = dist_max(e2e_ms, device)
    e2e_eager_ms = dist_max(e2e_eager_ms, device)
    if not torch.equal(ho.to(device), step.o):
        raise RuntimeError("the output read back to the host differs from the device output")
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = ho.numel() * ho.element_size()
    if rank != 0:
        return None
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = oracle_prefill_sample(step, args.cpu_seconds)
    return {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded normal rounded to bf16)",
        "config": dict(step.describe(), parallelism=f"replicas x{world}", l2=res["l2"]),
        "roofline": {"bound": "tensor", "kernel": KERNEL_NAMES[step.kernel()],
                     "achieved": res["tflops"], "peak": res["peak"],
                     "peak_kind": res["peak_kind"], "unit": "TFLOP/s",
                     "frac": res["frac_of_measured"], "frac_of_burst": res["frac_of_burst"],
                     "frac_of_spec_2250": res["frac_of_spec_2250"],
                     "flops_per_launch": step.flops, "avg_launch_us": round(res["ms"] * 1e3, 2),
                     "launches_per_pass": res["launches_per_pass"], "passes": res["passes"],
                     "traffic": args.traffic if args.traffic is not None else
                     captured_traffic(w.name, "prefill", window, args.hkv)},
        "e2e": {"value": round(aggregate_rate(step.flops, K_e2e, world, e2e_ms) / 1e12, 2),
                "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "mode": "CUDA graph of the public-API step (pinned host->device copies of q, k "
                        "and v, gqa_prefill, device->host copy of o), replayed once per step",
                "eager": round(aggregate_rate(step.flops, K_e2e, world, e2e_eager_ms) / 1e12, 2),
                "eager_mode": "the same step issued from Python each step", "steps": K_e2e},
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
        "cpu_baseline": cpu,
    }


def run_reference(args, world, rank):
    """The oracle as the reference arm: fp64 on the host cores, bounded."""
    if rank != 0:
        return None
    w = workloads.BY_NAME[args.workload]
    step = DecodeStep.__new__(DecodeStep)
    step.w = w
    step.Hkv = args.hkv or w.Hkv
    step.window, step.cached, step.C = decode_shape(w, args.window)
    B, Hq, d = w.B, w.Hq, w.d
    C = step.C
    step.q, step.kc, step.vc = synthetic.decode_inputs(B, Hq, step.Hkv, C, d, w.seed, std=w.std)
    budget = max(1.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_decode_sample(step, budget, single=False)
    samples = [oracle_decode_sample(step, budget, single=False) for _ in range(args.steps)]
    secs = sum(s["seconds"] for s in samples)
    value = statistics.mean(s["value"] for s in samples)
    n = np.array(step.cached) + 1
    desc = {"workload": w.name, "B": B, "Hq": Hq, "Hkv": step.Hkv, "d": d, "window": step.window,
            "capacity": C, "parallelism": "oracle on host cores"}
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / max(1, args.steps) * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": desc,
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "kind": "oracle",
                         "cores": samples[0]["cores"], "sample": samples[0]["sample"]},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["own", "reference"], default="own")
    ap.add_argument("--workload", default=workloads.DECODE_B8_N8000.name)
    ap.add_argument("--hkv", type=int, default=None, help="override Hkv (ragged MQA/MHA endpoints)")
    ap.add_argument("--window", type=int, default=None)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--phase", choices=["decode", "prefill"], default="decode")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the prefill figures on the decode line")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other decode workloads on the decode line")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per launch for the roofline (default: the "
                         "captured figure while the kernel is unchanged, else null)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    return args


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        # The oracle runs on rank 0 only; the other ranks exit without work.
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = dist_setup(args)
    try:
        if args.phase == "prefill":
            line = run_gpu_prefill(args, world, rank, local)
        else:
            line = run_gpu(args, world, rank, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
