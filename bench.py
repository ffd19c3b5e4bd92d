"""Benchmark of the GQA hot path on B200 (one JSON line on rank 0).

A step is one pass of the decode hot path over one batch: reset the lengths
to the cached count, then one gqa_decode_append call, which appends the new
token's K/V row to the cache and decodes it against the cache in the same
kernel (head map, permitted window, scores, online softmax, value mix,
split-K merge).  The same step unfused (gqa_cache_append, then gqa_decode)
is reported beside it.  The default workload is bf16 decode with B=8, Hq=32,
Hkv=8, d=128 and 8000 cached cells per sequence (8001 keys read with the
new token).

value  = algorithmic bytes per step x steps x ranks / max-over-ranks time,
         algorithmic bytes = K+V of every permitted cell + Q + O + the
         appended rows (read and written)
e2e    = the same through the public API with host buffers: the pinned
         host->device copy of the step's q and new K/V (one packed buffer)
         and the device->host read of o inside the timed region; the step is
         captured in a CUDA graph and replayed (the eager figure is beside it)
roofline = the fused split-K decode kernel against the measured HBM copy
         bandwidth
cpu_baseline = the fp64 oracle on this host's cores on a bounded sample

Usage: python bench.py [--gpus N --steps K --warmup W] [--impl reference]
                       [--workload NAME]
Multi-GPU (torchrun): every rank runs its own independent batch (replicas,
weak scaling; the path has no exchange step), timing is max over ranks.
"""
import argparse
import json
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
FALLBACK_HBM_GBS = 6650.0


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


# DRAM bytes (read + write) per launch of the dominant kernel, from the ncu
# captures summarised in profiles/, keyed by (workload, phase).  Each holds
# the SHA-256 of the kernel's source files at capture time, comments and
# blank lines stripped: once the code changes the figure no longer describes
# the kernel and is reported as null (a comment edit does not count).
CAPTURED_TRAFFIC = {
    ("decode_b8_n8000", "decode"): {
        "bytes": 268_888_576, "window": None, "hkv": None,
        "sources": ["decode_splitk.cuh", "common.cuh", "tc_ptx.cuh"],
        "sha256": "469e7abd4723ef10c25be45c3b3cbd9aa34bb86e61b8ae0969f0048e75fed2f6",
        "profile": "profiles/decode_split_kernel_b8_n8000.md"},
    ("swa_t32768", "prefill"): {
        "bytes": 692_894_976, "window": 4096, "hkv": None,
        "sources": ["prefill_pair.cuh", "common.cuh", "tc_ptx.cuh"],
        "sha256": "8c21ff11fc3aa0eda24d66f6c45b5c1a8fec2dec9750684743198082896bf26a",
        "profile": "profiles/prefill_pair_kernel_swa_t32768.md"},
}


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
    c = CAPTURED_TRAFFIC.get((workload, phase))
    if c is None or window != c["window"] or hkv != c["hkv"]:
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


class DecodeStep:
    """Append one token per sequence and decode it; the lengths are reset to
    the cached count first so every step reads the same number of cells.

    The step is one gqa_decode_append call (the append fused into the decode
    kernel); run_separate() is the same step as gqa_cache_append followed by
    gqa_decode, reported beside it."""

    def __init__(self, w, device, Hkv=None, window=None, extra=0):
        from grouped_query_attention_03_b200 import gqa
        self.gqa = gqa
        self.w = w
        self.Hkv = Hkv or w.Hkv
        self.window, self.cached, C = decode_shape(w, window)
        # `extra` spare cells of capacity let the fused call run back to back
        # (each call appends one cell) when it is timed alone
        self.extra = extra
        self.C = C + extra
        B, Hq, d = w.B, w.Hq, w.d
        C = self.C
        q, kc, vc = synthetic.decode_inputs(B, Hq, self.Hkv, C, d, w.seed, std=w.std)
        self.kc, self.vc = kc.to(device), vc.to(device)
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
        self.lens = self.lens0.clone()
        self.o = torch.empty_like(self.q)
        self.ws = gqa.decode_workspace(self.q, self.kc)
        self.status = gqa.new_status(device)
        self.kv_bytes = self.kv_bytes_at(0)
        e = 2  # bf16
        self.qo_bytes = int(2 * B * Hq * d * e)
        # the new K/V rows are read once (counted in kv_bytes) and written once
        self.write_bytes = int(2 * B * self.Hkv * d * e)
        self.decode_bytes = self.kv_bytes + self.qo_bytes
        self.step_bytes = self.decode_bytes + self.write_bytes
        self.launches_per_step = 1  # the fused kernel (plus a lengths copy and a counter memset)
        self.launches_separate = 3  # append copy + commit, split kernel

    def kv_bytes_at(self, grown):
        """K+V bytes one step reads when `grown` cells were appended since the
        lengths were reset (the window caps the cells read)."""
        n = np.array(self.cached) + 1 + grown
        eff = np.minimum(n, self.window) if self.window else n
        return int(2 * self.Hkv * eff.sum() * self.w.d * 2)

    def step_bytes_at(self, grown):
        return self.kv_bytes_at(grown) + self.qo_bytes + self.write_bytes

    def reset(self):
        self.lens.copy_(self.lens0, non_blocking=True)

    def run_kernel(self):
        self.gqa.decode_append(self.q, self.kc, self.vc, self.kn, self.vn, self.lens,
                               window=self.window, out=self.o, workspace=self.ws,
                               status=self.status)

    def run(self):
        self.reset()
        self.run_kernel()

    def run_separate(self):
        self.reset()
        self.gqa.cache_append(self.kc, self.vc, self.kn, self.vn, self.lens, status=self.status)
        self.gqa.decode(self.q, self.kc, self.vc, self.lens, window=self.window, out=self.o,
                        workspace=self.ws, status=self.status)

    def run_host(self, hin, ho):
        """One step through the public API: the step's inputs from a pinned
        host buffer (q, k_new, v_new packed), the output back to pinned host
        memory."""
        self.inbuf.copy_(hin, non_blocking=True)
        self.run()
        ho.copy_(self.o, non_blocking=True)

    def describe(self):
        w = self.w
        d = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": self.Hkv, "d": w.d,
             "window": self.window, "capacity": self.C - self.extra,
             "keys_read_per_seq": "cached+1 (the appended token)",
             "l2": "inputs exceed the 126 MB L2; no flush" if self.kv_bytes > 126e6
             else "L2 flushed before every step by reading a 256 MB buffer (outside the timed interval)",
             "timing": "CUDA graph of one step replayed K times; CUDA events on the launching stream"}
        if w.ragged:
            d["cached_lengths"] = f"uniform [{w.ragged[0]}, {w.ragged[1]}], seed {w.seed}"
        else:
            d["cached"] = w.cached
        return d


class PrefillStep:
    """One gqa_prefill over a whole prompt batch."""

    def __init__(self, w, device, window, Hkv=None):
        from grouped_query_attention_03_b200 import gqa
        self.gqa, self.w, self.window = gqa, w, window
        self.Hkv = Hkv or w.Hkv
        self.q, self.k, self.v = [t.to(device) for t in synthetic.qkv_prefill(
            w.B, w.Hq, self.Hkv, w.T, w.d, w.seed, std=w.std)]
        self.o = torch.empty_like(self.q)
        t = np.arange(w.T)
        lo = np.maximum(0, t - (window - 1)) if window else np.zeros_like(t)
        self.pairs = int((t - lo + 1).sum())          # permitted pairs per (b, h)
        self.flops = 4 * w.d * self.pairs * w.B * w.Hq  # QK^T + PV, 2 flops per MAC
        self.in_bytes = sum(x.numel() * x.element_size() for x in (self.q, self.k, self.v))

    def run(self):
        self.gqa.prefill(self.q, self.k, self.v, window=self.window, out=self.o)

    def describe(self):
        w = self.w
        return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": self.Hkv, "d": w.d, "T": w.T,
                "window": self.window, "permitted_pairs_per_head": self.pairs}

    def kernel(self):
        """The tensor-core kernel gqa_prefill dispatches to for this shape."""
        w = self.w
        if w.d in (64, 128) and (w.Hq // self.Hkv) % 2 == 0:
            return "pf2::prefill_pair_kernel (two query heads of one KV group per CTA)"
        return "pf::prefill_kernel (one query head per CTA)"


def measure_prefill(w, window, device, reps, warmup, Hkv=None):
    """Per-launch prefill time (CUDA events), L2 flushed between launches
    when the inputs fit in L2."""
    step = PrefillStep(w, device, window, Hkv)
    flush = make_flush(device) if step.in_bytes <= 126e6 else None
    for _ in range(warmup):
        step.run()
    graph = capture(step.run, device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for a, b in evs:
        if flush is not None:
            flush_l2(flush)
        a.record()
        graph.replay()
        b.record()
    torch.cuda.synchronize(device)
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    peaks, kind = measured_peaks()
    tflops = step.flops / (ms / 1e3) / 1e12
    return step, {
        **step.describe(), "kernel": step.kernel(), "tflops": round(tflops, 2), "ms": round(ms, 4),
        "flops": step.flops, "frac_of_measured": round(tflops / peaks["bf16_tflops"], 4),
        "peak_kind": f"{kind} bf16 matmul (burst)", "frac_of_spec_2250": round(tflops / 2250.0, 4),
        "l2": "inputs exceed L2" if flush is None else "L2 flushed between launches"}


def oracle_decode_sample(step, max_seconds, single=True):
    """Time the fp64 oracle on a bounded sample of the same decode step (on
    all host cores, and with `single` also on one thread)."""
    import oracle
    cores = oracle.set_threads(0)
    B = step.w.B
    nb = B
    q = step.q.float().cpu().double().numpy()
    kc = step.kc.float().cpu().double().numpy()
    vc = step.vc.float().cpu().double().numpy()
    lens = np.array(step.cached) + 1
    # one calibration call on a single sequence, then size the sample
    t0 = time.perf_counter()
    oracle.decode(q[:1], kc[:1], vc[:1], lens[:1], window=step.window)
    per_seq = max(time.perf_counter() - t0, 1e-4)
    nb = int(max(1, min(B, max_seconds / per_seq)))
    reps = max(1, int(max_seconds / (per_seq * nb)))
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


def make_flush(device):
    """A 256 MB buffer whose read evicts the 126 MB L2 with clean lines (a
    write-based flush would leave dirty lines whose write-back the next
    kernel would pay for)."""
    return torch.ones(64 << 20, dtype=torch.float32, device=device)


def flush_l2(buf):
    return buf.sum()


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


def run_gpu(args, world, rank, local):
    from grouped_query_attention_03_b200 import build as gbuild
    gbuild.build()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = workloads.BY_NAME[args.workload]
    K2 = min(args.steps, 100)  # back-to-back calls of the fused kernel alone
    step = DecodeStep(w, device, Hkv=args.hkv, window=args.window, extra=K2 + 2)
    stream = torch.cuda.current_stream(device)
    need_flush = step.kv_bytes <= 126e6
    flush = make_flush(device) if need_flush else None
    for _ in range(args.warmup):
        if flush is not None:
            flush_l2(flush)
        step.run()
    torch.cuda.synchronize(device)
    if int(step.status.item()) != 0:
        raise RuntimeError(f"device status {int(step.status.item())} after warm-up")
    # The step (fused), the same step unfused, and the gqa_decode_append call
    # alone, captured once and replayed: the timed regions hold only device
    # work (no per-call host overhead).
    g_step = capture(step.run, device)
    g_sep = capture(step.run_separate, device)
    g_reset = capture(step.reset, device)
    step.reset()
    g_dec = capture(step.run_kernel, device)

    def events(n):
        return [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(n)]

    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(local) as clocks:
        if flush is None:
            # inputs exceed L2: steps back to back
            start.record(stream)
            for i in range(K):
                g_step.replay()
            end.record(stream)
            torch.cuda.synchronize(device)
            total_ms = start.elapsed_time(end)
            start.record(stream)
            for i in range(K):
                g_sep.replay()
            end.record(stream)
            torch.cuda.synchronize(device)
            sep_ms = start.elapsed_time(end)
        else:
            # L2 flushed (outside the timed intervals) before every step
            step_ev, sep_ev = events(K), events(K)
            for i in range(K):
                flush_l2(flush)
                step_ev[i][0].record(stream)
                g_step.replay()
                step_ev[i][1].record(stream)
            for i in range(K):
                flush_l2(flush)
                sep_ev[i][0].record(stream)
                g_sep.replay()
                sep_ev[i][1].record(stream)
            torch.cuda.synchronize(device)
            total_ms = sum(a.elapsed_time(b) for a, b in step_ev)
            sep_ms = sum(a.elapsed_time(b) for a, b in sep_ev)
        # the gqa_decode_append call alone, K2 calls in a row from the reset
        # lengths (call i reads i more cells; its bytes are counted so)
        g_reset.replay()
        if flush is None:
            # inputs exceed L2: the calls back to back, one event pair
            start.record(stream)
            for i in range(K2):
                g_dec.replay()
            end.record(stream)
            torch.cuda.synchronize(device)
            dec_ms = [start.elapsed_time(end)]
        else:
            dec_ev = events(K2)
            for i in range(K2):
                flush_l2(flush)
                dec_ev[i][0].record(stream)
                g_dec.replay()
                dec_ev[i][1].record(stream)
            torch.cuda.synchronize(device)
            dec_ms = [a.elapsed_time(b) for a, b in dec_ev]
        g_reset.replay()
        torch.cuda.synchronize(device)
    dec_bytes = [step.step_bytes_at(i) for i in range(K2)]
    barrier()
    sep_ms = dist_max(sep_ms, device)
    total_ms = dist_max(total_ms, device)
    dec_avg_ms = sum(dec_ms) / K2

    # End to end through the public API with pinned host buffers: the step
    # (host->device copy of the inputs, the fused call, device->host copy of
    # the output) captured once in a CUDA graph and replayed per step, as a
    # serving loop runs it; and the same step issued eagerly from Python.
    hin = step.inbuf.cpu().pin_memory()
    ho = torch.empty(step.o.shape, dtype=step.o.dtype).pin_memory()
    for _ in range(2):
        step.run_host(hin, ho)
    torch.cuda.synchronize(device)
    g_host = capture(lambda: step.run_host(hin, ho), device)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = e2e_eager_ms = 0.0
    for i in range(K):
        if flush is not None:
            flush_l2(flush)
        e0.record(stream)
        g_host.replay()
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_ms += e0.elapsed_time(e1)
    for i in range(K):
        if flush is not None:
            flush_l2(flush)
        e0.record(stream)
        step.run_host(hin, ho)
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_eager_ms += e0.elapsed_time(e1)
    e2e_ms = dist_max(e2e_ms, device)
    e2e_eager_ms = dist_max(e2e_eager_ms, device)
    if not torch.equal(ho.to(device), step.o):
        raise RuntimeError("the output read back to the host differs from the device output")
    if int(step.status.item()) != 0:
        raise RuntimeError(f"device status {int(step.status.item())} after timing")

    prefill_extra = None
    if rank == 0 and not args.no_prefill:
        prefill_extra = [measure_prefill(workloads.SWA_T32768, 4096, device, 10, 3)[1],
                         measure_prefill(workloads.PREFILL_B4_T1024, None, device, 20, 3)[1],
                         measure_prefill(workloads.PREFILL_B4_T1024, 256, device, 20, 3)[1]]
    peaks, peak_kind = measured_peaks()
    value = aggregate_rate(step.step_bytes, K, world, total_ms) / 1e9
    achieved = sum(dec_bytes) / (sum(dec_ms) / 1e3) / 1e9
    h2d = hin.numel() * hin.element_size()
    d2h = ho.numel() * ho.element_size()
    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = oracle_decode_sample(step, args.cpu_seconds)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": round(total_ms / K, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded N(0,1) rounded to bf16)",
            "config": dict(step.describe(), parallelism=f"replicas x{world}"),
            "frac_of_spec_8TBs": round(value / SPEC_HBM_GBS, 4),
            "separate_step": {"what": "gqa_cache_append then gqa_decode (same step, not fused)",
                              "value": round(aggregate_rate(step.step_bytes, K, world, sep_ms) / 1e9, 2),
                              "ms_per_step": round(sep_ms / K, 5),
                              "gpu_launches_per_step": step.launches_separate},
            "roofline": {"bound": "hbm",
                         "kernel": "gqa_decode_append (counter memset + dec::split_kernel: fused append, in-kernel merge)",
                         "achieved": round(achieved, 2), "peak": peaks["hbm_gbs"],
                         "peak_kind": f"{peak_kind} copy bandwidth", "unit": "GB/s",
                         "frac": round(achieved / peaks["hbm_gbs"], 4),
                         "frac_of_spec_8TBs": round(achieved / SPEC_HBM_GBS, 4),
                         "bytes_per_launch": round(statistics.mean(dec_bytes)),
                         "launches_timed": K2,
                         "avg_launch_us": round(dec_avg_ms * 1e3, 3),
                         "traffic": args.traffic if args.traffic is not None else
                         captured_traffic(w.name, "decode", args.window, args.hkv)},
            "e2e": {"value": round(aggregate_rate(step.step_bytes, K, world, e2e_ms) / 1e9, 2),
                    "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "mode": "CUDA graph of the public-API step (pinned host->device copy of "
                            "q/k_new/v_new, gqa_decode_append, device->host copy of o), "
                            "replayed once per step",
                    "eager": round(aggregate_rate(step.step_bytes, K, world, e2e_eager_ms) / 1e9, 2),
                    "eager_mode": "the same step issued from Python each step"},
            "gpu_launches": step.launches_per_step * K,
            "clocks": clocks.summary(),
            "cpu_baseline": cpu,
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
        "roofline": {"bound": "tensor", "kernel": step.kernel(),
                     "achieved": res["tflops"], "peak": peaks["bf16_tflops"],
                     "peak_kind": f"{kind} bf16 matmul (burst)", "unit": "TFLOP/s",
                     "frac": res["frac_of_measured"], "frac_of_spec_2250": res["frac_of_spec_2250"],
                     "flops_per_launch": step.flops, "avg_launch_us": round(res["ms"] * 1e3, 2),
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
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["own", "reference"], default="own")
    ap.add_argument("--workload", default=workloads.DECODE_B8_N8000.name)
    ap.add_argument("--hkv", type=int, default=None, help="override Hkv (ragged MQA/MHA endpoints)")
    ap.add_argument("--window", type=int, default=None)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--phase", choices=["decode", "prefill"], default="decode")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the prefill figures on the decode line")
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
