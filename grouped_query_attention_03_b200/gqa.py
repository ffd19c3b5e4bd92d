"""ctypes binding of the C ABI in ``include/gqa.h`` (argument marshalling only).

Every computation runs in the CUDA library ``libgqa_b200.so``; this module
checks tensor dtypes, devices and contiguity, passes raw device pointers and
the current CUDA stream, and turns a non-zero ``gqa_status`` into
``GQAError``.  There is no fallback: if the library is missing, every call
raises.  PyTorch provides device memory and streams, nothing else.
"""
import ctypes
import os

import torch

from . import build as _build

LIB_PATH = _build.LIB

GQA_F32, GQA_BF16 = 0, 1
NO_WINDOW = -1

STATUS_NAMES = {
    0: "GQA_OK", 1: "GQA_ERR_NULL", 2: "GQA_ERR_SHAPE", 3: "GQA_ERR_GROUPS",
    4: "GQA_ERR_WINDOW", 5: "GQA_ERR_CAPACITY", 6: "GQA_ERR_OVERFLOW",
    7: "GQA_ERR_UNSUPPORTED", 8: "GQA_ERR_WORKSPACE", 9: "GQA_ERR_CUDA",
    10: "GQA_ERR_DEVICE", 11: "GQA_ERR_TIMEOUT", 12: "GQA_ERR_SEGMENT",
}

# Every symbol include/gqa.h declares.
EXPORTS = ("gqa_prefill", "gqa_prefill_packed", "gqa_decode", "gqa_decode_workspace_bytes",
           "gqa_decode_append", "gqa_decode_multi", "gqa_decode_noalloc", "gqa_cache_append", "gqa_cache_bytes",
           "gqa_ring_append", "gqa_ring_decode_append", "gqa_kv_head_for_query", "gqa_window_start", "gqa_prefill_kernel", "gqa_status_string",
           "gqa_version", "gqa_selftest_wait_timeout")

NOALLOC_SCRATCH_BYTES = 8 << 20  # GQA_NOALLOC_SCRATCH_BYTES in include/gqa.h


class GQAError(RuntimeError):
    def __init__(self, status, what):
        self.status = int(status)
        name = STATUS_NAMES.get(self.status, str(status))
        super().__init__(f"{what}: {name} ({_status_string(self.status)})")


_lib = None


def lib():
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"CUDA library {LIB_PATH} is missing; build it with "
                "grouped_query_attention_03_b200.build.build()")
        _lib = _declare(ctypes.CDLL(LIB_PATH))
    return _lib


def _declare(L):
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    sz, i64 = ctypes.c_size_t, ctypes.c_int64
    L.gqa_prefill.argtypes = [i32, vp, vp, vp, vp, vp] + [i32] * 6 + [f32, vp, vp]
    L.gqa_prefill.restype = i32
    L.gqa_prefill_packed.argtypes = [i32, vp, vp, vp, vp, vp, vp] + [i32] * 6 + [f32, vp, vp]
    L.gqa_prefill_packed.restype = i32
    L.gqa_decode.argtypes = [i32, vp, vp, vp, vp, vp] + [i32] * 6 + [f32, vp, sz, vp, vp]
    L.gqa_decode.restype = i32
    L.gqa_decode_append.argtypes = [i32] + [vp] * 7 + [i32] * 6 + [f32, vp, sz, vp, vp]
    L.gqa_decode_append.restype = i32
    L.gqa_decode_multi.argtypes = [i32, vp, vp, vp, vp, vp] + [i32] * 7 + [f32, vp, vp]
    L.gqa_decode_multi.restype = i32
    L.gqa_decode_noalloc.argtypes = [i32, vp, vp, vp, vp, vp] + [i32] * 6 + [f32, vp, vp]
    L.gqa_decode_noalloc.restype = i32
    L.gqa_decode_workspace_bytes.argtypes = [i32] * 6
    L.gqa_decode_workspace_bytes.restype = sz
    L.gqa_cache_append.argtypes = [i32, vp, vp, vp, vp, vp] + [i32] * 5 + [vp, vp]
    L.gqa_cache_append.restype = i32
    L.gqa_ring_append.argtypes = [i32, vp, vp, vp, vp, vp] + [i32] * 5 + [vp, vp]
    L.gqa_ring_append.restype = i32
    L.gqa_ring_decode_append.argtypes = [i32] + [vp] * 7 + [i32] * 5 + [f32, vp, sz, vp, vp]
    L.gqa_ring_decode_append.restype = i32
    L.gqa_cache_bytes.argtypes = [i64] * 6
    L.gqa_cache_bytes.restype = ctypes.c_uint64
    L.gqa_kv_head_for_query.argtypes = [i32] * 3
    L.gqa_kv_head_for_query.restype = i32
    L.gqa_prefill_kernel.argtypes = [i32] * 7
    L.gqa_prefill_kernel.restype = i32
    L.gqa_window_start.argtypes = [i32, i32]
    L.gqa_window_start.restype = i32
    L.gqa_status_string.argtypes = [i32]
    L.gqa_status_string.restype = ctypes.c_char_p
    L.gqa_version.argtypes = []
    L.gqa_version.restype = ctypes.c_char_p
    L.gqa_selftest_wait_timeout.argtypes = [i64, i32, vp, vp, vp]
    L.gqa_selftest_wait_timeout.restype = i32
    return L


def _status_string(s):
    try:
        return lib().gqa_status_string(int(s)).decode()
    except Exception:  # pragma: no cover - only while reporting another error
        return "?"


def _check(status, what):
    if status != 0:
        raise GQAError(status, what)


def _run(dev, what, fn, *args):
    """Call a C entry point with `dev` (the tensors' device) current: the
    library looks up per-device state (SM count, fixed scratch address) on
    the current device."""
    with torch.cuda.device(dev):
        _check(fn(*args), what)


def _dtype_code(t):
    if t.dtype == torch.float32:
        return GQA_F32
    if t.dtype == torch.bfloat16:
        return GQA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _ptr(t, name, dtype=None, device=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must live in CUDA device memory")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _window(window):
    return NO_WINDOW if window is None else int(window)


def ring_append(k_ring, v_ring, k_new, v_new, seq_lens, *, status=None, stream=None):
    """Rolling buffer of W slots (k_ring [B,Hkv,W,d]): write positions
    [len_b, len_b + t_new) at slots p mod W (the last W of them survive) and
    advance seq_lens in place."""
    B, Hkv, W, d = k_ring.shape
    t_new = k_new.shape[2]
    if k_new.shape != (B, Hkv, t_new, d) or v_new.shape != k_new.shape:
        raise ValueError("new K/V shape mismatch")
    dev = k_ring.device
    st = new_status(dev) if status is None else status
    _run(dev, "gqa_ring_append", lib().gqa_ring_append,
         _dtype_code(k_ring), _ptr(k_ring, "k_ring"), _ptr(v_ring, "v_ring", k_ring.dtype, dev),
         _ptr(k_new, "k_new", k_ring.dtype, dev), _ptr(v_new, "v_new", k_ring.dtype, dev),
         _ptr(seq_lens, "seq_lens", torch.int32, dev), B, Hkv, W, d, t_new,
         _ptr(st, "status", torch.int32, dev), _stream(stream, dev))


def ring_decode_append(q, k_ring, v_ring, k_new, v_new, seq_lens, *, scale=None, out=None,
                       workspace=None, status=None, stream=None):
    """The decode step against a rolling buffer of W slots, the step's row
    appended in the same call: the query at position len_b reads the last W
    positions; seq_lens (positions before the step) grows by one."""
    B, Hq, d = q.shape
    Hkv, W = k_ring.shape[1], k_ring.shape[2]
    if k_ring.shape != (B, Hkv, W, d) or v_ring.shape != k_ring.shape:
        raise ValueError("ring shape mismatch")
    if k_new.shape != (B, Hkv, 1, d) or v_new.shape != k_new.shape:
        raise ValueError("new K/V must be [B,Hkv,1,d]")
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    dev = q.device
    if workspace is None:
        workspace = decode_workspace(q, k_ring)
    st = new_status(dev) if status is None else status
    _run(dev, "gqa_ring_decode_append", lib().gqa_ring_decode_append,
         _dtype_code(q), _ptr(q, "q"), _ptr(k_ring, "k_ring", q.dtype, dev),
         _ptr(v_ring, "v_ring", q.dtype, dev), _ptr(k_new, "k_new", q.dtype, dev),
         _ptr(v_new, "v_new", q.dtype, dev), _ptr(out, "out", q.dtype, dev),
         _ptr(seq_lens, "seq_lens", torch.int32, dev), B, Hq, Hkv, W, d, float(scale),
         _ptr(workspace, "workspace", torch.uint8, dev), workspace.numel(),
         _ptr(st, "status", torch.int32, dev), _stream(stream, dev))
    return out


def new_status(device):
    """A zeroed device int32 status word."""
    return torch.zeros(1, dtype=torch.int32, device=device)


def prefill(q, k, v, *, window=None, scale=None, seq_lens=None, out=None,
            status=None, stream=None):
    """o = GQA(q, k, v) over whole prompts.  q [B,Hq,T,d], k/v [B,Hkv,T,d]."""
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, T, d) or v.shape != k.shape:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)} k {tuple(k.shape)} v {tuple(v.shape)}")
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    dev = q.device
    st = status
    _run(dev, "gqa_prefill", lib().gqa_prefill,
         _dtype_code(q), _ptr(q, "q"), _ptr(k, "k", q.dtype, dev), _ptr(v, "v", q.dtype, dev),
         _ptr(out, "out", q.dtype, dev), _ptr(seq_lens, "seq_lens", torch.int32, dev),
         B, Hq, Hkv, T, d, _window(window), float(scale),
         _ptr(st, "status", torch.int32, dev), _stream(stream, dev))
    return out


def prefill_packed(q, k, v, seg_start, *, window=None, scale=None, seq_lens=None,
                   out=None, status=None, stream=None):
    """prefill() over packed sequences: seg_start [B,T] int32 holds each
    cell's segment start; cell t attends [max(seg_start, t-(w-1)), t]."""
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, T, d) or v.shape != k.shape:
        raise ValueError("shape mismatch")
    if tuple(seg_start.shape) != (B, T):
        raise ValueError("seg_start must be [B, T]")
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    dev = q.device
    st = new_status(dev) if status is None else status
    _run(dev, "gqa_prefill_packed", lib().gqa_prefill_packed,
         _dtype_code(q), _ptr(q, "q"), _ptr(k, "k", q.dtype, dev), _ptr(v, "v", q.dtype, dev),
         _ptr(out, "out", q.dtype, dev), _ptr(seq_lens, "seq_lens", torch.int32, dev),
         _ptr(seg_start, "seg_start", torch.int32, dev),
         B, Hq, Hkv, T, d, _window(window), float(scale), _ptr(st, "status", torch.int32, dev),
         _stream(stream, dev))
    return out


def decode_workspace_bytes(dtype, B, Hq, Hkv, C, d):
    code = GQA_BF16 if dtype == torch.bfloat16 else GQA_F32
    return int(lib().gqa_decode_workspace_bytes(code, B, Hq, Hkv, C, d))


def decode_workspace(q, k_cache):
    """A zero-filled device workspace large enough for decode on these
    shapes (reusable by later calls of any shape that fits)."""
    B, Hq, d = q.shape
    Hkv, C = k_cache.shape[1], k_cache.shape[2]
    n = decode_workspace_bytes(q.dtype, B, Hq, Hkv, C, d)
    # zero-filled once; every completed call leaves it ready for the next
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=q.device)


def decode(q, k_cache, v_cache, seq_lens, *, window=None, scale=None, out=None,
           workspace=None, status=None, stream=None):
    """One new token per sequence: q [B,Hq,d], caches [B,Hkv,C,d],
    seq_lens [B] int32 counting the cached cells including the new token."""
    B, Hq, d = q.shape
    Hkv, C = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (B, Hkv, C, d) or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape mismatch")
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    dev = q.device
    if workspace is None:
        workspace = decode_workspace(q, k_cache)
    st = new_status(dev) if status is None else status
    _run(dev, "gqa_decode", lib().gqa_decode,
         _dtype_code(q), _ptr(q, "q"), _ptr(k_cache, "k_cache", q.dtype, dev),
         _ptr(v_cache, "v_cache", q.dtype, dev), _ptr(out, "out", q.dtype, dev),
         _ptr(seq_lens, "seq_lens", torch.int32, dev), B, Hq, Hkv, C, d,
         _window(window), float(scale), _ptr(workspace, "workspace", torch.uint8, dev),
         workspace.numel(), _ptr(st, "status", torch.int32, dev), _stream(stream, dev))
    return out


def decode_append(q, k_cache, v_cache, k_new, v_new, seq_lens, *, window=None, scale=None,
                  out=None, workspace=None, status=None, stream=None):
    """The decode step with its cache append fused in: seq_lens [B] int32
    counts the cells cached BEFORE the step; k_new/v_new [B,Hkv,1,d] are the
    step's key and value rows.  Attends over the cached cells plus the new
    row, writes the new row at cell seq_lens[b] and advances seq_lens in
    place (all-or-nothing on the device)."""
    B, Hq, d = q.shape
    Hkv, C = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (B, Hkv, C, d) or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape mismatch")
    if k_new.shape != (B, Hkv, 1, d) or v_new.shape != k_new.shape:
        raise ValueError("new K/V must be [B,Hkv,1,d]")
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    dev = q.device
    if workspace is None:
        workspace = decode_workspace(q, k_cache)
    st = new_status(dev) if status is None else status
    _run(dev, "gqa_decode_append", lib().gqa_decode_append,
         _dtype_code(q), _ptr(q, "q"), _ptr(k_cache, "k_cache", q.dtype, dev),
         _ptr(v_cache, "v_cache", q.dtype, dev), _ptr(k_new, "k_new", q.dtype, dev),
         _ptr(v_new, "v_new", q.dtype, dev), _ptr(out, "out", q.dtype, dev),
         _ptr(seq_lens, "seq_lens", torch.int32, dev), B, Hq, Hkv, C, d,
         _window(window), float(scale), _ptr(workspace, "workspace", torch.uint8, dev),
         workspace.numel(), _ptr(st, "status", torch.int32, dev), _stream(stream, dev))
    return out


def decode_multi(q, k_cache, v_cache, seq_lens, *, window=None, scale=None, out=None,
                 status=None, stream=None):
    """t_new new query rows per sequence against the cache: q [B,Hq,t_new,d],
    caches [B,Hkv,C,d], seq_lens [B] int32 counting the cached cells
    including the t_new new ones (query row i sits at cell n_b - t_new + i)."""
    B, Hq, t_new, d = q.shape
    Hkv, C = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (B, Hkv, C, d) or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape mismatch")
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    dev = q.device
    st = new_status(dev) if status is None else status
    _run(dev, "gqa_decode_multi", lib().gqa_decode_multi,
         _dtype_code(q), _ptr(q, "q"), _ptr(k_cache, "k_cache", q.dtype, dev),
         _ptr(v_cache, "v_cache", q.dtype, dev), _ptr(out, "out", q.dtype, dev),
         _ptr(seq_lens, "seq_lens", torch.int32, dev), B, Hq, Hkv, C, d, t_new,
         _window(window), float(scale), _ptr(st, "status", torch.int32, dev),
         _stream(stream, dev))
    return out


def decode_noalloc(q, k_cache, v_cache, seq_lens, *, window=None, scale=None, out=None,
                   status=None, stream=None):
    """decode() without a workspace argument, for callers that cannot
    allocate device memory: the library's fixed device array serves as the
    workspace (see gqa_decode_noalloc in include/gqa.h)."""
    B, Hq, d = q.shape
    Hkv, C = k_cache.shape[1], k_cache.shape[2]
    if k_cache.shape != (B, Hkv, C, d) or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape mismatch")
    if scale is None:
        scale = d ** -0.5
    if out is None:
        out = torch.empty_like(q)
    dev = q.device
    st = new_status(dev) if status is None else status
    _run(dev, "gqa_decode_noalloc", lib().gqa_decode_noalloc,
         _dtype_code(q), _ptr(q, "q"), _ptr(k_cache, "k_cache", q.dtype, dev),
         _ptr(v_cache, "v_cache", q.dtype, dev), _ptr(out, "out", q.dtype, dev),
         _ptr(seq_lens, "seq_lens", torch.int32, dev), B, Hq, Hkv, C, d,
         _window(window), float(scale), _ptr(st, "status", torch.int32, dev),
         _stream(stream, dev))
    return out


def cache_append(k_cache, v_cache, k_new, v_new, seq_lens, *, status=None, stream=None):
    """Write k_new/v_new [B,Hkv,t_new,d] at cells [len_b, len_b+t_new) and
    advance seq_lens in place (all-or-nothing on the device)."""
    B, Hkv, C, d = k_cache.shape
    t_new = k_new.shape[2]
    if k_new.shape != (B, Hkv, t_new, d) or v_new.shape != k_new.shape:
        raise ValueError("new K/V shape mismatch")
    dev = k_cache.device
    st = new_status(dev) if status is None else status
    _run(dev, "gqa_cache_append", lib().gqa_cache_append,
         _dtype_code(k_cache), _ptr(k_cache, "k_cache"), _ptr(v_cache, "v_cache", k_cache.dtype, dev),
         _ptr(k_new, "k_new", k_cache.dtype, dev), _ptr(v_new, "v_new", k_cache.dtype, dev),
         _ptr(seq_lens, "seq_lens", torch.int32, dev), B, Hkv, C, d, t_new,
         _ptr(st, "status", torch.int32, dev), _stream(stream, dev))
    return st


def cache_bytes(L, B, T, Hkv, d, elem_bytes):
    return int(lib().gqa_cache_bytes(L, B, T, Hkv, d, elem_bytes))


def prefill_kernel(B, Hq, Hkv, T, d, window=None, sms=None):
    """Which kernel gqa_prefill runs for a bf16 prompt of this shape: "pair"
    (two heads of a KV group per CTA), "split" (one head per CTA) or "simt"
    (CUDA cores).  `sms` defaults to the current device's SM count."""
    if sms is None:
        sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    r = lib().gqa_prefill_kernel(B, Hq, Hkv, T, d, -1 if window is None else window, sms)
    if r < 0:
        raise ValueError(f"prefill_kernel: invalid arguments {(B, Hq, Hkv, T, d, window, sms)}")
    return ("simt", "pair", "split")[r]


def kv_head_for_query(h, Hq, Hkv):
    g = lib().gqa_kv_head_for_query(h, Hq, Hkv)
    return None if g < 0 else g


def window_start(t, window):
    s = lib().gqa_window_start(t, _window(window))
    return None if s < 0 else s


def version():
    return lib().gqa_version().decode()


def selftest_wait_timeout(limit_us, *, arrive=False, device=None, status=None, stream=None):
    """Run the kernels' two bounded wait routines on mbarriers nobody
    arrives on (arrive=False: both give up after limit_us and the kernel
    records GQA_ERR_TIMEOUT) or that one thread completes first (arrive=True:
    both succeed).  Returns (status, gave_up) device tensors."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    st = new_status(dev) if status is None else status
    gave_up = torch.zeros(2, dtype=torch.int32, device=dev)
    _run(dev, "gqa_selftest_wait_timeout", lib().gqa_selftest_wait_timeout,
         int(limit_us), 1 if arrive else 0, _ptr(st, "status", torch.int32, dev),
         _ptr(gave_up, "gave_up", torch.int32, dev), _stream(stream, dev))
    return st, gave_up
