"""B200-native LCSA (locality-constrained sparse attention) library binding.

A thin ctypes face of ``liblcsa.so`` (declared in include/lcsa.h): the same
entry-point names, argument marshalling only. Every step of the call runs in
the library's CUDA kernels; there is no Python or CPU fallback, and using the
binding without the built library raises ``LcsaLibraryMissing``.

Tensors are passed as torch CUDA tensors (bf16 q, k, v, out; fp32 gains) or
as raw device addresses (int).
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblcsa.so")

ABI_VERSION = 2  # the LCSA_ABI_VERSION of include/lcsa.h this binding's structures follow
LCSA_OK = 0
LCSA_ERR_INVALID_ARG = 1
LCSA_ERR_SHAPE = 2
LCSA_ERR_ALIGNMENT = 3
LCSA_ERR_UNSUPPORTED = 4
LCSA_ERR_OOM = 5
LCSA_ERR_CUDA = 6
LCSA_ERR_DEVICE_TIMEOUT = 7
LCSA_ERR_DEVICE_BOUNDS = 8
LCSA_UNBOUNDED = 0
LCSA_NORM_TOKEN = 0
LCSA_NORM_HEAD = 1


class LcsaLibraryMissing(ImportError):
    pass


class LcsaError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__("%s: %s (%s)" % (where, _status_name(status), detail))


class lcsa_config_t(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
        ("q_frames", ctypes.c_int), ("kv_frames", ctypes.c_int),
        ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
        ("block_t", ctypes.c_int), ("block_h", ctypes.c_int), ("block_w", ctypes.c_int),
        ("local_range", ctypes.c_int), ("topk", ctypes.c_int), ("sparse_ratio", ctypes.c_float),
        ("kv_frame_offset", ctypes.c_int), ("norm_scope", ctypes.c_int),
        ("rms_eps", ctypes.c_float), ("softmax_scale", ctypes.c_float), ("host_io", ctypes.c_int),
        ("heads_total", ctypes.c_int),
    ]


class lcsa_geometry_t(ctypes.Structure):
    _fields_ = [
        ("q_tokens", ctypes.c_int64), ("kv_tokens", ctypes.c_int64), ("channels", ctypes.c_int64),
        ("block_tokens", ctypes.c_int64), ("blocks_per_frame", ctypes.c_int64),
        ("q_blocks", ctypes.c_int64), ("kv_blocks", ctypes.c_int64), ("rows", ctypes.c_int64),
        ("nnz", ctypes.c_int64), ("topk", ctypes.c_int), ("window_radius", ctypes.c_int),
        ("min_window", ctypes.c_int), ("max_window", ctypes.c_int),
        ("selected_flops", ctypes.c_double), ("prologue_bytes", ctypes.c_double),
        ("attention_min_bytes", ctypes.c_double), ("workspace_bytes", ctypes.c_size_t),
    ]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


# (name, restype, argtypes) of every entry point in include/lcsa.h
_VP = ctypes.c_void_p
_I = ctypes.c_int
_PLAN = ctypes.c_void_p
SIGNATURES = [
    ("lcsa_config_default", None, [ctypes.POINTER(lcsa_config_t)]),
    ("lcsa_config_resolve", _I, [ctypes.POINTER(lcsa_config_t), ctypes.POINTER(lcsa_geometry_t)]),
    ("lcsa_plan_create", _I, [ctypes.POINTER(lcsa_config_t), _I, ctypes.POINTER(_PLAN)]),
    ("lcsa_plan_destroy", None, [_PLAN]),
    ("lcsa_forward", _I, [_PLAN, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    ("lcsa_forward_host", _I, [_PLAN, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    ("lcsa_forward_noalloc", _I, [ctypes.POINTER(lcsa_config_t), _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    ("lcsa_noalloc_check_device_error", _I, [_VP]),
    ("lcsa_plan_create_stream", _I, [ctypes.POINTER(lcsa_config_t), _I, ctypes.POINTER(_PLAN)]),
    ("lcsa_stream_push", _I, [_PLAN, _VP, _VP, _VP, _I, _VP]),
    ("lcsa_forward_stream", _I, [_PLAN, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    ("lcsa_sumsq", _I, [_PLAN, _VP, _VP, _VP, _VP]),
    ("lcsa_plan_set_threshold_reuse", _I, [_PLAN, _I]),
    ("lcsa_selection_nnz", _I, [_PLAN, ctypes.POINTER(ctypes.c_int64)]),
    ("lcsa_forward_sharded", _I, [_PLAN, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    ("lcsa_plan_geometry", _I, [_PLAN, ctypes.POINTER(lcsa_geometry_t)]),
    ("lcsa_plan_topk", _I, [_PLAN, ctypes.POINTER(_I)]),
    ("lcsa_get_selection", _I, [_PLAN, _VP, ctypes.c_size_t, _VP, ctypes.c_size_t]),
    ("lcsa_get_intermediates", _I, [_PLAN, _VP, _VP, _VP, _VP]),
    ("lcsa_check_device_error", _I, [_PLAN, _VP]),
    ("lcsa_plan_set_timing", _I, [_PLAN, _I]),
    ("lcsa_get_kernel_times", _I, [_PLAN, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(_I)]),
    ("lcsa_selftest_exp2", _I, [_VP, _VP, _I, _VP]),
    ("lcsa_status_string", ctypes.c_char_p, [_I]),
    ("lcsa_last_error_message", ctypes.c_char_p, []),
    ("lcsa_abi_version", _I, []),
]

_lib = None


def lib():
    """The loaded liblcsa.so (raises LcsaLibraryMissing if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise LcsaLibraryMissing(
                "liblcsa.so is not built (python -m block_sparse_video_lcsa_b200.build); "
                "there is no fallback implementation")
        L = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        if L.lcsa_abi_version() != ABI_VERSION:
            raise LcsaLibraryMissing("liblcsa.so has ABI version %d, this binding needs %d: rebuild it"
                                     % (L.lcsa_abi_version(), ABI_VERSION))
        _lib = L
    return _lib


def _status_name(st: int) -> str:
    try:
        return lib().lcsa_status_string(st).decode()
    except Exception:  # noqa: BLE001 - only used to format an error
        return "status %d" % st


def _check(st: int, where: str):
    if st != LCSA_OK:
        raise LcsaError(st, where, lib().lcsa_last_error_message().decode())


def _addr(x) -> int:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ---- entry points, same names as the C ABI --------------------------------

def lcsa_config_default() -> lcsa_config_t:
    c = lcsa_config_t()
    lib().lcsa_config_default(ctypes.byref(c))
    return c


def lcsa_config_resolve(cfg: lcsa_config_t) -> lcsa_geometry_t:
    g = lcsa_geometry_t()
    _check(lib().lcsa_config_resolve(ctypes.byref(cfg), ctypes.byref(g)), "lcsa_config_resolve")
    return g


def _expect_tensor(t, dtype, shape, name, device):
    """`t` must be a contiguous tensor of `dtype` and `shape` (None: any) on
    CUDA device `device` (an index) or, with device "cpu", in host memory.
    Integers pass through as raw addresses. The C ABI cannot see dtypes,
    strides or devices, so a mismatch is refused here before any call."""
    if isinstance(t, int):
        return
    on_it = (not t.is_cuda) if device == "cpu" else (t.is_cuda and t.device.index == device)
    if (t.dtype != dtype or not on_it or not t.is_contiguous() or
            (shape is not None and tuple(t.shape) != tuple(shape))):
        raise ValueError("%s: want a contiguous %s tensor%s on %s, got %s %s on %s%s" % (
            name, dtype, "" if shape is None else " of shape %s" % (tuple(shape),),
            "the host" if device == "cpu" else "cuda:%d" % device, t.dtype, tuple(t.shape), t.device,
            "" if t.is_contiguous() else " (not contiguous)"))


def lcsa_plan_create(cfg: lcsa_config_t, device: int = 0) -> "Plan":
    h = _PLAN()
    _check(lib().lcsa_plan_create(ctypes.byref(cfg), int(device), ctypes.byref(h)), "lcsa_plan_create")
    return Plan(h, cfg, int(device))


def lcsa_plan_create_stream(cfg: lcsa_config_t, device: int = 0) -> "Plan":
    """A stream plan: the last kv_frames frames of k^, pooled k and v stay in a
    ring; feed it with Plan.lcsa_stream_push and Plan.lcsa_forward_stream."""
    h = _PLAN()
    _check(lib().lcsa_plan_create_stream(ctypes.byref(cfg), int(device), ctypes.byref(h)), "lcsa_plan_create_stream")
    return Plan(h, cfg, int(device))


LCSA_NOALLOC_WORKSPACE_BYTES = 64 << 20


def lcsa_forward_noalloc(cfg: lcsa_config_t, q, k, v, gamma_q, gamma_k, out, stream=None) -> int:
    """Plan-free call for callers that may not allocate device memory: every
    intermediate lives in the library's static device workspace. Returns the
    status code (LCSA_ERR_UNSUPPORTED when the problem does not fit). Tensors
    must be contiguous, of the right dtype and on the current CUDA device;
    their sizes are the caller's contract, as in the C ABI."""
    if any(t is not None and not isinstance(t, int) for t in (q, k, v, gamma_q, gamma_k, out)):
        import torch
        dev = torch.cuda.current_device()
        for t, dt, name in ((q, torch.bfloat16, "q"), (k, torch.bfloat16, "k"), (v, torch.bfloat16, "v"),
                            (out, torch.bfloat16, "out"), (gamma_q, torch.float32, "gamma_q"),
                            (gamma_k, torch.float32, "gamma_k")):
            if t is not None:
                _expect_tensor(t, dt, None, name, dev)
    return int(lib().lcsa_forward_noalloc(ctypes.byref(cfg), _addr(q), _addr(k), _addr(v), _addr(gamma_q),
                                          _addr(gamma_k), _addr(out), _stream(stream)))


def lcsa_noalloc_check_device_error(stream=None) -> int:
    """Status of the device error word of lcsa_forward_noalloc's static
    workspace in the current context (synchronises the stream, reads and
    clears the word): LCSA_OK, LCSA_ERR_DEVICE_TIMEOUT or LCSA_ERR_DEVICE_BOUNDS."""
    return int(lib().lcsa_noalloc_check_device_error(_stream(stream)))


def config_from_workload(wl, **over) -> lcsa_config_t:
    """lcsa_config_t of a named workload (synth.WORKLOADS entry)."""
    c = lcsa_config_default()
    for name in ("batch", "heads", "head_dim", "q_frames", "kv_frames", "grid_h", "grid_w", "block_t", "block_h",
                 "block_w", "local_range", "topk", "sparse_ratio", "kv_frame_offset"):
        setattr(c, name, getattr(wl, name))
    for k, v in over.items():
        setattr(c, k, v)
    return c


class Plan:
    """Owner of an lcsa_plan_t; every method maps to one C entry point."""

    def __init__(self, handle, cfg, device: int = 0):
        self._h = handle
        self.cfg = cfg
        self.device = device  # the CUDA device the plan's memory and kernels live on
        g = lcsa_geometry_t()
        _check(lib().lcsa_plan_geometry(self._h, ctypes.byref(g)), "lcsa_plan_geometry")
        self.geometry = g

    @property
    def handle(self):
        return self._h

    def destroy(self):
        if self._h is not None and self._h.value:
            lib().lcsa_plan_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:  # noqa: BLE001 - interpreter shutdown
            pass

    def _expect(self, t, dtype, shape, name, host=False):
        _expect_tensor(t, dtype, shape, name, "cpu" if host else self.device)

    def lcsa_forward(self, q, k, v, gamma_q, gamma_k, out, stream=None):
        import torch
        c, g = self.cfg, self.geometry
        self._expect(q, torch.bfloat16, (c.batch, g.q_tokens, g.channels), "q")
        self._expect(k, torch.bfloat16, (c.batch, g.kv_tokens, g.channels), "k")
        self._expect(v, torch.bfloat16, (c.batch, g.kv_tokens, g.channels), "v")
        self._expect(out, torch.bfloat16, (c.batch, g.q_tokens, g.channels), "out")
        self._expect(gamma_q, torch.float32, (g.channels,), "gamma_q")
        self._expect(gamma_k, torch.float32, (g.channels,), "gamma_k")
        _check(lib().lcsa_forward(self._h, _addr(q), _addr(k), _addr(v), _addr(gamma_q), _addr(gamma_k),
                                  _addr(out), _stream(stream)), "lcsa_forward")
        return out

    forward = lcsa_forward

    def lcsa_stream_push(self, k, v, gamma_k, frames, stream=None):
        """Append `frames` frames of k and v ([batch, frames * H' * W', heads*d]) to the window."""
        import torch
        c, g = self.cfg, self.geometry
        toks = frames * c.grid_h * c.grid_w
        self._expect(k, torch.bfloat16, (c.batch, toks, g.channels), "k")
        self._expect(v, torch.bfloat16, (c.batch, toks, g.channels), "v")
        self._expect(gamma_k, torch.float32, (g.channels,), "gamma_k")
        _check(lib().lcsa_stream_push(self._h, _addr(k), _addr(v), _addr(gamma_k), int(frames), _stream(stream)),
               "lcsa_stream_push")

    def lcsa_forward_stream(self, q, k, v, gamma_q, gamma_k, out, stream=None):
        """One stream chunk: q, k, v of the q_frames new frames ([batch, q_tokens, heads*d])."""
        import torch
        c, g = self.cfg, self.geometry
        for t, name in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
            self._expect(t, torch.bfloat16, (c.batch, g.q_tokens, g.channels), name)
        self._expect(gamma_q, torch.float32, (g.channels,), "gamma_q")
        self._expect(gamma_k, torch.float32, (g.channels,), "gamma_k")
        _check(lib().lcsa_forward_stream(self._h, _addr(q), _addr(k), _addr(v), _addr(gamma_q), _addr(gamma_k),
                                         _addr(out), _stream(stream)), "lcsa_forward_stream")
        return out

    def lcsa_sumsq(self, q, k, ssq, stream=None):
        """Per-token sums of squares of this plan's q then k channels into ssq
        (fp32 [batch*(q_tokens + kv_tokens)]), for a head-sharded layer."""
        import torch
        c, g = self.cfg, self.geometry
        self._expect(q, torch.bfloat16, (c.batch, g.q_tokens, g.channels), "q")
        self._expect(k, torch.bfloat16, (c.batch, g.kv_tokens, g.channels), "k")
        self._expect(ssq, torch.float32, (c.batch * (g.q_tokens + g.kv_tokens),), "ssq")
        _check(lib().lcsa_sumsq(self._h, _addr(q), _addr(k), _addr(ssq), _stream(stream)), "lcsa_sumsq")
        return ssq

    def lcsa_forward_sharded(self, q, k, v, gamma_q, gamma_k, ssq, out, stream=None):
        """lcsa_forward of a head-sharded plan, the RMS norm taken from ssq
        (the sums of lcsa_sumsq over all ranks)."""
        import torch
        c, g = self.cfg, self.geometry
        self._expect(q, torch.bfloat16, (c.batch, g.q_tokens, g.channels), "q")
        self._expect(k, torch.bfloat16, (c.batch, g.kv_tokens, g.channels), "k")
        self._expect(v, torch.bfloat16, (c.batch, g.kv_tokens, g.channels), "v")
        self._expect(out, torch.bfloat16, (c.batch, g.q_tokens, g.channels), "out")
        self._expect(gamma_q, torch.float32, (g.channels,), "gamma_q")
        self._expect(gamma_k, torch.float32, (g.channels,), "gamma_k")
        self._expect(ssq, torch.float32, (c.batch * (g.q_tokens + g.kv_tokens),), "ssq")
        _check(lib().lcsa_forward_sharded(self._h, _addr(q), _addr(k), _addr(v), _addr(gamma_q), _addr(gamma_k),
                                          _addr(ssq), _addr(out), _stream(stream)), "lcsa_forward_sharded")
        return out

    def lcsa_forward_host(self, q, k, v, gamma_q, gamma_k, out, stream=None):
        """Host (preferably pinned) tensors in and out; copies are inside the call."""
        import torch
        c, g = self.cfg, self.geometry
        self._expect(q, torch.bfloat16, (c.batch, g.q_tokens, g.channels), "q", host=True)
        self._expect(k, torch.bfloat16, (c.batch, g.kv_tokens, g.channels), "k", host=True)
        self._expect(v, torch.bfloat16, (c.batch, g.kv_tokens, g.channels), "v", host=True)
        self._expect(out, torch.bfloat16, (c.batch, g.q_tokens, g.channels), "out", host=True)
        self._expect(gamma_q, torch.float32, (g.channels,), "gamma_q", host=True)
        self._expect(gamma_k, torch.float32, (g.channels,), "gamma_k", host=True)
        _check(lib().lcsa_forward_host(self._h, _addr(q), _addr(k), _addr(v), _addr(gamma_q), _addr(gamma_k),
                                       _addr(out), _stream(stream)), "lcsa_forward_host")
        return out

    def lcsa_plan_topk(self) -> int:
        k = ctypes.c_int()
        _check(lib().lcsa_plan_topk(self._h, ctypes.byref(k)), "lcsa_plan_topk")
        return k.value

    def lcsa_plan_set_threshold_reuse(self, on: bool):
        """Later calls keep blocks by the recorded per-row thresholds instead of selecting the top k."""
        _check(lib().lcsa_plan_set_threshold_reuse(self._h, 1 if on else 0), "lcsa_plan_set_threshold_reuse")

    def lcsa_selection_nnz(self) -> int:
        n = ctypes.c_int64()
        _check(lib().lcsa_selection_nnz(self._h, ctypes.byref(n)), "lcsa_selection_nnz")
        return n.value

    def lcsa_get_selection(self):
        import numpy as np
        g = self.geometry
        nnz = self.lcsa_selection_nnz()
        rp = np.empty(g.rows + 1, dtype=np.int32)
        ci = np.empty(max(1, nnz), dtype=np.int32)
        _check(lib().lcsa_get_selection(self._h, rp.ctypes.data, rp.size, ci.ctypes.data, ci.size),
               "lcsa_get_selection")
        return rp, ci[:nnz]

    def lcsa_get_intermediates(self):
        """(q^, k^ as uint16 bf16 bits, pooled q, pooled k) in the plan's layouts."""
        import numpy as np
        c, g = self.cfg, self.geometry
        qh = np.empty((c.batch, c.heads, g.q_blocks, g.block_tokens, c.head_dim), dtype=np.uint16)
        kh = np.empty((c.batch, c.heads, g.kv_blocks, g.block_tokens, c.head_dim), dtype=np.uint16)
        pq = np.empty((c.batch, c.heads, g.q_blocks, c.head_dim), dtype=np.float32)
        pk = np.empty((c.batch, c.heads, g.kv_blocks, c.head_dim), dtype=np.float32)
        _check(lib().lcsa_get_intermediates(self._h, qh.ctypes.data, kh.ctypes.data, pq.ctypes.data,
                                            pk.ctypes.data), "lcsa_get_intermediates")
        return qh, kh, pq, pk

    def lcsa_check_device_error(self, stream=None):
        _check(lib().lcsa_check_device_error(self._h, _stream(stream)), "lcsa_check_device_error")

    def lcsa_plan_set_timing(self, capacity: int):
        _check(lib().lcsa_plan_set_timing(self._h, int(capacity)), "lcsa_plan_set_timing")

    def lcsa_get_kernel_times(self):
        """(mean ms of prologue, select, attention; number of calls averaged)."""
        ms = (ctypes.c_float * 3)()
        n = ctypes.c_int()
        _check(lib().lcsa_get_kernel_times(self._h, ms, ctypes.byref(n)), "lcsa_get_kernel_times")
        return list(ms), n.value


def lcsa_selftest_exp2(x, y, stream=None):
    """y = 2^x through the attention kernel's FMA-pipe exponential (fp32 CUDA tensors)."""
    _check(lib().lcsa_selftest_exp2(_addr(x), _addr(y), int(x.numel()), _stream(stream)), "lcsa_selftest_exp2")
    return y


def lcsa_status_string(status: int) -> str:
    return lib().lcsa_status_string(int(status)).decode()


def lcsa_last_error_message() -> str:
    return lib().lcsa_last_error_message().decode()


def lcsa_abi_version() -> int:
    return int(lib().lcsa_abi_version())
