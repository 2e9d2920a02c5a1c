"""Python binding of the SRNL four-direction scan C ABI (``include/srnl_scan.h``).

Argument marshalling only: every step of the forward and the backward runs in the CUDA
kernels of ``libsrnl_scan.so``.  There is no CPU fallback; importing works without a GPU,
but creating a handle needs the built library and a CUDA device.

    from self_referential_nested_b200 import srnl_scan_create, srnl_scan_forward
    h = srnl_scan_create(cfg_dict, params_dict)      # params: float32 numpy arrays
    srnl_scan_forward(h, x, y)                      # x, y: CUDA tensors [B,H,W,C]
    srnl_scan_backward(h, x, dy, dx, grads)         # fp32-generation handles; grads: GRAD_KEYS
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsrnl_scan.so")

SRNL_OK, SRNL_E_INVAL, SRNL_E_UNSUPPORTED, SRNL_E_CUDA, SRNL_E_NOMEM, SRNL_E_TIMEOUT = 0, -1, -2, -3, -4, -5
SRNL_F32, SRNL_BF16 = 0, 1
SRNL_CAP_SOFT, SRNL_CAP_HARD = 0, 1
STATE_FLOATS_D32 = 3 * 32 * 32 + 2 * 32

NOALLOC_SCRATCH_BYTES = 32 << 20

EXPORTED = ("srnl_scan_create", "srnl_scan_forward", "srnl_scan_forward_host",
            "srnl_scan_forward_noalloc",
            "srnl_scan_route_index", "srnl_scan_gather", "srnl_scan_enable_stage_timing",
            "srnl_scan_stage_times", "srnl_scan_device_status", "srnl_scan_workspace_bytes",
            "srnl_scan_last_error", "srnl_status_string", "srnl_scan_destroy",
            "srnl_seq_create", "srnl_seq_forward", "srnl_seq_device_status", "srnl_seq_last_error",
            "srnl_seq_destroy", "srnl_scan_cap_count", "srnl_seq_cap_count",
            "srnl_scan_forward_host_async", "srnl_scan_host_join", "srnl_scan_host_sync",
            "srnl_scan_backward", "srnl_seq_backward", "srnl_selftest_wait_timeout",
            "srnl_scan_noalloc_status", "srnl_selftest_noalloc_wait_timeout",
            "srnl_block_create", "srnl_block_forward", "srnl_block_device_status", "srnl_block_last_error",
            "srnl_block_destroy")


class SrnlError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        self.status = status
        super().__init__(f"{where}: {message} [status {status}]")


BLOCK_KEYS = ("ln1_g", "ln1_b", "W_in", "b_in", "dw_w", "dw_b", "W_out", "b_out", "ln2_g", "ln2_b",
              "W_1", "b_1", "W_2", "b_2")
OP_KEYS = ("W_q", "scales", "M_mem0", "M_k0", "M_v0", "m_eta0", "m_alpha0")


class _BlockConfig(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int), ("dim", ctypes.c_int),
                ("mixer_dim", ctypes.c_int), ("head_dim", ctypes.c_int), ("alpha", ctypes.c_float),
                ("eps", ctypes.c_float), ("chunk_row", ctypes.c_int), ("chunk_col", ctypes.c_int),
                ("act_dtype", ctypes.c_int), ("gen_dtype", ctypes.c_int), ("injection_cap", ctypes.c_int),
                ("ln_eps", ctypes.c_float)]


class _Config(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int), ("C", ctypes.c_int),
                ("heads", ctypes.c_int), ("d", ctypes.c_int), ("alpha", ctypes.c_float),
                ("eps", ctypes.c_float), ("chunk_row", ctypes.c_int), ("chunk_col", ctypes.c_int),
                ("act_dtype", ctypes.c_int), ("gen_dtype", ctypes.c_int), ("injection_cap", ctypes.c_int)]


class _Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("W_q", "scales", "M_mem0", "M_k0", "M_v0",
                                                "m_eta0", "m_alpha0")]


class _BlockParams(ctypes.Structure):
    _fields_ = ([(n, ctypes.c_void_p) for n in ("ln1_g", "ln1_b", "W_in", "b_in", "dw_w", "dw_b")]
                + [("op", _Params)]
                + [(n, ctypes.c_void_p) for n in ("W_out", "b_out", "ln2_g", "ln2_b", "W_1", "b_1", "W_2", "b_2")])


class _Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("W_q", "scales", "M_mem0", "M_k0", "M_v0",
                                                "m_eta0", "m_alpha0")]


GRAD_KEYS = ("W_q", "scales", "M_mem0", "M_k0", "M_v0", "m_eta0", "m_alpha0")
SEQ_GRAD_KEYS = ("M_mem0", "M_k0", "M_v0", "m_eta0", "m_alpha0")


class _SeqGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in SEQ_GRAD_KEYS]


class _SeqConfig(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("D", ctypes.c_int), ("heads", ctypes.c_int),
                ("d", ctypes.c_int), ("alpha", ctypes.c_float), ("eps", ctypes.c_float),
                ("chunk", ctypes.c_int), ("act_dtype", ctypes.c_int), ("gen_dtype", ctypes.c_int),
                ("injection_cap", ctypes.c_int)]


class _SeqParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("M_mem0", "M_k0", "M_v0", "m_eta0", "m_alpha0")]


_lib: Optional[ctypes.CDLL] = None


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load ``libsrnl_scan.so``; raises if it has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m self_referential_nested_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.srnl_scan_create.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(_Config), ctypes.POINTER(_Params)]
    lib.srnl_scan_forward.argtypes = [vp, vp, vp, vp, vp]
    lib.srnl_scan_forward_host.argtypes = [vp, vp, vp, vp]
    lib.srnl_scan_forward_noalloc.argtypes = [ctypes.POINTER(_Config), ctypes.POINTER(_Params), vp, vp, vp]
    lib.srnl_scan_route_index.argtypes = [vp, i, vp, vp]
    lib.srnl_scan_gather.argtypes = [vp, i, vp, vp, vp]
    lib.srnl_scan_enable_stage_timing.argtypes = [vp, i]
    lib.srnl_scan_stage_times.argtypes = [vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int)]
    lib.srnl_scan_device_status.argtypes = [vp]
    lib.srnl_scan_workspace_bytes.argtypes = [vp]
    lib.srnl_scan_workspace_bytes.restype = ctypes.c_size_t
    lib.srnl_scan_last_error.argtypes = [vp]
    lib.srnl_scan_last_error.restype = ctypes.c_char_p
    lib.srnl_status_string.argtypes = [i]
    lib.srnl_status_string.restype = ctypes.c_char_p
    lib.srnl_scan_destroy.argtypes = [vp]
    lib.srnl_scan_destroy.restype = None
    lib.srnl_seq_create.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(_SeqConfig), ctypes.POINTER(_SeqParams)]
    lib.srnl_seq_forward.argtypes = [vp, vp, vp, vp, vp, vp]
    lib.srnl_seq_device_status.argtypes = [vp]
    lib.srnl_seq_last_error.argtypes = [vp]
    lib.srnl_seq_last_error.restype = ctypes.c_char_p
    lib.srnl_seq_destroy.argtypes = [vp]
    lib.srnl_seq_destroy.restype = None
    lib.srnl_scan_cap_count.argtypes = [vp, ctypes.POINTER(ctypes.c_ulonglong)]
    lib.srnl_scan_forward_host_async.argtypes = [vp, vp, vp, vp]
    lib.srnl_scan_host_join.argtypes = [vp, vp]
    lib.srnl_scan_host_sync.argtypes = [vp]
    lib.srnl_seq_cap_count.argtypes = [vp, ctypes.POINTER(ctypes.c_ulonglong)]
    lib.srnl_scan_backward.argtypes = [vp, vp, vp, vp, ctypes.POINTER(_Grads), vp]
    lib.srnl_seq_backward.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.POINTER(_SeqGrads), vp]
    lib.srnl_selftest_wait_timeout.argtypes = [i]
    lib.srnl_scan_noalloc_status.argtypes = [vp]
    lib.srnl_block_create.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(_BlockConfig), ctypes.POINTER(_BlockParams)]
    lib.srnl_block_forward.argtypes = [vp, vp, vp, vp]
    lib.srnl_block_device_status.argtypes = [vp]
    lib.srnl_block_last_error.argtypes = [vp]
    lib.srnl_block_last_error.restype = ctypes.c_char_p
    lib.srnl_block_destroy.argtypes = [vp]
    lib.srnl_block_destroy.restype = None
    lib.srnl_selftest_noalloc_wait_timeout.argtypes = [i, vp]
    for name in ("srnl_scan_create", "srnl_scan_forward", "srnl_scan_forward_host", "srnl_scan_forward_noalloc",
                 "srnl_scan_route_index", "srnl_scan_gather", "srnl_scan_enable_stage_timing",
                 "srnl_scan_stage_times", "srnl_scan_device_status", "srnl_seq_create", "srnl_seq_forward",
                 "srnl_seq_device_status", "srnl_scan_cap_count", "srnl_seq_cap_count",
                 "srnl_scan_forward_host_async", "srnl_scan_host_join", "srnl_scan_host_sync",
                 "srnl_scan_backward", "srnl_seq_backward", "srnl_selftest_wait_timeout",
                 "srnl_scan_noalloc_status", "srnl_selftest_noalloc_wait_timeout", "srnl_block_create",
                 "srnl_block_forward", "srnl_block_device_status"):
        getattr(lib, name).restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def _ptr(t) -> int:
    """Raw address of a torch tensor, a numpy array or an int (0 for None)."""
    if t is None:
        return 0
    if isinstance(t, int):
        return t
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class SrnlScan:
    """Owns one ``srnl_scan*`` handle; ``close()`` (or GC) destroys it."""

    def __init__(self, handle: int, cfg: Dict):
        self._h = handle
        self.cfg = dict(cfg)

    @property
    def handle(self) -> int:
        if not self._h:
            raise RuntimeError("srnl_scan handle is closed")
        return self._h

    def _check(self, status: int, where: str):
        if status != SRNL_OK:
            msg = load_library().srnl_scan_last_error(self._h).decode()
            raise SrnlError(status, where, msg)

    def close(self):
        if self._h:
            load_library().srnl_scan_destroy(self._h)
            self._h = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace_bytes(self) -> int:
        return int(load_library().srnl_scan_workspace_bytes(self.handle))


def _cap(v) -> int:
    return {"soft": SRNL_CAP_SOFT, "hard": SRNL_CAP_HARD}.get(v, v)


def _config_struct(cfg: Dict) -> _Config:
    def dt(v):
        return {"f32": SRNL_F32, "bf16": SRNL_BF16}.get(v, v)

    return _Config(B=cfg["B"], H=cfg["H"], W=cfg["W"], C=cfg["C"], heads=cfg["heads"], d=cfg["d"],
                   alpha=cfg["alpha"], eps=cfg.get("eps", 1e-6), chunk_row=cfg.get("chunk_row", 0),
                   chunk_col=cfg.get("chunk_col", 0), act_dtype=dt(cfg["act_dtype"]),
                   gen_dtype=dt(cfg.get("gen_dtype", cfg["act_dtype"])),
                   injection_cap=_cap(cfg.get("injection_cap", "soft")))


def srnl_scan_create(cfg: Dict, params: Dict[str, np.ndarray]) -> SrnlScan:
    """cfg keys: B, H, W, C, heads, d, alpha, eps, chunk_row, chunk_col,
    act_dtype, gen_dtype ("f32"/"bf16" or SRNL_F32/SRNL_BF16).  params: float32
    host arrays W_q, scales, M_mem0, M_k0, M_v0, m_eta0, m_alpha0."""
    lib = load_library()
    c = _config_struct(cfg)
    keep = {k: np.ascontiguousarray(params[k], dtype=np.float32)
            for k in ("W_q", "scales", "M_mem0", "M_k0", "M_v0", "m_eta0", "m_alpha0")}
    p = _Params(**{k: v.ctypes.data for k, v in keep.items()})
    h = ctypes.c_void_p()
    st = lib.srnl_scan_create(ctypes.byref(h), ctypes.byref(c), ctypes.byref(p))
    if st != SRNL_OK:
        raise SrnlError(st, "srnl_scan_create", lib.srnl_scan_last_error(None).decode())
    return SrnlScan(h.value, cfg)


def srnl_scan_forward(h: SrnlScan, x, y, final_states=None, stream=None) -> None:
    st = load_library().srnl_scan_forward(h.handle, _ptr(x), _ptr(y), _ptr(final_states), _stream(stream))
    h._check(st, "srnl_scan_forward")


def srnl_scan_backward(h: SrnlScan, x, dy, dx, grads: Optional[Dict] = None, stream=None) -> None:
    """Backward pass: dx <- dL/dx for upstream dy = dL/dy (CUDA tensors [B,H,W,C] of the handle's
    act dtype); ``grads`` maps any of GRAD_KEYS to fp32 CUDA tensors in the parameter layouts,
    which are overwritten with the parameter gradients (missing keys are skipped)."""
    g = grads or {}
    gs = _Grads(**{k: _ptr(g.get(k)) for k in GRAD_KEYS})
    st = load_library().srnl_scan_backward(h.handle, _ptr(x), _ptr(dy), _ptr(dx),
                                           ctypes.byref(gs) if grads is not None else None, _stream(stream))
    h._check(st, "srnl_scan_backward")


def srnl_scan_forward_host(h: SrnlScan, x_host, y_host, stream=None) -> None:
    st = load_library().srnl_scan_forward_host(h.handle, _ptr(x_host), _ptr(y_host), _stream(stream))
    h._check(st, "srnl_scan_forward_host")


def srnl_scan_forward_host_async(h: SrnlScan, x_host, y_host, stream=None) -> None:
    """Pipelined host-buffer forward (pinned tensors); y_host is ready after srnl_scan_host_sync."""
    st = load_library().srnl_scan_forward_host_async(h.handle, _ptr(x_host), _ptr(y_host), _stream(stream))
    h._check(st, "srnl_scan_forward_host_async")


def srnl_scan_host_join(h: SrnlScan, stream=None) -> None:
    h._check(load_library().srnl_scan_host_join(h.handle, _stream(stream)), "srnl_scan_host_join")


def srnl_scan_host_sync(h: SrnlScan) -> None:
    h._check(load_library().srnl_scan_host_sync(h.handle), "srnl_scan_host_sync")


def srnl_scan_forward_noalloc(cfg: Dict, params_dev: Dict, x, y, stream=None) -> None:
    """Allocation-free forward: no handle, no device allocation.

    For callers that must not call cudaMalloc (a host framework that owns all
    device memory through its own pool; latency-critical loops).  params_dev:
    the seven parameter arrays as DEVICE buffers (torch CUDA tensors or raw
    addresses) in the srnl_scan_params layouts.  Scratch is a fixed
    NOALLOC_SCRATCH_BYTES device array inside the library, shared by all calls.
    """
    lib = load_library()
    c = _config_struct(cfg)
    p = _Params(**{k: _ptr(params_dev[k]) for k in ("W_q", "scales", "M_mem0", "M_k0", "M_v0",
                                                     "m_eta0", "m_alpha0")})
    st = lib.srnl_scan_forward_noalloc(ctypes.byref(c), ctypes.byref(p), _ptr(x), _ptr(y), _stream(stream))
    if st != SRNL_OK:
        raise SrnlError(st, "srnl_scan_forward_noalloc", lib.srnl_scan_last_error(None).decode())


def srnl_scan_noalloc_status(stream=None) -> None:
    """Raise SrnlError if a bounded in-kernel wait of the last allocation-free forward on the
    current device gave up (waits for ``stream`` first)."""
    lib = load_library()
    st = lib.srnl_scan_noalloc_status(_stream(stream))
    if st != SRNL_OK:
        raise SrnlError(st, "srnl_scan_noalloc_status", lib.srnl_scan_last_error(None).decode())


def srnl_selftest_noalloc_wait_timeout(wait_ms: int = 50, stream=None) -> None:
    """Run a bounded wait that must give up, recording its status where the allocation-free
    forward records its own (asynchronous)."""
    lib = load_library()
    st = lib.srnl_selftest_noalloc_wait_timeout(int(wait_ms), _stream(stream))
    if st != SRNL_OK:
        raise SrnlError(st, "srnl_selftest_noalloc_wait_timeout", lib.srnl_scan_last_error(None).decode())


def srnl_scan_route_index(h: SrnlScan, route: int, out, stream=None) -> None:
    st = load_library().srnl_scan_route_index(h.handle, route, _ptr(out), _stream(stream))
    h._check(st, "srnl_scan_route_index")


def srnl_scan_gather(h: SrnlScan, route: int, x, xr, stream=None) -> None:
    st = load_library().srnl_scan_gather(h.handle, route, _ptr(x), _ptr(xr), _stream(stream))
    h._check(st, "srnl_scan_gather")


def srnl_scan_enable_stage_timing(h: SrnlScan, ring: int = 256) -> None:
    """Keep per-kernel events of the last ``ring`` forwards (0 turns timing off)."""
    h._check(load_library().srnl_scan_enable_stage_timing(h.handle, int(ring)),
             "srnl_scan_enable_stage_timing")


def srnl_scan_stage_times(h: SrnlScan):
    """Mean (query projection, scan, fusion) kernel ms over the window, and its size."""
    out = (ctypes.c_float * 3)()
    n = ctypes.c_int(0)
    h._check(load_library().srnl_scan_stage_times(h.handle, out, ctypes.byref(n)), "srnl_scan_stage_times")
    return tuple(float(v) for v in out), int(n.value)


def srnl_scan_device_status(h: SrnlScan) -> None:
    """Raise SrnlError if a bounded in-kernel wait of this handle ever gave up."""
    h._check(load_library().srnl_scan_device_status(h.handle), "srnl_scan_device_status")


def srnl_scan_cap_count(h: SrnlScan) -> int:
    """Token updates of the last forward on which the hard clamp was active (synchronises)."""
    v = ctypes.c_ulonglong(0)
    h._check(load_library().srnl_scan_cap_count(h.handle, ctypes.byref(v)), "srnl_scan_cap_count")
    return int(v.value)


def srnl_scan_destroy(h: SrnlScan) -> None:
    h.close()


def srnl_status_string(status: int) -> str:
    return load_library().srnl_status_string(status).decode()


def srnl_scan_last_error(h: Optional[SrnlScan] = None) -> str:
    return load_library().srnl_scan_last_error(h._h if h is not None else None).decode()


# ------------------------------------------------ standalone sequence layer
class SrnlSeq:
    """Owns one ``srnl_seq*`` handle (the standalone SRNL layer on [B, T, D])."""

    def __init__(self, handle: int, cfg: Dict):
        self._h = handle
        self.cfg = dict(cfg)

    @property
    def handle(self) -> int:
        if not self._h:
            raise RuntimeError("srnl_seq handle is closed")
        return self._h

    def _check(self, status: int, where: str):
        if status != SRNL_OK:
            raise SrnlError(status, where, load_library().srnl_seq_last_error(self._h).decode())

    def close(self):
        if self._h:
            load_library().srnl_seq_destroy(self._h)
            self._h = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def srnl_seq_create(cfg: Dict, params: Dict[str, np.ndarray]) -> SrnlSeq:
    """cfg keys: B, T, D, heads, d, alpha, eps, chunk (0 = 64), act_dtype, gen_dtype.
    params: float32 host arrays M_mem0, M_k0, M_v0 [heads, d, d], m_eta0, m_alpha0 [heads, d]."""
    lib = load_library()

    def dt(v):
        return {"f32": SRNL_F32, "bf16": SRNL_BF16}.get(v, v)

    c = _SeqConfig(B=cfg["B"], T=cfg["T"], D=cfg["D"], heads=cfg["heads"], d=cfg["d"], alpha=cfg["alpha"],
                   eps=cfg.get("eps", 1e-6), chunk=cfg.get("chunk", 0), act_dtype=dt(cfg["act_dtype"]),
                   gen_dtype=dt(cfg.get("gen_dtype", cfg["act_dtype"])),
                   injection_cap=_cap(cfg.get("injection_cap", "soft")))
    keep = {k: np.ascontiguousarray(params[k], dtype=np.float32)
            for k in ("M_mem0", "M_k0", "M_v0", "m_eta0", "m_alpha0")}
    p = _SeqParams(**{k: v.ctypes.data for k, v in keep.items()})
    h = ctypes.c_void_p()
    st = lib.srnl_seq_create(ctypes.byref(h), ctypes.byref(c), ctypes.byref(p))
    if st != SRNL_OK:
        raise SrnlError(st, "srnl_seq_create", lib.srnl_seq_last_error(None).decode())
    return SrnlSeq(h.value, cfg)


def srnl_seq_forward(h: SrnlSeq, x, y, q=None, final_states=None, stream=None) -> None:
    """x, q, y: CUDA tensors [B, T, D] of act_dtype; q None means x is the query."""
    h._check(load_library().srnl_seq_forward(h.handle, _ptr(x), _ptr(q), _ptr(y), _ptr(final_states),
                                             _stream(stream)), "srnl_seq_forward")


def srnl_seq_backward(h: SrnlSeq, x, dy, dx, q=None, dq=None, grads: Optional[Dict] = None, stream=None) -> None:
    """Backward of the sequence layer: dx <- dL/dx (including the query path when q is None),
    dq <- dL/dq when q and dq are given; ``grads`` maps any of SEQ_GRAD_KEYS to fp32 CUDA
    tensors [heads, d, d] / [heads, d], overwritten with the initial-state gradients."""
    g = grads or {}
    gs = _SeqGrads(**{k: _ptr(g.get(k)) for k in SEQ_GRAD_KEYS})
    h._check(load_library().srnl_seq_backward(h.handle, _ptr(x), _ptr(q), _ptr(dy), _ptr(dx), _ptr(dq),
                                              ctypes.byref(gs) if grads is not None else None, _stream(stream)),
             "srnl_seq_backward")


def srnl_selftest_wait_timeout(wait_ms: int = 50) -> int:
    """Run the bounded-wait self-test on the current device; returns the status code
    (SRNL_E_TIMEOUT is the expected, passing result)."""
    return int(load_library().srnl_selftest_wait_timeout(int(wait_ms)))


def srnl_seq_device_status(h: SrnlSeq) -> None:
    h._check(load_library().srnl_seq_device_status(h.handle), "srnl_seq_device_status")


def srnl_seq_cap_count(h: SrnlSeq) -> int:
    """Token updates of the last forward on which the hard clamp was active (synchronises)."""
    v = ctypes.c_ulonglong(0)
    h._check(load_library().srnl_seq_cap_count(h.handle, ctypes.byref(v)), "srnl_seq_cap_count")
    return int(v.value)


def srnl_seq_destroy(h: SrnlSeq) -> None:
    h.close()


# ------------------------------------------------ residual block around the operator
class SrnlBlock:
    """Owns one ``srnl_block*`` handle (the VisionHOPE residual block, bf16 [B, H, W, dim])."""

    def __init__(self, handle: int, cfg: Dict):
        self._h = handle
        self.cfg = dict(cfg)

    @property
    def handle(self) -> int:
        if not self._h:
            raise RuntimeError("srnl_block handle is closed")
        return self._h

    def _check(self, status: int, where: str):
        if status != SRNL_OK:
            raise SrnlError(status, where, load_library().srnl_block_last_error(self._h).decode())

    def close(self):
        if self._h:
            load_library().srnl_block_destroy(self._h)
            self._h = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def srnl_block_create(cfg: Dict, params: Dict[str, np.ndarray]) -> SrnlBlock:
    """cfg keys: B, H, W, dim, mixer_dim, head_dim, alpha, eps, chunk_row, chunk_col, gen_dtype,
    injection_cap, ln_eps (act_dtype is bf16).  params: float32 host arrays BLOCK_KEYS and the
    operator's OP_KEYS at width mixer_dim."""
    lib = load_library()

    def dt(v):
        return {"f32": SRNL_F32, "bf16": SRNL_BF16}.get(v, v)

    c = _BlockConfig(B=cfg["B"], H=cfg["H"], W=cfg["W"], dim=cfg["dim"], mixer_dim=cfg["mixer_dim"],
                     head_dim=cfg["head_dim"], alpha=cfg["alpha"], eps=cfg.get("eps", 1e-6),
                     chunk_row=cfg.get("chunk_row", 0), chunk_col=cfg.get("chunk_col", 0),
                     act_dtype=dt(cfg.get("act_dtype", "bf16")), gen_dtype=dt(cfg.get("gen_dtype", "bf16")),
                     injection_cap=_cap(cfg.get("injection_cap", "soft")), ln_eps=cfg.get("ln_eps", 1e-6))
    keep = {k: np.ascontiguousarray(params[k], dtype=np.float32) for k in BLOCK_KEYS + OP_KEYS}
    op = _Params(**{k: keep[k].ctypes.data for k in OP_KEYS})
    p = _BlockParams(op=op, **{k: keep[k].ctypes.data for k in BLOCK_KEYS})
    h = ctypes.c_void_p()
    st = lib.srnl_block_create(ctypes.byref(h), ctypes.byref(c), ctypes.byref(p))
    if st != SRNL_OK:
        raise SrnlError(st, "srnl_block_create", lib.srnl_block_last_error(None).decode())
    return SrnlBlock(h.value, cfg)


def srnl_block_forward(h: SrnlBlock, x, y, stream=None) -> None:
    """y <- block(x): bf16 CUDA tensors [B, H, W, dim], 16-byte aligned, not overlapping."""
    h._check(load_library().srnl_block_forward(h.handle, _ptr(x), _ptr(y), _stream(stream)), "srnl_block_forward")


def srnl_block_device_status(h: SrnlBlock) -> None:
    """Raise SrnlError if a bounded in-kernel wait of the block or its operator gave up."""
    h._check(load_library().srnl_block_device_status(h.handle), "srnl_block_device_status")


def srnl_block_destroy(h: SrnlBlock) -> None:
    h.close()
