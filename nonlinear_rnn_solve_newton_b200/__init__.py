"""Python binding of libpararnn.so: Newton solves of nonlinear RNNs on a B200.

Argument marshalling only.  Every step of the computation runs in the CUDA
kernels of ``libpararnn.so`` (C ABI in ``include/pararnn.h``); torch provides
device memory (outputs, workspace, the info struct) and the current stream.
There is no CPU fallback: if the library is missing or the tensors are not on a
CUDA device, the calls raise.

Entry points (same names as the C ABI, without the ``pararnn_`` prefix):

* ``scan_diag(A, b, h0=None)``      h_t = A_t h_{t-1} + b_t           [B, L, D]
* ``scan_block2(A, b, x0=None)``    x_t = A_t x_{t-1} + b_t, 2x2 blocks  [B, L, D, 2]
* ``solve_gru(P, a, h0=None, tol=1e-4, max_iters=32)``   ParaGRU Newton solve
* ``solve_lstm(P, a, c0=None, h0=None, tol=1e-4, max_iters=32)``  ParaLSTM Newton solve
* ``solve_gru_backward`` / ``solve_lstm_backward``  gradients through the solution
* ``solve_mhgru(P, U, h0=None)``     multi-head GRU, dense 8x8 recurrence blocks
* ``solve_mhgru_strided(P, U, strides, h0=None)``  the same with a time stride per head
* ``input_projection(x, W, bias=None)``  P = x W^T + bias on the tensor cores
* ``solve_gru_projected(x, W, bias, a, h0=None)``  the projection fused with the
  ParaGRU Newton solve (P never reaches HBM)
* ``step_gru`` / ``step_lstm``      one decode step;  ``rollout_gru`` / ``rollout_lstm``
  the sequential application on the GPU

The workspace the solves and scans need comes from torch's allocator and is
reused between calls on the same thread, device and stream.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

__all__ = ["scan_diag", "scan_block2", "solve_gru", "solve_lstm", "solve_gru_noalloc", "solve_gru_projected", "solve_mhgru_strided",
           "solve_gru_backward", "solve_lstm_backward", "solve_mhgru", "input_projection",
           "step_gru", "step_lstm", "rollout_gru", "rollout_lstm",
           "workspace_size", "probe_rate", "PROBE_MUFU", "PROBE_FMA",
           "SolveInfo", "Options", "PararnnError", "library_path", "load", "MAX_ITERS"]

MAX_ITERS = 127
_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libpararnn.so")

OP_SCAN_DIAG, OP_SCAN_BLOCK2, OP_GRU, OP_LSTM = 0, 1, 2, 3
OP_GRU_BACKWARD, OP_LSTM_BACKWARD = 4, 5
OP_MHGRU = 6
OP_GRU_PROJECTED = 7
OP_MHGRU_STRIDED = 8
F32, BF16 = 0, 1

_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported device", 3: "CUDA runtime error",
           4: "device-side wait timed out", 5: "non-finite residual",
           6: "workspace missing, too small or misaligned"}


class PararnnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {_STATUS.get(self.status, 'unknown status')} ({self.status})")


class _Info(ctypes.Structure):
    _fields_ = [("iterations", ctypes.c_int32), ("converged", ctypes.c_int32),
                ("status", ctypes.c_int32), ("updates", ctypes.c_int32),
                ("passes", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("max_residual", ctypes.c_float), ("rho", ctypes.c_float * (MAX_ITERS + 1))]


class Options(ctypes.Structure):
    """Tuning and test hooks (see pararnn_options_t)."""
    _fields_ = [("iters_first", ctypes.c_int32), ("iters_next", ctypes.c_int32),
                ("wait_timeout_ns", ctypes.c_int64), ("debug_stall_unit", ctypes.c_int64),
                ("regime", ctypes.c_int32), ("walk_warps", ctypes.c_int32),
                ("walk_width", ctypes.c_int32), ("reserved", ctypes.c_int32)]

    AUTO, LOOKBACK, WALK = 0, 1, 2

    def __init__(self, iters_first=0, iters_next=0, wait_timeout_ns=0, debug_stall_unit=-1,
                 regime=0, walk_warps=0, walk_width=0):
        super().__init__(iters_first, iters_next, wait_timeout_ns, debug_stall_unit, regime,
                         walk_warps, walk_width, 0)


INFO_BYTES = ctypes.sizeof(_Info)

_lock = threading.Lock()
_lib = None
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64


def load(build_if_missing: bool = True):
    """Load libpararnn.so (building it in-tree with nvcc if it is missing or stale)."""
    global _lib
    lib = _lib
    if lib is not None:  # loaded: no lock on the per-call path
        return lib
    with _lock:
        if _lib is None:
            if build_if_missing and _build.needs_build():
                _build.build()
            if not os.path.exists(library_path):
                raise RuntimeError(f"libpararnn.so not found at {library_path}")
            lib = ctypes.CDLL(library_path)
            lib.pararnn_workspace_size.argtypes = [ctypes.c_int, _i64, _i64, _i64, ctypes.c_int32,
                                                   _vp]
            lib.pararnn_workspace_size.restype = ctypes.c_size_t
            for name in ("pararnn_scan_diag", "pararnn_scan_block2"):
                f = getattr(lib, name)
                f.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, ctypes.c_size_t, _vp, _vp,
                              _vp]
                f.restype = ctypes.c_int
            lib.pararnn_solve_gru.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, _i64, _i64, _i64,
                                              ctypes.c_float, ctypes.c_int32, _vp, ctypes.c_size_t,
                                              _vp, _vp, _vp]
            lib.pararnn_solve_gru.restype = ctypes.c_int
            lib.pararnn_solve_lstm.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _i64,
                                               _i64, _i64, ctypes.c_float, ctypes.c_int32, _vp,
                                               ctypes.c_size_t, _vp, _vp, _vp]
            lib.pararnn_solve_lstm.restype = ctypes.c_int
            lib.pararnn_solve_gru_backward.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp,
                                                       _vp, _vp, _i64, _i64, _i64, _vp,
                                                       ctypes.c_size_t, _vp, _vp, _vp]
            lib.pararnn_solve_gru_backward.restype = ctypes.c_int
            lib.pararnn_solve_lstm_backward.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp,
                                                        _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64,
                                                        _i64, _vp, ctypes.c_size_t, _vp, _vp, _vp]
            lib.pararnn_solve_lstm_backward.restype = ctypes.c_int
            lib.pararnn_step_gru.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, _i64, _i64, _vp]
            lib.pararnn_step_gru.restype = ctypes.c_int
            lib.pararnn_step_lstm.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _i64,
                                              _i64, _vp]
            lib.pararnn_step_lstm.restype = ctypes.c_int
            lib.pararnn_rollout_gru.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, _i64, _i64, _i64,
                                                _vp]
            lib.pararnn_rollout_gru.restype = ctypes.c_int
            lib.pararnn_rollout_lstm.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _i64,
                                                 _i64, _i64, _vp]
            lib.pararnn_rollout_lstm.restype = ctypes.c_int
            lib.pararnn_rollout_mhgru.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, _i64, _i64,
                                                  _i64, _vp]
            lib.pararnn_rollout_mhgru.restype = ctypes.c_int
            lib.pararnn_step_mhgru.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, _i64, _i64, _vp]
            lib.pararnn_step_mhgru.restype = ctypes.c_int
            lib.pararnn_solve_gru_noalloc.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, _i64,
                                                      _i64, _i64, ctypes.c_float, ctypes.c_int32,
                                                      _vp, _vp, _vp]
            lib.pararnn_solve_gru_noalloc.restype = ctypes.c_int
            lib.pararnn_solve_mhgru.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, _i64, _i64,
                                                _i64, ctypes.c_float, ctypes.c_int32, _vp,
                                                ctypes.c_size_t, _vp, _vp, _vp]
            lib.pararnn_solve_mhgru.restype = ctypes.c_int
            lib.pararnn_solve_mhgru_strided.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, _vp,
                                                        _i64, _i64, _i64, ctypes.c_float,
                                                        ctypes.c_int32, _vp, ctypes.c_size_t,
                                                        _vp, _vp, _vp]
            lib.pararnn_solve_mhgru_strided.restype = ctypes.c_int
            lib.pararnn_input_projection.argtypes = [_vp, _vp, _vp, _vp, ctypes.c_int, _i64,
                                                     _i64, _i64, _vp, _vp]
            lib.pararnn_input_projection.restype = ctypes.c_int
            lib.pararnn_solve_gru_projected.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64,
                                                        _i64, _i64, ctypes.c_float,
                                                        ctypes.c_int32, _vp, ctypes.c_size_t,
                                                        _vp, _vp, _vp]
            lib.pararnn_solve_gru_projected.restype = ctypes.c_int
            lib.pararnn_probe_rate.argtypes = [ctypes.c_int32, ctypes.c_int32, _vp, _vp, _vp]
            lib.pararnn_probe_rate.restype = ctypes.c_int
            lib.pararnn_status_string.argtypes = [ctypes.c_int]
            lib.pararnn_status_string.restype = ctypes.c_char_p
            lib.pararnn_version.restype = ctypes.c_int32
            _ws_sizes.clear()  # sizes are the loaded library's answers
            _lib = lib
    return _lib


_ws_sizes = {}


def workspace_size(op: int, B: int, L: int, D: int, max_iters: int = 0, opts: Options | None = None):
    """Workspace bytes of a call: the library's answer, remembered per distinct
    argument tuple (options included) until another library is loaded."""
    lib = load()
    key = (int(op), int(B), int(L), int(D), int(max_iters), None if opts is None else bytes(opts))
    n = _ws_sizes.get(key)
    if n is None:
        n = lib.pararnn_workspace_size(int(op), int(B), int(L), int(D), int(max_iters),
                                       ctypes.byref(opts) if opts is not None else None)
        if n == 0:
            raise PararnnError(1, "workspace_size")
        n = int(n)
        if len(_ws_sizes) > 4096:
            _ws_sizes.clear()
        _ws_sizes[key] = n
    return n


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_dev(name, t, dtype, shape):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _one_device(**named):
    """The one CUDA device every given tensor lives on.  The library resolves
    the launch (stream, scratch, occupancy) against the current device, so
    tensors on a device other than the one the call runs on, or on several
    devices, are refused here."""
    dev = None
    first = None
    for name, t in named.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
        if dev is None:
            dev, first = t.device, name
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device} but {first} is on {dev}: "
                             "all arguments of a call must be on one device")
    if dev is None:
        raise ValueError("no tensor argument")
    return dev


def _device_guard(dev):
    """Makes `dev` the current device for the duration of one library call."""
    return torch.cuda.device(dev)


def _stream_handle(stream, dev=None):
    """The stream a call is enqueued on: the given one (which must belong to
    the tensors' device) or that device's current stream."""
    if stream is None:
        s = torch.cuda.current_stream(dev)
    else:
        s = stream
        if dev is not None and s.device != dev:
            raise ValueError(f"stream is on {s.device} but the tensors are on {dev}")
    return ctypes.c_void_p(s.cuda_stream)


_ws_cache = threading.local()


def _workspace(nbytes, device, stream=None):
    """Workspace from torch's allocator, reused between calls on the same thread,
    device and stream (calls on one stream run in order, so they can share it;
    calls on different streams get their own)."""
    cache = getattr(_ws_cache, "bufs", None)
    if cache is None:
        cache = _ws_cache.bufs = {}
    dev = device.index if device.index is not None else torch.cuda.current_device()
    s = torch.cuda.current_stream(dev) if stream is None else stream
    key = (dev, s.cuda_stream)
    buf = cache.get(key)
    if buf is None or buf.numel() < nbytes:
        with torch.cuda.stream(s):
            buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        cache[key] = buf
    return buf


class SolveInfo:
    """Device-side outcome of a solve; fields are read (one device->host copy) on first access."""

    def __init__(self, dev_tensor: torch.Tensor):
        self.tensor = dev_tensor
        self._host = None

    def _get(self):
        if self._host is None:
            raw = self.tensor.cpu().numpy().tobytes()
            self._host = _Info.from_buffer_copy(raw)
        return self._host

    @property
    def iterations(self):
        return int(self._get().iterations)

    @property
    def converged(self):
        return bool(self._get().converged)

    @property
    def status(self):
        return int(self._get().status)

    @property
    def updates(self):
        return int(self._get().updates)

    @property
    def passes(self):
        return int(self._get().passes)

    @property
    def max_residual(self):
        return float(self._get().max_residual)

    @property
    def rho(self):
        h = self._get()
        return [float(h.rho[k]) for k in range(MAX_ITERS + 1)]

    def as_dict(self):
        return dict(iterations=self.iterations, converged=self.converged, status=self.status,
                    updates=self.updates, passes=self.passes, max_residual=self.max_residual)


def _raise(st, where):
    if st != 0:
        raise PararnnError(st, where)


def scan_diag(A, b, h0=None, out=None, status=None, opts: Options | None = None, stream=None):
    """h[b, t, d] = A[b, t, d] * h[b, t-1, d] + b[b, t, d] (fp32, [B, L, D])."""
    lib = load()
    B, L, D = A.shape
    _check_dev("A", A, torch.float32, (B, L, D))
    _check_dev("b", b, torch.float32, (B, L, D))
    _check_dev("h0", h0, torch.float32, (B, D))
    h = torch.empty_like(A) if out is None else out
    _check_dev("out", h, torch.float32, (B, L, D))
    _check_dev("status", status, torch.int32, (1,))
    dev = _one_device(A=A, b=b, h0=h0, out=h, status=status)
    n = workspace_size(OP_SCAN_DIAG, B, L, D, 0, opts)
    ws = _workspace(n, dev, stream)
    with _device_guard(dev):
        st = lib.pararnn_scan_diag(_ptr(A), _ptr(b), _ptr(h0), _ptr(h), B, L, D, _ptr(ws),
                                   ws.numel(), _ptr(status),
                                   ctypes.byref(opts) if opts is not None else None,
                                   _stream_handle(stream, dev))
    _raise(st, "pararnn_scan_diag")
    return h


def scan_block2(A, b, x0=None, out=None, status=None, opts: Options | None = None, stream=None):
    """x_t = A_t x_{t-1} + b_t with A [B, L, D, 2, 2] (row-major) and x, b [B, L, D, 2]."""
    lib = load()
    B, L, D = A.shape[:3]
    _check_dev("A", A, torch.float32, (B, L, D, 2, 2))
    _check_dev("b", b, torch.float32, (B, L, D, 2))
    _check_dev("x0", x0, torch.float32, (B, D, 2))
    x = torch.empty_like(b) if out is None else out
    _check_dev("out", x, torch.float32, (B, L, D, 2))
    _check_dev("status", status, torch.int32, (1,))
    dev = _one_device(A=A, b=b, x0=x0, out=x, status=status)
    n = workspace_size(OP_SCAN_BLOCK2, B, L, D, 0, opts)
    ws = _workspace(n, dev, stream)
    with _device_guard(dev):
        st = lib.pararnn_scan_block2(_ptr(A), _ptr(b), _ptr(x0), _ptr(x), B, L, D, _ptr(ws),
                                     ws.numel(), _ptr(status),
                                     ctypes.byref(opts) if opts is not None else None,
                                     _stream_handle(stream, dev))
    _raise(st, "pararnn_scan_block2")
    return x


def _p_dtype(P):
    if P.dtype == torch.float32:
        return F32
    if P.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"P must be float32 or bfloat16, got {P.dtype}")


def solve_gru(P, a, h0=None, tol=1e-4, max_iters=32, out=None, info=None,
              opts: Options | None = None, stream=None):
    """ParaGRU Newton solve.  P [B, L, 3, D] (z, r, c), a [3, D] -> (h [B, L, D], SolveInfo)."""
    lib = load()
    B, L, G, D = P.shape
    if G != 3:
        raise ValueError("P must be [B, L, 3, D]")
    dt = _p_dtype(P)
    _check_dev("P", P, P.dtype, (B, L, 3, D))
    _check_dev("a", a, torch.float32, (3, D))
    _check_dev("h0", h0, torch.float32, (B, D))
    h = torch.empty((B, L, D), dtype=torch.float32, device=P.device) if out is None else out
    _check_dev("out", h, torch.float32, (B, L, D))
    if info is None:
        info = torch.empty(INFO_BYTES // 4, dtype=torch.int32, device=P.device)
    _check_dev("info", info, torch.int32, (INFO_BYTES // 4,))
    dev = _one_device(P=P, a=a, h0=h0, out=h, info=info)
    n = workspace_size(OP_GRU, B, L, D, max_iters, opts)
    ws = _workspace(n, dev, stream)
    with _device_guard(dev):
        st = lib.pararnn_solve_gru(_ptr(P), dt, _ptr(a), _ptr(h0), _ptr(h), B, L, D, float(tol),
                                   int(max_iters), _ptr(ws), ws.numel(), _ptr(info),
                                   ctypes.byref(opts) if opts is not None else None,
                                   _stream_handle(stream, dev))
    _raise(st, "pararnn_solve_gru")
    return h, SolveInfo(info)


def solve_mhgru(P, U, h0=None, tol=1e-4, max_iters=32, out=None, info=None,
                opts: Options | None = None, stream=None):
    """Multi-head GRU (dense 8x8 recurrence blocks) Newton solve.  P [B, L, 3, D]
    (z, r, c), U [3, H, 8, 8] with D = 8 H -> (h [B, L, D], SolveInfo)."""
    lib = load()
    B, L, G, D = P.shape
    if G != 3 or U.dim() != 4 or tuple(U.shape[2:]) != (8, 8) or D != 8 * U.shape[1]:
        raise ValueError("P must be [B, L, 3, 8 H] and U [3, H, 8, 8]")
    H = U.shape[1]
    dt = _p_dtype(P)
    _check_dev("P", P, P.dtype, (B, L, 3, D))
    _check_dev("U", U, torch.float32, (3, H, 8, 8))
    _check_dev("h0", h0, torch.float32, (B, D))
    h = torch.empty((B, L, D), dtype=torch.float32, device=P.device) if out is None else out
    _check_dev("out", h, torch.float32, (B, L, D))
    if info is None:
        info = torch.empty(INFO_BYTES // 4, dtype=torch.int32, device=P.device)
    _check_dev("info", info, torch.int32, (INFO_BYTES // 4,))
    dev = _one_device(P=P, U=U, h0=h0, out=h, info=info)
    n = workspace_size(OP_MHGRU, B, L, D, max_iters, opts)
    ws = _workspace(n, dev, stream)
    with _device_guard(dev):
        st = lib.pararnn_solve_mhgru(_ptr(P), dt, _ptr(U), _ptr(h0), _ptr(h), B, L, H,
                                     float(tol), int(max_iters), _ptr(ws), ws.numel(),
                                     _ptr(info), ctypes.byref(opts) if opts is not None else None,
                                     _stream_handle(stream, dev))
    _raise(st, "pararnn_solve_mhgru")
    return h, SolveInfo(info)


def solve_mhgru_strided(P, U, strides, h0=None, tol=1e-4, max_iters=32, out=None, info=None,
                        opts: Options | None = None, stream=None):
    """Multi-head GRU with a time stride per head: head g recurs on h_{t - strides[g]}.
    P [B, L, 3, D] (z, r, c), U [3, H, 8, 8], strides [H] int32 (device, each >= 1)
    -> (h [B, L, D], SolveInfo)."""
    lib = load()
    B, L, G, D = P.shape
    if G != 3 or U.dim() != 4 or tuple(U.shape[2:]) != (8, 8) or D != 8 * U.shape[1]:
        raise ValueError("P must be [B, L, 3, 8 H] and U [3, H, 8, 8]")
    H = U.shape[1]
    dt = _p_dtype(P)
    _check_dev("P", P, P.dtype, (B, L, 3, D))
    _check_dev("U", U, torch.float32, (3, H, 8, 8))
    _check_dev("strides", strides, torch.int32, (H,))
    _check_dev("h0", h0, torch.float32, (B, D))
    h = torch.empty((B, L, D), dtype=torch.float32, device=P.device) if out is None else out
    _check_dev("out", h, torch.float32, (B, L, D))
    if info is None:
        info = torch.empty(INFO_BYTES // 4, dtype=torch.int32, device=P.device)
    _check_dev("info", info, torch.int32, (INFO_BYTES // 4,))
    dev = _one_device(P=P, U=U, strides=strides, h0=h0, out=h, info=info)
    n = workspace_size(OP_MHGRU_STRIDED, B, L, D, max_iters, opts)
    ws = _workspace(n, dev, stream)
    with _device_guard(dev):
        st = lib.pararnn_solve_mhgru_strided(_ptr(P), dt, _ptr(U), _ptr(strides), _ptr(h0),
                                             _ptr(h), B, L, H, float(tol), int(max_iters),
                                             _ptr(ws), ws.numel(), _ptr(info),
                                             ctypes.byref(opts) if opts is not None else None,
                                             _stream_handle(stream, dev))
    _raise(st, "pararnn_solve_mhgru_strided")
    return h, SolveInfo(info)


def solve_lstm(P, a, c0=None, h0=None, tol=1e-4, max_iters=32, out=None, info=None,
               opts: Options | None = None, stream=None):
    """ParaLSTM Newton solve.  P [B, L, 4, D] (i, f, g, o), a [4, D] -> (c, h, SolveInfo)."""
    lib = load()
    B, L, G, D = P.shape
    if G != 4:
        raise ValueError("P must be [B, L, 4, D]")
    dt = _p_dtype(P)
    _check_dev("P", P, P.dtype, (B, L, 4, D))
    _check_dev("a", a, torch.float32, (4, D))
    _check_dev("c0", c0, torch.float32, (B, D))
    _check_dev("h0", h0, torch.float32, (B, D))
    if out is None:
        c = torch.empty((B, L, D), dtype=torch.float32, device=P.device)
        h = torch.empty((B, L, D), dtype=torch.float32, device=P.device)
    else:
        c, h = out
    _check_dev("c", c, torch.float32, (B, L, D))
    _check_dev("h", h, torch.float32, (B, L, D))
    if info is None:
        info = torch.empty(INFO_BYTES // 4, dtype=torch.int32, device=P.device)
    _check_dev("info", info, torch.int32, (INFO_BYTES // 4,))
    dev = _one_device(P=P, a=a, c0=c0, h0=h0, c=c, h=h, info=info)
    n = workspace_size(OP_LSTM, B, L, D, max_iters, opts)
    ws = _workspace(n, dev, stream)
    with _device_guard(dev):
        st = lib.pararnn_solve_lstm(_ptr(P), dt, _ptr(a), _ptr(c0), _ptr(h0), _ptr(c), _ptr(h),
                                    B, L, D, float(tol), int(max_iters), _ptr(ws), ws.numel(),
                                    _ptr(info), ctypes.byref(opts) if opts is not None else None,
                                    _stream_handle(stream, dev))
    _raise(st, "pararnn_solve_lstm")
    return c, h, SolveInfo(info)


def solve_gru_projected(x, W, bias, a, h0=None, tol=1e-4, max_iters=32, out=None, info=None,
                        opts: Options | None = None, stream=None):
    """ParaGRU layer from its inputs: P = x W^T + bias on the tensor cores, fused
    with the Newton solve so that P never reaches HBM.  x [B, L, K] bf16, W
    [3 D, K] bf16 (rows z, r, c), bias [3 D] fp32 or None, a [3, D] ->
    (h [B, L, D], SolveInfo)."""
    lib = load()
    if x.dim() != 3 or W.dim() != 2 or x.shape[-1] != W.shape[1] or W.shape[0] % 3 != 0:
        raise ValueError(f"x [B, L, K] and W [3 D, K] do not match: {tuple(x.shape)}, "
                         f"{tuple(W.shape)}")
    B, L, K = x.shape
    D = W.shape[0] // 3
    _check_dev("x", x, torch.bfloat16, (B, L, K))
    _check_dev("W", W, torch.bfloat16, (3 * D, K))
    _check_dev("bias", bias, torch.float32, (3 * D,))
    _check_dev("a", a, torch.float32, (3, D))
    _check_dev("h0", h0, torch.float32, (B, D))
    h = torch.empty((B, L, D), dtype=torch.float32, device=x.device) if out is None else out
    _check_dev("out", h, torch.float32, (B, L, D))
    if info is None:
        info = torch.empty(INFO_BYTES // 4, dtype=torch.int32, device=x.device)
    _check_dev("info", info, torch.int32, (INFO_BYTES // 4,))
    dev = _one_device(x=x, W=W, bias=bias, a=a, h0=h0, out=h, info=info)
    n = workspace_size(OP_GRU_PROJECTED, B, L, D, max_iters, opts)
    ws = _workspace(n, dev, stream)
    with _device_guard(dev):
        st = lib.pararnn_solve_gru_projected(_ptr(x), _ptr(W), _ptr(bias), _ptr(a), _ptr(h0),
                                             _ptr(h), B, L, D, K, float(tol), int(max_iters),
                                             _ptr(ws), ws.numel(), _ptr(info),
                                             ctypes.byref(opts) if opts is not None else None,
                                             _stream_handle(stream, dev))
    _raise(st, "pararnn_solve_gru_projected")
    return h, SolveInfo(info)


NOALLOC_SCRATCH_BYTES = 4 << 20


def solve_gru_noalloc(P, a, h0=None, tol=1e-4, max_iters=32, out=None, info=None,
                      opts: Options | None = None, stream=None):
    """ParaGRU Newton solve through ``pararnn_solve_gru_noalloc``: the library
    allocates nothing and uses its own fixed device scratch array instead of a
    workspace (for callers that cannot allocate device memory where they
    solve).  Calls on one device share that array, so they must not overlap on
    the GPU.  ``out`` and ``info`` may be passed to keep this call itself free
    of allocations."""
    lib = load()
    B, L, G, D = P.shape
    if G != 3:
        raise ValueError("P must be [B, L, 3, D]")
    dt = _p_dtype(P)
    _check_dev("P", P, P.dtype, (B, L, 3, D))
    _check_dev("a", a, torch.float32, (3, D))
    _check_dev("h0", h0, torch.float32, (B, D))
    h = torch.empty((B, L, D), dtype=torch.float32, device=P.device) if out is None else out
    _check_dev("out", h, torch.float32, (B, L, D))
    if info is None:
        info = torch.empty(INFO_BYTES // 4, dtype=torch.int32, device=P.device)
    _check_dev("info", info, torch.int32, (INFO_BYTES // 4,))
    dev = _one_device(P=P, a=a, h0=h0, out=h, info=info)
    with _device_guard(dev):
        st = lib.pararnn_solve_gru_noalloc(_ptr(P), dt, _ptr(a), _ptr(h0), _ptr(h), B, L, D,
                                           float(tol), int(max_iters), _ptr(info),
                                           ctypes.byref(opts) if opts is not None else None,
                                           _stream_handle(stream, dev))
    _raise(st, "pararnn_solve_gru_noalloc")
    return h, SolveInfo(info)


def solve_gru_backward(P, a, h, dh, h0=None, out=None, status=None,
                       opts: Options | None = None, stream=None):
    """Gradients of a loss through the ParaGRU solution h, given dh = dl/dh.

    Returns (dP [B, L, 3, D] fp32, da [3, D], dh0 [B, D])."""
    lib = load()
    B, L, G, D = P.shape
    if G != 3:
        raise ValueError("P must be [B, L, 3, D]")
    dt = _p_dtype(P)
    _check_dev("P", P, P.dtype, (B, L, 3, D))
    _check_dev("a", a, torch.float32, (3, D))
    _check_dev("h0", h0, torch.float32, (B, D))
    _check_dev("h", h, torch.float32, (B, L, D))
    _check_dev("dh", dh, torch.float32, (B, L, D))
    if out is None:
        dP = torch.empty((B, L, 3, D), dtype=torch.float32, device=P.device)
        da = torch.empty((3, D), dtype=torch.float32, device=P.device)
        dh0 = torch.empty((B, D), dtype=torch.float32, device=P.device)
    else:
        dP, da, dh0 = out
    _check_dev("dP", dP, torch.float32, (B, L, 3, D))
    _check_dev("da", da, torch.float32, (3, D))
    _check_dev("dh0", dh0, torch.float32, (B, D))
    _check_dev("status", status, torch.int32, (1,))
    dev = _one_device(P=P, a=a, h0=h0, h=h, dh=dh, dP=dP, da=da, dh0=dh0, status=status)
    n = workspace_size(OP_GRU_BACKWARD, B, L, D, 0, opts)
    ws = _workspace(n, dev, stream)
    with _device_guard(dev):
        st = lib.pararnn_solve_gru_backward(_ptr(P), dt, _ptr(a), _ptr(h0), _ptr(h), _ptr(dh),
                                            _ptr(dP), _ptr(da), _ptr(dh0), B, L, D, _ptr(ws),
                                            ws.numel(), _ptr(status),
                                            ctypes.byref(opts) if opts is not None else None,
                                            _stream_handle(stream, dev))
    _raise(st, "pararnn_solve_gru_backward")
    return dP, da, dh0


def solve_lstm_backward(P, a, c, h, dc, dh, c0=None, h0=None, out=None, status=None,
                        opts: Options | None = None, stream=None):
    """Gradients through the ParaLSTM solution (c, h), given dc = dl/dc and dh = dl/dh
    (either may be None).  Returns (dP [B, L, 4, D], da [4, D], dc0 [B, D], dh0 [B, D])."""
    lib = load()
    B, L, G, D = P.shape
    if G != 4:
        raise ValueError("P must be [B, L, 4, D]")
    dt = _p_dtype(P)
    _check_dev("P", P, P.dtype, (B, L, 4, D))
    _check_dev("a", a, torch.float32, (4, D))
    for nm, t in (("c0", c0), ("h0", h0)):
        _check_dev(nm, t, torch.float32, (B, D))
    for nm, t in (("c", c), ("h", h), ("dc", dc), ("dh", dh)):
        _check_dev(nm, t, torch.float32, (B, L, D))
    if out is None:
        dP = torch.empty((B, L, 4, D), dtype=torch.float32, device=P.device)
        da = torch.empty((4, D), dtype=torch.float32, device=P.device)
        dc0 = torch.empty((B, D), dtype=torch.float32, device=P.device)
        dh0 = torch.empty((B, D), dtype=torch.float32, device=P.device)
    else:
        dP, da, dc0, dh0 = out
    _check_dev("dP", dP, torch.float32, (B, L, 4, D))
    _check_dev("da", da, torch.float32, (4, D))
    _check_dev("dc0", dc0, torch.float32, (B, D))
    _check_dev("dh0", dh0, torch.float32, (B, D))
    _check_dev("status", status, torch.int32, (1,))
    dev = _one_device(P=P, a=a, c0=c0, h0=h0, c=c, h=h, dc=dc, dh=dh, dP=dP, da=da, dc0=dc0,
                      dh0=dh0, status=status)
    n = workspace_size(OP_LSTM_BACKWARD, B, L, D, 0, opts)
    ws = _workspace(n, dev, stream)
    with _device_guard(dev):
        st = lib.pararnn_solve_lstm_backward(_ptr(P), dt, _ptr(a), _ptr(c0), _ptr(h0), _ptr(c),
                                             _ptr(h), _ptr(dc), _ptr(dh), _ptr(dP), _ptr(da),
                                             _ptr(dc0), _ptr(dh0), B, L, D, _ptr(ws), ws.numel(),
                                             _ptr(status),
                                             ctypes.byref(opts) if opts is not None else None,
                                             _stream_handle(stream, dev))
    _raise(st, "pararnn_solve_lstm_backward")
    return dP, da, dc0, dh0


def step_gru(P, a, h_prev=None, out=None, stream=None):
    """One ParaGRU step for every channel (decode): P [B, 3, D] -> h_next [B, D]."""
    lib = load()
    B, G, D = P.shape
    if G != 3:
        raise ValueError("P must be [B, 3, D]")
    dt = _p_dtype(P)
    _check_dev("P", P, P.dtype, (B, 3, D))
    _check_dev("a", a, torch.float32, (3, D))
    _check_dev("h_prev", h_prev, torch.float32, (B, D))
    h = torch.empty((B, D), dtype=torch.float32, device=P.device) if out is None else out
    _check_dev("out", h, torch.float32, (B, D))
    dev = _one_device(P=P, a=a, h_prev=h_prev, out=h)
    with _device_guard(dev):
        st = lib.pararnn_step_gru(_ptr(P), dt, _ptr(a), _ptr(h_prev), _ptr(h), B, D,
                                  _stream_handle(stream, dev))
    _raise(st, "pararnn_step_gru")
    return h


def step_mhgru(P, U, h_prev=None, out=None, stream=None):
    """One multi-head GRU step (decode): P [B, 3, D] (z, r, c), U [3, H, 8, 8],
    D = 8 H -> h_next [B, D]."""
    lib = load()
    B, G, D = P.shape
    if G != 3 or U.dim() != 4 or tuple(U.shape[2:]) != (8, 8) or D != 8 * U.shape[1]:
        raise ValueError("P must be [B, 3, 8 H] and U [3, H, 8, 8]")
    H = U.shape[1]
    dt = _p_dtype(P)
    _check_dev("P", P, P.dtype, (B, 3, D))
    _check_dev("U", U, torch.float32, (3, H, 8, 8))
    _check_dev("h_prev", h_prev, torch.float32, (B, D))
    h = torch.empty((B, D), dtype=torch.float32, device=P.device) if out is None else out
    _check_dev("out", h, torch.float32, (B, D))
    dev = _one_device(P=P, U=U, h_prev=h_prev, out=h)
    with _device_guard(dev):
        st = lib.pararnn_step_mhgru(_ptr(P), dt, _ptr(U), _ptr(h_prev), _ptr(h), B, H,
                                    _stream_handle(stream, dev))
    _raise(st, "pararnn_step_mhgru")
    return h


def input_projection(x, W, bias=None, out=None, out_dtype=torch.float32, status=None,
                     stream=None):
    """P = x W^T + bias on the tensor cores: x [..., K] bf16, W [N, K] bf16,
    bias [N] fp32 or None -> P [..., N] (fp32 or bf16).  With N = G * D and x
    [B, L, K], P.view(B, L, G, D) is the solve's input."""
    lib = load()
    if x.dtype != torch.bfloat16 or W.dtype != torch.bfloat16:
        raise TypeError("x and W must be bf16")
    if W.dim() != 2 or x.shape[-1] != W.shape[1]:
        raise ValueError(f"x [..., K] and W [N, K] do not match: {tuple(x.shape)}, {tuple(W.shape)}")
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("out_dtype must be float32 or bfloat16")
    N, K = W.shape
    lead = tuple(x.shape[:-1])
    M = 1
    for n in lead:
        M *= n
    if not x.is_contiguous() or not W.is_contiguous():
        raise ValueError("x and W must be contiguous")
    _check_dev("x", x, torch.bfloat16, lead + (K,))
    _check_dev("W", W, torch.bfloat16, (N, K))
    _check_dev("bias", bias, torch.float32, (N,))
    P = torch.empty(lead + (N,), dtype=out_dtype, device=x.device) if out is None else out
    _check_dev("out", P, out_dtype, lead + (N,))
    _check_dev("status", status, torch.int32, (1,))
    dt = BF16 if out_dtype == torch.bfloat16 else F32
    dev = _one_device(x=x, W=W, bias=bias, out=P, status=status)
    with _device_guard(dev):
        st = lib.pararnn_input_projection(_ptr(x), _ptr(W), _ptr(bias), _ptr(P), dt, M, N, K,
                                          _ptr(status), _stream_handle(stream, dev))
    _raise(st, "pararnn_input_projection")
    return P


def step_lstm(P, a, c_prev=None, h_prev=None, out=None, stream=None):
    """One ParaLSTM step for every channel: P [B, 4, D] -> (c_next, h_next)."""
    lib = load()
    B, G, D = P.shape
    if G != 4:
        raise ValueError("P must be [B, 4, D]")
    dt = _p_dtype(P)
    _check_dev("P", P, P.dtype, (B, 4, D))
    _check_dev("a", a, torch.float32, (4, D))
    _check_dev("c_prev", c_prev, torch.float32, (B, D))
    _check_dev("h_prev", h_prev, torch.float32, (B, D))
    if out is None:
        c = torch.empty((B, D), dtype=torch.float32, device=P.device)
        h = torch.empty((B, D), dtype=torch.float32, device=P.device)
    else:
        c, h = out
    _check_dev("c", c, torch.float32, (B, D))
    _check_dev("h", h, torch.float32, (B, D))
    dev = _one_device(P=P, a=a, c_prev=c_prev, h_prev=h_prev, c=c, h=h)
    with _device_guard(dev):
        st = lib.pararnn_step_lstm(_ptr(P), dt, _ptr(a), _ptr(c_prev), _ptr(h_prev), _ptr(c),
                                   _ptr(h), B, D, _stream_handle(stream, dev))
    _raise(st, "pararnn_step_lstm")
    return c, h


def rollout_gru(P, a, h0=None, out=None, stream=None):
    """Sequential ParaGRU application on the GPU (one thread per channel)."""
    lib = load()
    B, L, G, D = P.shape
    if G != 3:
        raise ValueError("P must be [B, L, 3, D]")
    dt = _p_dtype(P)
    _check_dev("P", P, P.dtype, (B, L, 3, D))
    _check_dev("a", a, torch.float32, (3, D))
    _check_dev("h0", h0, torch.float32, (B, D))
    h = torch.empty((B, L, D), dtype=torch.float32, device=P.device) if out is None else out
    _check_dev("out", h, torch.float32, (B, L, D))
    dev = _one_device(P=P, a=a, h0=h0, out=h)
    with _device_guard(dev):
        st = lib.pararnn_rollout_gru(_ptr(P), dt, _ptr(a), _ptr(h0), _ptr(h), B, L, D,
                                     _stream_handle(stream, dev))
    _raise(st, "pararnn_rollout_gru")
    return h


def rollout_mhgru(P, U, h0=None, out=None, stream=None):
    """Sequential multi-head GRU application on the GPU (8 lanes per head
    sequence).  P [B, L, 3, D] (z, r, c), U [3, H, 8, 8], D = 8 H -> h [B, L, D]."""
    lib = load()
    B, L, G, D = P.shape
    if G != 3 or U.dim() != 4 or tuple(U.shape[2:]) != (8, 8) or D != 8 * U.shape[1]:
        raise ValueError("P must be [B, L, 3, 8 H] and U [3, H, 8, 8]")
    H = U.shape[1]
    dt = _p_dtype(P)
    _check_dev("P", P, P.dtype, (B, L, 3, D))
    _check_dev("U", U, torch.float32, (3, H, 8, 8))
    _check_dev("h0", h0, torch.float32, (B, D))
    h = torch.empty((B, L, D), dtype=torch.float32, device=P.device) if out is None else out
    _check_dev("out", h, torch.float32, (B, L, D))
    dev = _one_device(P=P, U=U, h0=h0, out=h)
    with _device_guard(dev):
        st = lib.pararnn_rollout_mhgru(_ptr(P), dt, _ptr(U), _ptr(h0), _ptr(h), B, L, H,
                                       _stream_handle(stream, dev))
    _raise(st, "pararnn_rollout_mhgru")
    return h


def rollout_lstm(P, a, c0=None, h0=None, out=None, stream=None):
    """Sequential ParaLSTM application on the GPU (one thread per channel)."""
    lib = load()
    B, L, G, D = P.shape
    if G != 4:
        raise ValueError("P must be [B, L, 4, D]")
    dt = _p_dtype(P)
    _check_dev("P", P, P.dtype, (B, L, 4, D))
    _check_dev("a", a, torch.float32, (4, D))
    _check_dev("c0", c0, torch.float32, (B, D))
    _check_dev("h0", h0, torch.float32, (B, D))
    if out is None:
        c = torch.empty((B, L, D), dtype=torch.float32, device=P.device)
        h = torch.empty((B, L, D), dtype=torch.float32, device=P.device)
    else:
        c, h = out
    _check_dev("c", c, torch.float32, (B, L, D))
    _check_dev("h", h, torch.float32, (B, L, D))
    dev = _one_device(P=P, a=a, c0=c0, h0=h0, c=c, h=h)
    with _device_guard(dev):
        st = lib.pararnn_rollout_lstm(_ptr(P), dt, _ptr(a), _ptr(c0), _ptr(h0), _ptr(c), _ptr(h),
                                      B, L, D, _stream_handle(stream, dev))
    _raise(st, "pararnn_rollout_lstm")
    return c, h


PROBE_MUFU, PROBE_FMA = 0, 1


def probe_rate(pipe, iters, sink, stream=None):
    """Enqueue one throughput-probe launch (``pararnn_probe_rate``) and return
    the number of operations it performs: ex2 + rcp for ``PROBE_MUFU``, FMAs
    for ``PROBE_FMA``.  ``sink`` is a device tensor of at least 4 bytes."""
    lib = load()
    if not sink.is_cuda or sink.numel() * sink.element_size() < 4:
        raise ValueError("sink must be a CUDA tensor of at least 4 bytes")
    ops = ctypes.c_int64(0)
    with _device_guard(sink.device):
        st = lib.pararnn_probe_rate(int(pipe), int(iters), _ptr(sink), ctypes.byref(ops),
                                    _stream_handle(stream, sink.device))
    _raise(st, "pararnn_probe_rate")
    return int(ops.value)
