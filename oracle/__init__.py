"""fp64 CPU oracle for the ParaRNN / DEER Newton solve (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``oracle.c`` (plain C, fp64,
threads across independent channels only) through ctypes and shares no code with the
CUDA library in ``nonlinear_rnn_solve_newton_b200``.

What each function computes, and the passage it follows:

* ``scan_diag`` / ``scan_block2``: the block bi-diagonal linear system
  h_t = A_t h_{t-1} + b_t solved sequentially in t (ParaRNN TL;DR: the Newton
  step is a block bi-diagonal system; Figure 2 caption: diagonal and 2x2
  block-diagonal variants).
* ``rollout_gru`` / ``rollout_lstm``: the sequential application of the cell,
  the plain definition of the result that Newton must reproduce (ParaRNN
  abstract, "naive sequential application"; DEER summary: outputs agree with
  sequential evaluation).
* ``newton_gru`` / ``newton_lstm``: Newton's method on the stacked system,
  serial, with the max-abs residual over the whole batch as the stopping
  test (ParaRNN abstract and Figure 4 caption; DEER summary: tolerance 1e-4).
* ``gru_cell`` / ``lstm_cell``: one cell step and its Jacobian.
* ``backward_gru`` / ``backward_lstm``: gradients of a loss through the solved
  trajectory by the adjoint (reverse-time, transposed bi-diagonal) recursion.
* ``mhgru_cell`` / ``rollout_mhgru`` / ``newton_mhgru``: the multi-head GRU
  whose recurrence is block-diagonal with dense 8x8 blocks (the dense-block
  case the DEER summary's caveats price at O(n^3) per step), reducing to the
  ParaGRU cell when every block is diagonal.
* ``input_projection``: P = x W^T + bias, the projected gate inputs of the
  cells (ParaRNN TL;DR: dense weights act on the inputs, the recurrence keeps
  diagonal ones), as plain fp64 sums.

Parity status: every function above is pinned in ``tests/test_oracle_pins.py``
against closed forms, brute force, PyTorch's fp64 ``GRUCell``/``LSTMCell`` and
autograd, and Newton's own invariants.  The iteration count has no printed
value to pin against (Figure 4 survived only as a caption): parity unpinned for
the count itself; it is checked only through the invariants (one iteration for
an affine recurrence, two for an LSTM with no recurrence, at most L).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_intp = ctypes.POINTER(ctypes.c_int)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-std=c11", _SRC, "-o", _LIB + ".tmp", "-lm", "-lpthread"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _bind(lib):
    """Declare the C signatures on a loaded oracle library."""
    lib.oracle_scan_diag.argtypes = [_f64p, _f64p, _f64p, _f64p, _i64, _i64, _i64]
    lib.oracle_scan_block2.argtypes = [_f64p, _f64p, _f64p, _f64p, _i64, _i64, _i64]
    lib.oracle_gru_cell.argtypes = [_f64p, _f64p, ctypes.c_double, _f64p, _f64p]
    lib.oracle_lstm_cell.argtypes = [_f64p, _f64p, ctypes.c_double, ctypes.c_double,
                                     _f64p, _f64p, _f64p]
    lib.oracle_rollout_gru.argtypes = [_f64p, _f64p, _f64p, _f64p, _i64, _i64, _i64]
    lib.oracle_rollout_lstm.argtypes = [_f64p, _f64p, _f64p, _f64p, _f64p, _f64p,
                                        _i64, _i64, _i64]
    lib.oracle_newton_gru.argtypes = [_f64p, _f64p, _f64p, ctypes.c_double, ctypes.c_int,
                                      _i64, _i64, _i64, _f64p, _f64p, _i32p, _intp, _intp]
    lib.oracle_newton_gru.restype = ctypes.c_int
    lib.oracle_newton_lstm.argtypes = [_f64p, _f64p, _f64p, _f64p, ctypes.c_double,
                                       ctypes.c_int, _i64, _i64, _i64, _f64p, _f64p,
                                       _f64p, _i32p, _intp, _intp]
    lib.oracle_newton_lstm.restype = ctypes.c_int
    lib.oracle_residual_gru.argtypes = [_f64p, _f64p, _f64p, _f64p, _i64, _i64, _i64]
    lib.oracle_residual_gru.restype = ctypes.c_double
    lib.oracle_backward_gru.argtypes = [_f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p,
                                        _i64, _i64, _i64]
    lib.oracle_backward_lstm.argtypes = [_f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p, _f64p,
                                         _f64p, _f64p, _f64p, _f64p, _i64, _i64, _i64]
    lib.oracle_mhgru_cell.argtypes = [_f64p, _f64p, _f64p, _f64p, _f64p]
    lib.oracle_rollout_mhgru.argtypes = [_f64p, _f64p, _f64p, _f64p, _i64, _i64, _i64, _intp]
    lib.oracle_newton_mhgru.argtypes = [_f64p, _f64p, _f64p, ctypes.c_double, ctypes.c_int,
                                        _i64, _i64, _i64, _f64p, _f64p, _intp, _intp, _intp]
    lib.oracle_newton_mhgru.restype = ctypes.c_int
    lib.oracle_input_projection.argtypes = [_f64p, _f64p, _f64p, _f64p, _i64, _i64, _i64]
    lib.oracle_set_threads.argtypes = [ctypes.c_int]
    lib.oracle_get_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def compile_variant(src_path: str, out_path: str):
    """Build and bind another copy of oracle.c (used by the tests that plant a
    mistake in the oracle to check that the pins catch it)."""
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math",
                           "-ffp-contract=off", "-std=c11", src_path, "-o", out_path, "-lm",
                           "-lpthread"])
    return _bind(ctypes.CDLL(out_path))


def set_threads(n: int) -> None:
    """Number of host threads the oracle uses (0 = every CPU in the affinity mask)."""
    _load().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_load().oracle_get_threads())


def _d(x):
    """Contiguous fp64 copy (widening is exact for fp32 and bf16-valued inputs)."""
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(x):
    return None if x is None else x.ctypes.data_as(_f64p)


def scan_diag(A, b, h0=None):
    """h[b,t,d] = A[b,t,d] * h[b,t-1,d] + b[b,t,d]; A, b: [B,L,D]; h0: [B,D] or None (= 0)."""
    A, b = _d(A), _d(b)
    B, L, D = A.shape
    h0 = None if h0 is None else _d(h0).reshape(B, D)
    h = np.empty_like(A)
    _load().oracle_scan_diag(_p(A), _p(b), _p(h0), _p(h), B, L, D)
    return h


def scan_block2(A, b, x0=None):
    """x_t = A_t x_{t-1} + b_t; A: [B,L,D,2,2] row-major, b: [B,L,D,2], x0: [B,D,2] or None."""
    A, b = _d(A), _d(b)
    B, L, D = A.shape[:3]
    x0 = None if x0 is None else _d(x0).reshape(B, D, 2)
    x = np.empty_like(b)
    _load().oracle_scan_block2(_p(A), _p(b), _p(x0), _p(x), B, L, D)
    return x


def gru_cell(p, w, h):
    """One ParaGRU step: p = (Pz, Pr, Pc), w = (az, ar, ac) -> (h', dh'/dh)."""
    p, w = _d(p), _d(w)
    f = ctypes.c_double()
    J = ctypes.c_double()
    _load().oracle_gru_cell(_p(p), _p(w), float(h), ctypes.byref(f), ctypes.byref(J))
    return f.value, J.value


def lstm_cell(p, w, c, h):
    """One ParaLSTM step: p = (Pi, Pf, Pg, Po) -> (c', h', J 2x2 d(c',h')/d(c,h))."""
    p, w = _d(p), _d(w)
    fc = ctypes.c_double()
    fh = ctypes.c_double()
    J = np.zeros(4)
    _load().oracle_lstm_cell(_p(p), _p(w), float(c), float(h), ctypes.byref(fc),
                             ctypes.byref(fh), _p(J))
    return fc.value, fh.value, J.reshape(2, 2)


def rollout_gru(P, a, h0=None):
    """Sequential ParaGRU rollout. P: [B,L,3,D], a: [3,D], h0: [B,D] or None -> h [B,L,D]."""
    P, a = _d(P), _d(a)
    B, L, G, D = P.shape
    assert G == 3
    h0 = None if h0 is None else _d(h0).reshape(B, D)
    h = np.empty((B, L, D))
    _load().oracle_rollout_gru(_p(P), _p(a), _p(h0), _p(h), B, L, D)
    return h


def rollout_lstm(P, a, c0=None, h0=None):
    """Sequential ParaLSTM rollout. P: [B,L,4,D], a: [4,D] -> (c, h) each [B,L,D]."""
    P, a = _d(P), _d(a)
    B, L, G, D = P.shape
    assert G == 4
    c0 = None if c0 is None else _d(c0).reshape(B, D)
    h0 = None if h0 is None else _d(h0).reshape(B, D)
    c = np.empty((B, L, D))
    h = np.empty((B, L, D))
    _load().oracle_rollout_lstm(_p(P), _p(a), _p(c0), _p(h0), _p(c), _p(h), B, L, D)
    return c, h


class NewtonResult:
    def __init__(self, iterations, converged, nonfinite, rho, chan_iters, **states):
        self.iterations = iterations
        self.converged = bool(converged)
        self.nonfinite = bool(nonfinite)
        self.rho = rho                  # rho_0 .. rho_iterations
        self.chan_iters = chan_iters    # per channel [B, D]
        for k, v in states.items():
            setattr(self, k, v)


def newton_gru(P, a, h0=None, tol=1e-4, max_iters=32):
    """Serial Newton for the ParaGRU system from h^0 = 0 (see oracle.c)."""
    P, a = _d(P), _d(a)
    B, L, G, D = P.shape
    assert G == 3
    h0 = None if h0 is None else _d(h0).reshape(B, D)
    h = np.empty((B, L, D))
    rho = np.full(max_iters + 1, np.nan)
    ci = np.empty((B, D), dtype=np.int32)
    conv = ctypes.c_int()
    nf = ctypes.c_int()
    k = _load().oracle_newton_gru(_p(P), _p(a), _p(h0), float(tol), int(max_iters), B, L, D,
                                  _p(h), _p(rho), ci.ctypes.data_as(_i32p), ctypes.byref(conv),
                                  ctypes.byref(nf))
    return NewtonResult(k, conv.value, nf.value, rho[: k + 1], ci, h=h)


def newton_lstm(P, a, c0=None, h0=None, tol=1e-4, max_iters=32):
    """Serial Newton for the ParaLSTM system from (c, h)^0 = 0 (see oracle.c)."""
    P, a = _d(P), _d(a)
    B, L, G, D = P.shape
    assert G == 4
    c0 = None if c0 is None else _d(c0).reshape(B, D)
    h0 = None if h0 is None else _d(h0).reshape(B, D)
    c = np.empty((B, L, D))
    h = np.empty((B, L, D))
    rho = np.full(max_iters + 1, np.nan)
    ci = np.empty((B, D), dtype=np.int32)
    conv = ctypes.c_int()
    nf = ctypes.c_int()
    k = _load().oracle_newton_lstm(_p(P), _p(a), _p(c0), _p(h0), float(tol), int(max_iters),
                                   B, L, D, _p(c), _p(h), _p(rho), ci.ctypes.data_as(_i32p),
                                   ctypes.byref(conv), ctypes.byref(nf))
    return NewtonResult(k, conv.value, nf.value, rho[: k + 1], ci, c=c, h=h)


def residual_gru(P, a, h, h0=None):
    """fp64 max_t |f(h_{t-1}, P_t) - h_t| of a given trajectory h [B,L,D]."""
    P, a, h = _d(P), _d(a), _d(h)
    B, L, G, D = P.shape
    h0 = None if h0 is None else _d(h0).reshape(B, D)
    return _load().oracle_residual_gru(_p(P), _p(a), _p(h0), _p(h), B, L, D)


def backward_gru(P, a, h, gh, h0=None):
    """Gradients of a loss through the ParaGRU trajectory h (the forward solution).

    gh = dl/dh [B,L,D].  Returns (dP [B,L,3,D], da [3,D], dh0 [B,D]) by the adjoint
    recursion lambda_t = g_t + J_{t+1}^T lambda_{t+1}, evaluated backwards in time."""
    P, a, h, gh = _d(P), _d(a), _d(h), _d(gh)
    B, L, G, D = P.shape
    h0 = None if h0 is None else _d(h0).reshape(B, D)
    dP = np.empty_like(P)
    da = np.empty((3, D))
    dh0 = np.empty((B, D))
    _load().oracle_backward_gru(_p(P), _p(a), _p(h0), _p(h), _p(gh), _p(dP), _p(da), _p(dh0),
                                B, L, D)
    return dP, da, dh0


def backward_lstm(P, a, c, h, gc, gh, c0=None, h0=None):
    """Gradients through the ParaLSTM trajectory (c, h): gc = dl/dc, gh = dl/dh (either
    may be None = 0).  Returns (dP [B,L,4,D], da [4,D], dc0 [B,D], dh0 [B,D])."""
    P, a, c, h = _d(P), _d(a), _d(c), _d(h)
    B, L, G, D = P.shape
    gc = None if gc is None else _d(gc)
    gh = None if gh is None else _d(gh)
    c0 = None if c0 is None else _d(c0).reshape(B, D)
    h0 = None if h0 is None else _d(h0).reshape(B, D)
    dP = np.empty_like(P)
    da = np.empty((4, D))
    dc0 = np.empty((B, D))
    dh0 = np.empty((B, D))
    _load().oracle_backward_lstm(_p(P), _p(a), _p(c0), _p(h0), _p(c), _p(h), _p(gc), _p(gh),
                                 _p(dP), _p(da), _p(dc0), _p(dh0), B, L, D)
    return dP, da, dc0, dh0


def input_projection(x, W, bias=None):
    """P = x W^T + bias in fp64: x [..., K], W [N, K], bias [N] or None -> P [..., N]."""
    x, W = _d(x), _d(W)
    N, K = W.shape
    lead = x.shape[:-1]
    M = int(np.prod(lead, dtype=np.int64))
    x2 = np.ascontiguousarray(x.reshape(M, K))
    bias = None if bias is None else _d(bias).reshape(N)
    P = np.empty((M, N))
    _load().oracle_input_projection(_p(x2), _p(W), _p(bias), _p(P), M, N, K)
    return P.reshape(lead + (N,))


def mhgru_cell(p, U, h):
    """One multi-head GRU step of one head: p [3, 8] (z, r, c), U [3, 8, 8] (that
    head's blocks), h [8] -> (h' [8], J = dh'/dh [8, 8])."""
    p, U, h = _d(p).reshape(3, 8), _d(U).reshape(3, 8, 8), _d(h).reshape(8)
    f = np.empty(8)
    J = np.empty((8, 8))
    _load().oracle_mhgru_cell(_p(p), _p(U), _p(h), _p(f), _p(J))
    return f, J


def _strides(strides, H):
    if strides is None:
        return None, None
    st = np.ascontiguousarray(strides, dtype=np.int32).reshape(H)
    assert np.all(st >= 1), "strides must be >= 1"
    return st, st.ctypes.data_as(_intp)


def rollout_mhgru(P, U, h0=None, strides=None):
    """Sequential multi-head GRU rollout.  P [B, L, 3, D], U [3, H, 8, 8], D = 8 H;
    strides [H] (optional): head g recurs on h_{t - strides[g]}."""
    P, U = _d(P), _d(U)
    B, L, G, D = P.shape
    H = U.shape[1]
    assert G == 3 and U.shape == (3, H, 8, 8) and D == 8 * H
    h0 = None if h0 is None else _d(h0).reshape(B, D)
    h = np.empty((B, L, D))
    keep, sp = _strides(strides, H)
    _load().oracle_rollout_mhgru(_p(P), _p(U), _p(h0), _p(h), B, L, H, sp)
    return h


def newton_mhgru(P, U, h0=None, tol=1e-4, max_iters=32, strides=None):
    """Serial Newton for the multi-head GRU system from h^0 = 0, 8x8 block
    bi-diagonal solve per head (see oracle.c); strides as in rollout_mhgru."""
    P, U = _d(P), _d(U)
    B, L, G, D = P.shape
    H = U.shape[1]
    assert G == 3 and U.shape == (3, H, 8, 8) and D == 8 * H
    h0 = None if h0 is None else _d(h0).reshape(B, D)
    h = np.empty((B, L, D))
    rho = np.full(max_iters + 1, np.nan)
    conv = ctypes.c_int()
    nf = ctypes.c_int()
    keep, sp = _strides(strides, H)
    k = _load().oracle_newton_mhgru(_p(P), _p(U), _p(h0), float(tol), int(max_iters), B, L, H,
                                    _p(h), _p(rho), ctypes.byref(conv), ctypes.byref(nf), sp)
    return NewtonResult(k, conv.value, nf.value, rho[: k + 1], None, h=h)
