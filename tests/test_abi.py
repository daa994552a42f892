"""CPU-side checks of the C ABI: the library builds, loads, exports every symbol
that include/pararnn.h declares, sizes workspaces and rejects bad arguments on
the host (no CUDA work is issued by any call here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pararnn.h")


@pytest.fixture(scope="module")
def lib():
    import nonlinear_rnn_solve_newton_b200 as pr

    return pr.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pararnn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_four_entry_points():
    names = declared_functions()
    for n in ("pararnn_scan_diag", "pararnn_scan_block2", "pararnn_solve_gru",
              "pararnn_solve_lstm", "pararnn_workspace_size", "pararnn_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_version_and_status_strings(lib):
    assert lib.pararnn_version() == 1
    for code in range(7):
        s = lib.pararnn_status_string(code)
        assert isinstance(s, bytes) and len(s) > 0
    assert lib.pararnn_status_string(99) == b"unknown status"


def test_info_struct_layout():
    import nonlinear_rnn_solve_newton_b200 as pr

    # 6 int32 + 1 float + 128 floats
    assert pr.INFO_BYTES == 4 * (6 + 1 + 128)


def _header_define(name):
    m = re.search(r"#define\s+" + name + r"\s+\(?\s*(\d+)u?\s*(?:<<\s*(\d+))?\s*\)?",
                  open(HEADER).read())
    assert m, name
    v = int(m.group(1))
    return v << int(m.group(2)) if m.group(2) else v


def test_binding_constants_match_the_header():
    # the binding keeps its own copies of these limits; a stale copy would let
    # the binding accept what the library rejects (or the reverse)
    import nonlinear_rnn_solve_newton_b200 as pr

    assert pr.NOALLOC_SCRATCH_BYTES == _header_define("PARARNN_NOALLOC_SCRATCH_BYTES")
    assert pr.MAX_ITERS == _header_define("PARARNN_MAX_ITERS")


def test_workspace_size_host_only():
    import nonlinear_rnn_solve_newton_b200 as pr

    lb = pr.Options(regime=pr.Options.LOOKBACK)
    n1 = pr.workspace_size(pr.OP_GRU, 8, 4096, 1024, 32, lb)
    n2 = pr.workspace_size(pr.OP_GRU, 8, 8192, 1024, 32, lb)
    assert n1 > 0 and n2 > n1 and n1 % 256 == 0
    assert pr.workspace_size(pr.OP_SCAN_DIAG, 1, 1, 1) > 0
    assert pr.workspace_size(pr.OP_LSTM, 2, 7, 3, 0) > 0
    # more iterations per sweep -> more look-back slots
    o = pr.Options(iters_first=8, regime=pr.Options.LOOKBACK)
    assert pr.workspace_size(pr.OP_GRU, 8, 4096, 1024, 32, o) > n1
    # a CTA walking its tile needs no look-back slots: only the control block
    walk = pr.Options(regime=pr.Options.WALK)
    assert pr.workspace_size(pr.OP_GRU, 8, 4096, 1024, 32, walk) <= 4096
    with pytest.raises(pr.PararnnError):
        pr.workspace_size(pr.OP_GRU, 8, 4096, 1024, 500)   # above the iteration cap
    with pytest.raises(pr.PararnnError):
        pr.workspace_size(9, 1, 1, 1)


def test_host_validation_rejects_before_any_cuda_call(lib):
    vp = ctypes.c_void_p
    fake = vp(4096)  # never dereferenced: validation fails first
    info = vp(8192)
    # NULL inputs
    assert lib.pararnn_solve_gru(None, 0, fake, None, fake, 2, 8, 4, ctypes.c_float(1e-4), 4,
                                 fake, 1 << 20, info, None, None) == 1
    # bad dtype
    assert lib.pararnn_solve_gru(fake, 7, fake, None, fake, 2, 8, 4, ctypes.c_float(1e-4), 4,
                                 fake, 1 << 20, info, None, None) == 1
    # max_iters out of range, NaN tolerance, missing info
    assert lib.pararnn_solve_gru(fake, 0, fake, None, fake, 2, 8, 4, ctypes.c_float(1e-4), 128,
                                 fake, 1 << 20, info, None, None) == 1
    assert lib.pararnn_solve_gru(fake, 0, fake, None, fake, 2, 8, 4, ctypes.c_float(float("nan")),
                                 4, fake, 1 << 20, info, None, None) == 1
    assert lib.pararnn_solve_gru(fake, 0, fake, None, fake, 2, 8, 4, ctypes.c_float(1e-4), 4,
                                 fake, 1 << 20, None, None, None) == 1
    # negative sizes
    assert lib.pararnn_scan_diag(fake, fake, None, fake, -1, 8, 4, fake, 1 << 20, None, None,
                                 None) == 1
    # misaligned fp32 pointer
    assert lib.pararnn_scan_diag(vp(4098), fake, None, fake, 1, 8, 4, fake, 1 << 20, None, None,
                                 None) == 1
    # 2x2 scan needs 16-byte aligned A
    assert lib.pararnn_scan_block2(vp(4104), fake, None, fake, 1, 8, 4, fake, 1 << 20, None, None,
                                   None) == 1
    # workspace too small / misaligned / missing
    assert lib.pararnn_scan_diag(fake, fake, None, fake, 1, 8, 4, fake, 16, None, None, None) == 6
    assert lib.pararnn_scan_diag(fake, fake, None, fake, 1, 8, 4, vp(4100), 1 << 20, None, None,
                                 None) == 6
    assert lib.pararnn_scan_diag(fake, fake, None, fake, 1, 8, 4, None, 1 << 20, None, None,
                                 None) == 6
    # LSTM needs both outputs
    assert lib.pararnn_solve_lstm(fake, 0, fake, None, None, fake, None, 2, 8, 4,
                                  ctypes.c_float(1e-4), 4, fake, 1 << 20, info, None, None) == 1


def test_input_projection_host_validation(lib):
    vp = ctypes.c_void_p
    fake = vp(4096)  # never dereferenced: validation fails first
    # N and K must be multiples of 8
    assert lib.pararnn_input_projection(fake, fake, None, fake, 0, 16, 12, 64, None, None) == 1
    assert lib.pararnn_input_projection(fake, fake, None, fake, 0, 16, 16, 60, None, None) == 1
    # negative sizes, unknown dtype, misaligned P / x
    assert lib.pararnn_input_projection(fake, fake, None, fake, 0, -1, 16, 64, None, None) == 1
    assert lib.pararnn_input_projection(fake, fake, None, fake, 3, 16, 16, 64, None, None) == 1
    assert lib.pararnn_input_projection(fake, fake, None, vp(4104), 0, 16, 16, 64, None,
                                        None) == 1
    assert lib.pararnn_input_projection(vp(4100), fake, None, fake, 0, 16, 16, 64, None,
                                        None) == 1
    assert lib.pararnn_input_projection(fake, fake, vp(4100), fake, 0, 16, 16, 64, None,
                                        None) == 1
    # M = 0 or N = 0: nothing to do, nothing launched
    assert lib.pararnn_input_projection(fake, fake, None, fake, 0, 0, 16, 64, None, None) == 0
    assert lib.pararnn_input_projection(fake, fake, None, fake, 1, 16, 0, 64, None, None) == 0


def test_other_entry_points_validate_on_the_host(lib):
    """The backward passes, decode steps, rollouts, the multi-head solve and the
    allocation-free solve reject bad arguments before any CUDA call."""
    vp = ctypes.c_void_p
    fake, info, ws = vp(4096), vp(8192), vp(1 << 20)
    f1e4 = ctypes.c_float(1e-4)
    # GRU backward: (P, dtype, a, h0, h, dh, dP, da, dh0, B, L, D, ws, ws_bytes, status, opts, s)
    gb = lib.pararnn_solve_gru_backward
    assert gb(fake, 0, fake, None, fake, fake, fake, fake, None, -1, 8, 4, ws, 1 << 20, None, None,
              None) == 1
    assert gb(fake, 7, fake, None, fake, fake, fake, fake, None, 2, 8, 4, ws, 1 << 20, None, None,
              None) == 1
    assert gb(None, 0, fake, None, fake, fake, fake, fake, None, 2, 8, 4, ws, 1 << 20, None, None,
              None) == 1
    assert gb(fake, 0, fake, None, fake, None, fake, fake, None, 2, 8, 4, ws, 1 << 20, None, None,
              None) == 1                                   # no upstream gradient
    assert gb(fake, 0, vp(4098), None, fake, fake, fake, fake, None, 2, 8, 4, ws, 1 << 20, None,
              None, None) == 1                             # misaligned fp32 weights
    assert gb(vp(4097), 1, fake, None, fake, fake, fake, fake, None, 2, 8, 4, ws, 1 << 20, None,
              None, None) == 1                             # misaligned bf16 P
    # LSTM backward: neither dc nor dh given, or c missing
    lb = lib.pararnn_solve_lstm_backward
    assert lb(fake, 0, fake, None, None, fake, fake, None, None, fake, fake, None, None, 2, 8, 4,
              ws, 1 << 20, None, None, None) == 1
    assert lb(fake, 0, fake, None, None, None, fake, fake, fake, fake, fake, None, None, 2, 8, 4,
              ws, 1 << 20, None, None, None) == 1
    # decode steps and rollouts
    assert lib.pararnn_step_gru(fake, 0, fake, None, fake, -1, 4, None) == 1
    assert lib.pararnn_step_gru(fake, 3, fake, None, fake, 2, 4, None) == 1
    assert lib.pararnn_step_gru(None, 0, fake, None, fake, 2, 4, None) == 1
    assert lib.pararnn_step_gru(fake, 0, fake, None, fake, 0, 4, None) == 0   # nothing to do
    assert lib.pararnn_step_lstm(fake, 0, fake, None, None, fake, None, 2, 4, None) == 1
    assert lib.pararnn_rollout_gru(fake, 0, fake, vp(4098), fake, 2, 8, 4, None) == 1
    assert lib.pararnn_rollout_gru(fake, 0, fake, None, fake, 2, 0, 4, None) == 0
    assert lib.pararnn_rollout_lstm(fake, 0, fake, None, None, fake, None, 2, 8, 4, None) == 1
    # multi-head rollout: (P, dtype, U, h0, h, B, L, H, stream)
    mr = lib.pararnn_rollout_mhgru
    assert mr(fake, 0, fake, None, fake, -1, 8, 2, None) == 1          # negative size
    assert mr(fake, 3, fake, None, fake, 2, 8, 2, None) == 1           # unknown dtype
    assert mr(None, 0, fake, None, fake, 2, 8, 2, None) == 1           # P missing
    assert mr(fake, 0, None, None, fake, 2, 8, 2, None) == 1           # U missing
    assert mr(vp(4098), 0, fake, None, fake, 2, 8, 2, None) == 1       # fp32 P misaligned
    assert mr(fake, 0, fake, vp(4098), fake, 2, 8, 2, None) == 1       # h0 misaligned
    assert mr(fake, 0, fake, None, fake, 2, 0, 2, None) == 0           # nothing to do
    sm = lib.pararnn_step_mhgru  # (P, dtype, U, h_prev, h_next, B, H, stream)
    assert sm(fake, 0, fake, None, fake, -1, 2, None) == 1
    assert sm(fake, 0, None, None, fake, 2, 2, None) == 1
    assert sm(fake, 0, fake, None, fake, 0, 2, None) == 0
    # multi-head solve: (P, dtype, U, h0, h, B, L, H, tol, max_iters, ws, ws_bytes, info, opts, s)
    mh = lib.pararnn_solve_mhgru
    assert mh(fake, 0, fake, None, fake, -1, 8, 2, f1e4, 4, ws, 1 << 20, info, None, None) == 1
    assert mh(fake, 0, fake, None, fake, 2, 8, 2, f1e4, 4, ws, 1 << 20, None, None, None) == 1
    assert mh(fake, 0, fake, None, fake, 2, 8, 2, f1e4, 200, ws, 1 << 20, info, None, None) == 1
    assert mh(fake, 0, fake, None, fake, 2, 8, 2, ctypes.c_float(float("nan")), 4, ws, 1 << 20,
              info, None, None) == 1
    assert mh(fake, 5, fake, None, fake, 2, 8, 2, f1e4, 4, ws, 1 << 20, info, None, None) == 1
    assert mh(None, 0, fake, None, fake, 2, 8, 2, f1e4, 4, ws, 1 << 20, info, None, None) == 1
    assert mh(vp(4100), 0, fake, None, fake, 2, 8, 2, f1e4, 4, ws, 1 << 20, info, None,
              None) == 1                                   # P must be 16-byte aligned
    assert mh(fake, 0, fake, None, fake, 2, 8, 2, f1e4, 4, ws, 16, info, None, None) == 6
    assert mh(fake, 0, fake, None, fake, 2, 8, 2, f1e4, 4, None, 1 << 20, info, None, None) == 6
    # allocation-free solve: negative sizes, and a problem beyond its fixed scratch
    na = lib.pararnn_solve_gru_noalloc
    assert na(fake, 0, fake, None, fake, -1, 8, 4, f1e4, 4, info, None, None) == 1
    import nonlinear_rnn_solve_newton_b200 as pr

    o = ctypes.byref(pr.Options(regime=pr.Options.LOOKBACK, iters_first=8))
    assert lib.pararnn_workspace_size(2, 64, 1 << 16, 1024, 32, o) > pr.NOALLOC_SCRATCH_BYTES
    assert na(fake, 0, fake, None, fake, 64, 1 << 16, 1024, f1e4, 32, info, o, None) == 6


def test_binding_refuses_cpu_tensors():
    import torch

    import nonlinear_rnn_solve_newton_b200 as pr

    A = torch.zeros(1, 4, 2, dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        pr.scan_diag(A, A)
    P = torch.zeros(1, 4, 3, 2, dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        pr.solve_gru(P, torch.zeros(3, 2, dtype=torch.float32))


def test_workspace_size_remembered_per_argument_tuple():
    """The binding remembers sizes per (op, B, L, D, max_iters, options bytes):
    changing an Options object in place must give the size of its new value."""
    import nonlinear_rnn_solve_newton_b200 as pr

    o = pr.Options(regime=1)
    lookback = pr.workspace_size(pr.OP_GRU, 8, 4096, 1024, 32, o)
    assert pr.workspace_size(pr.OP_GRU, 8, 4096, 1024, 32, o) == lookback
    o.regime = 2
    walk = pr.workspace_size(pr.OP_GRU, 8, 4096, 1024, 32, o)
    assert walk == pr.load().pararnn_workspace_size(pr.OP_GRU, 8, 4096, 1024, 32,
                                                     ctypes.byref(pr.Options(regime=2)))
    assert walk != lookback
    with pytest.raises(pr.PararnnError):
        pr.workspace_size(pr.OP_GRU, 8, 4096, 1024, 500, o)


def test_probe_rate_host_validation(lib):
    """The throughput probe refuses a bad pipe, a non-positive length and NULL
    pointers on the host, before any CUDA call."""
    ops = ctypes.c_int64(-1)
    fake = ctypes.c_void_p(0x1000)
    for pipe, iters, sink, out in ((2, 10, fake, ctypes.byref(ops)),
                                   (-1, 10, fake, ctypes.byref(ops)),
                                   (0, 0, fake, ctypes.byref(ops)),
                                   (1, -5, fake, ctypes.byref(ops)),
                                   (0, 10, None, ctypes.byref(ops)),
                                   (0, 10, fake, None)):
        assert lib.pararnn_probe_rate(pipe, iters, sink, out, None) == 1
    assert ops.value == -1
