"""The allocation-free ParaGRU entry point, pararnn_solve_gru_noalloc.

It exists for callers that cannot allocate device memory where they solve
(memory fully reserved by another allocator, a plug-in interface with no
workspace, a loop where an allocation is not allowed).  It must give the same
trajectory as pararnn_solve_gru -- and, like it, the oracle's -- call after
call, although every call reuses the library's one scratch array: including
calls that follow one which left that array dirty (an unconverged solve, or
one whose bounded waits ran out).  This file is collected last so that a run
stopping at the first failure has already run every other test; it also
passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests import inputs

pytestmark = pytest.mark.gpu

SOLVE_ATOL = 1e-4   # the tolerance of the solve parity tests


@pytest.fixture(scope="module")
def pr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nonlinear_rnn_solve_newton_b200 as m

    m.load()
    return m


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def gates(pr, x, bf16):
    """P on the device: the bf16 bits when bf16, else the fp32 values."""
    if bf16:
        return torch.from_numpy(x["P_bits"].view(np.int16)).cuda().view(torch.bfloat16)
    return dev(x["P"])


def call_noalloc(pr, P, a, h0, out, info, tol=1e-4, max_iters=32, opts=None):
    """Straight through the C ABI (ctypes), with caller-owned output and info."""
    lib = pr.load()
    B, L, _, D = P.shape
    dt = 1 if P.dtype == torch.bfloat16 else 0
    st = lib.pararnn_solve_gru_noalloc(
        ctypes.c_void_p(P.data_ptr()), dt, ctypes.c_void_p(a.data_ptr()),
        ctypes.c_void_p(h0.data_ptr()), ctypes.c_void_p(out.data_ptr()), B, L, D,
        ctypes.c_float(tol), max_iters, ctypes.c_void_p(info.data_ptr()),
        ctypes.byref(opts) if opts is not None else None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def fresh(pr, B, L, D):
    out = torch.full((B, L, D), float("nan"), device="cuda")
    info = torch.zeros(pr.INFO_BYTES // 4, dtype=torch.int32, device="cuda")
    return out, info


@pytest.mark.parametrize("shape,regime,bf16", [((8, 1024, 1024), 0, False),   # walk regime
                                               ((2, 3000, 16), 0, False),     # look-back regime
                                               ((3, 700, 64), 1, False),      # look-back, forced
                                               ((4, 2048, 256), 0, True)])    # bf16 gates
def test_noalloc_matches_workspace_entry_point_and_oracle_twice(pr, oracle, shape, regime, bf16):
    B, L, D = shape
    x = inputs.gru_inputs(B, L, D, seed=[900, B, L, D], bf16=bf16, h0_normal=True)
    P, a, h0 = gates(pr, x, bf16), dev(x["a"]), dev(x["h0"])
    opts = pr.Options(regime=regime)
    ref, ref_info = pr.solve_gru(P, a, h0, opts=opts)
    torch.cuda.synchronize()
    assert ref_info.status == 0 and ref_info.converged
    # the oracle: fp64 sequential rollout on the same (bf16-rounded) values,
    # and its serial Newton's iteration count
    roll = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    orc = oracle.newton_gru(x["P"], x["a"], x["h0"], tol=1e-4, max_iters=32)
    for _ in range(2):
        out, info = fresh(pr, B, L, D)
        assert call_noalloc(pr, P, a, h0, out, info, opts=opts) == 0
        torch.cuda.synchronize()
        got = pr.SolveInfo(info)
        assert got.status == 0 and got.converged
        assert got.iterations == ref_info.iterations
        assert abs(got.iterations - orc.iterations) <= 1
        assert float(torch.max(torch.abs(out - ref)).item()) <= SOLVE_ATOL
        assert np.max(np.abs(out.cpu().numpy() - roll)) <= SOLVE_ATOL


@pytest.mark.parametrize("dirty", ["unconverged", "timed_out"])
def test_noalloc_call_after_a_call_that_left_the_scratch_dirty(pr, dirty):
    """The scratch keeps whatever the previous call left: look-back records of an
    unconverged solve, or of one whose waits ran out part-way.  The next call
    clears what must start at zero, so it still matches pararnn_solve_gru."""
    B, L, D = 2, 4096, 32
    lb = pr.Options(regime=pr.Options.LOOKBACK)
    x = inputs.gru_inputs(B, L, D, seed=[901, B, L, D], h0_normal=True)
    P, a, h0 = dev(x["P"]), dev(x["a"]), dev(x["h0"])
    ref, ref_info = pr.solve_gru(P, a, h0, opts=lb)
    torch.cuda.synchronize()
    assert ref_info.converged

    out, info = fresh(pr, B, L, D)
    if dirty == "unconverged":
        assert call_noalloc(pr, P, a, h0, out, info, max_iters=1, opts=lb) == 0
        torch.cuda.synchronize()
        first = pr.SolveInfo(info)
        assert first.status == 0 and not first.converged and first.iterations == 1
    else:
        stall = pr.Options(regime=pr.Options.LOOKBACK, wait_timeout_ns=20_000_000,
                           debug_stall_unit=1)
        assert call_noalloc(pr, P, a, h0, out, info, opts=stall) == 0
        torch.cuda.synchronize()
        first = pr.SolveInfo(info)
        assert first.status == 4 and not first.converged

    for _ in range(2):
        out, info = fresh(pr, B, L, D)
        assert call_noalloc(pr, P, a, h0, out, info, opts=lb) == 0
        torch.cuda.synchronize()
        got = pr.SolveInfo(info)
        assert got.status == 0 and got.converged
        assert got.iterations == ref_info.iterations
        assert float(torch.max(torch.abs(out - ref)).item()) <= SOLVE_ATOL


def test_noalloc_rejects_problems_beyond_the_scratch(pr):
    # look-back regime over many chunks needs more than the fixed scratch
    o = pr.Options(regime=pr.Options.LOOKBACK, iters_first=8)
    need = pr.workspace_size(pr.OP_GRU, 64, 1 << 16, 1024, 32, o)
    assert need > pr.NOALLOC_SCRATCH_BYTES
    fake = torch.empty(4, device="cuda")
    info = torch.zeros(pr.INFO_BYTES // 4, dtype=torch.int32, device="cuda")
    lib = pr.load()
    st = lib.pararnn_solve_gru_noalloc(
        ctypes.c_void_p(fake.data_ptr()), 0, ctypes.c_void_p(fake.data_ptr()), None,
        ctypes.c_void_p(fake.data_ptr()), 64, 1 << 16, 1024, ctypes.c_float(1e-4), 32,
        ctypes.c_void_p(info.data_ptr()), ctypes.byref(o), None)
    assert st == 6   # PARARNN_ERR_WORKSPACE, nothing enqueued
