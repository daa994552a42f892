"""The allocation-free ParaGRU entry point, pararnn_solve_gru_noalloc.

It exists for callers that cannot allocate device memory where they solve
(memory fully reserved by another allocator, a plug-in interface with no
workspace, a loop where an allocation is not allowed).  It must give the same
trajectory as pararnn_solve_gru, call after call, although every call reuses
the library's one scratch array.  This file is collected last so that a run
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


def call_noalloc(pr, P, a, h0, out, info, tol=1e-4, max_iters=32, opts=None):
    """Straight through the C ABI (ctypes), with caller-owned output and info."""
    lib = pr.load()
    B, L, _, D = P.shape
    st = lib.pararnn_solve_gru_noalloc(
        ctypes.c_void_p(P.data_ptr()), 0, ctypes.c_void_p(a.data_ptr()),
        ctypes.c_void_p(h0.data_ptr()), ctypes.c_void_p(out.data_ptr()), B, L, D,
        ctypes.c_float(tol), max_iters, ctypes.c_void_p(info.data_ptr()),
        ctypes.byref(opts) if opts is not None else None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


@pytest.mark.parametrize("shape,regime", [((8, 1024, 1024), 0),   # walk regime
                                          ((2, 3000, 16), 0),     # look-back regime
                                          ((3, 700, 64), 1)])     # look-back, forced
def test_noalloc_matches_workspace_entry_point_twice(pr, shape, regime):
    B, L, D = shape
    x = inputs.gru_inputs(B, L, D, seed=[900, B, L, D], h0_normal=True)
    P, a, h0 = dev(x["P"]), dev(x["a"]), dev(x["h0"])
    opts = pr.Options(regime=regime)
    ref, ref_info = pr.solve_gru(P, a, h0, opts=opts)
    torch.cuda.synchronize()
    assert ref_info.status == 0 and ref_info.converged
    for _ in range(2):
        out = torch.full((B, L, D), float("nan"), device="cuda")
        info = torch.zeros(pr.INFO_BYTES // 4, dtype=torch.int32, device="cuda")
        assert call_noalloc(pr, P, a, h0, out, info, opts=opts) == 0
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
