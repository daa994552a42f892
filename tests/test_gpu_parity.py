"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tolerances (written here, derived from the arithmetic):
* scans: |x - ref| <= 1e-5 * max(1, |ref|) elementwise (fp32 affine scan with
  contractive maps; rounding of a few ulp per combine does not accumulate).
* Newton solves: max-abs <= 1e-4 on the whole trajectory against the fp64
  sequential rollout of the same (bf16-rounded where applicable) inputs --
  the DEER summary's float32 tolerance.
* iteration counts: equal to the oracle's serial Newton up to +-1 (a residual
  that lands within fp32 rounding of tol may fall on either side).
"""
import numpy as np
import pytest
import torch

import oracle
from tests import inputs

pytestmark = pytest.mark.gpu

SCAN_RTOL = 1e-5
SOLVE_ATOL = 1e-4


@pytest.fixture(scope="module")
def pr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nonlinear_rnn_solve_newton_b200 as m

    m.load()
    return m


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def scan_err(got, ref):
    return np.max(np.abs(got - ref) / np.maximum(1.0, np.abs(ref)))


SCAN_SHAPES = [(1, 1, 1), (2, 3, 5), (3, 31, 3), (2, 33, 16), (1, 2049, 1), (2, 1000, 7),
               (2, 4096 + 17, 64), (1, 300, 33), (4, 129, 1024)]


@pytest.mark.parametrize("shape", SCAN_SHAPES)
def test_scan_diag_parity(pr, shape):
    B, L, D = shape
    x = inputs.scan_diag_inputs(B, L, D, seed=[100, B, L, D])
    h = pr.scan_diag(dev(x["A"]), dev(x["b"]), dev(x["h0"]))
    torch.cuda.synchronize()
    ref = oracle.scan_diag(x["A"], x["b"], x["h0"])
    assert scan_err(h.cpu().numpy(), ref) <= SCAN_RTOL


def test_scan_diag_no_h0_and_long_sequence(pr):
    x = inputs.scan_diag_inputs(2, 40000, 3, seed=101)
    h = pr.scan_diag(dev(x["A"]), dev(x["b"]))
    torch.cuda.synchronize()
    ref = oracle.scan_diag(x["A"], x["b"])
    assert scan_err(h.cpu().numpy(), ref) <= SCAN_RTOL


@pytest.mark.parametrize("shape", SCAN_SHAPES)
def test_scan_block2_parity(pr, shape):
    B, L, D = shape
    x = inputs.scan_block2_inputs(B, L, D, seed=[102, B, L, D])
    out = pr.scan_block2(dev(x["A"]), dev(x["b"]), dev(x["x0"]))
    torch.cuda.synchronize()
    ref = oracle.scan_block2(x["A"], x["b"], x["x0"])
    assert scan_err(out.cpu().numpy(), ref) <= SCAN_RTOL


def test_scan_output_canaries(pr):
    """Nothing is written outside the output."""
    B, L, D = 2, 777, 48
    x = inputs.scan_diag_inputs(B, L, D, seed=103)
    n = B * L * D
    buf = torch.full((n + 2048,), 12345.0, device="cuda")
    out = buf[1024:1024 + n].view(B, L, D)
    pr.scan_diag(dev(x["A"]), dev(x["b"]), dev(x["h0"]), out=out)
    torch.cuda.synchronize()
    b = buf.cpu().numpy()
    assert np.all(b[:1024] == 12345.0) and np.all(b[1024 + n:] == 12345.0)


# --------------------------------------------------------------------------
# Newton solves
# --------------------------------------------------------------------------
GRU_SHAPES = [(2, 512, 16), (1, 1, 1), (2, 3, 5), (3, 31, 3), (1, 2049, 1), (2, 1000, 7),
              (2, 1100, 64), (1, 300, 33), (4, 257, 128)]


@pytest.mark.parametrize("shape", GRU_SHAPES)
def test_gru_solve_parity(pr, shape):
    B, L, D = shape
    x = inputs.gru_inputs(B, L, D, seed=[200, B, L, D])
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), dev(x["h0"]), tol=1e-4, max_iters=32)
    torch.cuda.synchronize()
    ref = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    assert info.status == 0 and info.converged
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= SOLVE_ATOL
    orc = oracle.newton_gru(x["P"], x["a"], x["h0"], tol=1e-4, max_iters=32)
    assert abs(info.iterations - orc.iterations) <= 1, (info.iterations, orc.iterations)
    assert info.max_residual <= 1e-4


def test_gru_solve_nonzero_h0_and_bf16(pr):
    B, L, D = 3, 700, 40
    x = inputs.gru_inputs(B, L, D, seed=201, bf16=True, h0_normal=True)
    P16 = dev(x["P_bits"].view(np.int16)).view(torch.bfloat16)
    h, info = pr.solve_gru(P16, dev(x["a"]), dev(x["h0"]))
    torch.cuda.synchronize()
    ref = oracle.rollout_gru(x["P"], x["a"], x["h0"])   # same bf16-rounded values, in fp64
    assert info.converged
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= SOLVE_ATOL


def test_gru_unconverged_matches_oracle_iterate(pr):
    """tol = 0, max_iters = 2: both sides return h^2 and report no convergence."""
    B, L, D = 2, 300, 8
    x = inputs.gru_inputs(B, L, D, seed=202)
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), tol=0.0, max_iters=2)
    torch.cuda.synchronize()
    orc = oracle.newton_gru(x["P"], x["a"], tol=0.0, max_iters=2)
    assert not info.converged and info.iterations == 2 and info.updates == 2
    assert np.max(np.abs(h.cpu().numpy() - orc.h)) <= 1e-5
    np.testing.assert_allclose(info.rho[:3], orc.rho, rtol=1e-4, atol=1e-6)


def test_gru_max_iters_zero_returns_initial_guess(pr):
    x = inputs.gru_inputs(2, 50, 4, seed=203)
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), tol=1e-4, max_iters=0)
    torch.cuda.synchronize()
    assert info.iterations == 0 and not info.converged and info.updates == 0
    assert np.all(h.cpu().numpy() == 0.0)
    orc = oracle.newton_gru(x["P"], x["a"], tol=1e-4, max_iters=0)
    assert abs(info.rho[0] - orc.rho[0]) <= 1e-5


def test_gru_mingru_one_iteration(pr):
    """a = 0: the cell is affine in h, Newton needs one update and equals a single scan."""
    B, L, D = 2, 900, 32
    x = inputs.gru_inputs(B, L, D, seed=204, h0_normal=True)
    a0 = np.zeros_like(x["a"])
    h, info = pr.solve_gru(dev(x["P"]), dev(a0), dev(x["h0"]), tol=1e-5)
    torch.cuda.synchronize()
    assert info.converged and info.iterations == 1
    ref = oracle.rollout_gru(x["P"], a0, x["h0"])
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= 1e-5


def test_gru_iterations_per_sweep_do_not_change_result(pr):
    B, L, D = 2, 2000, 32
    x = inputs.gru_inputs(B, L, D, seed=205)
    ref = oracle.rollout_gru(x["P"], x["a"])
    counts = set()
    for first, nxt in ((1, 1), (2, 1), (4, 2), (8, 8)):
        o = pr.Options(iters_first=first, iters_next=nxt)
        h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), opts=o)
        torch.cuda.synchronize()
        assert info.converged
        assert np.max(np.abs(h.cpu().numpy() - ref)) <= SOLVE_ATOL
        counts.add(info.iterations)
    assert len(counts) == 1   # the stop decision is the same global rule


def test_gru_nonfinite_reported(pr):
    x = inputs.gru_inputs(1, 200, 8, seed=206)
    P = x["P"].copy()
    P[0, 77, 1, 3] = np.nan
    h, info = pr.solve_gru(dev(P), dev(x["a"]))
    torch.cuda.synchronize()
    assert info.status == 5 and not info.converged


def test_gru_empty_inputs(pr):
    P = torch.zeros((2, 0, 3, 4), device="cuda")
    h, info = pr.solve_gru(P, torch.zeros((3, 4), device="cuda"))
    torch.cuda.synchronize()
    assert h.shape == (2, 0, 4) and info.converged and info.iterations == 0


LSTM_SHAPES = [(2, 512, 16), (1, 1, 1), (2, 5, 3), (1, 1025, 1), (2, 600, 33), (2, 700, 128)]


@pytest.mark.parametrize("shape", LSTM_SHAPES)
def test_lstm_solve_parity(pr, shape):
    B, L, D = shape
    x = inputs.lstm_inputs(B, L, D, seed=[300, B, L, D])
    c, h, info = pr.solve_lstm(dev(x["P"]), dev(x["a"]), dev(x["c0"]), dev(x["h0"]))
    torch.cuda.synchronize()
    rc, rh = oracle.rollout_lstm(x["P"], x["a"], x["c0"], x["h0"])
    assert info.status == 0 and info.converged
    assert np.max(np.abs(c.cpu().numpy() - rc)) <= SOLVE_ATOL
    assert np.max(np.abs(h.cpu().numpy() - rh)) <= SOLVE_ATOL
    orc = oracle.newton_lstm(x["P"], x["a"], x["c0"], x["h0"], tol=1e-4, max_iters=32)
    assert abs(info.iterations - orc.iterations) <= 1


def test_lstm_no_recurrence_two_iterations(pr):
    x = inputs.lstm_inputs(2, 500, 24, seed=301, h0_normal=True)
    a0 = np.zeros_like(x["a"])
    c, h, info = pr.solve_lstm(dev(x["P"]), dev(a0), dev(x["c0"]), dev(x["h0"]), tol=1e-5)
    torch.cuda.synchronize()
    assert info.converged and info.iterations == 2


def test_lstm_bf16(pr):
    B, L, D = 2, 400, 64
    x = inputs.lstm_inputs(B, L, D, seed=302, bf16=True)
    P16 = dev(x["P_bits"].view(np.int16)).view(torch.bfloat16)
    c, h, info = pr.solve_lstm(P16, dev(x["a"]))
    torch.cuda.synchronize()
    rc, rh = oracle.rollout_lstm(x["P"], x["a"])
    assert info.converged
    assert np.max(np.abs(h.cpu().numpy() - rh)) <= SOLVE_ATOL
    assert np.max(np.abs(c.cpu().numpy() - rc)) <= SOLVE_ATOL


# --------------------------------------------------------------------------
# Failure detection: a bounded wait that runs out
# --------------------------------------------------------------------------
def test_stalled_unit_times_out_and_context_survives(pr):
    """A unit that never publishes (test hook) makes its successors' bounded waits
    expire: the kernel returns DEVICE_TIMEOUT and the context stays usable."""
    B, L, D = 1, 4096, 32
    x = inputs.gru_inputs(B, L, D, seed=400)
    o = pr.Options(wait_timeout_ns=20_000_000, debug_stall_unit=1)
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), opts=o)
    torch.cuda.synchronize()
    assert info.status == 4 and not info.converged
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    xs = inputs.scan_diag_inputs(1, 4096, 32, seed=401)
    pr.scan_diag(dev(xs["A"]), dev(xs["b"]), status=st, opts=o)
    torch.cuda.synchronize()
    assert int(st.item()) == 4
    # the next normal call is unaffected
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]))
    torch.cuda.synchronize()
    assert info.status == 0 and info.converged
    ref = oracle.rollout_gru(x["P"], x["a"])
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= SOLVE_ATOL


# --------------------------------------------------------------------------
# Both ways of chaining time chunks (look-back across CTAs, or one CTA walking
# a tile) must give the oracle's result.
# --------------------------------------------------------------------------
REGIME_SHAPES = [(2, 700, 64), (1, 2049, 1), (3, 300, 33), (2, 1500, 96)]


@pytest.mark.parametrize("regime", [1, 2])
@pytest.mark.parametrize("shape", REGIME_SHAPES)
def test_regimes_gru(pr, regime, shape):
    B, L, D = shape
    x = inputs.gru_inputs(B, L, D, seed=[500, B, L, D], h0_normal=True)
    o = pr.Options(regime=regime)
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), dev(x["h0"]), opts=o)
    torch.cuda.synchronize()
    ref = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    assert info.converged
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= SOLVE_ATOL
    orc = oracle.newton_gru(x["P"], x["a"], x["h0"], tol=1e-4, max_iters=32)
    assert abs(info.iterations - orc.iterations) <= 1


@pytest.mark.parametrize("regime", [1, 2])
@pytest.mark.parametrize("shape", REGIME_SHAPES)
def test_regimes_lstm(pr, regime, shape):
    B, L, D = shape
    x = inputs.lstm_inputs(B, L, D, seed=[501, B, L, D])
    o = pr.Options(regime=regime)
    c, h, info = pr.solve_lstm(dev(x["P"]), dev(x["a"]), opts=o)
    torch.cuda.synchronize()
    rc, rh = oracle.rollout_lstm(x["P"], x["a"])
    assert info.converged
    assert np.max(np.abs(h.cpu().numpy() - rh)) <= SOLVE_ATOL
    assert np.max(np.abs(c.cpu().numpy() - rc)) <= SOLVE_ATOL


@pytest.mark.parametrize("regime", [1, 2])
@pytest.mark.parametrize("shape", REGIME_SHAPES)
def test_regimes_scans(pr, regime, shape):
    B, L, D = shape
    o = pr.Options(regime=regime)
    x = inputs.scan_diag_inputs(B, L, D, seed=[502, B, L, D])
    h = pr.scan_diag(dev(x["A"]), dev(x["b"]), dev(x["h0"]), opts=o)
    y = inputs.scan_block2_inputs(B, L, D, seed=[503, B, L, D])
    xo = pr.scan_block2(dev(y["A"]), dev(y["b"]), dev(y["x0"]), opts=o)
    torch.cuda.synchronize()
    assert scan_err(h.cpu().numpy(), oracle.scan_diag(x["A"], x["b"], x["h0"])) <= SCAN_RTOL
    assert scan_err(xo.cpu().numpy(), oracle.scan_block2(y["A"], y["b"], y["x0"])) <= SCAN_RTOL


def test_walk_regime_unconverged_iterate(pr):
    """Walk regime, tol = 0, max_iters = 3: h^3 of the oracle's serial Newton."""
    B, L, D = 2, 900, 64
    x = inputs.gru_inputs(B, L, D, seed=504)
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), tol=0.0, max_iters=3,
                           opts=pr.Options(regime=2, iters_first=2, iters_next=1))
    torch.cuda.synchronize()
    orc = oracle.newton_gru(x["P"], x["a"], tol=0.0, max_iters=3)
    assert not info.converged and info.iterations == 3 and info.updates == 3
    assert np.max(np.abs(h.cpu().numpy() - orc.h)) <= 1e-5


# --------------------------------------------------------------------------
# The tensor-copy walker on 8- and 32-channel tiles (a warp = 8 channels x 4
# time segments, or 32 channels x 1): same results.  Shapes with D a multiple
# of 8 that is not of 32, a ragged last tile (D = 36), L not a multiple of the
# chunk, and bf16 gates.
# --------------------------------------------------------------------------
WIDTH_SHAPES = [(2, 1500, 64), (3, 700, 40), (1, 2100, 36), (2, 513, 96)]


@pytest.mark.parametrize("width", [8, 32])
@pytest.mark.parametrize("shape", WIDTH_SHAPES)
def test_walk_widths_gru(pr, shape, width):
    B, L, D = shape
    if width == 32 and D < 32:
        pytest.skip("32-channel tiles need D >= 32")
    x = inputs.gru_inputs(B, L, D, seed=[510, B, L, D], h0_normal=True)
    o = pr.Options(regime=2, walk_width=width)
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), dev(x["h0"]), opts=o)
    torch.cuda.synchronize()
    ref = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    assert info.converged
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= SOLVE_ATOL
    orc = oracle.newton_gru(x["P"], x["a"], x["h0"], tol=1e-4, max_iters=32)
    assert abs(info.iterations - orc.iterations) <= 1


@pytest.mark.parametrize("width", [8, 32])
@pytest.mark.parametrize("shape", WIDTH_SHAPES)
def test_walk_widths_lstm_bf16(pr, shape, width):
    B, L, D = shape
    if width == 32 and D < 32:
        pytest.skip("32-channel tiles need D >= 32")
    x = inputs.lstm_inputs(B, L, D, seed=[511, B, L, D], bf16=True)
    P16 = torch.from_numpy(x["P_bits"].view(np.int16)).cuda().view(torch.bfloat16)
    o = pr.Options(regime=2, walk_width=width)
    c, h, info = pr.solve_lstm(P16, dev(x["a"]), opts=o)
    torch.cuda.synchronize()
    rc, rh = oracle.rollout_lstm(x["P"], x["a"])
    assert info.converged
    assert np.max(np.abs(h.cpu().numpy() - rh)) <= SOLVE_ATOL
    assert np.max(np.abs(c.cpu().numpy() - rc)) <= SOLVE_ATOL


def test_walk_width_unconverged_iterate(pr):
    """8-channel walker, several sweeps (2 then 1 iterations), tol = 0: h^3 exactly."""
    B, L, D = 2, 1100, 48
    x = inputs.gru_inputs(B, L, D, seed=512, h0_normal=True)
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), dev(x["h0"]), tol=0.0, max_iters=3,
                           opts=pr.Options(regime=2, iters_first=2, iters_next=1,
                                           walk_width=8))
    torch.cuda.synchronize()
    orc = oracle.newton_gru(x["P"], x["a"], x["h0"], tol=0.0, max_iters=3)
    assert not info.converged and info.iterations == 3 and info.updates == 3
    assert np.max(np.abs(h.cpu().numpy() - orc.h)) <= 1e-5


def test_concurrent_solves_on_two_streams(pr):
    """Solves issued on two streams at once each get their own cached workspace:
    both results match the oracle."""
    B, L, D = 4, 2000, 64
    xs = [inputs.gru_inputs(B, L, D, seed=[520, i]) for i in range(2)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    Ps = [dev(x["P"]) for x in xs]
    As = [dev(x["a"]) for x in xs]
    torch.cuda.synchronize()
    outs = []
    for i in range(2):
        with torch.cuda.stream(streams[i]):
            outs.append(pr.solve_gru(Ps[i], As[i], stream=streams[i]))
    torch.cuda.synchronize()
    for (h, info), x in zip(outs, xs):
        assert info.converged
        assert np.max(np.abs(h.cpu().numpy() - oracle.rollout_gru(x["P"], x["a"]))) <= SOLVE_ATOL


def test_solve_replays_from_a_cuda_graph(pr):
    """A solve (workspace zeroing + cooperative launch) can be captured into a
    CUDA graph and replayed: the replays give the direct call's result, also
    after the inputs are overwritten in place."""
    B, L, D = 2, 512, 16
    x1 = inputs.gru_inputs(B, L, D, seed=530)
    x2 = inputs.gru_inputs(B, L, D, seed=531)
    P, a = dev(x1["P"]), dev(x1["a"])
    h = torch.empty((B, L, D), device="cuda")
    info_t = torch.empty(pr.INFO_BYTES // 4, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(2):                   # warm-up outside the capture
            pr.solve_gru(P, a, out=h, info=info_t, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        pr.solve_gru(P, a, out=h, info=info_t, stream=s)
    for x in (x1, x2):
        P.copy_(dev(x["P"]))
        a.copy_(dev(x["a"]))
        g.replay()
        torch.cuda.synchronize()
        ref = oracle.rollout_gru(x["P"], x["a"])
        assert np.max(np.abs(h.cpu().numpy() - ref)) <= SOLVE_ATOL
        assert pr.SolveInfo(info_t).converged


# --------------------------------------------------------------------------
# The GRU walker on 32-channel tiles: bf16 and fp32 gates, an unconverged
# iterate, agreement between 8- and 16-warp CTAs (different chunk splits, the
# same answer to rounding), and an odd D.
# --------------------------------------------------------------------------
WALK32_SHAPES = [(4, 1000, 128), (2, 333, 64), (1, 2100, 36)]


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("shape", WALK32_SHAPES)
def test_walk32_gru(pr, shape, bf16):
    B, L, D = shape
    x = inputs.gru_inputs(B, L, D, seed=[520, B, L, D], bf16=bf16, h0_normal=True)
    P = (torch.from_numpy(x["P_bits"].view(np.int16)).cuda().view(torch.bfloat16) if bf16
         else dev(x["P"]))
    o = pr.Options(regime=2, walk_width=32)
    h, info = pr.solve_gru(P, dev(x["a"]), dev(x["h0"]), opts=o)
    h1, info1 = pr.solve_gru(P, dev(x["a"]), dev(x["h0"]),
                             opts=pr.Options(regime=2, walk_width=32, walk_warps=16))
    torch.cuda.synchronize()
    ref = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    assert info.status == 0 and info.converged
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= SOLVE_ATOL
    orc = oracle.newton_gru(x["P"], x["a"], x["h0"], tol=1e-4, max_iters=32)
    assert abs(info.iterations - orc.iterations) <= 1
    assert info1.converged and info1.iterations == info.iterations
    assert float(torch.max(torch.abs(h - h1)).item()) <= 1e-5


def test_walk32_unconverged_iterate(pr):
    """tol = 0, max_iters = 3, two iterations per sweep: h^3 of the serial Newton."""
    B, L, D = 2, 900, 64
    x = inputs.gru_inputs(B, L, D, seed=521, h0_normal=True)
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), dev(x["h0"]), tol=0.0, max_iters=3,
                           opts=pr.Options(regime=2, walk_width=32, iters_first=2,
                                           iters_next=1))
    torch.cuda.synchronize()
    orc = oracle.newton_gru(x["P"], x["a"], x["h0"], tol=0.0, max_iters=3)
    assert not info.converged and info.iterations == 3 and info.updates == 3
    assert np.max(np.abs(h.cpu().numpy() - orc.h)) <= 1e-5
    np.testing.assert_allclose(info.rho[:4], orc.rho, rtol=1e-4, atol=1e-6)


def test_walk32_odd_width(pr):
    B, L, D = 2, 777, 33
    x = inputs.gru_inputs(B, L, D, seed=522, h0_normal=True)
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), dev(x["h0"]),
                           opts=pr.Options(regime=2, walk_width=32))
    torch.cuda.synchronize()
    assert info.converged
    ref = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= SOLVE_ATOL
