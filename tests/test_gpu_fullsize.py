"""Parity at the full workload sizes, in the launch configuration the benchmark
times.  Every channel's whole trajectory (t = 1..L) is compared element by
element with the fp64 oracle -- its sequential rollout for the solves (the
LM-width layer one batch row at a time, so host memory stays bounded), its
sequential scan for the scans -- and the Newton iteration count with the
oracle's serial Newton on the same full workload."""
import numpy as np
import pytest
import torch

import oracle
from tests import inputs

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SOLVE_ATOL = 1e-4     # trajectory vs fp64 rollout (fp32 solves)
SCAN_RTOL = 1e-5      # |x - ref| <= 1e-5 max(1, |ref|) (scans)


@pytest.fixture(scope="module")
def pr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nonlinear_rnn_solve_newton_b200 as m

    m.load()
    return m


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def max_err(got, ref):
    return float(np.max(np.abs(np.asarray(got, np.float64) - ref)))


def check_iterations(info, orc):
    """The GPU's count against the oracle's serial Newton on the same inputs:
    equal up to one (a residual within fp32 rounding of tol may fall on either
    side of it)."""
    assert orc.converged
    assert abs(info.iterations - orc.iterations) <= 1, (info.iterations, orc.iterations)


def test_scan_diag_fullsize(pr):
    x = inputs.workload_inputs("scan")
    h = pr.scan_diag(dev(x["A"]), dev(x["b"]), dev(x["h0"]))
    torch.cuda.synchronize()
    ref = oracle.scan_diag(x["A"], x["b"], x["h0"])
    got = h.cpu().numpy()
    assert np.max(np.abs(got - ref) / np.maximum(1, np.abs(ref))) <= SCAN_RTOL


def test_scan_diag_lm_width(pr):
    """The diagonal scan at the LM width (B=8, L=8192, D=4096), every channel,
    one batch row at a time on the host."""
    w = inputs.WORKLOADS["scan_lm"]
    x = inputs.workload_inputs("scan_lm")
    h = pr.scan_diag(dev(x["A"]), dev(x["b"]), dev(x["h0"]))
    torch.cuda.synchronize()
    for b in range(w["B"]):
        ref = oracle.scan_diag(x["A"][b:b + 1], x["b"][b:b + 1], x["h0"][b:b + 1])[0]
        got = h[b].cpu().numpy()
        assert np.max(np.abs(got - ref) / np.maximum(1, np.abs(ref))) <= SCAN_RTOL, b


def test_scan_block2_fullsize(pr):
    x = inputs.workload_inputs("block2")
    out = pr.scan_block2(dev(x["A"]), dev(x["b"]), dev(x["x0"]))
    torch.cuda.synchronize()
    ref = oracle.scan_block2(x["A"], x["b"], x["x0"])
    got = out.cpu().numpy()
    assert np.max(np.abs(got - ref) / np.maximum(1, np.abs(ref))) <= SCAN_RTOL


def test_gru_fullsize_fp32(pr):
    x = inputs.workload_inputs("gru_l")
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), dev(x["h0"]), tol=1e-4, max_iters=32)
    torch.cuda.synchronize()
    assert info.status == 0 and info.converged
    got = h.cpu().numpy()
    ref = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    assert max_err(got, ref) <= SOLVE_ATOL
    check_iterations(info, oracle.newton_gru(x["P"], x["a"], x["h0"], tol=1e-4, max_iters=32))
    # certificate: the fp64 residual of the GPU trajectory itself
    assert oracle.residual_gru(x["P"], x["a"], got, x["h0"]) <= 1e-4


@pytest.mark.parametrize("L", inputs.L_SWEEP)
def test_gru_length_sweep(pr, L):
    x = inputs.workload_inputs("gru_l", L=L)
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), dev(x["h0"]))
    torch.cuda.synchronize()
    assert info.converged
    ref = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    assert max_err(h.cpu().numpy(), ref) <= SOLVE_ATOL
    check_iterations(info, oracle.newton_gru(x["P"], x["a"], x["h0"], tol=1e-4, max_iters=32))


def test_gru_deer_shape_full(pr):
    x = inputs.workload_inputs("deer")
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), dev(x["h0"]))
    torch.cuda.synchronize()
    assert info.status == 0 and info.converged
    ref = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    assert max_err(h.cpu().numpy(), ref) <= SOLVE_ATOL
    check_iterations(info, oracle.newton_gru(x["P"], x["a"], x["h0"], tol=1e-4, max_iters=32))


def test_gru_lm_width_bf16(pr):
    """Every channel of the LM-width layer (bf16 gates), one batch row at a time.
    The global iteration count is the largest of the rows' counts: each row's
    serial Newton stops at its own first residual <= tol, and the residuals stay
    below tol once there."""
    w = inputs.WORKLOADS["lm"]
    x = inputs.workload_inputs("lm")
    P16 = dev(x["P_bits"].view(np.int16)).view(torch.bfloat16)
    h, info = pr.solve_gru(P16, dev(x["a"]), dev(x["h0"]))
    torch.cuda.synchronize()
    assert info.status == 0 and info.converged
    row_iters = []
    cert = 0.0
    for b in range(w["B"]):
        Pb, h0b = x["P"][b:b + 1], x["h0"][b:b + 1]
        got = h[b:b + 1].cpu().numpy()
        ref = oracle.rollout_gru(Pb, x["a"], h0b)
        assert max_err(got, ref) <= SOLVE_ATOL, b
        cert = max(cert, oracle.residual_gru(Pb, x["a"], got, h0b))
        orc = oracle.newton_gru(Pb, x["a"], h0b, tol=1e-4, max_iters=32)
        assert orc.converged
        row_iters.append(orc.iterations)
    assert abs(info.iterations - max(row_iters)) <= 1, (info.iterations, row_iters)
    assert cert <= 1e-4


def test_lstm_fullsize(pr):
    x = inputs.workload_inputs("lstm")
    c, h, info = pr.solve_lstm(dev(x["P"]), dev(x["a"]), dev(x["c0"]), dev(x["h0"]))
    torch.cuda.synchronize()
    assert info.status == 0 and info.converged
    rc, rh = oracle.rollout_lstm(x["P"], x["a"], x["c0"], x["h0"])
    assert max_err(c.cpu().numpy(), rc) <= SOLVE_ATOL
    assert max_err(h.cpu().numpy(), rh) <= SOLVE_ATOL
    check_iterations(info, oracle.newton_lstm(x["P"], x["a"], x["c0"], x["h0"], tol=1e-4,
                                              max_iters=32))


def sample_channels(B, D, n, seed):
    rng = np.random.default_rng(seed)
    idx = rng.choice(B * D, size=min(n, B * D), replace=False)
    # always include the first and last channel
    idx = np.unique(np.concatenate([idx, [0, B * D - 1]]))
    return [(int(i // D), int(i % D)) for i in idx]


def test_gru_backward_fullsize(pr):
    """Backward pass at the B=8, L=4096, D=1024 shape: the GPU differentiates its own
    forward solution; sampled channels are compared with the oracle's adjoint on the
    same (fp32) trajectory and gradients."""
    w = inputs.WORKLOADS["gru_bwd"]
    B, L, D = w["B"], w["L"], w["D"]
    x = inputs.gru_inputs(B, L, D, w["seed"])
    (gh,) = inputs.upstream_gradients(B, L, D, w["seed"], 1)
    P, a = dev(x["P"]), dev(x["a"])
    h, info = pr.solve_gru(P, a)
    dP, da, dh0 = pr.solve_gru_backward(P, a, h, dev(gh))
    torch.cuda.synchronize()
    assert info.converged and bool(torch.isfinite(dP).all())
    hh = h.cpu().numpy()
    for b, d in sample_channels(B, D, 32, 7):
        Pc = x["P"][b, :, :, d][None, :, :, None]
        rP, ra, rh0 = oracle.backward_gru(Pc, x["a"][:, d:d + 1], hh[b, :, d][None, :, None],
                                          gh[b, :, d][None, :, None])
        got = dP[b, :, :, d].cpu().numpy()
        assert np.max(np.abs(got - rP[0, :, :, 0]) / np.maximum(1, np.abs(rP[0, :, :, 0]))) <= 1e-4
        assert abs(float(dh0[b, d]) - rh0[0, 0]) <= 1e-4 * max(1.0, abs(rh0[0, 0]))
