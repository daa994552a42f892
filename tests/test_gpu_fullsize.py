"""Parity at the full workload sizes, in the launch configuration the benchmark
times: sampled channels are recomputed one by one by the fp64 oracle (the whole
trajectory of each sampled channel, t = 1..L), and every output is checked to be
finite.  The DEER-shaped workload (16 channels) is compared in full."""
import numpy as np
import pytest
import torch

import oracle
from tests import inputs

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

N_SAMPLE = 48


@pytest.fixture(scope="module")
def pr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nonlinear_rnn_solve_newton_b200 as m

    m.load()
    return m


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def sample_channels(B, D, n, seed):
    rng = np.random.default_rng(seed)
    idx = rng.choice(B * D, size=min(n, B * D), replace=False)
    # always include the first and last channel
    idx = np.unique(np.concatenate([idx, [0, B * D - 1]]))
    return [(int(i // D), int(i % D)) for i in idx]


def check_gru(h_dev, x, chans, atol=1e-4):
    worst = 0.0
    cert = 0.0
    for b, d in chans:
        got = h_dev[b, :, d].cpu().numpy()
        P = x["P"][b, :, :, d][None, :, :, None]
        a = x["a"][:, d:d + 1]
        h0 = x["h0"][b:b + 1, d:d + 1]
        ref = oracle.rollout_gru(P, a, h0)[0, :, 0]
        worst = max(worst, float(np.max(np.abs(got - ref))))
        cert = max(cert, oracle.residual_gru(P, a, got[None, :, None], h0))
    assert worst <= atol, worst
    return worst, cert


def test_scan_diag_fullsize(pr):
    w = inputs.WORKLOADS["scan"]
    x = inputs.workload_inputs("scan")
    h = pr.scan_diag(dev(x["A"]), dev(x["b"]), dev(x["h0"]))
    torch.cuda.synchronize()
    assert bool(torch.isfinite(h).all())
    for b, d in sample_channels(w["B"], w["D"], N_SAMPLE, 1):
        ref = oracle.scan_diag(x["A"][b:b + 1, :, d:d + 1], x["b"][b:b + 1, :, d:d + 1],
                               x["h0"][b:b + 1, d:d + 1])[0, :, 0]
        got = h[b, :, d].cpu().numpy()
        assert np.max(np.abs(got - ref) / np.maximum(1, np.abs(ref))) <= 1e-5


def test_scan_block2_fullsize(pr):
    w = inputs.WORKLOADS["block2"]
    x = inputs.workload_inputs("block2")
    out = pr.scan_block2(dev(x["A"]), dev(x["b"]), dev(x["x0"]))
    torch.cuda.synchronize()
    assert bool(torch.isfinite(out).all())
    for b, d in sample_channels(w["B"], w["D"], N_SAMPLE, 2):
        ref = oracle.scan_block2(x["A"][b:b + 1, :, d:d + 1], x["b"][b:b + 1, :, d:d + 1],
                                 x["x0"][b:b + 1, d:d + 1])[0, :, 0]
        got = out[b, :, d].cpu().numpy()
        assert np.max(np.abs(got - ref) / np.maximum(1, np.abs(ref))) <= 1e-5


def test_gru_fullsize_fp32(pr):
    w = inputs.WORKLOADS["gru_l"]
    x = inputs.workload_inputs("gru_l")
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), dev(x["h0"]), tol=1e-4, max_iters=32)
    torch.cuda.synchronize()
    assert info.status == 0 and info.converged
    assert bool(torch.isfinite(h).all())
    _, cert = check_gru(h, x, sample_channels(w["B"], w["D"], N_SAMPLE, 3))
    assert cert <= 1e-4


@pytest.mark.parametrize("L", inputs.L_SWEEP)
def test_gru_length_sweep(pr, L):
    w = inputs.WORKLOADS["gru_l"]
    x = inputs.workload_inputs("gru_l", L=L)
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), dev(x["h0"]))
    torch.cuda.synchronize()
    assert info.converged
    check_gru(h, x, sample_channels(w["B"], w["D"], 16, L))


def test_gru_deer_shape_full(pr):
    x = inputs.workload_inputs("deer")
    h, info = pr.solve_gru(dev(x["P"]), dev(x["a"]), dev(x["h0"]))
    torch.cuda.synchronize()
    assert info.status == 0 and info.converged
    ref = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= 1e-4


def test_gru_lm_width_bf16(pr):
    w = inputs.WORKLOADS["lm"]
    x = inputs.workload_inputs("lm")
    P16 = dev(x["P_bits"].view(np.int16)).view(torch.bfloat16)
    h, info = pr.solve_gru(P16, dev(x["a"]), dev(x["h0"]))
    torch.cuda.synchronize()
    assert info.status == 0 and info.converged
    assert bool(torch.isfinite(h).all())
    _, cert = check_gru(h, x, sample_channels(w["B"], w["D"], 24, 5))
    assert cert <= 1e-4


def test_lstm_fullsize(pr):
    w = inputs.WORKLOADS["lstm"]
    x = inputs.workload_inputs("lstm")
    c, h, info = pr.solve_lstm(dev(x["P"]), dev(x["a"]), dev(x["c0"]), dev(x["h0"]))
    torch.cuda.synchronize()
    assert info.status == 0 and info.converged
    for b, d in sample_channels(w["B"], w["D"], N_SAMPLE, 6):
        P = x["P"][b, :, :, d][None, :, :, None]
        rc, rh = oracle.rollout_lstm(P, x["a"][:, d:d + 1])
        assert np.max(np.abs(c[b, :, d].cpu().numpy() - rc[0, :, 0])) <= 1e-4
        assert np.max(np.abs(h[b, :, d].cpu().numpy() - rh[0, :, 0])) <= 1e-4


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
