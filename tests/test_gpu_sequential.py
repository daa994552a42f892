"""The sequential application on the GPU (one decode step; the one-thread-per-
channel rollout) against the fp64 oracle's cell and rollout."""
import numpy as np
import pytest
import torch

import oracle
from tests import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nonlinear_rnn_solve_newton_b200 as m

    m.load()
    return m


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


@pytest.mark.parametrize("shape", [(1, 1), (3, 5), (4, 1000), (8, 4096)])
def test_step_gru_matches_cell(pr, shape):
    B, D = shape
    x = inputs.gru_inputs(B, 1, D, seed=[700, B, D], h0_normal=True)
    P = x["P"][:, 0]                                   # [B, 3, D]
    h = pr.step_gru(dev(P), dev(x["a"]), dev(x["h0"]))
    torch.cuda.synchronize()
    ref = oracle.rollout_gru(x["P"], x["a"], x["h0"])[:, 0]
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= 2e-6


@pytest.mark.parametrize("shape", [(1, 1), (3, 5), (4, 1000)])
def test_step_lstm_matches_cell(pr, shape):
    B, D = shape
    x = inputs.lstm_inputs(B, 1, D, seed=[701, B, D], h0_normal=True)
    c, h = pr.step_lstm(dev(x["P"][:, 0]), dev(x["a"]), dev(x["c0"]), dev(x["h0"]))
    torch.cuda.synchronize()
    rc, rh = oracle.rollout_lstm(x["P"], x["a"], x["c0"], x["h0"])
    assert np.max(np.abs(c.cpu().numpy() - rc[:, 0])) <= 2e-6
    assert np.max(np.abs(h.cpu().numpy() - rh[:, 0])) <= 2e-6


@pytest.mark.parametrize("shape", [(2, 512, 16), (1, 1, 1), (3, 17, 5), (2, 3000, 64), (1, 5000, 1)])
def test_rollout_gru_matches_oracle(pr, shape):
    B, L, D = shape
    x = inputs.gru_inputs(B, L, D, seed=[702, B, L, D], h0_normal=True)
    h = pr.rollout_gru(dev(x["P"]), dev(x["a"]), dev(x["h0"]))
    torch.cuda.synchronize()
    ref = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= 1e-4


@pytest.mark.parametrize("shape", [(2, 512, 16), (1, 1, 1), (2, 1200, 33), (2, 700, 64)])
def test_rollout_lstm_matches_oracle(pr, shape):
    B, L, D = shape
    x = inputs.lstm_inputs(B, L, D, seed=[703, B, L, D], h0_normal=True)
    c, h = pr.rollout_lstm(dev(x["P"]), dev(x["a"]), dev(x["c0"]), dev(x["h0"]))
    torch.cuda.synchronize()
    rc, rh = oracle.rollout_lstm(x["P"], x["a"], x["c0"], x["h0"])
    assert np.max(np.abs(h.cpu().numpy() - rh)) <= 1e-4
    assert np.max(np.abs(c.cpu().numpy() - rc)) <= 1e-4


def test_step_loop_equals_rollout_and_newton(pr):
    """L launches of the decode step reproduce the rollout; both agree with the
    Newton solve within the solve's tolerance."""
    B, L, D = 2, 300, 32
    x = inputs.gru_inputs(B, L, D, seed=704)
    Pt = dev(np.ascontiguousarray(np.transpose(x["P"], (1, 0, 2, 3))))   # [L, B, 3, D]
    a = dev(x["a"])
    hs = torch.empty((L, B, D), device="cuda")
    prev = None
    for t in range(L):
        pr.step_gru(Pt[t], a, prev, out=hs[t])
        prev = hs[t]
    roll = pr.rollout_gru(dev(x["P"]), a)
    newt, info = pr.solve_gru(dev(x["P"]), a)
    torch.cuda.synchronize()
    loop = hs.permute(1, 0, 2).cpu().numpy()
    assert np.max(np.abs(loop - roll.cpu().numpy())) <= 1e-6
    assert info.converged and np.max(np.abs(newt.cpu().numpy() - loop)) <= 1e-4


@pytest.mark.parametrize("cell", ["gru", "lstm"])
def test_rollout_bf16_staged_matches_oracle(pr, cell):
    """bf16 gates with D a multiple of 32 (inputs staged through shared memory)
    against the oracle's rollout of the rounded gates."""
    B, L, D = 2, 1000, 96
    gen = inputs.gru_inputs if cell == "gru" else inputs.lstm_inputs
    x = gen(B, L, D, seed=[704, B, L, D], bf16=True, h0_normal=True)
    P16 = torch.from_numpy(x["P_bits"].view(np.int16)).cuda().view(torch.bfloat16)
    if cell == "gru":
        h = pr.rollout_gru(P16, dev(x["a"]), dev(x["h0"]))
        ref = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    else:
        _, h = pr.rollout_lstm(P16, dev(x["a"]), dev(x["c0"]), dev(x["h0"]))
        ref = oracle.rollout_lstm(x["P"], x["a"], x["c0"], x["h0"])[1]
    torch.cuda.synchronize()
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= 1e-4


@pytest.mark.parametrize("cell,bf16,shape", [("gru", True, (4, 4000, 1)), ("gru", False, (3, 999, 1)),
                                             ("lstm", False, (3, 999, 1)), ("lstm", True, (2, 1000, 1))])
def test_rollout_one_channel_staged(pr, cell, bf16, shape):
    """One channel per batch row (each thread stages its own contiguous inputs)."""
    B, L, D = shape
    gen = inputs.gru_inputs if cell == "gru" else inputs.lstm_inputs
    x = gen(B, L, D, seed=[705, B, L, D], bf16=bf16, h0_normal=True)
    P = (torch.from_numpy(x["P_bits"].view(np.int16)).cuda().view(torch.bfloat16) if bf16
         else dev(x["P"]))
    if cell == "gru":
        h = pr.rollout_gru(P, dev(x["a"]), dev(x["h0"]))
        ref = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    else:
        c, h = pr.rollout_lstm(P, dev(x["a"]), dev(x["c0"]), dev(x["h0"]))
        rc, ref = oracle.rollout_lstm(x["P"], x["a"], x["c0"], x["h0"])
        torch.cuda.synchronize()
        assert np.max(np.abs(c.cpu().numpy() - rc)) <= 1e-4
    torch.cuda.synchronize()
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= 1e-4
