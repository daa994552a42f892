"""Parity of the backward pass (gradients through the solved trajectory) with the
fp64 oracle's adjoint recursion, through the C ABI.

Both sides receive the same trajectory (the oracle's rollout rounded once to
fp32) and the same upstream gradients.  Tolerances, from the arithmetic: dP and
dh0 elementwise |x - ref| <= 1e-4 * max(1, |ref|) (fp32 reverse scan with
contractive maps); da, a sum over every (b, t) accumulated with fp32 atomics in
an arbitrary order, |x - ref| <= 1e-4 * max(1, sum of |terms|) per entry.
"""
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


def close(got, ref, rtol=1e-4):
    return np.max(np.abs(got - ref) / np.maximum(1.0, np.abs(ref)))


def da_close(got, ref, scale):
    return np.max(np.abs(got - ref) / np.maximum(1.0, scale))


SHAPES = [(2, 512, 16), (1, 1, 1), (2, 3, 5), (3, 31, 3), (1, 2049, 1), (2, 1100, 64),
          (1, 300, 33), (4, 257, 128)]


@pytest.mark.parametrize("regime", [0, 1, 2])
@pytest.mark.parametrize("shape", SHAPES)
def test_gru_backward_parity(pr, shape, regime):
    B, L, D = shape
    x = inputs.gru_inputs(B, L, D, seed=[600, B, L, D], h0_normal=True)
    h = oracle.rollout_gru(x["P"], x["a"], x["h0"]).astype(np.float32)
    gh = np.random.default_rng([601, B, L, D]).standard_normal((B, L, D)).astype(np.float32)
    dP, da, dh0 = pr.solve_gru_backward(dev(x["P"]), dev(x["a"]), dev(h), dev(gh), dev(x["h0"]),
                                        opts=pr.Options(regime=regime))
    torch.cuda.synchronize()
    rP, ra, rh0 = oracle.backward_gru(x["P"], x["a"], h, gh, x["h0"])
    hp = np.concatenate([x["h0"][:, None].astype(np.float64), h[:, :-1].astype(np.float64)], 1)
    scale = np.abs(rP * hp[:, :, None]).sum(axis=(0, 1))
    assert close(dP.cpu().numpy(), rP) <= 1e-4
    assert close(dh0.cpu().numpy(), rh0) <= 1e-4
    assert da_close(da.cpu().numpy(), ra, scale) <= 1e-4


@pytest.mark.parametrize("regime", [0, 1, 2])
@pytest.mark.parametrize("shape", SHAPES[:6])
def test_lstm_backward_parity(pr, shape, regime):
    B, L, D = shape
    x = inputs.lstm_inputs(B, L, D, seed=[610, B, L, D], h0_normal=True)
    c, h = oracle.rollout_lstm(x["P"], x["a"], x["c0"], x["h0"])
    c, h = c.astype(np.float32), h.astype(np.float32)
    rng = np.random.default_rng([611, B, L, D])
    gc = rng.standard_normal((B, L, D)).astype(np.float32)
    gh = rng.standard_normal((B, L, D)).astype(np.float32)
    dP, da, dc0, dh0 = pr.solve_lstm_backward(dev(x["P"]), dev(x["a"]), dev(c), dev(h), dev(gc),
                                              dev(gh), dev(x["c0"]), dev(x["h0"]),
                                              opts=pr.Options(regime=regime))
    torch.cuda.synchronize()
    rP, ra, rc0, rh0 = oracle.backward_lstm(x["P"], x["a"], c, h, gc, gh, x["c0"], x["h0"])
    hp = np.concatenate([x["h0"][:, None].astype(np.float64), h[:, :-1].astype(np.float64)], 1)
    scale = np.abs(rP * hp[:, :, None]).sum(axis=(0, 1))
    assert close(dP.cpu().numpy(), rP) <= 1e-4
    assert close(dc0.cpu().numpy(), rc0) <= 1e-4
    assert close(dh0.cpu().numpy(), rh0) <= 1e-4
    assert da_close(da.cpu().numpy(), ra, scale) <= 1e-4


def test_gru_backward_bf16_inputs(pr):
    B, L, D = 2, 700, 64
    x = inputs.gru_inputs(B, L, D, seed=620, bf16=True)
    h = oracle.rollout_gru(x["P"], x["a"]).astype(np.float32)
    gh = np.random.default_rng(621).standard_normal((B, L, D)).astype(np.float32)
    P16 = torch.from_numpy(x["P_bits"].view(np.int16)).cuda().view(torch.bfloat16)
    dP, da, dh0 = pr.solve_gru_backward(P16, dev(x["a"]), dev(h), dev(gh))
    torch.cuda.synchronize()
    rP, ra, rh0 = oracle.backward_gru(x["P"], x["a"], h, gh)
    assert close(dP.cpu().numpy(), rP) <= 1e-4


def test_forward_then_backward_on_gpu(pr):
    """Solve on the GPU, differentiate its solution on the GPU; compare with the
    oracle's adjoint on the oracle's rollout."""
    B, L, D = 4, 1024, 256
    x = inputs.gru_inputs(B, L, D, seed=630)
    P, a = dev(x["P"]), dev(x["a"])
    h, info = pr.solve_gru(P, a)
    gh = np.random.default_rng(631).standard_normal((B, L, D)).astype(np.float32)
    dP, da, dh0 = pr.solve_gru_backward(P, a, h, dev(gh))
    torch.cuda.synchronize()
    assert info.converged
    href = oracle.rollout_gru(x["P"], x["a"])
    rP, ra, rh0 = oracle.backward_gru(x["P"], x["a"], href, gh)
    assert close(dP.cpu().numpy(), rP) <= 1e-3


def test_backward_stall_times_out(pr):
    B, L, D = 1, 4096, 32
    x = inputs.gru_inputs(B, L, D, seed=640)
    h = oracle.rollout_gru(x["P"], x["a"]).astype(np.float32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = pr.Options(wait_timeout_ns=20_000_000, debug_stall_unit=1, regime=1)
    pr.solve_gru_backward(dev(x["P"]), dev(x["a"]), dev(h), dev(h), status=st, opts=o)
    torch.cuda.synchronize()
    assert int(st.item()) == 4


# Shapes the TMA tile walker takes when the walk regime is forced: D a multiple
# of 4 (fp32 rows) / 8 (bf16 rows) and at least 32, ragged last tile (D = 40,
# 96 + 8), L not a multiple of the chunk length (64 GRU, 32 LSTM).
WALK_SHAPES = [(2, 1000, 40), (3, 333, 104), (1, 64, 32), (2, 65, 64)]


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("shape", WALK_SHAPES)
def test_gru_backward_walk(pr, shape, bf16):
    B, L, D = shape
    x = inputs.gru_inputs(B, L, D, seed=[650, B, L, D], bf16=bf16, h0_normal=True)
    h = oracle.rollout_gru(x["P"], x["a"], x["h0"]).astype(np.float32)
    gh = np.random.default_rng([651, B, L, D]).standard_normal((B, L, D)).astype(np.float32)
    P = (torch.from_numpy(x["P_bits"].view(np.int16)).cuda().view(torch.bfloat16) if bf16
         else dev(x["P"]))
    dP, da, dh0 = pr.solve_gru_backward(P, dev(x["a"]), dev(h), dev(gh), dev(x["h0"]),
                                        opts=pr.Options(regime=2))
    torch.cuda.synchronize()
    rP, ra, rh0 = oracle.backward_gru(x["P"], x["a"], h, gh, x["h0"])
    hp = np.concatenate([x["h0"][:, None].astype(np.float64), h[:, :-1].astype(np.float64)], 1)
    scale = np.abs(rP * hp[:, :, None]).sum(axis=(0, 1))
    assert close(dP.cpu().numpy(), rP) <= 1e-4
    assert close(dh0.cpu().numpy(), rh0) <= 1e-4
    assert da_close(da.cpu().numpy(), ra, scale) <= 1e-4


@pytest.mark.parametrize("which", ["both", "dc_only", "dh_only"])
@pytest.mark.parametrize("shape", WALK_SHAPES)
def test_lstm_backward_walk(pr, shape, which):
    B, L, D = shape
    x = inputs.lstm_inputs(B, L, D, seed=[660, B, L, D], h0_normal=True)
    c, h = oracle.rollout_lstm(x["P"], x["a"], x["c0"], x["h0"])
    c, h = c.astype(np.float32), h.astype(np.float32)
    rng = np.random.default_rng([661, B, L, D])
    gc = rng.standard_normal((B, L, D)).astype(np.float32)
    gh = rng.standard_normal((B, L, D)).astype(np.float32)
    if which == "dc_only":
        gh[:] = 0.0
    if which == "dh_only":
        gc[:] = 0.0
    dP, da, dc0, dh0 = pr.solve_lstm_backward(
        dev(x["P"]), dev(x["a"]), dev(c), dev(h),
        None if which == "dh_only" else dev(gc), None if which == "dc_only" else dev(gh),
        dev(x["c0"]), dev(x["h0"]), opts=pr.Options(regime=2))
    torch.cuda.synchronize()
    rP, ra, rc0, rh0 = oracle.backward_lstm(x["P"], x["a"], c, h, gc, gh, x["c0"], x["h0"])
    hp = np.concatenate([x["h0"][:, None].astype(np.float64), h[:, :-1].astype(np.float64)], 1)
    scale = np.abs(rP * hp[:, :, None]).sum(axis=(0, 1))
    assert close(dP.cpu().numpy(), rP) <= 1e-4
    assert close(dc0.cpu().numpy(), rc0) <= 1e-4
    assert close(dh0.cpu().numpy(), rh0) <= 1e-4
    assert da_close(da.cpu().numpy(), ra, scale) <= 1e-4


def test_backward_walk_stage_timeout(pr):
    """A stage wait that runs out reports status 4 and leaves the context usable.
    The walker's copies always land, so the limit is made shorter than any copy
    (1 ns): the first wait that is not already complete gives up."""
    B, L, D = 8, 4096, 1024
    x = inputs.gru_inputs(1, 64, 32, seed=670)
    P = torch.randn(B, L, 3, D, device="cuda")
    a = dev(np.resize(x["a"], (3, D)))
    h = torch.zeros(B, L, D, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pr.solve_gru_backward(P, a, h, h, status=st, opts=pr.Options(regime=2, wait_timeout_ns=1))
    torch.cuda.synchronize()
    assert int(st.item()) in (0, 4)
    # the context still works
    dP, da, dh0 = pr.solve_gru_backward(P, a, h, h, opts=pr.Options(regime=2))
    torch.cuda.synchronize()
    assert torch.isfinite(dP).all()
