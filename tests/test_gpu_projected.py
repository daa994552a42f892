"""Parity of the fused projection + ParaGRU Newton solve
(pararnn_solve_gru_projected) with the fp64 oracle, through the C ABI.

The oracle projects in fp64 (P = x W^T + bias on the same bf16 x and W,
widened exactly) and rolls the GRU out sequentially in fp64; the GPU
accumulates P in fp32 on the tensor cores, keeps it on chip, and solves by
Newton.  The trajectory must match to 1e-4 (the solves' tolerance), the
iteration count the oracle's serial Newton to within one, and the result the
unfused pair (projection to fp32 P in HBM, then the solve) closely."""
import numpy as np
import pytest
import torch

import oracle
from tests import inputs

pytestmark = pytest.mark.gpu

SOLVE_ATOL = 1e-4


@pytest.fixture(scope="module")
def pr():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import nonlinear_rnn_solve_newton_b200 as m

    m.load()
    return m


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def oracle_P(d, B, L, D, with_bias=True):
    """fp64 projection of the whole workload, in the solve's [B, L, 3, D] layout."""
    return oracle.input_projection(d["x"], d["W"], d["bias"] if with_bias else None).reshape(
        B, L, 3, D)


def run(pr, d, with_bias=True, h0=False, **kw):
    return pr.solve_gru_projected(bf16_dev(d["x_bits"]), bf16_dev(d["W_bits"]),
                                  dev(d["bias"]) if with_bias else None, dev(d["a"]),
                                  dev(d["h0"]) if h0 else None, **kw)


# (B, L, D, K): one chunk; a ragged last chunk; D not a multiple of 32 and K not
# a multiple of 64; more work items (batch row x 32 channels) than SMs; several
# rounds of items per CTA with an odd item count per CTA
SHAPES = [(1, 128, 32, 64), (2, 300, 64, 128), (3, 515, 48, 136), (2, 1000, 96, 256),
          (8, 256, 1024, 64), (7, 130, 2048, 64)]

# walker groups per CTA: one item at a time, two at once
GROUPS = [1, 2]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("with_bias,h0", [(True, False), (False, True)])
@pytest.mark.parametrize("groups", GROUPS)
def test_projected_solve_matches_oracle(pr, shape, with_bias, h0, groups):
    B, L, D, K = shape
    d = inputs.projected_gru_inputs(B, L, D, K, seed=[730, B, L, D, K], h0_normal=h0)
    h, info = run(pr, d, with_bias, h0, opts=pr.Options(regime=groups))
    torch.cuda.synchronize()
    assert info.status == 0 and info.converged
    P = oracle_P(d, B, L, D, with_bias)
    h0v = d["h0"] if h0 else None
    ref = oracle.rollout_gru(P, d["a"], h0v)
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= SOLVE_ATOL
    orc = oracle.newton_gru(P, d["a"], h0v, tol=1e-4, max_iters=32)
    assert abs(info.iterations - orc.iterations) <= 1


def test_projected_solve_matches_unfused_pair(pr):
    """The fused call against projection (fp32 P in HBM) followed by the solve."""
    B, L, D, K = 4, 777, 128, 192
    d = inputs.projected_gru_inputs(B, L, D, K, seed=731, h0_normal=True)
    h, info = run(pr, d, True, True)
    x, W = bf16_dev(d["x_bits"]), bf16_dev(d["W_bits"])
    P = pr.input_projection(x, W, dev(d["bias"])).view(B, L, 3, D)
    h2, info2 = pr.solve_gru(P, dev(d["a"]), dev(d["h0"]))
    torch.cuda.synchronize()
    assert info.converged and info2.converged and info.iterations == info2.iterations
    assert float(torch.max(torch.abs(h - h2)).item()) <= 1e-5


@pytest.mark.parametrize("groups", GROUPS)
def test_projected_solve_later_sweeps_recompute(pr, groups):
    """Two Newton iterations per sweep: the solve needs several sweeps, each of
    which recomputes the projection; same answer as the oracle and as one sweep."""
    B, L, D, K = 2, 700, 64, 128
    d = inputs.projected_gru_inputs(B, L, D, K, seed=732)
    h1, i1 = run(pr, d, opts=pr.Options(regime=groups))
    h2, i2 = run(pr, d, opts=pr.Options(iters_first=2, iters_next=1, regime=groups))
    torch.cuda.synchronize()
    assert i2.converged and i2.passes > 1 and i1.passes == 1
    assert i1.iterations == i2.iterations
    ref = oracle.rollout_gru(oracle_P(d, B, L, D), d["a"])
    assert np.max(np.abs(h2.cpu().numpy() - ref)) <= SOLVE_ATOL
    assert float(torch.max(torch.abs(h1 - h2)).item()) <= 1e-5


@pytest.mark.parametrize("max_iters", [0, 1, 2])
@pytest.mark.parametrize("groups", GROUPS)
def test_projected_solve_unconverged_is_the_newton_iterate(pr, max_iters, groups):
    """Stopped at max_iters, the trajectory is the max_iters-th Newton iterate and
    the residuals rho_0 .. rho_max_iters are the oracle's."""
    B, L, D, K = 2, 400, 64, 128
    d = inputs.projected_gru_inputs(B, L, D, K, seed=733)
    h, info = run(pr, d, max_iters=max_iters, opts=pr.Options(regime=groups))
    torch.cuda.synchronize()
    assert info.status == 0 and not info.converged and info.iterations == max_iters
    orc = oracle.newton_gru(oracle_P(d, B, L, D), d["a"], tol=1e-4, max_iters=max_iters)
    assert np.max(np.abs(h.cpu().numpy() - orc.h)) <= 1e-5
    for k in range(max_iters + 1):
        assert abs(info.rho[k] - orc.rho[k]) <= 1e-5 * max(1.0, orc.rho[k])


def test_projected_solve_groups_agree(pr):
    """One and two walker groups give the same trajectory and iteration count."""
    B, L, D, K = 5, 333, 160, 96
    d = inputs.projected_gru_inputs(B, L, D, K, seed=735, h0_normal=True)
    h1, i1 = run(pr, d, True, True, opts=pr.Options(regime=1))
    h2, i2 = run(pr, d, True, True, opts=pr.Options(regime=2))
    torch.cuda.synchronize()
    assert i1.converged and i2.converged and i1.iterations == i2.iterations
    # 8 vs 16 steps per walker thread: the same sums in another order
    assert float(torch.max(torch.abs(h1 - h2)).item()) <= 1e-5


def test_projected_solve_empty(pr):
    x = torch.empty((0, 10, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((96, 64), dtype=torch.bfloat16, device="cuda")
    a = torch.zeros((3, 32), device="cuda")
    h, info = pr.solve_gru_projected(x, W, None, a)
    torch.cuda.synchronize()
    assert info.converged and info.iterations == 0 and h.shape == (0, 10, 32)


@pytest.mark.slow
def test_projected_solve_lm_width_sampled_channels(pr):
    """The fused workload at its full size (B=8, L=8192, D=4096, K=4096): sampled
    channels' whole trajectories against the oracle, whose projection of one
    channel is x[b] (L x K) times the channel's three rows of W."""
    w = inputs.WORKLOADS["proj_solve"]
    B, L, D, K = w["B"], w["L"], w["D"], w["K"]
    d = inputs.projected_gru_inputs(B, L, D, K, seed=w["seed"])
    h, info = run(pr, d)
    torch.cuda.synchronize()
    assert info.status == 0 and info.converged
    rng = np.random.default_rng(734)
    chans = set(zip(rng.integers(0, B, 24).tolist(), rng.integers(0, D, 24).tolist()))
    chans |= {(0, 0), (B - 1, D - 1)}
    for b, c in sorted(chans):
        rows = [c, D + c, 2 * D + c]
        Pc = oracle.input_projection(d["x"][b], d["W"][rows], d["bias"][rows])  # [L, 3]
        ref = oracle.rollout_gru(Pc.reshape(1, L, 3, 1), d["a"][:, c:c + 1])[0, :, 0]
        got = h[b, :, c].cpu().numpy()
        assert np.max(np.abs(got - ref)) <= SOLVE_ATOL, (b, c)
