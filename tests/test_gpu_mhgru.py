"""Parity of the multi-head GRU Newton solve (dense 8x8 recurrence blocks) with
the fp64 oracle, through the C ABI.

Tolerance as for the diagonal solves: the trajectory within 1e-4 (max-abs) of
the oracle's fp64 rollout once converged at tol = 1e-4; the iteration count
within one of the oracle's serial Newton (rho_k near tol under fp32 rounding);
an unconverged iterate h^k against the oracle's h^k within 1e-4.
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


# (B, L, H): one chunk, a chunk boundary with a 1-step tail (chunk = 512 steps),
# several chunks, one head, a single step, more sequences than one CTA holds
SHAPES = [(2, 100, 2), (1, 513, 3), (2, 1500, 4), (3, 37, 1), (2, 1, 2), (4, 300, 9)]


# the two layouts: one lane per time segment holding whole 8x8 maps (regime 1),
# 8 lanes per head and segment (regime 2); regime 0 chooses by the strides
LAYOUTS = [1, 2]


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("h0_normal", [False, True])
@pytest.mark.parametrize("shape", SHAPES)
def test_mhgru_matches_rollout(pr, shape, h0_normal, layout):
    B, L, H = shape
    x = inputs.mhgru_inputs(B, L, H, seed=[800, B, L, H], h0_normal=h0_normal)
    h, info = pr.solve_mhgru(dev(x["P"]), dev(x["U"]), dev(x["h0"]) if h0_normal else None,
                             opts=pr.Options(regime=layout))
    torch.cuda.synchronize()
    ref = oracle.rollout_mhgru(x["P"], x["U"], x["h0"])
    res = oracle.newton_mhgru(x["P"], x["U"], x["h0"])
    assert info.status == 0 and info.converged
    assert abs(info.iterations - res.iterations) <= 1
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= 1e-4


def test_mhgru_bf16_inputs(pr):
    B, L, H = 2, 700, 3
    x = inputs.mhgru_inputs(B, L, H, seed=801)
    bits, vals = inputs.round_to_bf16(x["P"])
    P16 = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    h, info = pr.solve_mhgru(P16, dev(x["U"]))
    torch.cuda.synchronize()
    assert info.converged
    assert np.max(np.abs(h.cpu().numpy() - oracle.rollout_mhgru(vals, x["U"]))) <= 1e-4


def test_mhgru_diagonal_blocks_match_paragru_solve(pr):
    """Diagonal blocks: the multi-head solve and the ParaGRU solve agree."""
    B, L, D = 2, 800, 32
    x = inputs.gru_inputs(B, L, D, seed=802)
    H = D // 8
    U = np.zeros((3, H, 8, 8), np.float32)
    for g in range(3):
        for k in range(H):
            U[g, k] = np.diag(x["a"][g, 8 * k: 8 * k + 8])
    hm, im = pr.solve_mhgru(dev(x["P"]), dev(U))
    hg, ig = pr.solve_gru(dev(x["P"]), dev(x["a"]))
    torch.cuda.synchronize()
    assert abs(im.iterations - ig.iterations) <= 1
    assert np.max(np.abs(hm.cpu().numpy() - hg.cpu().numpy())) <= 1e-4


@pytest.mark.parametrize("k", [1, 2])
def test_mhgru_unconverged_iterate(pr, k):
    """tol = 0 and max_iters = k: the result is Newton's h^k."""
    B, L, H = 2, 600, 2
    x = inputs.mhgru_inputs(B, L, H, seed=[803, k], h0_normal=True)
    h, info = pr.solve_mhgru(dev(x["P"]), dev(x["U"]), dev(x["h0"]), tol=0.0, max_iters=k)
    torch.cuda.synchronize()
    res = oracle.newton_mhgru(x["P"], x["U"], x["h0"], tol=0.0, max_iters=k)
    assert info.iterations == k and not info.converged and info.updates == k
    assert np.max(np.abs(h.cpu().numpy() - res.h)) <= 1e-4
    np.testing.assert_allclose(info.rho[: k + 1], res.rho, rtol=1e-3, atol=1e-6)


def test_mhgru_zero_iterations_returns_h0_iterate(pr):
    x = inputs.mhgru_inputs(1, 50, 1, seed=804)
    h, info = pr.solve_mhgru(dev(x["P"]), dev(x["U"]), max_iters=0)
    torch.cuda.synchronize()
    assert info.iterations == 0 and info.updates == 0
    assert not h.cpu().numpy().any()


def test_mhgru_nonfinite_reported(pr):
    x = inputs.mhgru_inputs(1, 200, 2, seed=805)
    x["P"][0, 77, 1, 3] = np.nan
    h, info = pr.solve_mhgru(dev(x["P"]), dev(x["U"]))
    torch.cuda.synchronize()
    assert info.status == 5 and not info.converged


def test_mhgru_empty(pr):
    P = torch.empty((0, 10, 3, 16), device="cuda")
    U = torch.zeros((3, 2, 8, 8), device="cuda")
    h, info = pr.solve_mhgru(P, U)
    torch.cuda.synchronize()
    assert info.converged and info.iterations == 0


def test_mhgru_full_size_every_head(pr):
    """The multi-head workload at full size (B = 8, L = 4096, 128 heads): every
    (batch row, head) sequence against the oracle's rollout, and the iteration
    count against its serial Newton on the same workload."""
    w = inputs.WORKLOADS["mhgru"]
    B, L, D = w["B"], w["L"], w["D"]
    H = D // 8
    x = inputs.mhgru_inputs(B, L, H, seed=w["seed"])
    h, info = pr.solve_mhgru(dev(x["P"]), dev(x["U"]))
    torch.cuda.synchronize()
    assert info.converged
    ref = oracle.rollout_mhgru(x["P"], x["U"])
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= 1e-4
    orc = oracle.newton_mhgru(x["P"], x["U"])
    assert orc.converged and abs(info.iterations - orc.iterations) <= 1


# --------------------------------------------------------------------------
# Per-head time strides (DEER summary, caveats: heads with exponentially
# increasing strides): head g recurs on h_{t - s_g}
# --------------------------------------------------------------------------
def sdev(strides):
    return torch.from_numpy(np.ascontiguousarray(strides, dtype=np.int32)).cuda()


# (B, L, strides): exponentially increasing strides; strides past the sequence
# end; stride 1 everywhere (= the unstrided solve); a long sequence whose
# residue sequences span several chunks; more units than one CTA holds
STRIDED = [(2, 300, [1, 2, 4, 8]), (1, 50, [1, 64, 3]), (2, 400, [1, 1, 1]),
           (1, 4000, [1, 2, 4, 8, 16, 32, 64, 128]), (4, 257, [1, 3, 5, 7, 2])]


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("h0_normal", [False, True])
@pytest.mark.parametrize("B,L,strides", STRIDED)
def test_mhgru_strided_matches_oracle(pr, B, L, strides, h0_normal, layout):
    H = len(strides)
    x = inputs.mhgru_inputs(B, L, H, seed=[810, B, L, H], h0_normal=h0_normal)
    h0 = dev(x["h0"]) if h0_normal else None
    h, info = pr.solve_mhgru_strided(dev(x["P"]), dev(x["U"]), sdev(strides), h0,
                                     opts=pr.Options(regime=layout))
    torch.cuda.synchronize()
    st = np.asarray(strides, np.int32)
    ref = oracle.rollout_mhgru(x["P"], x["U"], x["h0"], strides=st)
    res = oracle.newton_mhgru(x["P"], x["U"], x["h0"], strides=st)
    assert info.status == 0 and info.converged
    assert abs(info.iterations - res.iterations) <= 1
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= 1e-4


@pytest.mark.parametrize("layout", LAYOUTS)
def test_mhgru_strided_all_ones_is_the_unstrided_solve(pr, layout):
    """Within one layout, strides of 1 give the unstrided solve bit for bit; the
    automatic choice (which differs with and without strides) agrees to rounding."""
    x = inputs.mhgru_inputs(2, 700, 4, seed=811, h0_normal=True)
    P, U, h0 = dev(x["P"]), dev(x["U"]), dev(x["h0"])
    o = pr.Options(regime=layout)
    h1, i1 = pr.solve_mhgru(P, U, h0, opts=o)
    h2, i2 = pr.solve_mhgru_strided(P, U, sdev([1, 1, 1, 1]), h0, opts=o)
    h3, i3 = pr.solve_mhgru_strided(P, U, sdev([1, 1, 1, 1]), h0)
    torch.cuda.synchronize()
    assert i1.iterations == i2.iterations == i3.iterations
    assert float(torch.max(torch.abs(h1 - h2)).item()) == 0.0
    assert float(torch.max(torch.abs(h1 - h3)).item()) <= 1e-5


@pytest.mark.parametrize("k", [1, 2])
def test_mhgru_strided_unconverged_iterate(pr, k):
    B, L, strides = 2, 200, [1, 4, 9]
    x = inputs.mhgru_inputs(B, L, len(strides), seed=812, h0_normal=True)
    st = np.asarray(strides, np.int32)
    h, info = pr.solve_mhgru_strided(dev(x["P"]), dev(x["U"]), sdev(st), dev(x["h0"]), tol=0.0,
                                     max_iters=k)
    torch.cuda.synchronize()
    res = oracle.newton_mhgru(x["P"], x["U"], x["h0"], tol=0.0, max_iters=k, strides=st)
    assert info.status == 0 and not info.converged and info.iterations == k
    assert np.max(np.abs(h.cpu().numpy() - res.h)) <= 1e-4


def test_mhgru_stride_below_one_is_reported(pr):
    x = inputs.mhgru_inputs(1, 50, 3, seed=813)
    h, info = pr.solve_mhgru_strided(dev(x["P"]), dev(x["U"]), sdev([1, 0, 2]))
    torch.cuda.synchronize()
    assert info.status == 1 and not info.converged


def test_mhgru_strided_full_size_exponential_strides(pr):
    """The multi-head workload's full size (B = 8, L = 4096, 128 heads) with
    strides 2^(g mod 8): every sequence against the oracle's strided rollout."""
    w = inputs.WORKLOADS["mhgru"]
    B, L, D = w["B"], w["L"], w["D"]
    H = D // 8
    x = inputs.mhgru_inputs(B, L, H, seed=w["seed"])
    st = (2 ** (np.arange(H) % 8)).astype(np.int32)
    h, info = pr.solve_mhgru_strided(dev(x["P"]), dev(x["U"]), sdev(st))
    torch.cuda.synchronize()
    assert info.converged
    ref = oracle.rollout_mhgru(x["P"], x["U"], strides=st)
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= 1e-4


@pytest.mark.parametrize("shape", [(2, 100, 2), (1, 1, 1), (3, 517, 5), (1, 3000, 16)])
def test_rollout_mhgru_matches_oracle(pr, shape):
    """The sequential multi-head application (8 lanes per head) against the
    oracle's fp64 rollout."""
    B, L, H = shape
    x = inputs.mhgru_inputs(B, L, H, seed=[820, B, L, H], h0_normal=True)
    h = pr.rollout_mhgru(dev(x["P"]), dev(x["U"]), dev(x["h0"]))
    torch.cuda.synchronize()
    ref = oracle.rollout_mhgru(x["P"], x["U"], x["h0"])
    assert np.max(np.abs(h.cpu().numpy() - ref)) <= 1e-4


def test_rollout_mhgru_bf16_and_zero_state(pr):
    B, L, H = 2, 700, 3
    x = inputs.mhgru_inputs(B, L, H, seed=821)
    bits, vals = inputs.round_to_bf16(x["P"])
    P16 = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    h = pr.rollout_mhgru(P16, dev(x["U"]))
    torch.cuda.synchronize()
    assert np.max(np.abs(h.cpu().numpy() - oracle.rollout_mhgru(vals, x["U"]))) <= 1e-4


def test_rollout_mhgru_full_size_equals_newton(pr):
    """The multi-head workload's full size: every sequence of the rollout against
    the oracle, and the Newton solve against the rollout."""
    w = inputs.WORKLOADS["mhgru"]
    B, L, D = w["B"], w["L"], w["D"]
    H = D // 8
    x = inputs.mhgru_inputs(B, L, H, seed=w["seed"])
    P, U = dev(x["P"]), dev(x["U"])
    roll = pr.rollout_mhgru(P, U)
    h, info = pr.solve_mhgru(P, U)
    torch.cuda.synchronize()
    assert info.converged
    ref = oracle.rollout_mhgru(x["P"], x["U"])
    r = roll.cpu().numpy()
    assert np.max(np.abs(r - ref)) <= 1e-4
    assert np.max(np.abs(h.cpu().numpy() - r)) <= 1e-4


def test_step_mhgru_matches_oracle_cell_and_rollout(pr):
    """One decode step per head equals the oracle's cell; L steps equal the rollout."""
    B, L, H = 3, 40, 5
    x = inputs.mhgru_inputs(B, L, H, seed=822, h0_normal=True)
    P, U, h0 = dev(x["P"]), dev(x["U"]), dev(x["h0"])
    h1 = pr.step_mhgru(P[:, 0].contiguous(), U, h0)
    torch.cuda.synchronize()
    for b in range(B):
        for g in range(H):
            f, _ = oracle.mhgru_cell(x["P"][b, 0, :, 8 * g:8 * g + 8], x["U"][:, g],
                                     x["h0"][b, 8 * g:8 * g + 8])
            assert np.max(np.abs(h1[b, 8 * g:8 * g + 8].cpu().numpy() - f)) <= 2e-6
    hs, prev = [], h0
    for t in range(L):
        prev = pr.step_mhgru(P[:, t].contiguous(), U, prev)
        hs.append(prev)
    roll = pr.rollout_mhgru(P, U, h0)
    torch.cuda.synchronize()
    assert torch.equal(torch.stack(hs, 1), roll)
