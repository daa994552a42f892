"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test fixes one part of the oracle against something it does not share
code with: closed forms of linear recurrences, brute-force composition of
affine maps, PyTorch's fp64 ``GRUCell``/``LSTMCell`` (a library routine that the
ParaGRU / ParaLSTM cells reduce to once the recurrence weights are placed on a
diagonal), autograd Jacobians of those library cells, and the invariants of
Newton's method that the pages state or imply (converged Newton reproduces the
sequential rollout; a recurrence with no h-dependence in its gates is a single
scan; quadratic convergence).
"""
import math

import numpy as np
import pytest
import torch

from tests import inputs



@pytest.fixture(autouse=True)
def _fp64_default():
    old = torch.get_default_dtype()
    torch.set_default_dtype(torch.float64)
    yield
    torch.set_default_dtype(old)


# --------------------------------------------------------------------------
# Library stand-ins for the cells: PyTorch fp64 GRUCell / LSTMCell whose
# hidden-to-hidden weights are diagonal.  ParaGRU's z is torch's (1 - z).
# --------------------------------------------------------------------------
def torch_gru_cell(D, a):
    """GRUCell(3D -> D) that maps x = [Pr, -Pz, Pc] to the ParaGRU step."""
    a = torch.as_tensor(np.asarray(a, np.float64))
    cell = torch.nn.GRUCell(3 * D, D, bias=False).double()
    with torch.no_grad():
        cell.weight_ih.copy_(torch.eye(3 * D))
        cell.weight_hh.copy_(torch.cat([torch.diag(a[1]), torch.diag(-a[0]), torch.diag(a[2])]))
    return cell


def torch_gru_step(cell, p, h):
    """p: [N, 3, D] as (Pz, Pr, Pc), h: [N, D] -> h'."""
    p = torch.as_tensor(np.asarray(p, np.float64))
    assert p.dim() == 3 and h.dim() == 2
    x = torch.cat([p[..., 1, :], -p[..., 0, :], p[..., 2, :]], dim=-1)
    return cell(x, h)


def torch_lstm_cell(D, a):
    a = torch.as_tensor(np.asarray(a, np.float64))
    cell = torch.nn.LSTMCell(4 * D, D, bias=False).double()
    with torch.no_grad():
        cell.weight_ih.copy_(torch.eye(4 * D))
        cell.weight_hh.copy_(torch.cat([torch.diag(a[g]) for g in range(4)]))
    return cell


def torch_gru_rollout(P, a, h0=None):
    P = np.asarray(P, np.float64)
    B, L, _, D = P.shape
    cell = torch_gru_cell(D, a)
    h = torch.zeros(B, D) if h0 is None else torch.as_tensor(np.asarray(h0, np.float64))
    out = []
    with torch.no_grad():
        for t in range(L):
            h = torch_gru_step(cell, P[:, t], h)
            out.append(h)
    return torch.stack(out, 1).numpy()


def torch_lstm_rollout(P, a, c0=None, h0=None):
    P = torch.as_tensor(np.asarray(P, np.float64))
    B, L, _, D = P.shape
    cell = torch_lstm_cell(D, a)
    c = torch.zeros(B, D) if c0 is None else torch.as_tensor(np.asarray(c0, np.float64))
    h = torch.zeros(B, D) if h0 is None else torch.as_tensor(np.asarray(h0, np.float64))
    cs, hs = [], []
    with torch.no_grad():
        for t in range(L):
            h, c = cell(P[:, t].reshape(B, 4 * D), (h, c))
            cs.append(c)
            hs.append(h)
    return torch.stack(cs, 1).numpy(), torch.stack(hs, 1).numpy()


# --------------------------------------------------------------------------
# Diagonal scan
# --------------------------------------------------------------------------
def brute_force_diag(A, b, h0):
    """h_t = (prod_{s<=t} A_s) h0 + sum_s (prod_{s<u<=t} A_u) b_s, term by term."""
    L = len(A)
    out = []
    for t in range(L):
        acc = math.prod(A[: t + 1]) * h0
        for s in range(t + 1):
            acc += math.prod(A[s + 1: t + 1]) * b[s]
        out.append(acc)
    return np.array(out)


def test_scan_diag_brute_force(oracle):
    rng = np.random.default_rng(10)
    for L in (1, 2, 3, 7, 16):
        A = rng.uniform(-1.2, 1.2, (2, L, 3))
        b = rng.standard_normal((2, L, 3))
        h0 = rng.standard_normal((2, 3))
        h = oracle.scan_diag(A, b, h0)
        for bb in range(2):
            for d in range(3):
                ref = brute_force_diag(A[bb, :, d], b[bb, :, d], h0[bb, d])
                np.testing.assert_allclose(h[bb, :, d], ref, rtol=1e-13, atol=1e-13)


def test_scan_diag_closed_forms(oracle):
    L = 50
    alpha, beta, x0 = 0.9, 0.7, -1.3
    A = np.full((1, L, 1), alpha)
    b = np.full((1, L, 1), beta)
    h = oracle.scan_diag(A, b, np.array([[x0]]))[0, :, 0]
    t = np.arange(1, L + 1)
    np.testing.assert_allclose(h, alpha ** t * x0 + beta * (1 - alpha ** t) / (1 - alpha), rtol=1e-13)
    # A = 1: running sum (exact on small integers)
    bi = np.random.default_rng(0).integers(-5, 6, (2, 40, 3)).astype(np.float64)
    h = oracle.scan_diag(np.ones_like(bi), bi, np.full((2, 3), 2.0))
    np.testing.assert_array_equal(h, 2.0 + np.cumsum(bi, axis=1))
    # A = 0: h = b
    h = oracle.scan_diag(np.zeros_like(bi), bi, np.full((2, 3), 7.0))
    np.testing.assert_array_equal(h, bi)
    # h0 = None means zero
    h = oracle.scan_diag(np.ones_like(bi), bi)
    np.testing.assert_array_equal(h, np.cumsum(bi, axis=1))


# --------------------------------------------------------------------------
# 2x2 block scan
# --------------------------------------------------------------------------
def test_scan_block2_brute_force(oracle):
    rng = np.random.default_rng(11)
    B, L, D = 2, 9, 3
    A = rng.uniform(-0.9, 0.9, (B, L, D, 2, 2))
    b = rng.standard_normal((B, L, D, 2))
    x0 = rng.standard_normal((B, D, 2))
    x = oracle.scan_block2(A, b, x0)
    for bb in range(B):
        for d in range(D):
            for t in range(L):
                M = np.eye(2)
                for s in range(t + 1):
                    M = A[bb, s, d] @ M
                acc = M @ x0[bb, d]
                for s in range(t + 1):
                    N = np.eye(2)
                    for u in range(s + 1, t + 1):
                        N = A[bb, u, d] @ N
                    acc = acc + N @ b[bb, s, d]
                np.testing.assert_allclose(x[bb, t, d], acc, rtol=1e-12, atol=1e-12)


def test_scan_block2_rotation_power(oracle):
    """Constant A = s R(theta), b = 0: x_t = s^t R(t theta) x0 (a transposed A rotates backwards)."""
    L, s, th = 40, 0.97, 0.3
    R = np.array([[math.cos(th), -math.sin(th)], [math.sin(th), math.cos(th)]])
    A = np.broadcast_to(s * R, (1, L, 1, 2, 2)).copy()
    x0 = np.array([[[1.0, 0.25]]])
    x = oracle.scan_block2(A, np.zeros((1, L, 1, 2)), x0)[0, :, 0]
    for t in range(1, L + 1):
        Rt = np.array([[math.cos(t * th), -math.sin(t * th)], [math.sin(t * th), math.cos(t * th)]])
        np.testing.assert_allclose(x[t - 1], s ** t * Rt @ x0[0, 0], rtol=1e-12, atol=1e-14)


def test_scan_block2_diagonal_is_two_scans():
    """Diagonal blocks decouple into two running products; checked against np.cumprod sums."""
    import oracle

    rng = np.random.default_rng(12)
    B, L, D = 2, 30, 4
    a0 = rng.uniform(0, 1, (B, L, D))
    a1 = rng.uniform(0, 1, (B, L, D))
    A = np.zeros((B, L, D, 2, 2))
    A[..., 0, 0] = a0
    A[..., 1, 1] = a1
    b = rng.standard_normal((B, L, D, 2))
    x = oracle.scan_block2(A, b, np.zeros((B, D, 2)))
    for comp, a in ((0, a0), (1, a1)):
        for bb in range(B):
            for d in range(D):
                ref = brute_force_diag(a[bb, :, d], b[bb, :, d, comp], 0.0)
                np.testing.assert_allclose(x[bb, :, d, comp], ref, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# Cells and Jacobians against the library cells and autograd
# --------------------------------------------------------------------------
def test_gru_cell_matches_torch_gru_cell(oracle):
    rng = np.random.default_rng(13)
    D = 1
    for _ in range(50):
        p = rng.standard_normal(3) * 2
        w = rng.uniform(-1, 1, 3)
        h = rng.standard_normal() * 1.5
        f, J = oracle.gru_cell(p, w, h)
        cell = torch_gru_cell(D, w.reshape(3, 1))
        ht = torch.tensor([[h]], requires_grad=True)
        out = torch_gru_step(cell, p.reshape(1, 3, 1), ht)
        assert abs(out.item() - f) < 1e-14
        Jt = torch.autograd.functional.jacobian(lambda x: torch_gru_step(cell, p.reshape(1, 3, 1), x),
                                                ht)
        assert abs(Jt.item() - J) < 1e-12


def test_lstm_cell_matches_torch_lstm_cell(oracle):
    rng = np.random.default_rng(14)
    for _ in range(50):
        p = rng.standard_normal(4) * 2
        w = rng.uniform(-1, 1, 4)
        c, h = rng.standard_normal(2)
        fc, fh, J = oracle.lstm_cell(p, w, c, h)
        cell = torch_lstm_cell(1, w.reshape(4, 1))
        x = torch.tensor(p).reshape(1, 4)

        def step(state):
            hh, cc = cell(x, (state[1].reshape(1, 1), state[0].reshape(1, 1)))
            return torch.stack([cc.reshape(()), hh.reshape(())])

        st = torch.tensor([c, h])
        out = step(st)
        assert abs(out[0].item() - fc) < 1e-14 and abs(out[1].item() - fh) < 1e-14
        Jt = torch.autograd.functional.jacobian(step, st).numpy()
        np.testing.assert_allclose(J, Jt, atol=1e-12, rtol=0)


def test_gru_jacobian_finite_difference(oracle):
    """Central differences of the oracle's own step agree with its analytic Jacobian."""
    rng = np.random.default_rng(15)
    for _ in range(30):
        p = rng.standard_normal(3)
        w = rng.uniform(-0.5, 0.5, 3)
        h = rng.standard_normal()
        e = 1e-5
        fp, _ = oracle.gru_cell(p, w, h + e)
        fm, _ = oracle.gru_cell(p, w, h - e)
        _, J = oracle.gru_cell(p, w, h)
        assert abs((fp - fm) / (2 * e) - J) < 1e-8 * max(1, abs(J))


def test_lstm_jacobian_finite_difference(oracle):
    """Central differences of the oracle's own LSTM step in c and in h agree with
    all four entries of its analytic Jacobian (row-major d(c', h')/d(c, h))."""
    rng = np.random.default_rng(16)
    e = 1e-5
    for _ in range(30):
        p = rng.standard_normal(4)
        w = rng.uniform(-0.5, 0.5, 4)
        c, h = rng.standard_normal(2)
        _, _, J = oracle.lstm_cell(p, w, c, h)
        J = np.asarray(J).reshape(2, 2)
        cp, hp_, _ = oracle.lstm_cell(p, w, c + e, h)
        cm, hm, _ = oracle.lstm_cell(p, w, c - e, h)
        dc = np.array([(cp - cm) / (2 * e), (hp_ - hm) / (2 * e)])   # column d/dc
        cp, hp_, _ = oracle.lstm_cell(p, w, c, h + e)
        cm, hm, _ = oracle.lstm_cell(p, w, c, h - e)
        dh = np.array([(cp - cm) / (2 * e), (hp_ - hm) / (2 * e)])   # column d/dh
        fd = np.stack([dc, dh], axis=1)
        np.testing.assert_allclose(fd, J, atol=1e-8, rtol=1e-8)


def test_mhgru_jacobian_finite_difference(oracle):
    """Central differences of the oracle's own multi-head step, one input channel
    at a time, agree with its 8x8 Jacobian's columns."""
    rng = np.random.default_rng(17)
    e = 1e-5
    for _ in range(10):
        U = rng.uniform(-0.6, 0.6, (3, 8, 8))
        p = rng.standard_normal((3, 8))
        h = rng.standard_normal(8)
        _, J = oracle.mhgru_cell(p, U, h)
        for j in range(8):
            dh = np.zeros(8)
            dh[j] = e
            fp, _ = oracle.mhgru_cell(p, U, h + dh)
            fm, _ = oracle.mhgru_cell(p, U, h - dh)
            np.testing.assert_allclose((fp - fm) / (2 * e), J[:, j], atol=1e-8, rtol=1e-8)


# --------------------------------------------------------------------------
# Rollouts against the library cells
# --------------------------------------------------------------------------
def test_rollout_gru_matches_torch(oracle):
    x = inputs.gru_inputs(2, 40, 5, seed=20, h0_normal=True)
    h = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    ref = torch_gru_rollout(x["P"], x["a"], x["h0"])
    np.testing.assert_allclose(h, ref, atol=1e-13, rtol=0)


def test_rollout_lstm_matches_torch(oracle):
    x = inputs.lstm_inputs(2, 40, 5, seed=21, h0_normal=True)
    c, h = oracle.rollout_lstm(x["P"], x["a"], x["c0"], x["h0"])
    rc, rh = torch_lstm_rollout(x["P"], x["a"], x["c0"], x["h0"])
    np.testing.assert_allclose(c, rc, atol=1e-13, rtol=0)
    np.testing.assert_allclose(h, rh, atol=1e-13, rtol=0)


# --------------------------------------------------------------------------
# Newton
# --------------------------------------------------------------------------
def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def test_newton_gru_converges_to_rollout(oracle):
    x = inputs.gru_inputs(2, 200, 6, seed=22)
    res = oracle.newton_gru(x["P"], x["a"], x["h0"], tol=1e-12, max_iters=50)
    assert res.converged and not res.nonfinite
    ref = torch_gru_rollout(x["P"], x["a"], x["h0"])
    assert np.max(np.abs(res.h - ref)) < 1e-10


def test_newton_lstm_converges_to_rollout(oracle):
    x = inputs.lstm_inputs(2, 200, 6, seed=23)
    res = oracle.newton_lstm(x["P"], x["a"], x["c0"], x["h0"], tol=1e-12, max_iters=50)
    assert res.converged
    rc, rh = torch_lstm_rollout(x["P"], x["a"])
    assert np.max(np.abs(res.c - rc)) < 1e-10 and np.max(np.abs(res.h - rh)) < 1e-10


def test_newton_first_residual_is_max_of_first_step(oracle):
    """rho_0 at h^0 = 0 is max over (b, t, d) of |f(0, P_t)| (h0 = 0): the step from zero."""
    x = inputs.gru_inputs(3, 30, 4, seed=24)
    res = oracle.newton_gru(x["P"], x["a"], tol=1e-4, max_iters=3)
    cell = torch_gru_cell(4, x["a"])
    with torch.no_grad():
        f0 = torch_gru_step(cell, x["P"].astype(np.float64).reshape(90, 3, 4),
                            torch.zeros(90, 4)).numpy()
    assert abs(res.rho[0] - np.max(np.abs(f0))) < 1e-14


def test_newton_mingru_single_iteration(oracle):
    """a = 0 removes h from the gates (minGRU): the system is affine, one Newton step
    solves it, and the solution is the scan with A = 1 - z, b = z * tanh(Pc)."""
    x = inputs.gru_inputs(2, 300, 5, seed=25, h0_normal=True)
    a0 = np.zeros_like(x["a"])
    res = oracle.newton_gru(x["P"], a0, x["h0"], tol=1e-11, max_iters=10)
    assert res.converged and res.iterations == 1
    assert res.rho[1] < 1e-13
    P = x["P"].astype(np.float64)
    z = sigmoid(P[:, :, 0])
    c = np.tanh(P[:, :, 2])
    h_scan = oracle.scan_diag(1 - z, z * c, x["h0"])
    np.testing.assert_allclose(res.h, h_scan, atol=1e-13, rtol=0)


def test_newton_lstm_no_recurrence_two_iterations(oracle):
    """LSTM with a = 0: c' is affine in c (exact after one step), h' depends only on c',
    so the second step is exact too: exactly two iterations."""
    x = inputs.lstm_inputs(2, 100, 5, seed=26, h0_normal=True)
    res = oracle.newton_lstm(x["P"], np.zeros_like(x["a"]), x["c0"], x["h0"], tol=1e-11,
                             max_iters=10)
    assert res.converged and res.iterations == 2
    assert res.rho[1] > 1e-6


def test_newton_prefix_exactness_and_finite_termination(oracle):
    """After k updates the first k steps equal the rollout exactly (up to rounding);
    after L updates the whole trajectory does."""
    L = 8
    x = inputs.gru_inputs(2, L, 3, seed=27, h0_normal=True)
    ref = torch_gru_rollout(x["P"], x["a"], x["h0"])
    for k in range(1, L + 1):
        res = oracle.newton_gru(x["P"], x["a"], x["h0"], tol=0.0, max_iters=k)
        assert res.iterations == k
        np.testing.assert_allclose(res.h[:, :k], ref[:, :k], atol=1e-14, rtol=0)
    xl = inputs.lstm_inputs(2, L, 3, seed=28, h0_normal=True)
    rc, rh = torch_lstm_rollout(xl["P"], xl["a"], xl["c0"], xl["h0"])
    for k in range(1, L + 1):
        res = oracle.newton_lstm(xl["P"], xl["a"], xl["c0"], xl["h0"], tol=0.0, max_iters=k)
        np.testing.assert_allclose(res.h[:, :k], rh[:, :k], atol=1e-14, rtol=0)
        np.testing.assert_allclose(res.c[:, :k], rc[:, :k], atol=1e-14, rtol=0)


def test_newton_quadratic_convergence(oracle):
    """Newton converges quadratically: rho_{k+1} <= C rho_k^2 once rho_k is small.
    A wrong or missing Jacobian term degrades this to linear convergence."""
    for fn, mk in ((oracle.newton_gru, inputs.gru_inputs), (oracle.newton_lstm, inputs.lstm_inputs)):
        x = mk(4, 256, 8, seed=29)
        args = (x["P"], x["a"]) if fn is oracle.newton_gru else (x["P"], x["a"], x["c0"])
        res = fn(*args, tol=1e-13, max_iters=30)
        rho = res.rho
        assert res.converged
        checked = 0
        for k in range(len(rho) - 1):
            if 1e-9 < rho[k] < 0.05:
                assert rho[k + 1] <= 50.0 * rho[k] ** 2, (k, rho)
                checked += 1
        assert checked >= 1


def test_newton_steady_state_fixed_point(oracle):
    """Constant inputs over a long sequence: h_L reaches the scalar fixed point
    h* = f(h*), located by bisection on the library cell."""
    L = 400
    p = np.array([0.3, -0.4, 0.8])
    w = np.array([0.2, -0.3, 0.45])
    P = np.broadcast_to(p.reshape(1, 1, 3, 1), (1, L, 3, 1)).copy()
    res = oracle.newton_gru(P, w.reshape(3, 1), tol=1e-12, max_iters=60)
    cell = torch_gru_cell(1, w.reshape(3, 1))

    def g(hv):
        with torch.no_grad():
            return torch_gru_step(cell, p.reshape(1, 3, 1), torch.tensor([[hv]])).item() - hv

    lo, hi = -1.0, 1.0
    assert g(lo) * g(hi) < 0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if g(lo) * g(mid) <= 0:
            hi = mid
        else:
            lo = mid
    assert abs(res.h[0, -1, 0] - 0.5 * (lo + hi)) < 1e-11


def test_newton_nonconvergence_reported(oracle):
    x = inputs.gru_inputs(2, 64, 4, seed=30)
    res = oracle.newton_gru(x["P"], x["a"], tol=0.0, max_iters=2)
    assert not res.converged and res.iterations == 2 and len(res.rho) == 3


def test_newton_nonfinite_input_reported(oracle):
    x = inputs.gru_inputs(1, 16, 2, seed=31)
    P = x["P"].astype(np.float64)
    P[0, 5, 2, 1] = np.nan
    res = oracle.newton_gru(P, x["a"], tol=1e-4, max_iters=5)
    assert res.nonfinite and not res.converged


def test_channel_iteration_counts_bounded_by_global(oracle):
    x = inputs.gru_inputs(3, 128, 8, seed=32)
    res = oracle.newton_gru(x["P"], x["a"], tol=1e-6, max_iters=30)
    assert res.converged
    assert res.chan_iters.max() == res.iterations
    assert res.chan_iters.min() >= 0


def test_residual_certificate(oracle):
    x = inputs.gru_inputs(2, 50, 3, seed=33)
    ref = torch_gru_rollout(x["P"], x["a"])
    assert oracle.residual_gru(x["P"], x["a"], ref) < 1e-14
    bad = ref.copy()
    bad[1, -1, 2] += 3e-3          # the last step feeds nothing: residual equals the bump
    assert abs(oracle.residual_gru(x["P"], x["a"], bad) - 3e-3) < 1e-12


# --------------------------------------------------------------------------
# Seeded inputs
# --------------------------------------------------------------------------
def test_bf16_rounding_is_nearest_even():
    v = np.array([1.0, 1.00390625, 1.005859375, -2.5, 3.0e-3, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8],
                 np.float32)
    bits, vals = inputs.round_to_bf16(v)
    t = torch.tensor(v, dtype=torch.float32).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(vals, t)
    assert bits.dtype == np.uint16


def test_inputs_are_deterministic():
    a = inputs.gru_inputs(2, 10, 3, seed=5)
    b = inputs.gru_inputs(2, 10, 3, seed=5)
    np.testing.assert_array_equal(a["P"], b["P"])
    assert a["P"].dtype == np.float32 and a["P"].shape == (2, 10, 3, 3)
    assert np.all(np.abs(a["a"]) <= 0.5)


# --------------------------------------------------------------------------
# Backward pass: the adjoint recursion against autograd through the library cells
# --------------------------------------------------------------------------
def _autograd_gru(P, a, h0, gh):
    """dl/dP, dl/da, dl/dh0 for l = sum_t <gh_t, h_t>, with torch's GRU cell
    (weights built from a, so autograd reaches a through the diagonal)."""
    P = torch.tensor(np.asarray(P, np.float64), requires_grad=True)
    a = torch.tensor(np.asarray(a, np.float64), requires_grad=True)
    h = torch.tensor(np.asarray(h0, np.float64), requires_grad=True)
    B, L, _, D = P.shape
    w_ih = torch.eye(3 * D)
    w_hh = torch.cat([torch.diag(a[1]), torch.diag(-a[0]), torch.diag(a[2])])
    hs = []
    ht = h
    for t in range(L):
        x = torch.cat([P[:, t, 1], -P[:, t, 0], P[:, t, 2]], dim=-1)
        ht = torch._VF.gru_cell(x, ht, w_ih, w_hh, None, None)
        hs.append(ht)
    loss = (torch.stack(hs, 1) * torch.tensor(np.asarray(gh, np.float64))).sum()
    loss.backward()
    return P.grad.numpy(), a.grad.numpy(), h.grad.numpy()


def _autograd_lstm(P, a, c0, h0, gc, gh):
    P = torch.tensor(np.asarray(P, np.float64), requires_grad=True)
    a = torch.tensor(np.asarray(a, np.float64), requires_grad=True)
    c = torch.tensor(np.asarray(c0, np.float64), requires_grad=True)
    h = torch.tensor(np.asarray(h0, np.float64), requires_grad=True)
    B, L, _, D = P.shape
    w_ih = torch.eye(4 * D)
    w_hh = torch.cat([torch.diag(a[g]) for g in range(4)])
    cs, hs = [], []
    ct, ht = c, h
    for t in range(L):
        ht, ct = torch._VF.lstm_cell(P[:, t].reshape(B, 4 * D), (ht, ct), w_ih, w_hh, None, None)
        cs.append(ct)
        hs.append(ht)
    loss = (torch.stack(cs, 1) * torch.tensor(np.asarray(gc, np.float64))).sum() + \
        (torch.stack(hs, 1) * torch.tensor(np.asarray(gh, np.float64))).sum()
    loss.backward()
    return P.grad.numpy(), a.grad.numpy(), c.grad.numpy(), h.grad.numpy()


def test_backward_gru_matches_autograd(oracle):
    x = inputs.gru_inputs(2, 40, 5, seed=40, h0_normal=True)
    gh = np.random.default_rng(41).standard_normal((2, 40, 5))
    h = oracle.rollout_gru(x["P"], x["a"], x["h0"])
    dP, da, dh0 = oracle.backward_gru(x["P"], x["a"], h, gh, x["h0"])
    rP, ra, rh0 = _autograd_gru(x["P"], x["a"], x["h0"], gh)
    np.testing.assert_allclose(dP, rP, atol=1e-12, rtol=1e-10)
    np.testing.assert_allclose(da, ra, atol=1e-11, rtol=1e-10)
    np.testing.assert_allclose(dh0, rh0, atol=1e-12, rtol=1e-10)


def test_backward_lstm_matches_autograd(oracle):
    x = inputs.lstm_inputs(2, 40, 5, seed=42, h0_normal=True)
    rng = np.random.default_rng(43)
    gc = rng.standard_normal((2, 40, 5))
    gh = rng.standard_normal((2, 40, 5))
    c, h = oracle.rollout_lstm(x["P"], x["a"], x["c0"], x["h0"])
    dP, da, dc0, dh0 = oracle.backward_lstm(x["P"], x["a"], c, h, gc, gh, x["c0"], x["h0"])
    rP, ra, rc0, rh0 = _autograd_lstm(x["P"], x["a"], x["c0"], x["h0"], gc, gh)
    np.testing.assert_allclose(dP, rP, atol=1e-12, rtol=1e-10)
    np.testing.assert_allclose(da, ra, atol=1e-11, rtol=1e-10)
    np.testing.assert_allclose(dc0, rc0, atol=1e-12, rtol=1e-10)
    np.testing.assert_allclose(dh0, rh0, atol=1e-12, rtol=1e-10)


def test_backward_linear_recurrence_is_a_reverse_scan(oracle):
    """a = 0 (minGRU): J_t = 1 - z_t does not depend on h, so lambda is the reverse
    scan lambda_t = g_t + (1 - z_{t+1}) lambda_{t+1}, and dh0 = (1 - z_1) lambda_1."""
    x = inputs.gru_inputs(1, 25, 3, seed=44, h0_normal=True)
    a0 = np.zeros_like(x["a"])
    gh = np.random.default_rng(45).standard_normal((1, 25, 3))
    h = oracle.rollout_gru(x["P"], a0, x["h0"])
    dP, da, dh0 = oracle.backward_gru(x["P"], a0, h, gh, x["h0"])
    z = sigmoid(x["P"].astype(np.float64)[:, :, 0])                     # [1, L, D]
    # reverse scan as a forward scan over reversed time
    lam = oracle.scan_diag(np.concatenate([np.zeros((1, 1, 3)), (1 - z)[:, :0:-1]], 1),
                           gh[:, ::-1])[:, ::-1]
    np.testing.assert_allclose(dh0, (1 - z[:, 0]) * lam[:, 0], atol=1e-12)
    c = np.tanh(x["P"].astype(np.float64)[:, :, 2])
    hp = np.concatenate([x["h0"][:, None].astype(np.float64), h[:, :-1]], 1)
    np.testing.assert_allclose(dP[:, :, 0], lam * (c - hp) * z * (1 - z), atol=1e-12)


# --------------------------------------------------------------------------
# Input projection P = x W^T + bias
# --------------------------------------------------------------------------
def test_projection_selects_permuted_columns(oracle):
    """W with a single 1 per row, W[n, pi(n)] = 1, picks column pi(n) of x.  pi is
    a 7-cycle (not its own inverse), so a transposed W would pick pi^-1(n)."""
    rng = np.random.default_rng(700)
    K = 7
    pi = np.array([1, 2, 3, 4, 5, 6, 0])
    W = np.zeros((K, K))
    W[np.arange(K), pi] = 1.0
    x = rng.standard_normal((5, K))
    b = rng.standard_normal(K)
    assert np.array_equal(oracle.input_projection(x, W, b), x[:, pi] + b)


def test_projection_rectangular_selection(oracle):
    """N != K: each output feature is a scaled copy of one input feature."""
    rng = np.random.default_rng(701)
    M, N, K = 4, 3, 10
    W = np.zeros((N, K))
    W[[0, 1, 2], [7, 2, 9]] = [2.0, -1.0, 0.5]
    x = rng.standard_normal((M, K))
    expect = np.stack([2.0 * x[:, 7], -x[:, 2], 0.5 * x[:, 9]], axis=1)
    assert np.array_equal(oracle.input_projection(x, W), expect)


def test_projection_bias_only(oracle):
    rng = np.random.default_rng(702)
    b = rng.standard_normal(6)
    P = oracle.input_projection(rng.standard_normal((3, 5)), np.zeros((6, 5)), b)
    assert np.array_equal(P, np.broadcast_to(b, (3, 6)))
    P0 = oracle.input_projection(np.zeros((3, 0)), np.zeros((6, 0)), b)
    assert np.array_equal(P0, np.broadcast_to(b, (3, 6)))


def test_projection_small_integers_brute_force(oracle):
    """Integer operands: the sums are exact, so brute force in Python integers
    must agree bit for bit."""
    rng = np.random.default_rng(703)
    M, N, K = 3, 4, 5
    x = rng.integers(-3, 4, (M, K))
    W = rng.integers(-3, 4, (N, K))
    b = rng.integers(-5, 6, N)
    P = oracle.input_projection(x, W, b)
    for m in range(M):
        for n in range(N):
            s = int(b[n])
            for k in range(K):
                s += int(x[m, k]) * int(W[n, k])
            assert P[m, n] == s


def test_projection_rank_one(oracle):
    """x = u v^T  =>  P = u (W v)^T."""
    rng = np.random.default_rng(704)
    u, v = rng.standard_normal(6), rng.standard_normal(9)
    W = rng.standard_normal((5, 9))
    P = oracle.input_projection(np.outer(u, v), W)
    assert np.allclose(P, np.outer(u, W @ v), rtol=0, atol=1e-12)


def test_projection_matches_library_matmul(oracle):
    rng = np.random.default_rng(705)
    x, W, b = rng.standard_normal((33, 70)), rng.standard_normal((24, 70)), rng.standard_normal(24)
    assert np.allclose(oracle.input_projection(x, W, b), x @ W.T + b, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Multi-head GRU with dense 8x8 recurrence blocks
# --------------------------------------------------------------------------
def torch_mhgru_cell(U):
    """GRUCell(3D -> D) whose hidden-to-hidden weights are block-diagonal with the
    8x8 blocks of U [3, H, 8, 8]; x = [Pr, -Pz, Pc] as for ParaGRU (torch's z is
    1 - z, so its z-row gets -U_z)."""
    U = torch.as_tensor(np.asarray(U, np.float64))
    H = U.shape[1]
    D = 8 * H
    bd = [torch.block_diag(*[U[g, k] for k in range(H)]) for g in range(3)]
    cell = torch.nn.GRUCell(3 * D, D, bias=False).double()
    with torch.no_grad():
        cell.weight_ih.copy_(torch.eye(3 * D))
        cell.weight_hh.copy_(torch.cat([bd[1], -bd[0], bd[2]]))
    return cell


def test_mhgru_cell_matches_torch_gru_cell(oracle):
    rng = np.random.default_rng(720)
    for _ in range(20):
        U = rng.uniform(-0.8, 0.8, (3, 1, 8, 8))   # not symmetric: a transposed block fails
        p = rng.standard_normal((3, 8)) * 2
        h = rng.standard_normal(8)
        f, J = oracle.mhgru_cell(p, U[:, 0], h)
        cell = torch_mhgru_cell(U)
        ht = torch.tensor(h[None, :], requires_grad=True)
        out = torch_gru_step(cell, p[None], ht)
        np.testing.assert_allclose(out.detach().numpy()[0], f, atol=1e-14, rtol=0)
        Jt = torch.autograd.functional.jacobian(lambda x: torch_gru_step(cell, p[None], x), ht)
        np.testing.assert_allclose(Jt.numpy().reshape(8, 8), J, atol=1e-12, rtol=0)


def test_mhgru_rollout_matches_torch(oracle):
    x = inputs.mhgru_inputs(2, 40, 3, seed=721, h0_normal=True)
    cell = torch_mhgru_cell(x["U"])
    h = torch.as_tensor(x["h0"].astype(np.float64))
    ref = []
    with torch.no_grad():
        for t in range(40):
            h = torch_gru_step(cell, x["P"][:, t], h)
            ref.append(h)
    ref = torch.stack(ref, 1).numpy()
    np.testing.assert_allclose(oracle.rollout_mhgru(x["P"], x["U"], x["h0"]), ref, atol=1e-13,
                               rtol=0)


def test_mhgru_diagonal_blocks_are_paragru(oracle):
    """With every block diagonal the cell, the rollout and Newton's iterates are
    those of ParaGRU with a_g = the blocks' diagonals."""
    x = inputs.gru_inputs(2, 60, 16, seed=722)
    H = 2
    U = np.zeros((3, H, 8, 8))
    for g in range(3):
        for k in range(H):
            U[g, k] = np.diag(x["a"][g, 8 * k: 8 * k + 8])
    np.testing.assert_allclose(oracle.rollout_mhgru(x["P"], U), oracle.rollout_gru(x["P"], x["a"]),
                               atol=1e-14, rtol=0)
    rm = oracle.newton_mhgru(x["P"], U)
    rg = oracle.newton_gru(x["P"], x["a"])
    assert rm.iterations == rg.iterations
    np.testing.assert_allclose(rm.rho, rg.rho, rtol=0, atol=1e-14)
    np.testing.assert_allclose(rm.h, rg.h, atol=1e-14, rtol=0)


def test_mhgru_newton_converges_to_rollout(oracle):
    x = inputs.mhgru_inputs(2, 300, 2, seed=723, h0_normal=True)
    res = oracle.newton_mhgru(x["P"], x["U"], x["h0"], tol=1e-12, max_iters=50)
    assert res.converged
    np.testing.assert_allclose(res.h, oracle.rollout_mhgru(x["P"], x["U"], x["h0"]), atol=1e-10,
                               rtol=0)


def test_mhgru_no_recurrence_single_iteration(oracle):
    """U = 0: the gates do not depend on h, the step is affine in h, Newton is exact
    after one update."""
    x = inputs.mhgru_inputs(1, 100, 2, seed=724, h0_normal=True)
    U = np.zeros_like(x["U"])
    res = oracle.newton_mhgru(x["P"], U, x["h0"], tol=1e-12)
    assert res.iterations == 1 and res.rho[1] < 1e-13


def test_mhgru_newton_quadratic_convergence(oracle):
    """Newton on the dense-block system converges quadratically too (measured
    rho_{k+1} / rho_k^2 <= 0.22 at these seeds); a wrong or missing term of the
    8x8 Jacobian degrades it to linear convergence."""
    for seed, u_scale in ((726, 0.3), (728, 0.6)):
        x = inputs.mhgru_inputs(2, 256, 2, seed=seed, u_scale=u_scale)
        res = oracle.newton_mhgru(x["P"], x["U"], tol=1e-13, max_iters=30)
        assert res.converged
        rho = res.rho
        checked = 0
        for k in range(len(rho) - 1):
            if 1e-9 < rho[k] < 0.05:
                assert rho[k + 1] <= 50.0 * rho[k] ** 2, (k, rho)
                checked += 1
        assert checked >= 1


def test_mhgru_prefix_exactness(oracle):
    L = 6
    x = inputs.mhgru_inputs(2, L, 2, seed=725, u_scale=0.6, h0_normal=True)
    ref = oracle.rollout_mhgru(x["P"], x["U"], x["h0"])
    for k in range(1, L + 1):
        res = oracle.newton_mhgru(x["P"], x["U"], x["h0"], tol=0.0, max_iters=k)
        assert res.iterations == k
        np.testing.assert_allclose(res.h[:, :k], ref[:, :k], atol=1e-13, rtol=0)


# --------------------------------------------------------------------------
# Multi-head GRU with per-head time strides (DEER summary, caveats: heads with
# exponentially increasing strides): head g recurs on h_{t - s_g}
# --------------------------------------------------------------------------
def test_mhgru_strided_rollout_matches_torch(oracle):
    """A plain loop over torch's GRUCell in which each head reads its own lag."""
    B, L, H = 2, 37, 3
    strides = np.array([1, 2, 5], np.int32)
    x = inputs.mhgru_inputs(B, L, H, seed=724, h0_normal=True)
    cell = torch_mhgru_cell(x["U"])
    hist = []
    h0 = torch.as_tensor(x["h0"].astype(np.float64))
    with torch.no_grad():
        for t in range(L):
            # the state each head recurs on, assembled head by head
            prev = torch.cat([(hist[t - s] if t - s >= 0 else h0)[:, 8 * g:8 * g + 8]
                              for g, s in enumerate(strides)], 1)
            hist.append(torch_gru_step(cell, x["P"][:, t], prev))
    ref = torch.stack(hist, 1).numpy()
    got = oracle.rollout_mhgru(x["P"], x["U"], x["h0"], strides=strides)
    np.testing.assert_allclose(got, ref, atol=1e-13, rtol=0)


def test_mhgru_strided_head_is_interleaved_stride_one_sequences(oracle):
    """A head at stride s is s independent stride-1 sequences (t = r, r + s, ...):
    de-interleaving by slicing and solving each at stride 1 gives the same values."""
    B, L, H = 2, 50, 4
    strides = np.array([1, 3, 4, 7], np.int32)
    x = inputs.mhgru_inputs(B, L, H, seed=725, h0_normal=True)
    got = oracle.rollout_mhgru(x["P"], x["U"], x["h0"], strides=strides)
    for g, s in enumerate(strides):
        for r in range(s):
            sub = oracle.rollout_mhgru(x["P"][:, r::s, :, 8 * g:8 * g + 8], x["U"][:, g:g + 1],
                                       x["h0"][:, 8 * g:8 * g + 8])
            np.testing.assert_allclose(got[:, r::s, 8 * g:8 * g + 8], sub, atol=1e-14, rtol=0)
    # and the Newton solve at those strides reaches the same trajectory
    res = oracle.newton_mhgru(x["P"], x["U"], x["h0"], tol=1e-12, max_iters=50, strides=strides)
    assert res.converged
    np.testing.assert_allclose(res.h, got, atol=1e-10, rtol=0)


def test_mhgru_strides_beyond_the_sequence_are_one_explicit_step(oracle):
    """With every stride >= L each step depends on h0 only: the system is explicit,
    Newton is exact after one update, and h_t = cell(P_t, h0)."""
    B, L, H = 2, 9, 2
    x = inputs.mhgru_inputs(B, L, H, seed=726, h0_normal=True)
    strides = np.array([L, L + 5], np.int32)
    got = oracle.rollout_mhgru(x["P"], x["U"], x["h0"], strides=strides)
    for b in range(B):
        for t in range(L):
            for g in range(H):
                f, _ = oracle.mhgru_cell(x["P"][b, t][:, 8 * g:8 * g + 8], x["U"][:, g],
                                         x["h0"][b, 8 * g:8 * g + 8])
                np.testing.assert_allclose(got[b, t, 8 * g:8 * g + 8], f, atol=1e-15, rtol=0)
    res = oracle.newton_mhgru(x["P"], x["U"], x["h0"], tol=1e-12, max_iters=5, strides=strides)
    assert res.converged and res.iterations == 1
