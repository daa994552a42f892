"""Parity of the tensor-core input projection P = x W^T + bias with the fp64
oracle, through the C ABI.

Both sides read the same bf16 x and W (the oracle widens them exactly).  The
GPU multiplies bf16 pairs exactly and accumulates in fp32, so per element
|P - ref| <= 2 K 2^-23 sum_k |x_k W_nk| (a bound for K fp32 additions, doubled
to allow truncating accumulation); a bf16 output adds the rounding to nearest
even, at most 2^-8 |ref|.
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


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def check(P, x, W, b, out_bf16, rows=None):
    """P (numpy fp32) against the oracle on the given rows of x."""
    xs = x if rows is None else x[rows]
    ref = oracle.input_projection(xs, W, b)
    scale = oracle.input_projection(np.abs(xs), np.abs(W), None if b is None else np.abs(b))
    K = W.shape[1]
    tol = 2.0 * K * 2.0 ** -23 * scale + 1e-30
    if out_bf16:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    err = np.abs(P.astype(np.float64) - ref)
    assert np.all(err <= tol), (float(err.max()), float((err / tol).max()))


# K <= 2048 runs on CTA pairs, larger K on single CTAs: both kernels are covered
SHAPES = [(128, 256, 64), (300, 264, 200), (1, 8, 8), (37, 40, 1024), (129, 512, 136),
          (1000, 3072, 1024), (257, 384, 2056), (520, 264, 4096)]


@pytest.mark.parametrize("out_bf16", [False, True])
@pytest.mark.parametrize("with_bias", [False, True])
@pytest.mark.parametrize("shape", SHAPES)
def test_projection_parity(pr, shape, with_bias, out_bf16):
    M, N, K = shape
    d = inputs.projection_inputs(M, N, K, seed=[710, M, N, K])
    b = d["bias"] if with_bias else None
    P = pr.input_projection(bf16_dev(d["x_bits"]), bf16_dev(d["W_bits"]),
                            None if b is None else dev(b),
                            out_dtype=torch.bfloat16 if out_bf16 else torch.float32)
    torch.cuda.synchronize()
    check(P.float().cpu().numpy(), d["x"], d["W"], b, out_bf16)


def test_projection_batched_leading_dims(pr):
    """x [B, L, K] -> P [B, L, N] = [B, L, G, D]."""
    B, L, K, G, D = 2, 70, 96, 3, 40
    d = inputs.projection_inputs(B * L, G * D, K, seed=711)
    x = bf16_dev(d["x_bits"]).view(B, L, K)
    P = pr.input_projection(x, bf16_dev(d["W_bits"]), dev(d["bias"]))
    torch.cuda.synchronize()
    assert tuple(P.shape) == (B, L, G * D)
    check(P.cpu().numpy().reshape(B * L, G * D), d["x"], d["W"], d["bias"], False)


def test_projection_k_zero_writes_bias(pr):
    M, N = 5, 16
    b = np.arange(N, dtype=np.float32)
    x = torch.empty((M, 0), dtype=torch.bfloat16, device="cuda")
    W = torch.empty((N, 0), dtype=torch.bfloat16, device="cuda")
    P = pr.input_projection(x, W, dev(b))
    P0 = pr.input_projection(x, W)
    torch.cuda.synchronize()
    assert np.array_equal(P.cpu().numpy(), np.broadcast_to(b, (M, N)))
    assert not P0.cpu().numpy().any()


def test_projection_empty_m(pr):
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    st = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    P = pr.input_projection(x, W, status=st)
    torch.cuda.synchronize()
    assert P.shape == (0, 16) and int(st.item()) == 0


def test_projection_status_zero_on_success(pr):
    d = inputs.projection_inputs(256, 512, 128, seed=712)
    st = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    pr.input_projection(bf16_dev(d["x_bits"]), bf16_dev(d["W_bits"]), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def test_projection_full_size_sampled_rows(pr):
    """The projection workload at its full size (M = 8 * 4096, N = 3 * 1024,
    K = 1024), rows sampled across every M tile and the last one."""
    w = inputs.WORKLOADS["proj"]
    M, N, K = w["B"] * w["L"], w["G"] * w["D"], w["K"]
    d = inputs.projection_inputs(M, N, K, seed=w["seed"])
    P = pr.input_projection(bf16_dev(d["x_bits"]), bf16_dev(d["W_bits"]), dev(d["bias"]))
    torch.cuda.synchronize()
    rng = np.random.default_rng(713)
    rows = np.unique(np.concatenate([rng.integers(0, M, 96), np.arange(0, M, 4099), [M - 1]]))
    check(P[torch.from_numpy(rows).cuda()].cpu().numpy(), d["x"], d["W"], d["bias"], False, rows)


def test_projection_then_solve(pr):
    """x -> P on the tensor cores -> Newton solve on the GPU, against the
    oracle's fp64 projection followed by the fp64 sequential rollout."""
    B, L, K, D = 2, 600, 256, 64
    d = inputs.projection_inputs(B * L, 3 * D, K, seed=714)
    a = np.random.default_rng(715).uniform(-0.5, 0.5, (3, D)).astype(np.float32)
    x = bf16_dev(d["x_bits"]).view(B, L, K)
    P = pr.input_projection(x, bf16_dev(d["W_bits"]), dev(d["bias"])).view(B, L, 3, D)
    h, info = pr.solve_gru(P, dev(a))
    torch.cuda.synchronize()
    Pref = oracle.input_projection(d["x"], d["W"], d["bias"]).reshape(B, L, 3, D)
    href = oracle.rollout_gru(Pref, a)
    assert info.converged
    assert np.max(np.abs(h.cpu().numpy() - href)) <= 1e-4
