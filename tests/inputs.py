"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module holds no arithmetic of the method: it only draws random numbers
(numpy PCG64 ``default_rng``) in a fixed order and, for bf16 workloads, rounds
the fp32 draws to bf16 once (round to nearest even).  Both sides receive the
same bytes: the CUDA library reads the bf16 bits, the oracle reads the same
values widened exactly to fp64.

The pages measure on evaluation datasets and language-model corpora (ParaRNN
Figure 4 caption; DEER summary's task table).  None of those is used here:
these synthetic draws stand in for them, with the shapes of the workloads:

=======  =====================================  ==========================
name     operation                              shape (B, L, D)
=======  =====================================  ==========================
gru_s    ParaGRU solve, fp32                    2, 512, 16
scan     diagonal affine scan, fp32             8, 4096, 1024
gru_l    ParaGRU solve, fp32, L sweep 2^6..2^14 8, L, 1024
gru_bwd  ParaGRU backward pass, fp32           8, 4096, 1024
lstm_bwd ParaLSTM backward pass, fp32          8, 4096, 1024
lstm     ParaLSTM solve, fp32 (+ block scan)    8, 4096, 1024
deer     ParaGRU solve, fp32, DEER shape        16, 2^20, 1
lm       ParaGRU solve, bf16 P, fp32 state      8, 8192, 4096
scan_lm  diagonal affine scan, fp32, LM width   8, 8192, 4096
proj     input projection x W^T (+bias), G=3    8, 4096, 1024, K = 1024
proj_lm  input projection, LM width, G=3        8, 8192, 4096, K = 4096
proj_solve projection fused with the GRU solve   8, 8192, 4096, K = 4096
mhgru    multi-head GRU, 8x8 blocks, fp32       8, 4096, 1024 (128 heads)
=======  =====================================  ==========================

Distributions: projected gate inputs P ~ N(0, 1); diagonal recurrence weights
a ~ U(-0.5, 0.5); h0 = c0 = 0 for the solves.  Diagonal scan: A ~ U(0, 1),
b ~ N(0, 1), h0 ~ N(0, 1).  Block scan: A entries ~ U(-0.5, 0.5), b ~ N(0, 1),
x0 ~ N(0, 1).  Draw order: P (or A) first, then a (or b), then h0 (or x0).
Backward passes: the forward workload's inputs, and upstream gradients
dl/dh (and dl/dc) ~ N(0, 1) from their own generator.
Multi-head GRU: U blocks ~ U(-0.3, 0.3) (so that each 8x8 block has norm
below 1, like the diagonal a ~ U(-0.5, 0.5)).
Input projection: x ~ N(0, 1) and W ~ N(0, 1/K), both rounded to bf16 once,
bias ~ N(0, 0.1^2) fp32 (draw order x, W, bias), so that P = x W^T + bias has
about the N(0, 1) spread of the solves' P.
"""
from __future__ import annotations

import numpy as np

WORKLOADS = {
    "gru_s": dict(op="gru", B=2, L=512, D=16, seed=1, bf16=False),
    "scan": dict(op="scan_diag", B=8, L=4096, D=1024, seed=2, bf16=False),
    "gru_l": dict(op="gru", B=8, L=4096, D=1024, seed=2, bf16=False),
    "lstm": dict(op="lstm", B=8, L=4096, D=1024, seed=3, bf16=False),
    "block2": dict(op="scan_block2", B=8, L=4096, D=1024, seed=3, bf16=False),
    "deer": dict(op="gru", B=16, L=1 << 20, D=1, seed=4, bf16=False),
    "lm": dict(op="gru", B=8, L=8192, D=4096, seed=5, bf16=True),
    "scan_lm": dict(op="scan_diag", B=8, L=8192, D=4096, seed=9, bf16=False),
    "gru_bwd": dict(op="gru_bwd", B=8, L=4096, D=1024, seed=2, bf16=False),
    "lstm_bwd": dict(op="lstm_bwd", B=8, L=4096, D=1024, seed=3, bf16=False),
    "mhgru": dict(op="mhgru", B=8, L=4096, D=1024, seed=8, bf16=False),
    "proj": dict(op="proj", B=8, L=4096, D=1024, K=1024, G=3, seed=6, bf16=False),
    "proj_lm": dict(op="proj", B=8, L=8192, D=4096, K=4096, G=3, seed=7, bf16=True),
    "proj_solve": dict(op="proj_solve", B=8, L=8192, D=4096, K=4096, G=3, seed=10, bf16=True),
}

L_SWEEP = [1 << e for e in range(6, 15)]


def _rng(seed):
    return np.random.default_rng(seed)


def round_to_bf16(x32: np.ndarray):
    """Round fp32 values to bf16 (nearest even).  Returns (bits uint16, values fp32)."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    bits = ((u + bias) >> np.uint32(16)).astype(np.uint16)
    vals = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return bits, vals


def _normal(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


def _uniform(rng, lo, hi, shape):
    return (rng.random(size=shape, dtype=np.float32) * np.float32(hi - lo) + np.float32(lo)).astype(
        np.float32)


def gate_inputs(G, B, L, D, seed, bf16=False, h0_normal=False):
    """Projected pre-activations P [B,L,G,D], weights a [G,D], initial state.

    Returns a dict with ``P`` (fp32 values, already bf16-rounded if ``bf16``),
    ``P_bits`` (uint16 bf16 bits or None), ``a`` [G,D] fp32 and ``h0`` [B,D]
    (and ``c0`` for G == 4) fp32, zeros unless ``h0_normal``.
    """
    rng = _rng(seed)
    P = _normal(rng, (B, L, G, D))
    a = _uniform(rng, -0.5, 0.5, (G, D))
    out = {}
    if h0_normal:
        out["h0"] = _normal(rng, (B, D))
        if G == 4:
            out["c0"] = _normal(rng, (B, D))
    else:
        out["h0"] = np.zeros((B, D), np.float32)
        if G == 4:
            out["c0"] = np.zeros((B, D), np.float32)
    bits = None
    if bf16:
        bits, P = round_to_bf16(P)
    out.update(P=P, P_bits=bits, a=a)
    return out


def gru_inputs(B, L, D, seed, bf16=False, h0_normal=False):
    return gate_inputs(3, B, L, D, seed, bf16, h0_normal)


def lstm_inputs(B, L, D, seed, bf16=False, h0_normal=False):
    return gate_inputs(4, B, L, D, seed, bf16, h0_normal)


def scan_diag_inputs(B, L, D, seed, a_lo=0.0, a_hi=1.0):
    rng = _rng(seed)
    A = _uniform(rng, a_lo, a_hi, (B, L, D))
    b = _normal(rng, (B, L, D))
    h0 = _normal(rng, (B, D))
    return dict(A=A, b=b, h0=h0)


def scan_block2_inputs(B, L, D, seed, a_lo=-0.5, a_hi=0.5):
    rng = _rng(seed)
    A = _uniform(rng, a_lo, a_hi, (B, L, D, 2, 2))
    b = _normal(rng, (B, L, D, 2))
    x0 = _normal(rng, (B, D, 2))
    return dict(A=A, b=b, x0=x0)


def workload_inputs(name, L=None):
    """Inputs of a named workload (``L`` overrides the length for the sweep)."""
    w = dict(WORKLOADS[name])
    if L is not None:
        w["L"] = L
        seed = [w["seed"], L]
    else:
        seed = w["seed"]
    op = w["op"]
    if op == "gru":
        return gru_inputs(w["B"], w["L"], w["D"], seed, w["bf16"])
    if op == "lstm":
        return lstm_inputs(w["B"], w["L"], w["D"], seed, w["bf16"])
    if op == "scan_diag":
        return scan_diag_inputs(w["B"], w["L"], w["D"], seed)
    if op == "scan_block2":
        return scan_block2_inputs(w["B"], w["L"], w["D"], seed)
    raise KeyError(op)


def upstream_gradients(B, L, D, seed, n=1):
    """n arrays [B, L, D] of fp32 N(0, 1) draws: the upstream gradients dl/dh (, dl/dc)."""
    rng = _rng([seed, 97])
    return [_normal(rng, (B, L, D)) for _ in range(n)]


def projection_inputs(M, N, K, seed):
    """x [M, K] and W [N, K] as bf16 (bits uint16, values fp32), bias [N] fp32."""
    rng = _rng(seed)
    x_bits, x = round_to_bf16(_normal(rng, (M, K)))
    w32 = (_normal(rng, (N, K)) * np.float32(1.0 / np.sqrt(max(K, 1)))).astype(np.float32)
    w_bits, W = round_to_bf16(w32)
    bias = (_normal(rng, (N,)) * np.float32(0.1)).astype(np.float32)
    return dict(x=x, x_bits=x_bits, W=W, W_bits=w_bits, bias=bias)


def projected_gru_inputs(B, L, D, K, seed, h0_normal=False):
    """A ParaGRU layer from its inputs: x [B, L, K] and W [3 D, K] as bf16 (bits
    and values), bias [3 D] (as projection_inputs with M = B L, N = 3 D), then
    a [3, D] ~ U(-0.5, 0.5) and h0 [B, D] (zeros, or N(0, 1)).  Draw order x, W,
    bias, a, h0."""
    rng = _rng(seed)
    x_bits, x = round_to_bf16(_normal(rng, (B * L, K)))
    w32 = (_normal(rng, (3 * D, K)) * np.float32(1.0 / np.sqrt(max(K, 1)))).astype(np.float32)
    w_bits, W = round_to_bf16(w32)
    bias = (_normal(rng, (3 * D,)) * np.float32(0.1)).astype(np.float32)
    a = _uniform(rng, -0.5, 0.5, (3, D))
    h0 = _normal(rng, (B, D)) if h0_normal else np.zeros((B, D), np.float32)
    return dict(x=x.reshape(B, L, K), x_bits=x_bits.reshape(B, L, K), W=W, W_bits=w_bits,
                bias=bias, a=a, h0=h0)


def mhgru_inputs(B, L, H, seed, u_scale=0.3, h0_normal=False):
    """Multi-head GRU (dense 8x8 recurrence blocks): P [B, L, 3, 8H] ~ N(0, 1),
    U [3, H, 8, 8] ~ U(-u_scale, u_scale), h0 zeros (or N(0, 1)).  Draw order P, U, h0."""
    rng = _rng(seed)
    D = 8 * H
    P = _normal(rng, (B, L, 3, D))
    U = _uniform(rng, -u_scale, u_scale, (3, H, 8, 8))
    h0 = _normal(rng, (B, D)) if h0_normal else np.zeros((B, D), np.float32)
    return dict(P=P, U=U, h0=h0)
