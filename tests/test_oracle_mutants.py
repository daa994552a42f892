"""The pins catch plausible mistakes in the oracle (CPU only).

Each case plants one mistake in a copy of oracle.c -- a dropped Jacobian term,
a flipped sign, an index off by one step, a transposed 2x2 operand, swapped
LSTM gates, a forgotten initial state -- builds it, points the oracle package
at it and runs the pins of tests/test_oracle_pins.py.  At least one pin must
fail for every mistake; the unmodified oracle passes them all.
"""
import inspect
import os
import shutil

import pytest
import torch

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.abspath(oracle.__file__)), "oracle.c")

MUTANTS = {
    "gru_jacobian_drops_c_dz": ("*J = (1.0 - z) - h * dz + c * dz + z * dc;",
                                "*J = (1.0 - z) - h * dz + z * dc;"),
    "gru_jacobian_dr_sign": ("double du = w[2] * (r + h * dr);", "double du = w[2] * (r - h * dr);"),
    "newton_residual_sign": ("x->rt[i] = f - x->h[i];", "x->rt[i] = x->h[i] - f;"),
    "newton_previous_step_index": (
        "x->h[IDX3(bb, t - 1, d, L, D)];\n"
        "    double pg[3];\n"
        "    for (int g = 0; g < 3; ++g) pg[g] = x->P[IDXP(bb, t, g, d, L, 3, D)];\n"
        "    double f, J;",
        "x->h[IDX3(bb, t, d, L, D)];\n"
        "    double pg[3];\n"
        "    for (int g = 0; g < 3; ++g) pg[g] = x->P[IDXP(bb, t, g, d, L, 3, D)];\n"
        "    double f, J;"),
    "scan_diag_misplaced_offset": ("x = c->A[i] * x + c->b[i];", "x = c->A[i] * (x + c->b[i]);"),
    "scan_block2_transposed": (
        "double n0 = M[0] * u0 + M[1] * u1 + c->b[2 * i + 0];\n"
        "    double n1 = M[2] * u0 + M[3] * u1 + c->b[2 * i + 1];",
        "double n0 = M[0] * u0 + M[2] * u1 + c->b[2 * i + 0];\n"
        "    double n1 = M[1] * u0 + M[3] * u1 + c->b[2 * i + 1];"),
    "lstm_gates_swapped": ("double cn = f * c + i * g;", "double cn = i * c + f * g;"),
    "lstm_jacobian_drops_o": ("J[2] = o * dtc * dcn_dc;", "J[2] = dtc * dcn_dc;"),
    "gru_rollout_ignores_h0": ("double s = x->h0 ? x->h0[bb * D + d] : 0.0;", "double s = 0.0;"),
    "newton_solve_drops_carry": ("delta = x->Jt[i] * delta + x->rt[i];", "delta = x->rt[i];"),
    "backward_gru_drops_r_derivative": ("double dfdr = dfdu * w[2] * hp * r * (1.0 - r);",
                                        "double dfdr = dfdu * w[2] * hp * r;"),
    "backward_lstm_untransposed_jacobian": ("mc = J[0] * lc + J[2] * lh;\n    mh = J[1] * lc + J[3] * lh;",
                                            "mc = J[0] * lc + J[1] * lh;\n    mh = J[2] * lc + J[3] * lh;"),
    "mhgru_reset_gate_inside": ("double c = tanh(p[2 * NB + i] + r * uc[i]);",
                                "double c = tanh(p[2 * NB + i] + uc[i]);"),
    "mhgru_jacobian_drops_ur": ("uc[i] * r * (1.0 - r) * U[(1 * NB + i) * NB + j]);",
                                "0.0 * U[(1 * NB + i) * NB + j]);"),
    "mhgru_transposed_block": ("uz[i] += U[(0 * NB + i) * NB + j] * h[j];",
                               "uz[i] += U[(0 * NB + j) * NB + i] * h[j];"),
    "projection_transposed_w": ("s += c->x[m * c->K + k] * c->W[n * c->K + k];",
                                "s += c->x[m * c->K + k] * c->W[k * c->N + n];"),
    "projection_drops_bias": ("double s = c->bias ? c->bias[n] : 0.0;", "double s = 0.0;"),
    "projection_skips_first_k": ("for (int64_t k = 0; k < c->K; ++k) s +=",
                                 "for (int64_t k = 1; k < c->K; ++k) s +="),
    "backward_gru_forward_time": ("double lam = x->gh[IDX3(bb, t, d, L, D)] + lam_next;",
                                  "double lam = x->gh[IDX3(bb, t, d, L, D)];"),
    "rho_max_over_first_channel_only": (
        "  for (int64_t c = 0; c < n; ++c) {\n    if (!(cmax[c] <= rho)) rho = cmax[c];",
        "  for (int64_t c = 0; c < 1; ++c) {\n    if (!(cmax[c] <= rho)) rho = cmax[c];"),
    "rho_drops_nan": ("if (!(cmax[c] <= rho)) rho = cmax[c];", "if (cmax[c] > rho) rho = cmax[c];"),
    "scan_diag_ignores_h0": ("  double x = c->x0 ? c->x0[bb * c->D + d] : 0.0;", "  double x = 0.0;"),
    "lstm_rollout_ignores_c0": ("double sc = x->c0 ? x->c0[bb * D + d] : 0.0;", "double sc = 0.0;"),
    "newton_lstm_ignores_c0": (
        "  double m = 0.0;\n  for (int64_t t = 0; t < L; ++t) {\n    double cp, hp;\n    if (t == 0) {\n"
        "      cp = x->c0 ? x->c0[bb * D + d] : 0.0;",
        "  double m = 0.0;\n  for (int64_t t = 0; t < L; ++t) {\n    double cp, hp;\n    if (t == 0) {\n"
        "      cp = 0.0;"),
    "backward_gru_da_z_without_h": ("da[0] += lam * dfdz * hp;", "da[0] += lam * dfdz;"),
    "backward_lstm_dh0_from_c": ("if (x->dh0) x->dh0[bb * D + d] = mh;",
                                 "if (x->dh0) x->dh0[bb * D + d] = mc;"),
    "backward_lstm_da_without_h": ("      da[g] += v * hp;", "      da[g] += v;"),
    "mhgru_ignores_h0": ("hp[i] = (tp < 0) ? (x->h0 ? x->h0[bb * D + g * NB + i] : 0.0)",
                         "hp[i] = (tp < 0) ? 0.0"),
    "mhgru_stride_ignored": ("int64_t D = NB * x->H, tp = t - mh_stride(x, g);",
                             "int64_t D = NB * x->H, tp = t - 1;"),
    "mhgru_newton_delta_lag_one": (
        "prev[j] = (t - st < 0) ? 0.0 : x->dt[IDX3(bb, t - st, g * NB + j, L, D)];",
        "prev[j] = (t - 1 < 0) ? 0.0 : x->dt[IDX3(bb, t - 1, g * NB + j, L, D)];"),
}


def _pin_functions():
    out = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if name.startswith("test_") and "oracle" in inspect.signature(fn).parameters:
            out.append(fn)
    return out


def _failures_with(lib):
    saved = oracle._lib
    old_dtype = torch.get_default_dtype()
    failed = []
    try:
        oracle._lib = lib
        torch.set_default_dtype(torch.float64)
        for fn in _pin_functions():
            try:
                fn(oracle)
            except AssertionError:
                failed.append(fn.__name__)
    finally:
        oracle._lib = saved
        torch.set_default_dtype(old_dtype)
    return failed


def test_unmodified_oracle_passes_every_pin(tmp_path):
    shutil.copy(SRC, tmp_path / "o.c")
    lib = oracle.compile_variant(str(tmp_path / "o.c"), str(tmp_path / "o.so"))
    assert _failures_with(lib) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    (tmp_path / "o.c").write_text(src.replace(old, new))
    lib = oracle.compile_variant(str(tmp_path / "o.c"), str(tmp_path / "o.so"))
    failed = _failures_with(lib)
    assert failed, f"no pin caught the planted mistake {name}"
