"""Writes the text fixtures of this folder with the fp64 oracle, and nothing else.

    python tests/golden/make_golden.py        (from the repository root)

The pages print no worked example (ParaRNN's Figures 2-5 survive only as
captions; the DEER summary gives timings, not values), so no fixture here holds
a value quoted from them.  Each file holds the oracle's own result on a small
seeded case. That makes it a regression guard, not an independent pin: a later
change to the oracle's arithmetic changes these numbers, fails
``tests/test_golden.py`` and has to be justified when the fixtures are
rewritten.  The inputs are not stored: they are the seeded draws of
``tests/inputs.py`` named in each header.
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# name -> (what, B, L, D, seed)
CASES = {
    "newton_gru_b2_l16_d3.txt": ("newton_gru", 2, 16, 3, [300]),
    "newton_lstm_b2_l16_d3.txt": ("newton_lstm", 2, 16, 3, [301]),
    "scan_diag_b2_l16_d3.txt": ("scan_diag", 2, 16, 3, [302]),
    "scan_block2_b1_l12_d2.txt": ("scan_block2", 1, 12, 2, [303]),
}

TITLES = {
    "newton_gru": "ParaGRU Newton solve (ParaRNN, Abstract and Figure 4 caption), tol 1e-4, h^0 = 0",
    "newton_lstm": "ParaLSTM Newton solve (ParaRNN, Abstract and Figure 2 caption), tol 1e-4, h^0 = 0",
    "scan_diag": "diagonal affine scan h_t = A_t h_{t-1} + b_t (ParaRNN, TL;DR)",
    "scan_block2": "2x2 block affine scan x_t = A_t x_{t-1} + b_t (ParaRNN, Figure 2 caption)",
}

RECIPES = {
    "newton_gru": "tests/inputs.py gru_inputs(B, L, D, seed, h0_normal=True)",
    "newton_lstm": "tests/inputs.py lstm_inputs(B, L, D, seed, h0_normal=True)",
    "scan_diag": "tests/inputs.py scan_diag_inputs(B, L, D, seed)",
    "scan_block2": "tests/inputs.py scan_block2_inputs(B, L, D, seed)",
}


def compute(what, B, L, D, seed):
    """The oracle's result on the case, as named flat arrays."""
    import oracle
    from tests import inputs

    if what == "newton_gru":
        x = inputs.gru_inputs(B, L, D, seed, h0_normal=True)
        r = oracle.newton_gru(x["P"], x["a"], x["h0"], tol=1e-4, max_iters=32)
        return {"iterations": np.array([r.iterations]), "rho": r.rho, "h": r.h.ravel()}
    if what == "newton_lstm":
        x = inputs.lstm_inputs(B, L, D, seed, h0_normal=True)
        r = oracle.newton_lstm(x["P"], x["a"], x["c0"], x["h0"], tol=1e-4, max_iters=32)
        return {"iterations": np.array([r.iterations]), "rho": r.rho, "c": r.c.ravel(),
                "h": r.h.ravel()}
    if what == "scan_diag":
        x = inputs.scan_diag_inputs(B, L, D, seed)
        return {"h": oracle.scan_diag(x["A"], x["b"], x["h0"]).ravel()}
    if what == "scan_block2":
        x = inputs.scan_block2_inputs(B, L, D, seed)
        return {"x": oracle.scan_block2(x["A"], x["b"], x["x0"]).ravel()}
    raise ValueError(what)


def render(name):
    what, B, L, D, seed = CASES[name]
    vals = compute(what, B, L, D, seed)
    lines = [f"# {TITLES[what]}",
             f"# B={B} L={L} D={D}; inputs: {RECIPES[what]} with seed={seed}",
             "# written by tests/golden/make_golden.py with the fp64 oracle (a regression guard,",
             "# not a value from the pages); arrays flattened in C order, t = 1..L"]
    for key, arr in vals.items():
        if key == "iterations":
            lines.append(f"{key}: {int(arr[0])}")
        else:
            lines.append(f"{key}: " + " ".join(repr(float(v)) for v in np.asarray(arr, np.float64)))
    return "\n".join(lines) + "\n"


def parse(text):
    out = {}
    for line in text.splitlines():
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(":")
        vals = rest.split()
        out[key.strip()] = (int(vals[0]) if key.strip() == "iterations"
                            else np.array([float(v) for v in vals]))
    return out


def main():
    for name in CASES:
        with open(os.path.join(HERE, name), "w") as f:
            f.write(render(name))
        print("wrote", name)


if __name__ == "__main__":
    main()
