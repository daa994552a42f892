"""The oracle still reproduces the fixtures in tests/golden/ (CPU only).

The fixtures are the oracle's own results on small seeded cases, written by
tests/golden/make_golden.py: the pages print no worked example to store.  They
guard the oracle against unannounced changes of its arithmetic.  Tolerance:
1e-12 relative (a different libm may round exp/tanh differently in the last
bit); iteration counts exactly.
"""
import importlib.util
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
_spec = importlib.util.spec_from_file_location(
    "make_golden", os.path.join(HERE, "golden", "make_golden.py"))
mg = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(mg)


@pytest.mark.parametrize("name", sorted(mg.CASES))
def test_oracle_matches_golden_fixture(name):
    with open(os.path.join(HERE, "golden", name)) as f:
        text = f.read()
    assert text.startswith("# "), "fixture header (what it is, where it comes from)"
    stored = mg.parse(text)
    what, B, L, D, seed = mg.CASES[name]
    now = mg.compute(what, B, L, D, seed)
    assert set(stored) == set(now)
    for key, val in now.items():
        if key == "iterations":
            assert stored[key] == int(val[0])
        else:
            np.testing.assert_allclose(np.asarray(val, np.float64), stored[key], rtol=1e-12,
                                       atol=1e-14, err_msg=f"{name}: {key}")


def test_fixture_files_are_exactly_the_cases():
    files = sorted(f for f in os.listdir(os.path.join(HERE, "golden")) if f.endswith(".txt"))
    assert files == sorted(mg.CASES)
