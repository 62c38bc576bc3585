"""The oracle against its frozen output on one small problem (tests/golden/tiny_regression.json,
written by tests/golden/make_tiny_regression.py from the oracle itself).  The pages print no worked
example, so this pins the oracle only against unexplained changes; its agreement with the pages
rests on the closed forms and special cases in test_oracle_pins.py."""
import json
import os

import numpy as np

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_frozen_tiny_problem():
    with open(os.path.join(HERE, "golden", "tiny_regression.json")) as f:
        g = json.load(f)
    x = {k: np.asarray(v, dtype=np.float64) for k, v in g["inputs"].items()}
    o, S = oracle.recurrence(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"])
    np.testing.assert_allclose(o, np.asarray(g["o"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(S, np.asarray(g["S_T"]), rtol=0, atol=1e-13)
