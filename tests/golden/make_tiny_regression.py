"""Writes tiny_regression.json: the fp64 oracle's o and S_T on one small seeded problem.

The pages print no worked numeric example of the recurrence, so no fixture here holds a
value taken from them.  This file freezes the oracle's own output on a problem small enough
to read (B=1, H=1, T=5, d_k=3, d_v=2), so that any later change to the oracle's arithmetic
shows up as a test failure that its commit has to explain.  Run from the repository root:

    python tests/golden/make_tiny_regression.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402


def problem():
    rng = np.random.default_rng(20261202)
    T, K, V = 5, 3, 2
    q = rng.normal(size=(1, T, 1, K))
    k = rng.normal(size=(1, T, 1, K))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(1, T, 1, V))
    alpha = np.exp(-np.log1p(np.exp(rng.normal(size=(1, T, 1, K)))))
    b = 1.0 / (1.0 + np.exp(-rng.normal(size=(1, T, 1, K))))
    w = 1.0 / (1.0 + np.exp(-rng.normal(size=(1, T, 1, V))))
    S0 = rng.normal(scale=0.1, size=(1, 1, K, V))
    return dict(q=q, k=k, v=v, alpha=alpha, b=b, w=w, S0=S0)


def main():
    p = problem()
    o, S = oracle.recurrence(p["q"], p["k"], p["v"], p["alpha"], p["b"], p["w"], p["S0"])
    out = {"inputs": {key: val.tolist() for key, val in p.items()}, "o": np.asarray(o).tolist(),
           "S_T": np.asarray(S).tolist()}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_regression.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
