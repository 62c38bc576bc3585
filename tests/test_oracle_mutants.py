"""Plant one plausible mistake at a time in a COPY of the oracle (CPU only) and
check that the pins of test_oracle_pins.py catch every one of them.

Each mutant is a textual edit of oracle/gdn2_oracle.c compiled with gcc into a
temporary directory; the real oracle is never modified.
"""
import os

import numpy as np
import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn2_oracle.c")

# (name, text in the source, replacement)
MUTANTS = [
    ("decay_squared", "S[(size_t)c * V + j] *= at[c];", "S[(size_t)c * V + j] *= at[c] * at[c];"),
    ("decay_dropped", "S[(size_t)c * V + j] *= at[c];", "S[(size_t)c * V + j] *= 1.0;"),
    ("erase_gate_dropped", "const double e = bt[c] * kt[c];", "const double e = kt[c];"),
    ("erase_uses_q", "const double e = bt[c] * kt[c];", "const double e = bt[c] * qt[c];"),
    ("write_gate_dropped", "(wt[j] * vt[j] - r[j])", "(vt[j] - r[j])"),
    ("erase_sign", "(wt[j] * vt[j] - r[j])", "(wt[j] * vt[j] + r[j])"),
    ("outer_uses_b", "S[(size_t)c * V + j] += kt[c] * (", "S[(size_t)c * V + j] += bt[c] * kt[c] * ("),
    ("readout_uses_k", "ot[j] += qt[c] * S[(size_t)c * V + j];", "ot[j] += kt[c] * S[(size_t)c * V + j];"),
    ("readout_scaled", "ot[j] += qt[c] * S[(size_t)c * V + j];", "ot[j] += 0.5 * qt[c] * S[(size_t)c * V + j];"),
    ("state_reset_each_token", "        /* X = Diag(alpha_t) S_{t-1}: row c of S is scaled by alpha_t[c] */",
     "        if (t > 0 && t % 3 == 0) memset(S, 0, sizeof(double) * (size_t)K * V);\n"
     "        /* X = Diag(alpha_t) S_{t-1}: row c of S is scaled by alpha_t[c] */"),
    ("s0_ignored", "    if (J->S0)\n", "    if (0)\n"),
    ("erase_before_decay",
     "        /* X = Diag(alpha_t) S_{t-1}: row c of S is scaled by alpha_t[c] */\n"
     "        for (int c = 0; c < K; ++c)\n"
     "            for (int j = 0; j < V; ++j) S[(size_t)c * V + j] *= at[c];\n",
     ""),
    ("decay_after_update",
     "        /* o_t = S_t^T q_t */\n",
     "        for (int c = 0; c < K; ++c)\n"
     "            for (int j = 0; j < V; ++j) S[(size_t)c * V + j] *= at[c];\n"
     "        /* o_t = S_t^T q_t */\n"),
]


def _pin_suite(lib, rng):
    """Run a compact version of the pins against `lib`; return the names that fail."""
    failed = []

    def rec(*a):
        return oracle.recurrence(*a, lib=lib, threads=1)

    # brute force
    q, k, v, alpha, b, w, S0 = pins.rand_inputs(rng, 1, 6, 2, 5, 4, unit_k=False)
    o, ST = rec(q, k, v, alpha, b, w, S0)
    for hh in range(2):
        ob, Sb = pins.brute_force(q[0, :, hh], k[0, :, hh], v[0, :, hh], alpha[0, :, hh], b[0, :, hh],
                                  w[0, :, hh], S0[0, hh])
        if not (np.allclose(o[0, :, hh], ob, rtol=1e-10, atol=1e-12) and np.allclose(ST[0, hh], Sb, rtol=1e-10)):
            failed.append("brute_force")
            break
    # KDA
    q, k, v, alpha, _, _, S0 = pins.rand_inputs(rng, 1, 20, 1, 6, 5)
    beta = 1 / (1 + np.exp(-rng.standard_normal((1, 20, 1))))
    o, ST = rec(q, k, v, alpha, np.repeat(beta[..., None], 6, -1), np.repeat(beta[..., None], 5, -1), S0)
    ok, Sk = pins.kda_restatement(q[0, :, 0], k[0, :, 0], v[0, :, 0], alpha[0, :, 0], beta[0, :, 0], S0[0, 0])
    if not (np.allclose(o[0, :, 0], ok, rtol=1e-10) and np.allclose(ST[0, 0], Sk, rtol=1e-10)):
        failed.append("kda")
    # erase-then-write
    q, k, v, alpha, _, w, S0 = pins.rand_inputs(rng, 1, 9, 1, 6, 4)
    _, ST = rec(q, k, v, alpha, np.ones_like(k), w, S0)
    if not np.allclose(k[0, -1, 0] @ ST[0, 0], w[0, -1, 0] * v[0, -1, 0], rtol=1e-10, atol=1e-12):
        failed.append("erase_then_write")
    # frozen state
    q, k, v, _, _, _, S0 = pins.rand_inputs(rng, 1, 9, 1, 6, 4)
    o, ST = rec(q, k, v, np.ones_like(k), np.zeros_like(k), np.zeros_like(v), S0)
    if not (np.array_equal(ST, S0) and np.allclose(o, np.einsum("bthc,bhcv->bthv", q, S0))):
        failed.append("frozen")
    return failed


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, rng, name, old, new):
    src = open(SRC).read()
    assert old in src, f"mutation site for {name} not found in the oracle source"
    mutated = src.replace(old, new, 1)
    path = tmp_path / f"oracle_{name}.c"
    path.write_text(mutated)
    lib = oracle.load(oracle.build(force=True, src=str(path), out=str(tmp_path / f"lib_{name}.so")))
    failed = _pin_suite(lib, rng)
    assert failed, f"mutant {name} passed every pin"


def test_unmutated_oracle_passes_compact_suite(rng):
    assert _pin_suite(oracle.load(), rng) == []
