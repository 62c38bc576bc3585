"""Plant one plausible mistake at a time in a COPY of the backward oracle (CPU only)
and check that the finite-difference pin of test_oracle_backward.py catches each.

Each mutant is a textual edit of oracle/backward.py executed into a fresh
namespace; the real module is never modified.
"""
import inspect

import numpy as np
import pytest

from oracle import backward as ob
from tests import test_oracle_backward as pins

SRC = inspect.getsource(ob)

# (name, text in the source, replacement)
MUTANTS = [
    ("readout_uses_previous_state", "dq[t] = states[t + 1] @ dO[t]", "dq[t] = states[t] @ dO[t]"),
    ("readout_gradient_after_state", "        G = G + np.outer(q[t], dO[t])\n        # S_t",
     "        # S_t"),
    ("erase_term_dropped", "dSbar = G - np.outer(e, ddelta)", "dSbar = G"),
    ("erase_sign", "de = -(Sbar @ ddelta)", "de = (Sbar @ ddelta)"),
    ("erase_reads_new_state", "de = -(Sbar @ ddelta)", "de = -(states[t + 1] @ ddelta)"),
    ("key_write_term_dropped", "dk[t] = G @ deltas[t]", "dk[t] = 0.0 * k[t]"),
    ("key_erase_term_dropped", "dk[t] = dk[t] + b[t] * de", "dk[t] = dk[t]"),
    ("erase_gate_uses_q", "db[t] = k[t] * de", "db[t] = q[t] * de"),
    ("write_gate_swapped", "dw[t] = v[t] * du", "dw[t] = w[t] * du"),
    ("decay_reads_new_state", "dalpha[t] = np.sum(dSbar * states[t], axis=1)",
     "dalpha[t] = np.sum(dSbar * states[t + 1], axis=1)"),
    ("decay_uses_G", "dalpha[t] = np.sum(dSbar * states[t], axis=1)",
     "dalpha[t] = np.sum(G * states[t], axis=1)"),
    ("decay_not_propagated", "G = alpha[t][:, None] * dSbar", "G = dSbar"),
    ("state_gradient_ignored", "G = np.zeros((K, V)) if dST is None else np.array(dST, dtype=np.float64)",
     "G = np.zeros((K, V))"),
]


def mutant_module(old, new):
    assert SRC.count(old) >= 1, old
    ns = {"__name__": "oracle_backward_mutant"}
    exec(compile(SRC.replace(old, new, 1), "<mutant>", "exec"), ns)
    return ns


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(rng, name, old, new):
    ns = mutant_module(old, new)
    x, dO, dST = pins.problem(rng, 1, 5, 1, 4, 3)
    grads = ns["recurrence_backward"](*(x[n] for n in pins.NAMES), dO, dST)
    errs = pins.directional_errors(rng, x, dO, dST, grads)
    assert max(errs.values()) > 1e-4, f"{name} survived: {errs}"


def test_unmutated_copy_passes(rng):
    ns = mutant_module("import numpy as np", "import numpy as np")
    x, dO, dST = pins.problem(rng, 1, 5, 1, 4, 3)
    grads = ns["recurrence_backward"](*(x[n] for n in pins.NAMES), dO, dST)
    errs = pins.directional_errors(rng, x, dO, dST, grads)
    assert max(errs.values()) < 1e-8, errs
    assert np.isfinite(list(errs.values())).all()


# mistakes planted in the C version (oracle/gdn2_oracle.c, gdn2_oracle_backward)
import oracle  # noqa: E402

C_SRC = oracle._SRC
C_MUTANTS = [
    ("c_ddelta_uses_q", "dd[j] += G[(size_t)c * V + j] * kt[c];", "dd[j] += G[(size_t)c * V + j] * qt[c];"),
    ("c_erase_sign", "de[c] = -s;", "de[c] = s;"),
    ("c_erase_term_dropped", "dX[(size_t)c * V + j] = G[(size_t)c * V + j] - e * dd[j];",
     "dX[(size_t)c * V + j] = G[(size_t)c * V + j];"),
    ("c_decay_not_propagated", "G[(size_t)c * V + j] = at[c] * dX[(size_t)c * V + j];",
     "G[(size_t)c * V + j] = dX[(size_t)c * V + j];"),
    ("c_decay_reads_new_state", "s += dX[(size_t)c * V + j] * Sp[(size_t)c * V + j];",
     "s += dX[(size_t)c * V + j] * Sn[(size_t)c * V + j];"),
    ("c_readout_uses_previous_state", "s += Sn[(size_t)c * V + j] * gt[j];", "s += Sp[(size_t)c * V + j] * gt[j];"),
    ("c_erase_gate_uses_b", "dbt[c] = kt[c] * de[c];", "dbt[c] = bt[c] * de[c];"),
]


@pytest.mark.parametrize("name,old,new", C_MUTANTS, ids=[m[0] for m in C_MUTANTS])
def test_c_mutant_is_caught(tmp_path, rng, name, old, new):
    src = open(C_SRC).read()
    assert src.count(old) == 1, name
    path = tmp_path / f"oracle_{name}.c"
    path.write_text(src.replace(old, new))
    lib = oracle.load(oracle.build(force=True, src=str(path), out=str(tmp_path / f"lib_{name}.so")))
    x, dO, dST = pins.problem(rng, 1, 5, 1, 4, 3)
    grads = oracle.recurrence_backward_c(*(x[n] for n in pins.NAMES), dO, dST, lib=lib)
    errs = pins.directional_errors(rng, x, dO, dST, grads)
    assert max(errs.values()) > 1e-4, f"{name} survived: {errs}"
