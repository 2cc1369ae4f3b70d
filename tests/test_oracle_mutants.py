"""Plant plausible mistakes in copies of the C oracle and check a pin catches each.

Every mutant is the oracle source with one textual change (a dropped term, a
wrong sign, a wrong index, swapped operands, a reordered update), compiled
with gcc into a temporary directory.  The pins used are the ones of
``test_oracle.py`` that do not depend on the C oracle itself: the pages'
four-token example, the quadratic dual built from explicit products, and the
closed forms.  The unmodified source must pass them all.
"""
import json
import os
import subprocess

import numpy as np
import pytest

import oracle
from structured_state_space_ssd_b200.inputs import make_inputs

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssd_oracle.c")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "four_token_example.json")

MUTANTS = {
    "none": [],
    "dropped_skip_term": [("yt[p] = acc + j->D[h] * xv;", "yt[p] = acc;")],
    "decay_after_input": [("Sp[n] = a * Sp[n] + xv * Bt[n];", "Sp[n] = a * (Sp[n] + xv * Bt[n]);")],
    "swapped_B_and_C": [("const double *Bt = j->B", "const double *Bt = j->C"),
                        ("const double *Ct = j->C", "const double *Ct = j->B")],
    "group_map_modulo": [("const long g = h / (H / G);", "const long g = h % G;")],
    "wrong_exponent_sign": [("exp(j->dt[(b * T + t) * H + h] * j->A[h])",
                             "exp(-j->dt[(b * T + t) * H + h] * j->A[h])")],
    "reads_state_before_update": [
        ("Sp[n] = a * Sp[n] + xv * Bt[n];\n                acc += Sp[n] * Ct[n];",
         "acc += Sp[n] * Ct[n];\n                Sp[n] = a * Sp[n] + xv * Bt[n];")],
    "wrong_head_dt": [("exp(j->dt[(b * T + t) * H + h] * j->A[h])",
                       "exp(j->dt[(b * T + t) * H + (H - 1 - h)] * j->A[h])")],
    "initial_state_ignored": [("if (j->init) memcpy", "if (0) memcpy")],
    "x_time_head_transposed": [("j->x + ((b * T + t) * H + h) * P", "j->x + ((b * H + h) * T + t) * P")],
}


def _build(name, edits, tmpdir):
    src = open(SRC).read()
    for old, new in edits:
        assert old in src, (name, old)
        src = src.replace(old, new)
    cpath = os.path.join(tmpdir, f"{name}.c")
    with open(cpath, "w") as f:
        f.write(src)
    so = os.path.join(tmpdir, f"lib{name}.so")
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", so, cpath, "-lm", "-lpthread"])
    return so


def _pins_fail(so):
    """Return the names of the pins the build at ``so`` fails."""
    failed = []
    run = lambda *a, **k: oracle.ssd_ref_fwd(*a, _lib_path=so, **k)  # noqa: E731

    g = json.load(open(GOLDEN))
    a = np.array(g["inputs"]["a"])
    args = (np.array(g["inputs"]["x"]).reshape(1, 4, 1, 1), (-np.log(a)).reshape(1, 4, 1), np.array([-1.0]),
            np.array(g["inputs"]["B"], float).reshape(1, 4, 1, 2),
            np.array(g["inputs"]["C"], float).reshape(1, 4, 1, 2), np.array([0.0]))
    y, fin = run(*args)
    if not (np.allclose(y.ravel(), g["printed"]["y_recurrence"], atol=1e-12)
            and np.allclose(fin.ravel(), g["derived_by_hand"]["final_state"], atol=1e-12)):
        failed.append("four_token_example")

    for seed, shape in [(7, dict(batch=2, T=37, H=4, P=3, N=5, G=2)), (8, dict(batch=1, T=20, H=6, P=2, N=4, G=3))]:
        inp = make_inputs(**shape, dtype="f32", seed=seed, with_init=True)
        a6 = (inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"])
        y, fin = run(*a6, init_state=inp["init_state"] * 10)
        y2, fin2, _ = oracle.ssd_dual_fwd(*a6, init_state=inp["init_state"] * 10)
        if not (np.allclose(y, y2, atol=1e-11) and np.allclose(fin, fin2, atol=1e-11)):
            failed.append(f"dual_{seed}")
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    so = _build(name, MUTANTS[name], str(tmp_path))
    failed = _pins_fail(so)
    if name == "none":
        assert failed == []
    else:
        assert failed, f"mutant {name} passed every pin"
