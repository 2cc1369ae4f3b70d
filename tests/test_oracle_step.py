"""Pins of the oracle's single autoregressive step (the recurrent mode).

Expected values come from the pages' worked example stepped one token at a
time, closed forms of special decays, and the C oracle's full recurrence
(a separate implementation of the same definition, in another language).
"""
import json
import os

import numpy as np
import pytest

import oracle
from structured_state_space_ssd_b200.inputs import make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "four_token_example.json")


def test_four_tokens_stepped_one_at_a_time_match_the_printed_output():
    with open(GOLDEN) as f:
        g = json.load(f)
    inp = g["inputs"]
    a = np.array(inp["a"])
    Bs = np.array(inp["B"], dtype=float)
    Cs = np.array(inp["C"], dtype=float)
    state = np.zeros((1, 1, 1, 2))
    ys = []
    for t in range(4):
        state, y = oracle.ssd_ref_step(state, np.array(inp["x"][t]).reshape(1, 1, 1), np.array([[-np.log(a[t])]]),
                                       np.array([-1.0]), Bs[t].reshape(1, 1, 2), Cs[t].reshape(1, 1, 2),
                                       np.array([0.0]))
        ys.append(float(y.reshape(())))
    np.testing.assert_allclose(ys, g["printed"]["y_recurrence"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(state.reshape(2), g["derived_by_hand"]["final_state"], rtol=0, atol=1e-12)


def test_full_decay_forgets_the_state():
    # exp(dt * A) = 0: the new state is x B^T alone, y = (B . C) x + D x
    rng = np.random.default_rng(1)
    b, H, P, N, G = 2, 4, 3, 5, 2
    state = rng.standard_normal((b, H, P, N))
    x = rng.standard_normal((b, H, P))
    B = rng.standard_normal((b, G, N))
    C = rng.standard_normal((b, G, N))
    D = rng.standard_normal(H)
    dt = np.full((b, H), 1.0)
    A = np.full(H, -np.inf)
    new, y = oracle.ssd_ref_step(state, x, dt, A, B, C, D)
    for bb in range(b):
        for h in range(H):
            g = h // (H // G)
            np.testing.assert_allclose(new[bb, h], np.outer(x[bb, h], B[bb, g]), rtol=0, atol=0)
            np.testing.assert_allclose(y[bb, h], (B[bb, g] @ C[bb, g] + D[h]) * x[bb, h], rtol=1e-14, atol=1e-14)


def test_zero_step_keeps_the_state_and_adds_the_input():
    # dt = 0: a = 1, the state only accumulates
    rng = np.random.default_rng(2)
    state = rng.standard_normal((1, 2, 4, 3))
    x = rng.standard_normal((1, 2, 4))
    B = rng.standard_normal((1, 1, 3))
    C = rng.standard_normal((1, 1, 3))
    new, _ = oracle.ssd_ref_step(state, x, np.zeros((1, 2)), np.array([-0.7, -3.0]), B, C, np.zeros(2))
    for h in range(2):
        np.testing.assert_allclose(new[0, h] - state[0, h], np.outer(x[0, h], B[0, 0]), rtol=0, atol=1e-15)


@pytest.mark.parametrize("init", [False, True])
def test_chained_steps_equal_the_full_recurrence(init):
    inp = make_inputs(2, 9, 4, 3, 5, 2, "f32", seed=5, with_init=init)
    x, dt, A, B, C, D = (inp[k].double().numpy() for k in ("x", "dt", "A", "B", "C", "D"))
    y_ref, fin_ref = oracle.ssd_ref_fwd(x, dt, A, B, C, D, init_state=inp["init_state"])
    state = np.zeros((2, 4, 3, 5)) if inp["init_state"] is None else inp["init_state"].double().numpy()
    for t in range(9):
        state, y = oracle.ssd_ref_step(state, x[:, t], dt[:, t], A, B[:, t], C[:, t], D)
        np.testing.assert_allclose(y, y_ref[:, t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(state, fin_ref, rtol=1e-12, atol=1e-12)
