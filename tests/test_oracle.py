"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: every expected value comes from
the pages' worked example, a closed form, an independent evaluation order
(explicit products instead of the recurrence), or a structural property.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from structured_state_space_ssd_b200.inputs import make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "four_token_example.json")


def _four_token():
    with open(GOLDEN) as f:
        g = json.load(f)
    inp = g["inputs"]
    a = np.array(inp["a"])
    x = np.array(inp["x"]).reshape(1, 4, 1, 1)
    dt = (-np.log(a)).reshape(1, 4, 1)
    A = np.array([-1.0])
    B = np.array(inp["B"], dtype=float).reshape(1, 4, 1, 2)
    C = np.array(inp["C"], dtype=float).reshape(1, 4, 1, 2)
    D = np.array([0.0])
    return g, (x, dt, A, B, C, D)


def test_four_token_recurrence_matches_printed_output():
    g, args = _four_token()
    y, fin = oracle.ssd_ref_fwd(*args)
    np.testing.assert_allclose(y.reshape(4), g["printed"]["y_recurrence"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(fin.reshape(2), g["derived_by_hand"]["final_state"], rtol=0, atol=1e-12)


def test_four_token_mask_matches_printed_L():
    g, _ = _four_token()
    L = oracle.segsum_mask(g["inputs"]["a"])
    np.testing.assert_allclose(L, g["printed"]["L"], rtol=0, atol=1e-12)


def test_four_token_dual_matches_printed_output():
    g, args = _four_token()
    y, fin, M = oracle.ssd_dual_fwd(*args)
    np.testing.assert_allclose(y.reshape(4), g["printed"]["y_matrix"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(fin.reshape(2), g["derived_by_hand"]["final_state"], rtol=0, atol=1e-12)
    # M = L o (C B^T) with the printed L
    inp = g["inputs"]
    CB = np.array(inp["C"], float) @ np.array(inp["B"], float).T
    np.testing.assert_allclose(M[0, 0], np.array(g["printed"]["L"]) * CB, atol=1e-12)


@pytest.mark.parametrize("Q", [1, 2, 3, 4, 64])
def test_four_token_chunked_matches_printed_output(Q):
    g, args = _four_token()
    y, fin, _, _ = oracle.ssd_chunked_fwd(*args, Q=Q)
    np.testing.assert_allclose(y.reshape(4), g["printed"]["y_recurrence"], atol=1e-12)
    np.testing.assert_allclose(fin.reshape(2), g["derived_by_hand"]["final_state"], atol=1e-12)


def _rand(batch=2, T=37, H=4, P=3, N=5, G=2, seed=0, init=True):
    inp = make_inputs(batch, T, H, P, N, G, "f32", seed, with_init=init)
    # stronger init so its contribution is visible in the comparisons
    if inp["init_state"] is not None:
        inp["init_state"] = inp["init_state"] * 10
    return inp


def _args(inp):
    return (inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"])


@pytest.mark.parametrize("shape", [
    dict(batch=1, T=1, H=1, P=1, N=1, G=1),
    dict(batch=2, T=37, H=4, P=3, N=5, G=2),
    dict(batch=1, T=64, H=6, P=4, N=8, G=3),
    dict(batch=3, T=17, H=2, P=2, N=16, G=1),
])
@pytest.mark.parametrize("init", [False, True])
def test_recurrence_equals_quadratic_dual(shape, init):
    inp = _rand(**shape, seed=7, init=init)
    y, fin = oracle.ssd_ref_fwd(*_args(inp), init_state=inp["init_state"])
    y2, fin2, _ = oracle.ssd_dual_fwd(*_args(inp), init_state=inp["init_state"])
    np.testing.assert_allclose(y, y2, rtol=0, atol=1e-12 * max(1.0, np.abs(y2).max()))
    np.testing.assert_allclose(fin, fin2, rtol=0, atol=1e-12 * max(1.0, np.abs(fin2).max()))


@pytest.mark.parametrize("Q", [1, 2, 5, 16, 37, 64])
def test_block_decomposition_is_Q_invariant(Q):
    inp = _rand(seed=11)
    y, fin = oracle.ssd_ref_fwd(*_args(inp), init_state=inp["init_state"])
    y2, fin2, _, _ = oracle.ssd_chunked_fwd(*_args(inp), Q=Q, init_state=inp["init_state"])
    np.testing.assert_allclose(y2, y, atol=1e-11 * max(1.0, np.abs(y).max()))
    np.testing.assert_allclose(fin2, fin, atol=1e-11 * max(1.0, np.abs(fin).max()))


def test_A_zero_is_causal_linear_attention():
    """a_t = 1: y_t = C_t^T (sum_{s<=t} B_s x_s^T) + D x_t, a plain cumulative sum."""
    inp = _rand(seed=3, init=False)
    inp["A"] = inp["A"] * 0
    x, B, C, D = (inp[k].double().numpy() for k in ("x", "B", "C", "D"))
    H, G = x.shape[2], B.shape[2]
    g_of_h = np.arange(H) // (H // G)
    Bh, Ch = B[:, :, g_of_h, :], C[:, :, g_of_h, :]
    KV = np.cumsum(np.einsum("bthp,bthn->bthpn", x, Bh), axis=1)
    expect = np.einsum("bthpn,bthn->bthp", KV, Ch) + D[None, None, :, None] * x
    y, _ = oracle.ssd_ref_fwd(*_args(inp))
    np.testing.assert_allclose(y, expect, atol=1e-12 * np.abs(expect).max())


def test_zero_decay_is_diagonal_only():
    """a_t = 0 (exp underflows for dt*A <= -1000): y_t = (C_t . B_t) x_t + D x_t."""
    inp = _rand(seed=4, init=True)
    inp["A"] = inp["A"] * 0 - 1e8
    x, B, C, D = (inp[k].double().numpy() for k in ("x", "B", "C", "D"))
    assert float(inp["dt"].min()) * -1e8 <= -1000
    H, G = x.shape[2], B.shape[2]
    g_of_h = np.arange(H) // (H // G)
    cb = np.einsum("btgn,btgn->btg", C, B)[:, :, g_of_h]
    expect = cb[..., None] * x + D[None, None, :, None] * x
    y, fin = oracle.ssd_ref_fwd(*_args(inp), init_state=inp["init_state"])
    np.testing.assert_allclose(y, expect, atol=1e-13)
    # the final state is the last token's outer product alone
    last = np.einsum("bhp,bhn->bhpn", x[:, -1], B[:, -1][:, g_of_h])
    np.testing.assert_allclose(fin, last, atol=1e-13)


def test_constant_decay_is_toeplitz():
    """a_t = gamma for all t: M[t, s] = gamma^(t-s) C_t . B_s (the RetNet-style mask)."""
    inp = _rand(batch=1, T=23, H=2, P=2, N=3, G=1, seed=5, init=False)
    gamma = 0.83
    inp["dt"] = inp["dt"] * 0 + 0.5
    inp["A"] = inp["A"] * 0 + 2 * math.log(gamma)  # exp(0.5 * 2 ln gamma) = gamma
    gamma = math.exp(0.5 * float(inp["A"][0]))  # the fp32-rounded A's exact decay
    x, B, C, D = (inp[k].double().numpy() for k in ("x", "B", "C", "D"))
    T = x.shape[1]
    expect = np.zeros_like(x)
    for t in range(T):
        for s in range(t + 1):
            expect[0, t] += gamma ** (t - s) * float(C[0, t, 0] @ B[0, s, 0]) * x[0, s]
        expect[0, t] += D[:, None] * x[0, t]
    y, _ = oracle.ssd_ref_fwd(*_args(inp))
    np.testing.assert_allclose(y, expect, atol=1e-12)


def test_linearity_in_x_and_initial_state():
    i1, i2 = _rand(seed=21), _rand(seed=22)
    i2["dt"], i2["A"], i2["B"], i2["C"], i2["D"] = i1["dt"], i1["A"], i1["B"], i1["C"], i1["D"]
    al, be = 0.7, -1.9
    y1, f1 = oracle.ssd_ref_fwd(*_args(i1), init_state=i1["init_state"])
    y2, f2 = oracle.ssd_ref_fwd(*_args(i2), init_state=i2["init_state"])
    mix = dict(i1)
    mix["x"] = al * i1["x"].double() + be * i2["x"].double()
    mixinit = al * i1["init_state"].double() + be * i2["init_state"].double()
    y3, f3 = oracle.ssd_ref_fwd(*_args(mix), init_state=mixinit)
    np.testing.assert_allclose(y3, al * y1 + be * y2, atol=1e-11 * np.abs(y3).max())
    np.testing.assert_allclose(f3, al * f1 + be * f2, atol=1e-11 * np.abs(f3).max())


@pytest.mark.parametrize("split", [1, 16, 19, 36])
def test_sequence_continuation(split):
    """Running [0, s) then [s, T) seeded with the first final state = one run."""
    inp = _rand(T=37, seed=31)
    y, fin = oracle.ssd_ref_fwd(*_args(inp), init_state=inp["init_state"])
    first = {k: (v[:, :split] if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}
    second = {k: (v[:, split:] if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}
    ya, fa = oracle.ssd_ref_fwd(*_args(first), init_state=inp["init_state"])
    yb, fb = oracle.ssd_ref_fwd(*_args(second), init_state=fa)
    np.testing.assert_allclose(np.concatenate([ya, yb], axis=1), y, atol=1e-12 * np.abs(y).max())
    np.testing.assert_allclose(fb, fin, atol=1e-12 * np.abs(fin).max())


def test_off_diagonal_blocks_have_rank_at_most_N():
    """Semiseparable structure: every block strictly below the diagonal has rank <= N."""
    N = 3
    inp = _rand(batch=1, T=40, H=1, P=1, N=N, G=1, seed=41, init=False)
    _, _, M = oracle.ssd_dual_fwd(*_args(inp))
    M = M[0, 0]
    for k in (5, 13, 20, 33):
        sv = np.linalg.svd(M[k:, :k], compute_uv=False)
        assert (sv[N:] <= 1e-10 * sv[0]).all(), sv
        assert sv[N - 1] > 1e-6 * sv[0]


def test_head_to_group_map_is_contiguous():
    """G=2, H=4: heads 0,1 read group 0 and heads 2,3 read group 1."""
    inp = _rand(batch=1, T=12, H=4, P=2, N=3, G=2, seed=51, init=False)
    inp["B"][:, :, 1] = 0  # group 1 writes nothing into the state
    y, _ = oracle.ssd_ref_fwd(*_args(inp))
    x, D = inp["x"].double().numpy(), inp["D"].double().numpy()
    np.testing.assert_allclose(y[:, :, 2:], D[None, None, 2:, None] * x[:, :, 2:], atol=1e-14)
    assert np.abs(y[:, :, :2] - D[None, None, :2, None] * x[:, :, :2]).max() > 1e-3


def test_skip_term_alone_when_C_is_zero():
    inp = _rand(seed=61)
    inp["C"] = inp["C"] * 0
    y, _ = oracle.ssd_ref_fwd(*_args(inp), init_state=inp["init_state"])
    x, D = inp["x"].double().numpy(), inp["D"].double().numpy()
    np.testing.assert_allclose(y, D[None, None, :, None] * x, atol=1e-14)


def test_pairs_subset_and_thread_count_do_not_change_results():
    inp = _rand(batch=2, T=29, H=4, seed=71)
    y, fin = oracle.ssd_ref_fwd(*_args(inp), init_state=inp["init_state"], nthreads=1)
    y4, fin4 = oracle.ssd_ref_fwd(*_args(inp), init_state=inp["init_state"], nthreads=4)
    assert np.array_equal(y, y4) and np.array_equal(fin, fin4)
    pairs = [(1, 2), (0, 3)]
    ys, fs = oracle.ssd_ref_fwd(*_args(inp), init_state=inp["init_state"], pairs=pairs)
    for b, h in pairs:
        assert np.array_equal(ys[b, :, h], y[b, :, h]) and np.array_equal(fs[b, h], fin[b, h])
    assert np.abs(ys[0, :, 0]).max() == 0


def test_empty_sequence():
    inp = _rand(T=5, seed=81)
    empty = {k: (v[:, :0] if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}
    y, fin = oracle.ssd_ref_fwd(*_args(empty), init_state=inp["init_state"])
    assert y.shape[1] == 0
    np.testing.assert_array_equal(fin, inp["init_state"].double().numpy())


def test_input_generator_distributions():
    inp = make_inputs(2, 4096, 4, 8, 16, 1, "f32", seed=1000)
    dt = inp["dt"]
    frac = float(((dt >= 1e-3) & (dt <= 0.1)).float().mean())
    assert 0.96 < frac < 0.995, frac
    A = inp["A"]
    assert float(A.max()) <= -1.0 and float(A.min()) >= -16.0
    assert abs(float(inp["B"].std()) * 4 - 1) < 0.05
    again = make_inputs(2, 4096, 4, 8, 16, 1, "f32", seed=1000)
    assert all(torch_equal(inp[k], again[k]) for k in ("x", "dt", "A", "B", "C", "D"))


def torch_equal(a, b):
    return bool((a == b).all())
