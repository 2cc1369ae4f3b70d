"""Pins of the backward oracle (gradients of the SSD layer).

The pages print no backward, so nothing here compares against printed values;
the gradient of a function is unique, and these tests pin the oracle's
gradients to things that fix them independently of how it computes them:
central finite differences of the C forward oracle (a separate program in
another language), the bilinear adjoint identity of the map
(x, init) -> (y, final), closed forms when every decay is zero, the
explicit-sum evaluation at single tokens, and the head -> group sum.
"""
import numpy as np
import pytest

import oracle
from structured_state_space_ssd_b200.inputs import make_inputs, make_output_grads

NAMES = ("x", "dt", "A", "B", "C", "D", "init_state")


def _problem(batch=2, T=7, H=4, P=3, N=5, G=2, seed=0, init=True, dfinal=True):
    inp = make_inputs(batch, T, H, P, N, G, "f32", seed=seed, with_init=init)
    grads = make_output_grads(batch, T, H, P, N, "f32", seed=seed, with_dfinal=dfinal)
    arr = {k: (None if v is None else v.double().numpy()) for k, v in {**inp, **grads}.items()}
    return arr


def _loss(p):
    y, fin = oracle.ssd_ref_fwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], init_state=p["init_state"],
                                nthreads=1)
    val = float(np.sum(p["dy"] * y))
    if p["dfinal_state"] is not None:
        val += float(np.sum(p["dfinal_state"] * fin))
    return val


def _bwd(p):
    return oracle.ssd_ref_bwd(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["dy"],
                              init_state=p["init_state"], dfinal_state=p["dfinal_state"])


GRAD_OF = {"x": "dx", "dt": "ddt", "A": "dA", "B": "dB", "C": "dC", "D": "dD", "init_state": "dinit_state"}


@pytest.mark.parametrize("init,dfinal", [(True, True), (False, False), (True, False), (False, True)])
def test_every_gradient_matches_central_finite_differences(init, dfinal):
    p = _problem(init=init, dfinal=dfinal)
    g = _bwd(p)
    eps = 1e-6
    for name in NAMES:
        if p[name] is None:
            continue
        base = p[name]
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            keep = base[idx]
            base[idx] = keep + eps
            up = _loss(p)
            base[idx] = keep - eps
            dn = _loss(p)
            base[idx] = keep
            fd[idx] = (up - dn) / (2 * eps)
        got = g[GRAD_OF[name]]
        scale = max(np.abs(fd).max(), 1e-12)
        assert np.abs(got - fd).max() / scale < 1e-7, name
    if not init:
        # the gradient w.r.t. a zero initial state is still defined: check it the same way
        p["init_state"] = np.zeros_like(g["dinit_state"])
        base = p["init_state"]
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            base[idx] = eps
            up = _loss(p)
            base[idx] = -eps
            dn = _loss(p)
            base[idx] = 0.0
            fd[idx] = (up - dn) / (2 * eps)
        assert np.abs(g["dinit_state"] - fd).max() / max(np.abs(fd).max(), 1e-12) < 1e-7


def test_adjoint_identity_of_the_linear_map():
    # for fixed (dt, A, B, C, D) the map (x, init) -> (y, final) is linear, so
    # <dy, y(x', i')> + <dfinal, final(x', i')> = <dx, x'> + <dinit, i'> for any probe (x', i')
    p = _problem(batch=2, T=150, H=6, P=8, N=16, G=3, seed=4)
    g = _bwd(p)
    rng = np.random.default_rng(5)
    xp = rng.standard_normal(p["x"].shape)
    ip = rng.standard_normal(p["init_state"].shape)
    y, fin = oracle.ssd_ref_fwd(xp, p["dt"], p["A"], p["B"], p["C"], p["D"], init_state=ip)
    lhs = np.sum(p["dy"] * y) + np.sum(p["dfinal_state"] * fin)
    rhs = np.sum(g["dx"] * xp) + np.sum(g["dinit_state"] * ip)
    assert abs(lhs - rhs) <= 1e-11 * (abs(lhs) + np.abs(y).sum())


def test_zero_decay_closed_forms():
    # every a_t = exp(dt A) = 0 exactly: y_t = (C_t . B_t) x_t + D x_t, the state forgets, and
    # dx_t = (C_t . B_t + D) dy_t, dB_t = sum_h (dy_t . x_t) C_t, dC_t = sum_h (dy_t . x_t) B_t,
    # d(dt) = dA = dinit = 0
    p = _problem(batch=2, T=9, H=4, P=3, N=5, G=2, seed=6, init=True, dfinal=False)
    p["A"] = np.full_like(p["A"], -1e6)
    p["dt"] = np.maximum(p["dt"], 1e-3)
    g = _bwd(p)
    x, dy, B, C, D = p["x"], p["dy"], p["B"], p["C"], p["D"]
    grp = np.arange(4) // 2
    cb = np.einsum("btgn,btgn->btg", C, B)[:, :, grp]                     # [b,T,H]
    np.testing.assert_allclose(g["dx"], (cb + D)[..., None] * dy, rtol=1e-13, atol=1e-13)
    w = np.einsum("bthp,bthp->bth", dy, x)                               # [b,T,H]
    wg = w.reshape(2, 9, 2, 2).sum(axis=3)                               # per group
    np.testing.assert_allclose(g["dB"], wg[..., None] * C, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(g["dC"], wg[..., None] * B, rtol=1e-13, atol=1e-13)
    assert np.all(g["ddt"] == 0) and np.all(g["dA"] == 0) and np.all(g["dinit_state"] == 0)
    np.testing.assert_allclose(g["dD"], w.sum(axis=(0, 1)), rtol=1e-13)


def test_explicit_sums_at_tokens_equal_the_reverse_recurrence():
    p = _problem(batch=2, T=90, H=4, P=6, N=10, G=2, seed=8)
    g = _bwd(p)
    toks = [0, 1, 45, 88, 89]
    for b in range(2):
        at = oracle.ssd_ref_bwd_at(p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"], p["dy"], b, toks,
                                   init_state=p["init_state"], dfinal_state=p["dfinal_state"])
        for name in ("dx", "ddt", "dB", "dC"):
            ref = g[name][b, toks]
            assert np.abs(at[name] - ref).max() <= 1e-11 * max(np.abs(ref).max(), 1.0), name


def test_group_sum_equals_per_head_copies_of_B_and_C():
    # G = 2 groups of 3 heads vs the same problem with B, C repeated per head (G = H): the
    # group gradient is the sum of its heads' gradients, in the contiguous head -> group map
    p = _problem(batch=1, T=40, H=6, P=4, N=8, G=2, seed=9)
    g = _bwd(p)
    q = dict(p)
    grp = np.arange(6) // 3
    q["B"] = np.ascontiguousarray(p["B"][:, :, grp, :])
    q["C"] = np.ascontiguousarray(p["C"][:, :, grp, :])
    gq = _bwd(q)
    for name in ("dB", "dC"):
        np.testing.assert_allclose(g[name], gq[name].reshape(1, 40, 2, 3, 8).sum(axis=3), rtol=1e-12, atol=1e-12)
    for name in ("dx", "ddt", "dA", "dD", "dinit_state"):
        np.testing.assert_allclose(g[name], gq[name], rtol=1e-12, atol=1e-12)


def test_empty_sequence_passes_the_final_gradient_to_the_initial_state():
    p = _problem(batch=2, T=0, H=2, P=3, N=4, G=1, seed=10)
    g = _bwd(p)
    np.testing.assert_array_equal(g["dinit_state"], p["dfinal_state"])
    assert g["dx"].size == 0 and np.all(g["dA"] == 0) and np.all(g["dD"] == 0)


MUTANTS = {
    "decay factor dropped from d(log a)": ("dlog = a[t] * np.einsum", "dlog = np.einsum"),
    "dC from the previous state": ('np.einsum("hpn,hp->hn", states[t], dy[b, t])',
                                   'np.einsum("hpn,hp->hn", states[t - 1] if t > 0 else h0, dy[b, t])'),
    "skip term dropped from dx": ("+ D[:, None] * dy[b, t]", ""),
    "adjoint decayed one step early": ("g = g + dy[b, t][:, :, None]", "g = a[t][:, None, None] * g + dy[b, t][:, :, None]"),
    "dB contracted with dy": ('np.einsum("hpn,hp->hn", g, x[b, t])', 'np.einsum("hpn,hp->hn", g, dy[b, t])'),
    "sign of d(dt)": ('out["ddt"][b, t] = A * dlog', 'out["ddt"][b, t] = -A * dlog'),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_finite_differences_catch_planted_mistakes(mutant, monkeypatch):
    # plant one plausible mistake in a copy of the oracle's source (CPU only) and check that
    # the finite-difference pin rejects it
    import inspect
    src = inspect.getsource(oracle.ssd_ref_bwd)
    old, new = MUTANTS[mutant]
    assert old in src
    ns = dict(oracle.__dict__)
    exec(src.replace(old, new), ns)
    monkeypatch.setattr(oracle, "ssd_ref_bwd", ns["ssd_ref_bwd"])
    with pytest.raises(AssertionError):
        test_every_gradient_matches_central_finite_differences(True, True)
