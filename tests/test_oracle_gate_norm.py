"""Pins of the oracle's gate + GroupNorm (the Mamba-2 block's step after the layer).

Expected values come from a hand-worked two-channel example, the defining
property of the normalisation (zero mean, unit variance per group), its scale
invariance, and the limits of the Swish gate.
"""
import numpy as np
import pytest

import oracle


def test_two_channel_example_by_hand():
    # z = 40: silu(z) = z to double precision, so g = 40 y = [1, 3]: mean 2, variance 1
    y = np.array([[1.0 / 40, 3.0 / 40]])
    z = np.array([[40.0, 40.0]])
    out = oracle.ref_gate_norm(y, z, ngroups=1, eps=0.0)
    np.testing.assert_allclose(out, [[-1.0, 1.0]], rtol=0, atol=1e-13)
    out = oracle.ref_gate_norm(y, z, ngroups=1, eps=0.0, weight=np.array([2.0, 3.0]), bias=np.array([0.5, -1.0]))
    np.testing.assert_allclose(out, [[-1.5, 2.0]], rtol=0, atol=1e-13)


def test_gate_is_swish():
    # silu(0) = 0 kills the channel; for a very negative z the gate is ~0 too
    y = np.array([[2.0, 5.0, -1.0, 4.0]])
    z = np.array([[0.0, 40.0, 40.0, -80.0]])
    out = oracle.ref_gate_norm(y, z, ngroups=1, eps=0.0)
    g = np.array([0.0, 200.0, -40.0, 4.0 * -80.0 / (1 + np.exp(80.0))])
    np.testing.assert_allclose(out[0], (g - g.mean()) / g.std(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("ngroups", [1, 4, 80])
def test_each_group_has_zero_mean_and_unit_variance(ngroups):
    rng = np.random.default_rng(3)
    y = rng.standard_normal((3, 7, 320))
    z = rng.standard_normal((3, 7, 320))
    out = oracle.ref_gate_norm(y, z, ngroups=ngroups, eps=0.0).reshape(-1, ngroups, 320 // ngroups)
    np.testing.assert_allclose(out.mean(axis=2), 0.0, atol=1e-12)
    np.testing.assert_allclose(out.var(axis=2), 1.0, atol=1e-10)


def test_scale_of_the_layer_output_cancels():
    rng = np.random.default_rng(4)
    y = rng.standard_normal((5, 64))
    z = rng.standard_normal((5, 64))
    np.testing.assert_allclose(oracle.ref_gate_norm(3.5 * y, z, 8, eps=0.0), oracle.ref_gate_norm(y, z, 8, eps=0.0),
                               rtol=1e-12, atol=1e-12)


def test_groups_are_contiguous_channel_ranges():
    # perturbing one channel changes only its own group
    rng = np.random.default_rng(5)
    y = rng.standard_normal((1, 64))
    z = rng.standard_normal((1, 64))
    a = oracle.ref_gate_norm(y, z, 4)
    y2 = y.copy()
    y2[0, 20] += 1.0  # group 1 = channels 16..31
    b = oracle.ref_gate_norm(y2, z, 4)
    changed = np.nonzero(np.abs(a - b)[0] > 0)[0]
    assert changed.min() >= 16 and changed.max() <= 31
