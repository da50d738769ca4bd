"""Pins of the oracle's output epilogue ([W1 第六站]: per-head RMSNorm of the
read-out, then a per-channel output gate; reading: sigmoid gate, epsilon a
parameter).  Checks that follow from the definition: the normalised row has
unit RMS, positive scaling of the row does not change the result, the gate's
limits are the plain norm and zero, and the gate at zero halves it."""
import numpy as np

from oracle import output_epilogue

D = 16


def _row(seed, n=6):
    r = np.random.default_rng(seed)
    return r.standard_normal((n, 3, D)), r.standard_normal((n, 3, D)), 0.5 + r.random(D)


def test_unit_rms_without_weight_and_open_gate():
    o, _, _ = _row(0)
    y = output_epilogue(o, np.full(o.shape, 50.0), np.ones(D), eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-12)


def test_positive_scaling_of_the_row_is_invisible():
    o, z, w = _row(1)
    np.testing.assert_allclose(output_epilogue(7.5 * o, z, w, eps=0.0),
                               output_epilogue(o, z, w, eps=0.0), rtol=1e-12, atol=1e-15)


def test_gate_limits_and_midpoint():
    o, _, w = _row(2)
    plain = output_epilogue(o, np.full(o.shape, 1e4), w, eps=1e-5)
    closed = output_epilogue(o, np.full(o.shape, -1e4), w, eps=1e-5)
    half = output_epilogue(o, np.zeros(o.shape), w, eps=1e-5)
    assert np.all(closed == 0.0)
    np.testing.assert_allclose(half, 0.5 * plain, rtol=1e-15)
    np.testing.assert_allclose(plain / w, o / np.sqrt(np.mean(o * o, -1, keepdims=True) + 1e-5),
                               rtol=1e-12)


def test_epsilon_bounds_a_zero_row():
    o = np.zeros((2, 1, D))
    y = output_epilogue(o, np.zeros(o.shape), np.ones(D), eps=1e-5)
    assert np.all(y == 0.0)
