"""Pins of the oracle's bounded log-decay gate ([W1 彩蛋], the gate.py excerpt):
g = lower_bound * sigmoid(exp(A_log[h]) * (g_raw + dt_bias[h, :])), lower bound
-5 in K3.  Each check follows from the definition, not from retyping it: the
midpoint, the sigmoid's point symmetry, the limits, the inverse through the
logit, the neutral parameters and monotonicity."""
import numpy as np

from oracle import gate

H, D = 3, 5


def _params(seed):
    r = np.random.default_rng(seed)
    return (r.standard_normal((7, H, D)), 0.5 * r.standard_normal(H), r.standard_normal((H, D)))


def test_midpoint_is_half_the_bound_exactly():
    _, A_log, dt_bias = _params(0)
    g = gate(-dt_bias[None].repeat(4, 0), A_log, dt_bias, -5.0)
    assert np.all(g == -2.5)


def test_point_symmetry_of_the_sigmoid():
    g_raw, A_log, dt_bias = _params(1)
    z_pos = g_raw
    z_neg = -2.0 * dt_bias[None] - g_raw  # mirrors g_raw + dt_bias around zero
    total = gate(z_pos, A_log, dt_bias, -5.0) + gate(z_neg, A_log, dt_bias, -5.0)
    np.testing.assert_allclose(total, -5.0, rtol=0, atol=1e-14)


def test_limits_and_open_range():
    _, A_log, dt_bias = _params(2)
    big = np.full((1, H, D), 1e4)
    assert np.all(gate(big, A_log, dt_bias) == -5.0)
    assert np.all(gate(-big, A_log, dt_bias) == 0.0)
    g_raw, _, _ = _params(3)
    g = gate(g_raw, A_log, dt_bias)
    assert np.all((g > -5.0) & (g < 0.0))


def test_logit_recovers_the_scaled_preactivation():
    g_raw, A_log, dt_bias = _params(4)
    g = gate(g_raw, A_log, dt_bias, -5.0)
    p = g / -5.0  # the sigmoid's value
    z = np.log(p / (1.0 - p))
    np.testing.assert_allclose(z, np.exp(A_log)[:, None] * (g_raw + dt_bias), rtol=1e-10,
                               atol=1e-10)


def test_missing_parameters_are_neutral():
    g_raw, _, _ = _params(5)
    ref = gate(g_raw, np.zeros(H), np.zeros((H, D)), -5.0)
    np.testing.assert_array_equal(gate(g_raw, None, None, -5.0), ref)
    np.testing.assert_array_equal(gate(g_raw, None, np.zeros((H, D)), -5.0), ref)


def test_decreasing_in_the_preactivation_and_scaled_by_the_bound():
    g_raw, A_log, dt_bias = _params(6)
    g1 = gate(g_raw, A_log, dt_bias, -5.0)
    g2 = gate(g_raw + 0.1, A_log, dt_bias, -5.0)
    assert np.all(g2 < g1)
    np.testing.assert_allclose(gate(g_raw, A_log, dt_bias, -2.0), 0.4 * g1, rtol=1e-15)
