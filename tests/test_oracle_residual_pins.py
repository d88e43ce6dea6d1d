"""Pins of the oracle's _residual_core forms (layers page: _residual_core,
MuseSparkResidual) against what the page and mathematics fix.

The page states that the blend is "norm-preserving" and that eps is a "lower
bound on the squared residual coefficient"; the formula itself is a declared
reading (c^2 = max(sigmoid(gate/temperature), eps), s^2 = 1 - c^2, blend
c h + s branch, i.e. core 5's cos(theta) h + sin(theta) branch with
theta = atan2(s, c)).  Each check below is an identity, a limit or a closed
form of that reading, chosen so that a swapped coefficient, a missing square
root, the bound applied to the wrong coefficient, a multiplied temperature or
a flipped sigmoid fails at least one of them.
"""
import math

import numpy as np

import oracle


def rng(seed=0):
    return np.random.default_rng(seed)


def test_blend_zero_angle_returns_stream_bitwise():
    r = rng(1)
    h = r.standard_normal((7, 33)).astype(np.float32)
    b = r.standard_normal((7, 33)).astype(np.float32)
    out, lo, hi, mag = oracle.residual_blend(h, b, np.zeros(33, np.float32))
    assert np.array_equal(out.view(np.uint32), h.view(np.uint32))


def test_blend_unit_inputs_give_cos_and_sin():
    th = np.array([0.1, 0.7, 1.3, 1.5707964], np.float32)
    one, zero = np.ones((1, 4), np.float32), np.zeros((1, 4), np.float32)
    c = oracle.residual_blend(one, zero, th)[1][0]
    s = oracle.residual_blend(zero, one, th)[1][0]
    np.testing.assert_allclose(c * c + s * s, 1.0, rtol=0, atol=1e-15)
    assert np.all(s > 0) and np.all(np.diff(s) > 0)  # sin grows with theta on [0, pi/2]


def test_blend_reads_bf16_branch_exactly():
    # bf16 1 + 2^-7 is exact; the blend adds no cast of the branch
    th = np.array([0.5], np.float32)
    b = np.array([[0x3F81]], np.uint16)  # 1.0078125
    out, lo, hi, mag = oracle.residual_blend(np.zeros((1, 1), np.float32), b, th)
    assert lo[0, 0] == math.sin(float(th[0])) * 1.0078125


def test_gate_zero_balances_and_monotone_angle():
    g = np.linspace(-3, 3, 61).astype(np.float32)
    c, s, th = oracle.residual_gate_coefficients(g, 0.3, 1e-3)
    i0 = 30
    assert g[i0] == 0.0 and c[i0] == math.sqrt(0.5) and s[i0] == math.sqrt(0.5)
    assert th[i0] == math.atan2(math.sqrt(0.5), math.sqrt(0.5))
    # the angle falls as the gate rises, strictly above the lower bound and
    # flat where the squared residual coefficient sits at eps
    free = c[:-1] ** 2 > float(np.float32(1e-3)) * (1 + 1e-12)
    assert np.all(np.diff(c)[free] > 0) and np.all(np.diff(s)[free] < 0) and np.all(np.diff(th)[free] < 0)
    assert np.all(np.diff(th)[~free] <= 0) and np.any(~free)
    assert np.all((th >= 0) & (th <= math.pi / 2))


def test_gate_norm_preserving():
    # c^2 + s^2 = 1 for every gate, including the clamped and saturated ends
    g = np.concatenate([rng(2).standard_normal(1000) * 3, [-1e4, -50, 50, 1e4]]).astype(np.float32)
    for eps in (0.0, 1e-3, 0.25):
        c, s, _ = oracle.residual_gate_coefficients(g, 0.3, eps)
        np.testing.assert_allclose(c * c + s * s, 1.0, rtol=0, atol=4e-16)


def test_gate_lower_bound_on_squared_residual_coefficient():
    g = np.array([-1e4, -100.0, -30.0, 0.0, 30.0], np.float32)
    eps = np.float32(0.0625)
    c, s, _ = oracle.residual_gate_coefficients(g, 0.25, float(eps))
    assert np.all(c * c >= float(eps) * (1 - 1e-15))
    assert c[0] == 0.25 and c[1] == 0.25 and s[0] == math.sqrt(15) / 4
    # above the bound the sigmoid decides: sigmoid(0) = 1/2 > 1/16
    assert c[3] == math.sqrt(0.5)


def test_gate_temperature_scales_the_gate():
    # only gate / temperature matters (power-of-two rescaling is exact), and at
    # gate = temperature the squared coefficient is sigmoid(1) = e / (1 + e)
    g = rng(3).standard_normal(200).astype(np.float32)
    a = oracle.residual_gate_coefficients(g, 0.3, 1e-3)
    b = oracle.residual_gate_coefficients(g * np.float32(4), 1.2, 1e-3)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=4e-7, atol=0)  # 1.2 is 4 * f32(0.3) to within rounding
    c, s, _ = oracle.residual_gate_coefficients(np.array([0.5], np.float32), 0.5, 0.0)
    e = math.e
    assert abs(c[0] ** 2 - e / (1 + e)) < 1e-15 and abs(s[0] ** 2 - 1 / (1 + e)) < 1e-15
    # a sharper temperature pushes the same gate further from balance
    c1, _, _ = oracle.residual_gate_coefficients(np.array([0.2], np.float32), 1.0, 0.0)
    c2, _, _ = oracle.residual_gate_coefficients(np.array([0.2], np.float32), 0.1, 0.0)
    assert 0.5 < c1[0] ** 2 < c2[0] ** 2


def test_gate_saturation_keeps_branch_weight_relative_precision():
    # s = sqrt(sigmoid(-x)) = exp(-x/2) / sqrt(1 + exp(-x)) for large x
    c, s, th = oracle.residual_gate_coefficients(np.array([10.0, 25.0], np.float32), 0.25, 1e-3)
    for x, sj in zip((40.0, 100.0), s):
        want = math.exp(-x / 2) / math.sqrt(1 + math.exp(-x))
        assert abs(sj - want) <= 1e-14 * want
    assert c[1] == 1.0 and abs(th[1] - s[1]) < 1e-30


def test_gate_form_equals_angle_form():
    # _residual_core with the gate = the angle blend with theta = atan2(s, c)
    # (theta rounded to FP32, so within a few FP32 roundings of the terms)
    r = rng(4)
    g = (r.standard_normal(64) * 2).astype(np.float32)
    h = r.standard_normal((9, 64)).astype(np.float32)
    b = r.standard_normal((9, 64)).astype(np.float32)
    _, _, th = oracle.residual_gate_coefficients(g, 0.3, 1e-3)
    y1, l1, _, m1 = oracle.residual(h, b, g, 0.3, 1e-3)
    y2, l2, _, m2 = oracle.residual_blend(h, b, th.astype(np.float32))
    assert np.all(np.abs(l1 - l2) <= 1e-6 * m1 + 1e-30)


def test_blend_preserves_norm_of_independent_unit_inputs():
    # the "norm-preserving" property: independent zero-mean unit-variance
    # stream and branch give a unit-variance result for any gate
    r = rng(5)
    g = np.array([-8.0, -1.0, 0.0, 0.4, 2.0, 9.0], np.float32)
    n = 200000
    h = r.standard_normal((n, g.size)).astype(np.float32)
    b = r.standard_normal((n, g.size)).astype(np.float32)
    _, lo, _, _ = oracle.residual(h, b, g, 0.3, 1e-3)
    var = (lo ** 2).mean(axis=0)
    assert np.all(np.abs(var - 1.0) < 0.02), var
