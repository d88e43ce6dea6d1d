"""Pins of the _residual_core backward oracle (residual_blend_bwd,
residual_bwd) against torch.autograd in float64 on the forward definitions
(angle form: cos(theta) h + sin(theta) b; gate form under reading R29:
c = sqrt(clamp_min(sigmoid(gate / temperature), eps)), s = sqrt(1 - c^2)),
so autograd, not a retyped derivative, derives the reference; plus the
special cases the derivative must meet."""
import numpy as np
import pytest
import torch

import oracle


def rng(seed=0):
    return np.random.default_rng(seed)


def _inputs(seed, rows=6, hidden=40, bf16=False):
    r = rng(seed)
    h = r.standard_normal((rows, hidden)).astype(np.float32)
    b = r.standard_normal((rows, hidden)).astype(np.float32)
    dy = r.standard_normal((rows, hidden)).astype(np.float32)
    if bf16:
        b = torch.from_numpy(b).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return h, b, dy


def _b64(b):
    if b.dtype == np.uint16:
        return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return b.astype(np.float64)


def _autograd(h, b, dy, coef):
    th = torch.tensor(h, dtype=torch.float64, requires_grad=True)
    tb = torch.tensor(_b64(b), requires_grad=True)
    c, s, p = coef()
    y = c * th + s * tb
    (y * torch.tensor(dy, dtype=torch.float64)).sum().backward()
    return th.grad.numpy(), tb.grad.numpy(), p.grad.numpy()


@pytest.mark.parametrize("bf16", [False, True])
def test_angle_form_matches_autograd(bf16):
    h, b, dy = _inputs(1, bf16=bf16)
    theta = rng(2).uniform(0, np.pi / 2, h.shape[1]).astype(np.float32)

    def coef():
        t = torch.tensor(theta, dtype=torch.float64, requires_grad=True)
        return torch.cos(t), torch.sin(t), t
    gh, gb, gt = _autograd(h, b, dy, coef)
    (ds, sl, _, _), (db, bl, _, _), (pl, ph, pm) = oracle.residual_blend_bwd(h, b, dy, theta)
    np.testing.assert_allclose(sl, gh, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(bl, gb, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(pl, gt, rtol=1e-12, atol=1e-13)
    assert np.array_equal(pl, ph) and np.all(pm >= np.abs(pl))
    # the branch gradient is stored rounded to the branch dtype
    if bf16:
        want = torch.tensor(gb).to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(db, oracle.round_bf16(bl)) and np.mean(db == want) > 0.99


@pytest.mark.parametrize("temperature,eps", [(0.3, 1e-3), (1.0, 0.0), (0.1, 0.05)])
def test_gate_form_matches_autograd(temperature, eps):
    h, b, dy = _inputs(3, hidden=64)
    # gate / temperature within +-7: autograd's s = sqrt(1 - c^2) cancels as c
    # nears 1 (its own error grows like 1e-16 / s^2), so the reference is only
    # trusted where s^2 >= 1e-3
    g = (np.clip(rng(4).standard_normal(64) * 2.5, -7, 7) * temperature).astype(np.float32)
    eps32 = float(np.float32(eps))

    def coef():
        tg = torch.tensor(g, dtype=torch.float64, requires_grad=True)
        c2 = torch.clamp_min(torch.sigmoid(tg / float(np.float32(temperature))), eps32)
        return torch.sqrt(c2), torch.sqrt(1.0 - c2), tg
    gh, gb, gg = _autograd(h, b, dy, coef)
    (ds, sl, _, _), (db, bl, _, _), (pl, ph, pm) = oracle.residual_bwd(h, b, dy, g, temperature, eps32)
    np.testing.assert_allclose(sl, gh, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(bl, gb, rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(pl, gg, rtol=1e-9, atol=1e-12)


def test_gate_gradient_is_zero_where_the_bound_holds():
    h, b, dy = _inputs(5, hidden=8)
    g = np.array([-50.0, -20.0, -5.0, -1.0, 0.0, 1.0, 5.0, 20.0], np.float32)
    _, _, (pl, _, _) = oracle.residual_bwd(h, b, dy, g, 0.3, 0.01)
    # sigmoid(g / 0.3) < 0.01 for the first three gates (g / 0.3 < -4.6)
    assert np.all(pl[:3] == 0.0) and np.all(pl[3:7] != 0.0)


def test_zero_angle_and_quarter_turn():
    h, b, dy = _inputs(6, hidden=4)
    th = np.zeros(4, np.float32)
    (ds, sl, _, _), (_, bl, _, _), (pl, _, _) = oracle.residual_blend_bwd(h, b, dy, th)
    assert np.array_equal(ds.view(np.uint32), dy.view(np.uint32))  # cos 0 = 1: dstream = dy exactly
    assert np.all(bl == 0.0)                                       # sin 0 = 0
    np.testing.assert_allclose(pl, (dy.astype(np.float64) * b).sum(0), rtol=1e-15)  # d/dtheta = b at 0
    # a quarter turn: the stream's gradient vanishes, the branch takes dy, d/dtheta = -h
    th = np.full(4, np.pi / 2, np.float32)
    c, s = np.cos(np.float64(th[0])), np.sin(np.float64(th[0]))
    (ds, sl, _, _), (_, bl, _, _), (pl, _, _) = oracle.residual_blend_bwd(h, b, dy, th)
    assert np.all(np.abs(sl) <= 1e-7 * np.abs(dy)) and np.allclose(bl, s * dy, rtol=1e-15)
    np.testing.assert_allclose(pl, (dy.astype(np.float64) * (-s * h + c * b)).sum(0), rtol=1e-12)
    assert np.all(np.sign(pl) == np.sign(-(dy.astype(np.float64) * h).sum(0)))


def test_gate_and_angle_forms_chain():
    # dL/dgate = dL/dtheta * dtheta/dgate with dtheta/dgate = -c s / (2 temperature)
    h, b, dy = _inputs(7, hidden=32)
    g = (rng(8).standard_normal(32)).astype(np.float32)
    c, s, th = oracle.residual_gate_coefficients(g, 0.3, 1e-3)
    _, _, (pg, _, _) = oracle.residual_bwd(h, b, dy, g, 0.3, 1e-3)
    # the angle form at the same coefficients (theta rounded to FP32 moves c, s by 1e-8)
    _, _, (pt, _, pm) = oracle.residual_blend_bwd(h, b, dy, th.astype(np.float32))
    want = pt * (-c * s / (2 * float(np.float32(0.3))))
    free = 1 / (1 + np.exp(-g.astype(np.float64) / float(np.float32(0.3)))) >= float(np.float32(1e-3))
    assert np.any(~free) and np.all(pg[~free] == 0.0)
    assert np.all(np.abs(pg - want)[free] <= 1e-6 * pm[free] + 1e-12)
