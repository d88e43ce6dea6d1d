"""Pins of the oracle's backward (gradients of the five cores).

The oracle writes each gradient out by hand.  These tests check it against
torch.autograd in float64 on the forward definitions (autograd derives the
gradients itself, so a dropped term, a wrong sign or a transposed rotation in
the hand-written formulas fails here).  A forward cast is modelled for
autograd as a straight-through rounding (value rounded, gradient passed
unchanged), which is the oracle's round_grads = 0.  The gradient roundings
of round_grads = 1 are pinned by composition: the rounded gradient fed into
the separately pinned plain backward must give the same result.
"""
import math

import numpy as np
import pytest
import torch

import oracle

REL = 1e-12


def bf16_vals(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def rnd_bf16(shape, rng, scale=1.0):
    return oracle.round_bf16(rng.standard_normal(shape) * scale)


def ste(v):
    """Straight-through bf16 rounding: forward value rounded, gradient identity."""
    r = torch.from_numpy(bf16_vals(oracle.round_bf16(v.detach().numpy())))
    return v + (r - v).detach()


def close(a, b, mag, rel=REL):
    a, b, mag = np.asarray(a), np.asarray(b), np.asarray(mag)
    err = np.abs(a - b)
    bad = err > rel * (mag + 1e-300) + 1e-300
    assert not bad.any(), (np.argmax(err / (mag + 1e-300)), float(np.max(err / (mag + 1e-300))))


def rms(u, eps):
    return 1.0 / torch.sqrt((u * u).mean(-1, keepdim=True) + eps)


@pytest.mark.parametrize("offset", [0.0, 1.0])
@pytest.mark.parametrize("eps", [1e-6, 0.5])
def test_rms_norm_bwd_matches_autograd(offset, eps):
    rng = np.random.default_rng(1)
    R, H = 5, 48
    xb, dyb = rnd_bf16((R, H), rng), rnd_bf16((R, H), rng)
    gain = (rng.uniform(-0.5, 0.5, H) if offset else rng.uniform(0.5, 1.5, H)).astype(np.float32)
    (dx, lo, hi, mag), (glo, ghi, gmag) = oracle.rms_norm_bwd(xb, dyb, gain, offset, eps)
    x = torch.tensor(bf16_vals(xb), requires_grad=True)
    w = torch.tensor((gain + np.float32(offset)).astype(np.float32).astype(np.float64), requires_grad=True)
    y = x * rms(x, eps) * w
    (y * torch.tensor(bf16_vals(dyb))).sum().backward()
    assert np.array_equal(lo, hi)
    close(lo, x.grad.numpy(), mag)
    assert np.array_equal(dx, oracle.round_bf16(lo))
    close(glo, w.grad.numpy(), gmag)
    assert np.array_equal(glo, ghi)


def test_rms_norm_bwd_without_gain_is_orthogonal_to_x():
    # eps = 0, no gain: the Jacobian annihilates x, so sum_k x_k dx_k = 0
    rng = np.random.default_rng(2)
    xb, dyb = rnd_bf16((3, 64), rng), rnd_bf16((3, 64), rng)
    (_, lo, _, mag), dg = oracle.rms_norm_bwd(xb, dyb, None, 0.0, 0.0)
    assert dg is None
    x = bf16_vals(xb)
    dots = (x * lo).sum(-1)
    assert np.all(np.abs(dots) <= 1e-12 * (np.abs(x) * mag).sum(-1))


@pytest.mark.parametrize("offset", [0.0, 1.0])
def test_input_scale_norm_bwd_matches_autograd(offset):
    rng = np.random.default_rng(3)
    R, H, eps = 4, 40, 1e-6
    xb, dyb = rnd_bf16((R, H), rng), rnd_bf16((R, H), rng)
    gain = (rng.uniform(-0.5, 0.5, H) if offset else rng.uniform(0.5, 1.5, H)).astype(np.float32)
    (dx, lo, hi, mag), (glo, ghi, gmag) = oracle.input_scale_norm_bwd(xb, dyb, gain, offset, eps)
    x = torch.tensor(bf16_vals(xb), requires_grad=True)
    w = torch.tensor((gain + np.float32(offset)).astype(np.float32).astype(np.float64), requires_grad=True)
    z = x * w
    y = z * rms(z, eps)
    (y * torch.tensor(bf16_vals(dyb))).sum().backward()
    close(lo, x.grad.numpy(), mag)
    close(glo, w.grad.numpy(), gmag)


def test_input_scale_differs_from_rms_bwd():
    # the two forms coincide only for a unit gain
    rng = np.random.default_rng(4)
    xb, dyb = rnd_bf16((2, 32), rng), rnd_bf16((2, 32), rng)
    one = np.ones(32, np.float32)
    a = oracle.rms_norm_bwd(xb, dyb, one, 0.0, 1e-6)[0][1]
    b = oracle.input_scale_norm_bwd(xb, dyb, one, 0.0, 1e-6)[0][1]
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
    g = np.linspace(0.5, 1.5, 32).astype(np.float32)
    a = oracle.rms_norm_bwd(xb, dyb, g, 0.0, 1e-6)[0][1]
    b = oracle.input_scale_norm_bwd(xb, dyb, g, 0.0, 1e-6)[0][1]
    assert np.max(np.abs(a - b)) > 1e-3


@pytest.mark.parametrize("per_token", [False, True])
def test_output_norm_gate_bwd_matches_autograd(per_token):
    rng = np.random.default_rng(5)
    T, Hh, D, eps = 3, 4, 16, 1e-6
    ob, gb, dyb = rnd_bf16((T, Hh, D), rng), rnd_bf16((T, Hh, D), rng, 2.0), rnd_bf16((T, Hh, D), rng)
    ng = Hh * D if per_token else D
    (do, olo, ohi, omag), (dg, glo, ghi, gmag) = oracle.output_norm_gate_bwd(ob, gb, dyb, ng, eps)
    o = torch.tensor(bf16_vals(ob), requires_grad=True)
    g = torch.tensor(bf16_vals(gb), requires_grad=True)
    og = o.reshape(T, -1, ng)
    y = (og * rms(og, eps)).reshape(T, Hh, D) * torch.sigmoid(g)
    (y * torch.tensor(bf16_vals(dyb))).sum().backward()
    close(olo, o.grad.numpy(), omag)
    close(glo, g.grad.numpy(), gmag)


def test_output_norm_gate_bwd_saturated_gate():
    # sigmoid -> 1 for large gates: do becomes the plain norm backward, dg -> 0
    rng = np.random.default_rng(6)
    ob, dyb = rnd_bf16((2, 1, 32), rng), rnd_bf16((2, 1, 32), rng)
    gb = oracle.round_bf16(np.full((2, 1, 32), 60.0))
    (_, olo, _, _), (_, glo, _, _) = oracle.output_norm_gate_bwd(ob, gb, dyb, None, 1e-6)
    ref = oracle.rms_norm_bwd(ob.reshape(2, 32), dyb.reshape(2, 32), None, 0.0, 1e-6)[0][1]
    np.testing.assert_allclose(olo.reshape(2, 32), ref, rtol=1e-12, atol=1e-20)
    assert np.all(np.abs(glo) < 1e-20)


@pytest.mark.parametrize("input_scale", [False, True])
def test_norm_residual_bwd_matches_autograd(input_scale):
    rng = np.random.default_rng(7)
    R, H, eps = 4, 32, 1e-6
    hb = rng.standard_normal((R, H)).astype(np.float32)
    bb = rnd_bf16((R, H), rng)
    dh = rng.standard_normal((R, H)).astype(np.float32)
    theta = rng.uniform(0, math.pi / 2, H).astype(np.float32)
    gain = rng.uniform(0.5, 1.5, H).astype(np.float32)
    (ds, slo, _, smag), (db, blo, bhi, bmag), (glo, ghi, gmag), (tlo, thi, tmag) = \
        oracle.norm_residual_bwd(hb, bb, dh, theta, gain, 0.0, input_scale, eps, round_grads=False)
    h = torch.tensor(hb.astype(np.float64), requires_grad=True)
    b = torch.tensor(bf16_vals(bb), requires_grad=True)
    w = torch.tensor(gain.astype(np.float64), requires_grad=True)
    th = torch.tensor(theta.astype(np.float64), requires_grad=True)
    if input_scale:
        z = b * w
        v = z * rms(z, eps)
    else:
        v = b * rms(b, eps) * w
    nb = ste(v)
    out = torch.cos(th) * h + torch.sin(th) * nb
    (out * torch.tensor(dh.astype(np.float64))).sum().backward()
    close(slo, h.grad.numpy(), smag)
    close(blo, b.grad.numpy(), bmag)
    close(glo, w.grad.numpy(), gmag)
    # dtheta uses the forward's cast nb; its bracket is over nb's admissible casts
    close(tlo, th.grad.numpy(), tmag, rel=1e-9)


def test_norm_residual_bwd_rounded_gradient_composes():
    # round_grads: dnb = bf16(sin(theta) dh') fed to the pinned core 1 backward
    rng = np.random.default_rng(8)
    R, H, eps = 3, 32, 1e-6
    hb = rng.standard_normal((R, H)).astype(np.float32)
    bb = rnd_bf16((R, H), rng)
    dh = rng.standard_normal((R, H)).astype(np.float32)
    theta = rng.uniform(0, math.pi / 2, H).astype(np.float32)
    gain = rng.uniform(0.5, 1.5, H).astype(np.float32)
    _, (db, blo, bhi, _), (glo, ghi, _), _ = oracle.norm_residual_bwd(
        hb, bb, dh, theta, gain, 0.0, False, eps, round_grads=True)
    dnb = oracle.round_bf16(np.sin(theta.astype(np.float64)) * dh.astype(np.float64))
    (dx, lo, _, _), (g2, _, _) = oracle.rms_norm_bwd(bb, dnb, gain, 0.0, eps)
    assert np.array_equal(db, dx)
    assert np.all(blo <= lo) and np.all(lo <= bhi)
    assert np.all(glo <= g2 + 1e-12 * np.abs(g2)) and np.all(g2 <= ghi + 1e-12 * np.abs(g2))


def test_norm_residual_bwd_theta_zero():
    # theta = 0: dh = dh', no gradient reaches the branch, dtheta = sum dh' nb
    rng = np.random.default_rng(9)
    hb = rng.standard_normal((2, 16)).astype(np.float32)
    bb = rnd_bf16((2, 16), rng)
    dh = rng.standard_normal((2, 16)).astype(np.float32)
    theta = np.zeros(16, np.float32)
    (ds, *_), (db, *_), _, (tlo, thi, _) = oracle.norm_residual_bwd(hb, bb, dh, theta)
    assert np.array_equal(ds, dh)
    assert np.all(bf16_vals(db) == 0)
    nb = oracle.rms_norm(bb, None, 0.0, 1e-6)[0]
    ref = (dh.astype(np.float64) * bf16_vals(nb)).sum(0)
    tol = 1e-12 * np.abs(dh.astype(np.float64) * bf16_vals(nb)).sum(0)
    assert np.all(tlo - tol <= ref) and np.all(ref <= thi + tol)


@pytest.mark.parametrize("use_rope", [True, False])
def test_qk_norm_rope_bwd_matches_autograd(use_rope):
    rng = np.random.default_rng(10)
    T, hq, hkv, D, eps, qs, base = 3, 2, 1, 16, 1e-6, 0.125, 10000.0
    qb, kb = rnd_bf16((T, hq, D), rng), rnd_bf16((T, hkv, D), rng)
    dqb, dkb = rnd_bf16((T, hq, D), rng), rnd_bf16((T, hkv, D), rng)
    pos = np.array([0, 7, 1234], np.int32)
    (dq, qlo, qhi, qmag), (dk, klo, khi, kmag) = oracle.qk_norm_rope_bwd(
        qb, kb, dqb, dkb, pos, eps, qs, use_rope, base, round_grads=False)
    inv = oracle.inv_freq(D, base).astype(np.float32)
    phi = (pos.astype(np.float32)[:, None] * inv[None, :]).astype(np.float32).astype(np.float64)
    c = torch.tensor(np.cos(phi))[:, None, :]
    s = torch.tensor(np.sin(phi))[:, None, :]

    def fwd(x, scale):
        n = ste(x * rms(x, eps))
        if scale is not None:
            n = ste(n * scale)
        if not use_rope:
            return n
        a, b = n[..., 0::2], n[..., 1::2]
        return torch.stack([a * c - b * s, a * s + b * c], dim=-1).reshape(n.shape)

    q = torch.tensor(bf16_vals(qb), requires_grad=True)
    k = torch.tensor(bf16_vals(kb), requires_grad=True)
    loss = (fwd(q, qs) * torch.tensor(bf16_vals(dqb))).sum() + \
        (fwd(k, None) * torch.tensor(bf16_vals(dkb))).sum()
    loss.backward()
    close(qlo, q.grad.numpy(), qmag)
    close(klo, k.grad.numpy(), kmag)


def test_qk_norm_rope_bwd_rounded_gradient_composes():
    # round_grads: the key gradient is the plain norm backward of bf16(R^T dy),
    # the query gradient that of bf16(bf16(R^T dy) * query_scale), with R the
    # FP32-angle rotation
    rng = np.random.default_rng(11)
    T, D, eps, base, qs = 2, 32, 1e-6, 5e5, 0.3
    qb, kb = rnd_bf16((T, 1, D), rng), rnd_bf16((T, 1, D), rng)
    dqb, dkb = rnd_bf16((T, 1, D), rng), rnd_bf16((T, 1, D), rng)
    pos = np.array([3, 4000], np.int32)
    (dq, qlo, qhi, _), (dk, klo, khi, _) = oracle.qk_norm_rope_bwd(qb, kb, dqb, dkb, pos, eps, qs,
                                                                    True, base)
    inv = oracle.inv_freq(D, base).astype(np.float32)
    phi = (pos.astype(np.float32)[:, None] * inv[None, :]).astype(np.float32).astype(np.float64)

    def rt(dyb):
        dy = bf16_vals(dyb)[:, 0, :]
        a, b = dy[:, 0::2], dy[:, 1::2]
        m = np.stack([np.cos(phi) * a + np.sin(phi) * b, -np.sin(phi) * a + np.cos(phi) * b], -1)
        return oracle.round_bf16(m.reshape(T, D))

    dn = rt(dkb)
    (dx, lo, _, _), _ = oracle.rms_norm_bwd(kb[:, 0, :], dn, None, 0.0, eps)
    assert np.array_equal(dk[:, 0, :], dx)
    assert np.all(klo[:, 0, :] <= lo) and np.all(lo <= khi[:, 0, :])
    dn = oracle.round_bf16(bf16_vals(rt(dqb)) * qs)
    (dx, lo, _, _), _ = oracle.rms_norm_bwd(qb[:, 0, :], dn, None, 0.0, eps)
    assert np.array_equal(dq[:, 0, :], dx)
    assert np.all(qlo[:, 0, :] <= lo) and np.all(lo <= qhi[:, 0, :])


def _bf16_ok(gpu_bits, lo, hi, mag):
    from .parity import bf16_ok, BWD_EVAL_ULPS
    return bf16_ok(gpu_bits, lo, hi, mag, BWD_EVAL_ULPS)


@pytest.mark.parametrize("qs", [1.0, 0.3])
def test_qk_norm_rope_bwd_v2_matches_bf16_autograd(qs):
    # The v2 rotation on bf16 tensors, written with torch's own bf16 CPU
    # operations (each product and sum rounded to bf16, cos/sin cast to bf16);
    # torch.autograd then derives the backward through those bf16 operations
    # (a product's gradient rounded to bf16, the two gradients of a tensor used
    # twice added in bf16).  The oracle's v2 backward must agree within the
    # backward rule.
    rng = np.random.default_rng(21)
    T, hq, hkv, D, eps, base = 6, 4, 2, 64, 1e-6, 10000.0
    qb, kb = rnd_bf16((T, hq, D), rng, 3.0), rnd_bf16((T, hkv, D), rng, 3.0)
    dqb, dkb = rnd_bf16((T, hq, D), rng), rnd_bf16((T, hkv, D), rng)
    pos = np.array([0, 1, 17, 999, 4096, 31000], np.int32)
    (dq, qlo, qhi, qmag), (dk, klo, khi, kmag) = oracle.qk_norm_rope_bwd(
        qb, kb, dqb, dkb, pos, eps, qs, True, base, upcast_rope=False)
    inv = torch.tensor(oracle.inv_freq(D, base).astype(np.float32))
    phi = torch.tensor(pos).float()[:, None] * inv[None, :]          # FP32 angle
    C = torch.cos(phi).to(torch.bfloat16)[:, None, :]
    S = torch.sin(phi).to(torch.bfloat16)[:, None, :]

    def to_t(bits):
        return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)

    def fwd(x, scale):
        xf = x.float()
        n = (xf * torch.rsqrt((xf * xf).mean(-1, keepdim=True) + eps)).to(torch.bfloat16)
        if scale is not None:
            n = n * scale
        a, b = n[..., 0::2], n[..., 1::2]
        return torch.stack([a * C - b * S, a * S + b * C], dim=-1).reshape(n.shape)

    q = to_t(qb).requires_grad_(True)
    k = to_t(kb).requires_grad_(True)
    fwd(q, qs if qs != 1.0 else None).backward(to_t(dqb))
    fwd(k, None).backward(to_t(dkb))
    gq = q.grad.view(torch.int16).numpy().view(np.uint16)
    gk = k.grad.view(torch.int16).numpy().view(np.uint16)
    assert _bf16_ok(gq, qlo, qhi, qmag).all()
    assert _bf16_ok(gk, klo, khi, kmag).all()


def test_qk_norm_rope_bwd_v2_rounded_gradient_composes():
    # v2: the key gradient is the plain norm backward of the pairs
    # (bf16(bf16(dy0 C) + bf16(dy1 S)), bf16(bf16(dy1 C) - bf16(dy0 S))),
    # C, S the bf16 cos / sin of the FP32 angle; it differs from the FP32
    # rotation's gradient
    rng = np.random.default_rng(22)
    T, D, eps, base = 4, 32, 1e-6, 5e5
    kb = rnd_bf16((T, 1, D), rng)
    dkb = rnd_bf16((T, 1, D), rng)
    qb, dqb = kb.copy(), dkb.copy()
    pos = np.array([3, 77, 4000, 12345], np.int32)
    _, (dk, klo, khi, _) = oracle.qk_norm_rope_bwd(qb, kb, dqb, dkb, pos, eps, 1.0, True, base,
                                                   upcast_rope=False)
    _, (dk_legacy, *_) = oracle.qk_norm_rope_bwd(qb, kb, dqb, dkb, pos, eps, 1.0, True, base)
    inv = oracle.inv_freq(D, base).astype(np.float32)
    phi = (pos.astype(np.float32)[:, None] * inv[None, :]).astype(np.float32).astype(np.float64)
    C, S = bf16_vals(oracle.round_bf16(np.cos(phi))), bf16_vals(oracle.round_bf16(np.sin(phi)))
    r = lambda v: bf16_vals(oracle.round_bf16(v))
    dy = bf16_vals(dkb)[:, 0, :]
    a, b = dy[:, 0::2], dy[:, 1::2]
    dn = np.stack([r(r(a * C) + r(b * S)), r(r(b * C) - r(a * S))], -1).reshape(T, D)
    (dx, lo, _, _), _ = oracle.rms_norm_bwd(kb[:, 0, :], oracle.round_bf16(dn), None, 0.0, eps)
    assert np.array_equal(dk[:, 0, :], dx)
    assert np.all(klo[:, 0, :] <= lo) and np.all(lo <= khi[:, 0, :])
    assert not np.array_equal(dk, dk_legacy)
