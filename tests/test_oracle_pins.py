"""Pins of the CPU oracle against what the pages and mathematics fix.

None of these compares the oracle with a retyped copy of itself: each check is
a closed form worked out by hand (tests/golden/closed_forms.json), an
invariant of the definition, a special case that reduces to another core or to
a textbook routine, or an exhaustive/library cross-check of a rounding rule.
Each is chosen so that a plausible slip in the oracle (a dropped eps, gain on
the wrong side of the norm, a swapped RoPE sign or pairing, a missing cast, a
wrong sigmoid sign, a missing blend term) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from gate_cores_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def bf16(a):
    """float array -> bf16 bit patterns via torch (round to nearest even)."""
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def from_bf16(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def rng(seed=0):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------- rounding

def test_round_bf16_matches_torch_on_float32_values():
    r = rng(1)
    v = np.concatenate([
        r.standard_normal(200000).astype(np.float32),
        (r.standard_normal(20000) * 1e30).astype(np.float32),
        (r.standard_normal(20000) * 1e-38).astype(np.float32),  # subnormal range
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.3895314e38, -3.39e38,
                  np.inf, -np.inf], dtype=np.float32),
    ])
    # exact ties: bf16 value + half spacing, both parities
    base = from_bf16(np.arange(0x3F80, 0x3F90, dtype=np.uint16)).astype(np.float32)
    ties = (base * np.float32(1 + 2.0 ** -8)).astype(np.float32)
    v = np.concatenate([v, ties])
    got = oracle.round_bf16(v.astype(np.float64))
    want = bf16(v)
    assert np.array_equal(got, want)


def test_round_bf16_nearest_by_exhaustive_search_on_doubles():
    # Doubles that are not float32 values: the answer must be the nearest of all
    # finite bf16 values (ties to even), found by brute force.
    all_bits = np.arange(0, 0x7F80, dtype=np.uint16)  # non-negative finite bf16
    vals = from_bf16(all_bits)
    r = rng(2)
    v = np.abs(r.standard_normal(3000)) * 10.0 ** r.integers(-30, 30, 3000)
    v = np.concatenate([v, vals[1000:1100] + (vals[1001:1101] - vals[1000:1100]) / 2])  # ties
    got = oracle.round_bf16(v)
    idx = np.searchsorted(vals, v)
    for i, x in enumerate(v):
        j = idx[i]
        cands = [k for k in (j - 1, j) if 0 <= k < len(vals)]
        d = [abs(vals[k] - x) for k in cands]
        best = [cands[t] for t in range(len(cands)) if d[t] == min(d)]
        if len(best) == 2:  # tie: even mantissa
            best = [k for k in best if (all_bits[k] & 1) == 0]
        assert got[i] == all_bits[best[0]], (x, got[i], all_bits[best[0]])


# ------------------------------------------------------------ golden cases

def _eval(expr, eps):
    env = {k: getattr(math, k) for k in ("sqrt", "cos", "sin", "exp")}
    env["eps"] = eps
    env["f32"] = lambda v: float(np.float32(v))
    return float(eval(expr, {"__builtins__": {}}, env))


def _f32(a):
    return None if a is None else np.asarray(a, dtype=np.float32)


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_golden_closed_forms(case):
    core = case["core"]
    eps = float(np.float32(case.get("eps", case.get("norm_eps", 0.0))))
    if core in ("rms_norm", "input_scale_norm"):
        fn = getattr(oracle, core)
        out, lo, hi, mag = fn(_f32(case["x"]), _f32(case["gain"]), case["gain_offset"], eps)
        got = {"expect": lo.ravel()}
        assert np.array_equal(lo, hi)
    elif core == "qk_norm_rope":
        (qo, ql, qh, _), (ko, kl, kh, _) = oracle.qk_norm_rope(
            _f32(case["q"]), _f32(case["k"]), np.asarray(case["pos"], np.int32), eps,
            case["query_scale"], case["use_rope"], case["upcast_rope"], case["rope_base"])
        got = {"expect_q": ql.ravel(), "expect_k": kl.ravel()}
        assert np.array_equal(ql, qh) and np.array_equal(kl, kh)
    elif core == "output_norm_gate":
        out, lo, hi, mag = oracle.output_norm_gate(_f32(case["o"]), _f32(case["g"]),
                                                   case["norm_group"], eps)
        got = {"expect": lo.ravel()}
    elif core == "norm_residual":
        out, lo, hi, mag = oracle.norm_residual(
            _f32(case["stream"]), _f32(case["branch"]), _f32(case["theta"]), _f32(case["gain"]),
            case["gain_offset"], case["input_scale"], eps)
        got = {"expect": lo.ravel()}
    elif core == "residual_blend":
        out, lo, hi, mag = oracle.residual_blend(_f32(case["stream"]), _f32(case["branch"]),
                                                 _f32(case["theta"]))
        got = {"expect": lo.ravel()}
    elif core == "residual":
        out, lo, hi, mag = oracle.residual(_f32(case["stream"]), _f32(case["branch"]), _f32(case["gate"]),
                                           case["temperature"], float(np.float32(case["eps"])))
        got = {"expect": lo.ravel()}
    else:
        raise AssertionError(core)
    for key, vals in got.items():
        want = np.array([_eval(e, eps) for e in case[key]])
        np.testing.assert_allclose(vals, want, rtol=1e-14, atol=1e-15, err_msg=f"{case['name']} {key}")


# ------------------------------------------------------------ positions / freq

def test_positions_bshd_and_thd():
    assert oracle.positions(0, batch=2, seqlen=3).tolist() == [0, 1, 2, 0, 1, 2]
    cu = np.array([0, 2, 5, 5, 6], np.int32)
    assert oracle.positions(1, cu_seqlens=cu, total_tokens=6).tolist() == [0, 1, 0, 1, 2, 0]
    with pytest.raises(ValueError):
        oracle.positions(1, cu_seqlens=np.array([0, 3, 2], np.int32), total_tokens=2)
    with pytest.raises(ValueError):
        oracle.positions(1, cu_seqlens=np.array([0, 3, 5], np.int32), total_tokens=6)


def test_inv_freq_definition():
    # base 256, D 8: base^(-2i/D) = 2^(-2i) exactly
    assert oracle.inv_freq(8, 256.0).tolist() == [1.0, 0.25, 0.0625, 0.015625]
    f = oracle.inv_freq(128, 500000.0).astype(np.float64)
    assert f[0] == 1.0 and np.all(np.diff(f) < 0)
    # library cross-check: torch float64 power, rounded once to float32
    i = torch.arange(0, 64, dtype=torch.float64)
    want = (1.0 / torch.pow(torch.tensor(500000.0, dtype=torch.float64), 2 * i / 128)).float().numpy()
    assert np.array_equal(oracle.inv_freq(128, 500000.0), want)


# ------------------------------------------------------------------ core 1

def _rand_bf16(shape, seed, scale=1.0):
    return bf16(rng(seed).standard_normal(shape) * scale)


def test_rms_norm_unit_rms_and_eps_effect():
    x = _rand_bf16((16, 256), 3)
    _, lo, hi, _ = oracle.rms_norm(x, None, 0.0, 0.0)
    rms = np.sqrt(np.mean(lo ** 2, axis=1))
    np.testing.assert_allclose(rms, 1.0, rtol=1e-14)
    _, lo_e, _, _ = oracle.rms_norm(x, None, 0.0, 1e-6)
    rms_e = np.sqrt(np.mean(lo_e ** 2, axis=1))
    ms = np.mean(from_bf16(x) ** 2, axis=1)
    # RMS 1 up to the stabiliser: below 1 by about eps/(2 ms)
    assert np.all(rms_e < 1.0) and np.all(1.0 - rms_e < 1e-6 / ms)


def test_rms_norm_zero_centered_zero_gain_is_parameter_free():
    x = _rand_bf16((8, 512), 4)
    a = oracle.rms_norm(x, np.zeros(512, np.float32), 1.0, 1e-6)[0]
    b = oracle.rms_norm(x, None, 0.0, 1e-6)[0]
    assert np.array_equal(a, b)


def test_rms_norm_power_of_two_scale_invariance():
    x = _rand_bf16((8, 256), 5)
    x2 = bf16(from_bf16(x) * 4.0)
    assert np.array_equal(oracle.rms_norm(x, None, 0, 0.0)[0], oracle.rms_norm(x2, None, 0, 0.0)[0])


def test_rms_norm_constant_and_one_hot_rows():
    H = 64
    for c in (0.5, 3.0, -7.25):
        x = bf16(np.full((1, H), c))
        _, lo, _, _ = oracle.rms_norm(x, None, 0, 1e-6)
        eps = float(np.float32(1e-6))
        np.testing.assert_allclose(lo, c / math.sqrt(c * c + eps), rtol=1e-15)
        x = np.zeros((1, H), np.float32)
        x[0, 7] = c
        _, lo, _, _ = oracle.rms_norm(x, None, 0, 1e-6)
        np.testing.assert_allclose(lo[0, 7], c / math.sqrt(c * c / H + eps), rtol=1e-15)
        assert np.count_nonzero(lo) == 1


def test_rms_norm_gain_after_norm_does_not_change_scale():
    x = _rand_bf16((4, 128), 6)
    g = (rng(7).random(128) + 0.5).astype(np.float32)
    _, lo_g, _, _ = oracle.rms_norm(x, g, 0.0, 1e-6)
    _, lo_n, _, _ = oracle.rms_norm(x, None, 0.0, 1e-6)
    # the gain scales each channel of the normalised row; r(x) is unchanged
    np.testing.assert_allclose(lo_g / lo_n, np.broadcast_to(g.astype(np.float64), lo_g.shape), rtol=1e-15)


def test_rms_norm_f32_and_bf16_paths_agree_before_cast():
    x = _rand_bf16((4, 256), 8)
    _, lo_b, _, _ = oracle.rms_norm(x, None, 0, 1e-6)
    _, lo_f, _, _ = oracle.rms_norm(from_bf16(x).astype(np.float32), None, 0, 1e-6)
    assert np.array_equal(lo_b, lo_f)


# ------------------------------------------------------------------ core 2

def test_input_scale_unit_gain_equals_rms_norm():
    x = _rand_bf16((8, 256), 9)
    ones = np.ones(256, np.float32)
    assert np.array_equal(oracle.input_scale_norm(x, ones, 0, 1e-6)[0],
                          oracle.rms_norm(x, ones, 0, 1e-6)[0])


def test_input_scale_power_of_two_gains_equal_norm_of_scaled_input():
    x = _rand_bf16((8, 256), 10)
    w = (2.0 ** rng(11).integers(-3, 4, 256)).astype(np.float32)
    xs = bf16(from_bf16(x) * w)  # exact: power-of-two scaling of bf16 values
    a = oracle.input_scale_norm(x, w, 0.0, 1e-6)[0]
    b = oracle.rms_norm(xs, None, 0.0, 1e-6)[0]
    assert np.array_equal(a, b)
    # and it differs from the gain-after-norm core
    assert not np.array_equal(a, oracle.rms_norm(x, w, 0.0, 1e-6)[0])


def test_input_scale_eps_acts_on_scaled_mean_square():
    # tiny activations: eps dominates an unscaled mean square but not a scaled one
    x = bf16(np.full((1, 16), 1e-4))
    w = np.full(16, 1024.0, np.float32)
    _, lo, _, _ = oracle.input_scale_norm(x, w, 0.0, 1e-6)
    z = float(from_bf16(x)[0, 0]) * 1024.0
    np.testing.assert_allclose(lo, z / math.sqrt(z * z + float(np.float32(1e-6))), rtol=1e-15)


# ------------------------------------------------------------------ core 3

def _qk(seed, T=6, hq=4, hkv=2, d=16):
    return _rand_bf16((T, hq, d), seed), _rand_bf16((T, hkv, d), seed + 1)


@pytest.mark.parametrize("upcast", [True, False])
def test_qk_position_zero_is_identity(upcast):
    q, k = _qk(12)
    pos = np.zeros(q.shape[0], np.int32)
    (qa, *_), (ka, *_) = oracle.qk_norm_rope(q, k, pos, 1e-6, 1.0, True, upcast, 10000.0)
    (qb, *_), (kb, *_) = oracle.qk_norm_rope(q, k, pos, 1e-6, 1.0, False, upcast, 10000.0)
    assert np.array_equal(qa, qb) and np.array_equal(ka, kb)


def test_qk_without_rope_is_per_head_parameter_free_norm():
    q, k = _qk(13)
    pos = np.arange(q.shape[0], dtype=np.int32)
    (qo, *_), (ko, *_) = oracle.qk_norm_rope(q, k, pos, 1e-6, 1.0, False, True, 10000.0)
    assert np.array_equal(qo.reshape(-1, 16), oracle.rms_norm(q.reshape(-1, 16), None, 0, 1e-6)[0])
    assert np.array_equal(ko.reshape(-1, 16), oracle.rms_norm(k.reshape(-1, 16), None, 0, 1e-6)[0])


def test_qk_query_scale_only_scales_queries():
    q, k = _qk(14)
    pos = np.arange(q.shape[0], dtype=np.int32)
    (q1, *_), (k1, *_) = oracle.qk_norm_rope(q, k, pos, 1e-6, 1.0, True, True, 10000.0)
    (q2, *_), (k2, *_) = oracle.qk_norm_rope(q, k, pos, 1e-6, 2.0, True, True, 10000.0)
    assert np.array_equal(k1, k2)
    # power-of-two scale commutes exactly with the casts and the rotation
    assert np.array_equal(from_bf16(q2), 2.0 * from_bf16(q1))


def test_qk_rotation_preserves_pair_norm():
    q, k = _qk(15, T=32, d=64)
    pos = rng(16).integers(0, 32768, 32).astype(np.int32)
    (_, ql, qh, _), _ = oracle.qk_norm_rope(q, k, pos, 1e-6, 1.0, False, True, 10000.0)
    (_, rl, rh, _), _ = oracle.qk_norm_rope(q, k, pos, 1e-6, 1.0, True, True, 500000.0)
    ok = (ql == qh).reshape(32, 4, 32, 2).all(-1) & (rl == rh).reshape(32, 4, 32, 2).all(-1)
    n_in = (ql.reshape(32, 4, 32, 2) ** 2).sum(-1)
    n_out = (rl.reshape(32, 4, 32, 2) ** 2).sum(-1)
    np.testing.assert_allclose(n_out[ok], n_in[ok], rtol=1e-13)


def test_qk_relative_position_property():
    # base 256, D 8: FP32 angles are exact, so <R(q,m), R(k,n)> depends only on m - n
    q, k = _qk(17, T=1, hq=1, hkv=1, d=8)

    def rot(pos):
        (_, ql, qh, _), (_, kl, kh, _) = oracle.qk_norm_rope(
            q, k, np.array([pos], np.int32), 1e-6, 1.0, True, True, 256.0)
        assert np.array_equal(ql, qh) and np.array_equal(kl, kh)
        return ql.ravel(), kl.ravel()

    for m, n, dlt in [(3, 1, 5), (10, 4, 100), (7, 7, 33)]:
        qm, _ = rot(m)
        _, kn = rot(n)
        qmd, _ = rot(m + dlt)
        _, knd = rot(n + dlt)
        assert abs(qm @ kn - qmd @ knd) < 1e-12 * (np.abs(qm) @ np.abs(kn))


def test_qk_rotation_matrix_brute_force():
    # textbook 2x2 rotation of each adjacent pair by angle pos * 4^-i (exact in FP32)
    q, k = _qk(18, T=4, hq=2, hkv=1, d=8)
    pos = np.array([0, 1, 5, 123], np.int32)
    (_, ql, qh, _), _ = oracle.qk_norm_rope(q, k, pos, 1e-6, 1.0, True, True, 256.0)
    (_, nl, _, _), _ = oracle.qk_norm_rope(q, k, pos, 1e-6, 1.0, False, True, 256.0)
    for t in range(4):
        for h in range(2):
            for i in range(4):
                ang = float(pos[t]) * 4.0 ** (-i)
                R = np.array([[math.cos(ang), -math.sin(ang)], [math.sin(ang), math.cos(ang)]])
                want = R @ nl[t, h, 2 * i:2 * i + 2]
                if ql[t, h, 2 * i] == qh[t, h, 2 * i]:
                    np.testing.assert_allclose(ql[t, h, 2 * i:2 * i + 2], want, rtol=1e-15, atol=1e-16)


def test_qk_v2_rotation_close_to_fp32_rotation():
    q, k = _qk(19, T=16, d=64)
    pos = rng(20).integers(0, 4096, 16).astype(np.int32)
    (a, *_), _ = oracle.qk_norm_rope(q, k, pos, 1e-6, 1.0, True, True, 10000.0)
    (b, *_), _ = oracle.qk_norm_rope(q, k, pos, 1e-6, 1.0, True, False, 10000.0)
    fa, fb = from_bf16(a), from_bf16(b)
    # v2 rounds two products and cos/sin to bf16: a few bf16 ulps of the terms at most
    assert np.all(np.abs(fa - fb) <= 2.0 ** -6 * 2.0)
    assert np.mean(a != b) > 0.05  # but it is a different rounding path


def test_qk_candidates_bracket_primary():
    q, k = _qk(21, T=64, hq=8, d=64)
    pos = np.arange(64, dtype=np.int32)
    for upcast in (True, False):
        (qo, ql, qh, qm), _ = oracle.qk_norm_rope(q, k, pos, 1e-6, 0.125, True, upcast, 10000.0)
        v = from_bf16(qo)
        assert np.all(ql <= qh)
        # the primary output is the rounding of a value inside [lo, hi]
        assert np.all(v >= from_bf16(oracle.round_bf16(ql)) - 1e-30)
        assert np.all(v <= from_bf16(oracle.round_bf16(qh)) + 1e-30)
        frac = np.mean(ql != qh)
        assert frac < 0.01


# ------------------------------------------------------------------ core 4

def test_output_gate_zero_gate_halves_norm():
    o = _rand_bf16((4, 4, 32), 22)
    g = np.zeros_like(o)
    y = oracle.output_norm_gate(o, g)[0]
    n = oracle.rms_norm(o.reshape(-1, 32), None, 0, 1e-6)[0].reshape(o.shape)
    assert np.array_equal(from_bf16(y), from_bf16(n) / 2)


def test_output_gate_saturation_limits():
    o = _rand_bf16((4, 4, 32), 23)
    n = oracle.rms_norm(o.reshape(-1, 32), None, 0, 1e-6)[0].reshape(o.shape)
    y_pos = oracle.output_norm_gate(o, bf16(np.full(o.shape, 100.0)))[0]
    assert np.array_equal(y_pos, n)
    y_neg = oracle.output_norm_gate(o, bf16(np.full(o.shape, -100.0)))[0]
    assert np.all(from_bf16(y_neg) == 0.0)


def test_output_gate_sigmoid_in_unit_interval_and_sign():
    o = _rand_bf16((8, 4, 64), 24)
    g = _rand_bf16((8, 4, 64), 25, 2.0)
    _, lo, _, _ = oracle.output_norm_gate(o, g)
    _, nlo, _, _ = oracle.rms_norm(o.reshape(-1, 64), None, 0, 1e-6)
    ratio = lo.reshape(-1, 64) / nlo
    assert np.all((ratio > 0) & (ratio < 1))
    # larger gate logit -> larger gate (sigmoid increasing, not decreasing)
    gg = from_bf16(g).reshape(-1, 64)
    order = np.argsort(gg, axis=None)
    assert np.all(np.diff(ratio.ravel()[order]) >= -1e-15)


def test_output_gate_whole_token_group():
    o = _rand_bf16((4, 4, 32), 26)
    y = oracle.output_norm_gate(o, bf16(np.full(o.shape, 100.0)), norm_group=128)[0]
    n = oracle.rms_norm(o.reshape(4, 128), None, 0, 1e-6)[0]
    assert np.array_equal(y.reshape(4, 128), n)


# ------------------------------------------------------------------ core 5

def _res_inputs(seed, T=8, H=256):
    r = rng(seed)
    h = r.standard_normal((T, H)).astype(np.float32)
    b = _rand_bf16((T, H), seed + 1)
    th = (r.random(H) * math.pi / 2).astype(np.float32)
    g = (r.random(H) - 0.5).astype(np.float32)
    return h, b, th, g


def test_residual_zero_angle_returns_stream():
    h, b, th, g = _res_inputs(27)
    out = oracle.norm_residual(h, b, np.zeros_like(th), g, 1.0)[0]
    assert np.array_equal(out, h)


@pytest.mark.parametrize("input_scale", [False, True])
def test_residual_zero_stream_gives_sin_times_branch_norm(input_scale):
    h, b, th, g = _res_inputs(28)
    out = oracle.norm_residual(np.zeros_like(h), b, th, g, 1.0, input_scale)[0]
    core = oracle.input_scale_norm if input_scale else oracle.rms_norm
    nb = from_bf16(core(b, g, 1.0, 1e-6)[0])
    derived = out.astype(np.float64) / np.sin(th.astype(np.float64))
    # out = f32(sin * nb): dividing by sin recovers nb to 2^-23, which pins the bf16 value
    assert np.array_equal(oracle.round_bf16(derived), bf16(nb))


def test_residual_coefficients_are_cos_and_sin():
    h, b, th, g = _res_inputs(29)
    zero_b = np.zeros_like(b)
    c = oracle.norm_residual(h, zero_b, th, g, 1.0)[0].astype(np.float64) / h
    s = oracle.norm_residual(np.zeros_like(h), b, th, g, 1.0)[0].astype(np.float64)
    nb = from_bf16(oracle.rms_norm(b, g, 1.0, 1e-6)[0])
    s = s / nb
    np.testing.assert_allclose(c ** 2 + s ** 2, 1.0, atol=1e-6)
    assert np.all(c > 0) and np.all(s > 0)  # theta in (0, pi/2)


def test_residual_branch_cast_before_blend():
    # the blend uses the bf16-rounded normalised branch: with h = 0 and theta
    # near pi/2 the output is sin(theta) times a bf16 value, not an FP32 one
    h, b, th, g = _res_inputs(30, T=4, H=64)
    th[:] = np.float32(math.pi / 2)
    out, lo, hi, _ = oracle.norm_residual(np.zeros_like(h), b, th, None, 0.0)
    nb = from_bf16(oracle.rms_norm(b, None, 0, 1e-6)[0])
    np.testing.assert_allclose(lo, nb * math.sin(float(np.float32(math.pi / 2))), rtol=1e-15)


def test_workload_inputs_deterministic_and_shaped():
    a = inputs.make_inputs("tiny_t64_h256", "qk_norm_rope", seed=0)
    b = inputs.make_inputs("tiny_t64_h256", "qk_norm_rope", seed=0)
    assert torch.equal(a.tensors["q"], b.tensors["q"])
    assert a.tensors["q"].shape == (64, 4, 64) and a.tensors["k"].shape == (64, 2, 64)
    cu = inputs.cu_seqlens(inputs.WORKLOADS["thd16_h5120"])
    lens = np.diff(cu.numpy())
    assert len(lens) == 16 and lens.min() >= 512 and lens.max() <= 8192
    big = inputs.WORKLOADS["large_t32768_h8192"]
    x = inputs.activation(big, 0, "probe", (4, 8192))
    col_max = x.float().abs().amax(0)
    assert int((col_max > 50).sum()) == 82  # 1% of 8192 channels scaled by 1000


def test_qk_query_scale_applies_to_the_cast_query():
    # Q and K hold the same rows; K's output is the cast normalised row n.  The
    # query must be bf16(n * query_scale) - scaling after the cast - which for a
    # non-power-of-two scale differs from casting x*r*query_scale once.
    q, _ = _qk(31, T=32, hq=4, hkv=4, d=64)
    qs = float(np.float32(128 ** -0.5))
    pos = np.zeros(32, np.int32)
    (qo, ql, qh, _), (ko, *_) = oracle.qk_norm_rope(q, q.copy(), pos, 1e-6, qs, False, True, 1e4)
    want = oracle.round_bf16(from_bf16(ko) * qs)
    sure = ql == qh
    assert np.array_equal(qo[sure], want[sure])
    _, lo1, _, _ = oracle.rms_norm(q.reshape(-1, 64), None, 0, 1e-6)
    once = oracle.round_bf16(lo1.reshape(q.shape) * qs)
    assert np.mean(once != want) > 0.01  # the two orders are distinguishable


def test_rms_norm_to_output_cast():
    # FP32 input, bf16 output: a constant row normalises to sign * w exactly
    # (eps = 0), so the output is the bf16 rounding of the effective gain.
    H = 64
    rng = np.random.default_rng(12)
    gain = rng.uniform(0.5, 1.5, H).astype(np.float32)
    x = np.vstack([np.full(H, 3.25, np.float32), np.full(H, -0.125, np.float32)])
    out, lo, hi, _ = oracle.rms_norm_to(x, oracle.BF16, gain, 0.0, 0.0)
    assert out.dtype == np.uint16
    assert np.array_equal(out[0], oracle.round_bf16(gain.astype(np.float64)))
    assert np.array_equal(out[1], oracle.round_bf16(-gain.astype(np.float64)))
    assert np.array_equal(lo, hi)
    # same arithmetic as the FP32-output call; only the final cast differs
    o32, lo32, _, _ = oracle.rms_norm_to(x, oracle.F32, gain, 0.0, 0.0)
    assert np.array_equal(lo, lo32) and np.array_equal(o32, lo32.astype(np.float32))


def test_rms_norm_grouped_pins():
    # per-expert gains: a group whose gain is twice another's gives exactly
    # twice the outputs (power-of-two scaling is exact through every rounding);
    # an empty group shifts nothing; a single group is core 1
    rng = np.random.default_rng(13)
    H, rows = 32, 9
    x = oracle.round_bf16(rng.standard_normal((rows, H)))
    g = rng.uniform(0.5, 1.5, H).astype(np.float32)
    gains = np.stack([g, 0.5 * g, 2 * g])     # distinct rows: a shifted group index shows
    offs = np.array([0, 4, 4, 9], np.int32)   # groups of 4, 0 and 5 rows
    out, lo, hi, _ = oracle.rms_norm_grouped(x, gains, offs, 0.0, 1e-6)
    a = oracle.rms_norm(x[:4], g, 0.0, 1e-6)
    b = oracle.rms_norm(x[4:], 2 * g, 0.0, 1e-6)
    assert np.array_equal(out[:4], a[0]) and np.array_equal(out[4:], b[0])
    b1 = oracle.rms_norm(x[4:], g, 0.0, 1e-6)
    np.testing.assert_array_equal(lo[4:], 2 * b1[1])
    one, *_ = oracle.rms_norm_grouped(x, g[None, :], np.array([0, rows], np.int32), 0.0, 1e-6)
    assert np.array_equal(one, oracle.rms_norm(x, g, 0.0, 1e-6)[0])
    with pytest.raises(ValueError):
        oracle.rms_norm_grouped(x, gains, np.array([0, 3, 2, 9], np.int32))


# ------------------------------------------------------- vision 2-D RoPE

def _vision_inputs(seed, T=5, hq=3, hk=2, D=16, dtype="bf16"):
    r = rng(seed)
    q = r.standard_normal((T, hq, D)) * 2.0
    k = r.standard_normal((T, hk, D)) * 2.0
    if dtype == "bf16":
        return bf16(q), bf16(k)
    return q.astype(np.float32), k.astype(np.float32)


def _table(T, D, angles):
    f = np.empty((T, D // 2, 2), np.float32)
    f[..., 0] = np.cos(angles)
    f[..., 1] = np.sin(angles)
    return f


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_vision_rope_identity_and_quarter_turn(dtype):
    # (c, s) = (1, 0) leaves every element unchanged; (0, 1) maps (a, b) to (-b, a)
    q, k = _vision_inputs(30, dtype=dtype)
    T, D = q.shape[0], q.shape[2]
    ident = np.zeros((T, D // 2, 2), np.float32)
    ident[..., 0] = 1.0
    (qo, lo, hi, _), (ko, *_) = oracle.vision_rope(q, k, ident)
    assert np.array_equal(qo, q) and np.array_equal(ko, k) and np.array_equal(lo, hi)
    quarter = np.zeros_like(ident)
    quarter[..., 1] = 1.0
    (qo, *_), _ = oracle.vision_rope(q, k, quarter)
    val = from_bf16 if dtype == "bf16" else (lambda a: a.astype(np.float64))
    assert np.array_equal(val(qo)[..., 0::2], -val(q)[..., 1::2])
    assert np.array_equal(val(qo)[..., 1::2], val(q)[..., 0::2])


def test_vision_rope_is_complex_multiplication():
    # adjacent pairs (2i, 2i+1) as a + ib, the table's (c, s) as c + is:
    # the exact rotated value is their complex product (numpy complex128)
    q, k = _vision_inputs(31, T=7, D=24)
    T, D = q.shape[0], q.shape[2]
    ang = rng(32).uniform(-40.0, 40.0, (T, D // 2))
    f = _table(T, D, ang)
    (qo, lo, hi, mag), (ko, klo, _, _) = oracle.vision_rope(q, k, f)
    for x, l in ((q, lo), (k, klo)):
        xv = from_bf16(x)
        z = (xv[..., 0::2] + 1j * xv[..., 1::2]) * (f[None, :, :, 0].astype(np.float64).transpose(1, 0, 2)
                                                    + 1j * f[None, :, :, 1].astype(np.float64).transpose(1, 0, 2))
        ref = np.stack([z.real, z.imag], -1).reshape(x.shape)
        assert np.allclose(l, ref, rtol=1e-13, atol=1e-300)
    assert np.array_equal(lo, hi)
    assert np.all(mag >= np.abs(lo))


def test_vision_rope_preserves_pair_norms_and_composes():
    # a unit (c, s) keeps |(a, b)|; rotating by alpha then beta equals one
    # rotation by alpha + beta (exact arithmetic on the oracle's pre-cast values)
    q, k = _vision_inputs(33, dtype="f32")
    T, D = q.shape[0], q.shape[2]
    r = rng(34)
    al, be = r.uniform(-3, 3, (T, D // 2)), r.uniform(-3, 3, (T, D // 2))
    (_, lo1, _, _), _ = oracle.vision_rope(q, k, _table(T, D, al))
    n0 = q.astype(np.float64)[..., 0::2] ** 2 + q.astype(np.float64)[..., 1::2] ** 2
    n1 = lo1[..., 0::2] ** 2 + lo1[..., 1::2] ** 2
    assert np.allclose(n1, n0, rtol=1e-6)
    (q1, *_), _ = oracle.vision_rope(q, k, _table(T, D, al))
    (_, lo2, _, _), _ = oracle.vision_rope(q1, k, _table(T, D, be))
    (_, lo3, _, _), _ = oracle.vision_rope(q, k, _table(T, D, al + be))
    assert np.allclose(lo2, lo3, rtol=1e-5, atol=1e-5)


def test_vision_rope_frequencies_reading():
    # patch (0, 0): every angle 0; the first D/4 pairs vary with the row only,
    # the others with the column only; angles grow linearly with the index and
    # fall geometrically over the pairs (ratio theta^(-2/(D/2)))
    D, Hg, Wg, theta = 16, 3, 5, 100.0
    f = oracle.vision_rope_frequencies(D, Hg, Wg, theta).reshape(Hg, Wg, D // 2, 2)
    assert np.array_equal(f[0, 0, :, 0], np.ones(D // 2, np.float32))
    assert np.array_equal(f[0, 0, :, 1], np.zeros(D // 2, np.float32))
    assert np.allclose(f[..., 0] ** 2 + f[..., 1] ** 2, 1.0, atol=1e-6)
    q4 = D // 4
    assert np.all(f[:, :, :q4] == f[:, :1, :q4])   # row half: same along a row
    assert np.all(f[:, :, q4:] == f[:1, :, q4:])   # column half: same down a column
    ang = np.arctan2(f[..., 1].astype(np.float64), f[..., 0].astype(np.float64))
    # row 1 / column 1 give the frequencies themselves (all below pi)
    fr, fc = ang[1, 0, :q4], ang[0, 1, q4:]
    assert np.allclose(fr, fc, rtol=1e-6)
    assert np.allclose(fr[1:] / fr[:-1], theta ** (-2.0 / (D // 2)), rtol=1e-5)
    assert abs(fr[0] - 1.0) < 1e-6
    assert np.allclose(ang[2, 0, :q4], np.angle(np.exp(2j * fr)), rtol=1e-5, atol=1e-6)
