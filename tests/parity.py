"""Acceptance rules for comparing the CUDA cores with the oracle.

The oracle returns, per output element, the interval [lo, hi] of exact
pre-cast values (lo < hi only where an intermediate bf16 cast sits within
2^-20 of a rounding midpoint) and mag, the sum of the magnitudes of the terms.

  bf16 outputs: the GPU value must lie within one bf16 ulp (ordered-integer
    distance 1) of the rounding of some value in
    [lo - s, hi + s],  s = BF16_EVAL_ULPS * 2^-24 * mag.
    s is the allowance for evaluating the last FP32 expression (a rotation
    a*c - b*s, with cos/sin from FP32 sincosf) before the cast; for a plain
    product it is far below half an ulp and the rule is "within 1 ulp".
  FP32 outputs: |gpu - [lo, hi]| <= F32_REL * mag + F32_ABS   (2e-6 relative
    to the magnitudes of the terms, so a cancelling sum is not held to a
    relative bound it cannot meet; plus 16 FP32 subnormal spacings, 16 * 2^-149,
    because a result, or a factor of it such as a saturated sigmoid, below
    2^-126 carries an absolute rounding error of that order that no relative
    bound covers).
"""
from __future__ import annotations

import numpy as np

import oracle

BF16_EVAL_ULPS = 4.0
F32_REL = 2e-6
F32_ABS = 16 * 2.0 ** -149

# Backward (gradients).  The last expression of an input gradient,
# r w g - r^3 x C / H, carries the FP32 error of the row dot product C:
# at most 16 sequential products per thread, a 5-level warp butterfly and a
# 5-level butterfly over the warps' partials, i.e. about 26 units of 2^-24
# relative to the sum of the magnitudes of C's terms, which mag includes;
# BWD_EVAL_ULPS = 64 covers it with margin.  A parameter gradient (gain,
# theta) is an FP32 sum over all rows: each CTA sums its rows in order (a few
# dozen), a second kernel sums the CTAs' partials in 8 interleaved runs and
# adds the 8 results; PARAM_REL = 256 * 2^-24 of the sum of the magnitudes of
# the terms bounds those roundings with margin.
BWD_EVAL_ULPS = 64.0
BWD_F32_REL = 64 * 2.0 ** -24
PARAM_REL = 256 * 2.0 ** -24


def ordered_bf16(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_ok(gpu_bits, lo, hi, mag, eval_ulps=BF16_EVAL_ULPS):
    s = eval_ulps * 2.0 ** -24 * mag
    lo_b = ordered_bf16(oracle.round_bf16(lo - s)) - 1
    hi_b = ordered_bf16(oracle.round_bf16(hi + s)) + 1
    g = ordered_bf16(gpu_bits)
    return (g >= lo_b) & (g <= hi_b)


def f32_ok(gpu, lo, hi, mag, rel=F32_REL):
    g = gpu.astype(np.float64)
    tol = rel * mag + F32_ABS
    return (g >= lo - tol) & (g <= hi + tol)


def check(gpu: np.ndarray, ref, what: str = "", backward: bool = False) -> dict:
    """gpu: uint16 bf16 bits or float32 values; ref: oracle tuple (out, lo, hi, mag).
    backward selects the gradient allowances.  Raises AssertionError with the
    first failures; returns summary stats."""
    out, lo, hi, mag = ref
    assert gpu.shape == out.shape, (gpu.shape, out.shape)
    if gpu.dtype == np.uint16:
        ok = bf16_ok(gpu, lo, hi, mag, BWD_EVAL_ULPS if backward else BF16_EVAL_ULPS)
        dist = np.abs(ordered_bf16(gpu) - ordered_bf16(out))
        stats = {"max_ulp_vs_oracle_out": int(dist.max()) if dist.size else 0,
                 "exact_frac": float(np.mean(dist == 0)) if dist.size else 1.0}
    else:
        ok = f32_ok(gpu, lo, hi, mag, BWD_F32_REL if backward else F32_REL)
        with np.errstate(divide="ignore", invalid="ignore"):
            rel = np.abs(gpu.astype(np.float64) - out.astype(np.float64)) / np.maximum(mag, 1e-300)
        stats = {"max_rel_vs_mag": float(np.nanmax(rel)) if rel.size else 0.0}
    stats["ambiguous"] = int(np.count_nonzero(lo != hi))
    stats["n"] = int(gpu.size)
    bad = np.flatnonzero(~ok.ravel())
    if bad.size:
        i = bad[:8]
        gv = bf16_to_f64(gpu.ravel()[i]) if gpu.dtype == np.uint16 else gpu.ravel()[i]
        raise AssertionError(
            f"{what}: {bad.size}/{gpu.size} elements outside tolerance; first idx {i.tolist()} "
            f"gpu={np.asarray(gv).tolist()} lo={lo.ravel()[i].tolist()} hi={hi.ravel()[i].tolist()} "
            f"mag={mag.ravel()[i].tolist()}")
    return stats


def check_param(gpu: np.ndarray, ref, what: str = "") -> dict:
    """FP32 parameter gradient (a row sum) against the oracle's (lo, hi, mag)."""
    lo, hi, mag = ref
    g = gpu.astype(np.float64)
    tol = PARAM_REL * mag + F32_ABS
    ok = (g >= lo - tol) & (g <= hi + tol)
    bad = np.flatnonzero(~ok)
    with np.errstate(divide="ignore", invalid="ignore"):
        rel = np.abs(g - 0.5 * (lo + hi)) / np.maximum(mag, 1e-300)
    if bad.size:
        i = bad[:8]
        raise AssertionError(f"{what}: {bad.size}/{g.size} outside; idx {i.tolist()} gpu={g[i].tolist()} "
                             f"lo={lo[i].tolist()} hi={hi[i].tolist()} mag={mag[i].tolist()}")
    return {"max_rel_vs_mag": float(np.nanmax(rel)) if rel.size else 0.0,
            "median_rel_vs_mag": float(np.nanmedian(rel)) if rel.size else 0.0}
