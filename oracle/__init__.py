"""NumPy front end of the double-precision CPU oracle (``muse_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` import this package.  The product
path (``gate_cores_b200``) never imports it and shares no code with it.

Each wrapper takes contiguous NumPy arrays (bf16 as ``uint16`` bit patterns,
f32 as ``float32``) and returns ``(out, lo, hi, mag)``: the core's output in
its dtype plus the three double arrays described in ``muse_oracle.h``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "muse_oracle.c")
_LIB = os.path.join(_HERE, "libmuse_oracle.so")

BF16 = 0
F32 = 1

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, IEEE rounding, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "muse_oracle.h"))
    ):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra",
             "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            i64, i32, f32, c_int = ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_int
            lib.muse_oracle_version.restype = c_int
            lib.muse_oracle_round_bf16.argtypes = [P, P, i64]
            lib.muse_oracle_round_bf16.restype = None
            lib.muse_oracle_inv_freq.argtypes = [i32, f32, P]
            lib.muse_oracle_positions.argtypes = [c_int, i64, i64, P, i32, i64, P]
            lib.muse_oracle_rms_norm.argtypes = [c_int, P, i64, i64, P, f32, f32, P, P, P, P]
            lib.muse_oracle_input_scale_norm.argtypes = lib.muse_oracle_rms_norm.argtypes
            lib.muse_oracle_rms_norm_to.argtypes = [c_int, c_int, P, i64, i64, P, f32, f32, P, P, P, P]
            lib.muse_oracle_rms_norm_to.restype = c_int
            lib.muse_oracle_rms_norm_grouped.argtypes = [c_int, P, i64, i64, P, f32, P, i32, f32,
                                                         P, P, P, P]
            lib.muse_oracle_rms_norm_grouped.restype = c_int
            lib.muse_oracle_qk_norm_rope.argtypes = [
                c_int, P, P, i64, i32, i32, i32, P, f32, f32, c_int, c_int, f32,
                P, P, P, P, P, P, P, P]
            lib.muse_oracle_output_norm_gate.argtypes = [
                c_int, P, P, i64, i32, i32, i32, f32, P, P, P, P]
            lib.muse_oracle_norm_residual.argtypes = [
                P, c_int, P, i64, i64, P, f32, P, c_int, f32, P, P, P, P]
            lib.muse_oracle_rms_norm_bwd.argtypes = [c_int, P, P, i64, i64, P, f32, f32,
                                                     P, P, P, P, P, P, P]
            lib.muse_oracle_input_scale_norm_bwd.argtypes = lib.muse_oracle_rms_norm_bwd.argtypes
            lib.muse_oracle_qk_norm_rope_bwd.argtypes = [
                c_int, P, P, P, P, i64, i32, i32, i32, P, f32, f32, c_int, c_int, f32, c_int,
                P, P, P, P, P, P, P, P]
            lib.muse_oracle_output_norm_gate_bwd.argtypes = [
                c_int, P, P, P, i64, i32, i32, i32, f32, P, P, P, P, P, P, P, P]
            lib.muse_oracle_norm_residual_bwd.argtypes = [
                P, c_int, P, P, i64, i64, P, f32, P, c_int, f32, c_int,
                P, P, P, P, P, P, P, P, P, P, P, P, P, P]
            lib.muse_oracle_residual_blend.argtypes = [P, c_int, P, i64, i64, P, P, P, P, P]
            lib.muse_oracle_residual_gate_coefficients.argtypes = [P, i64, f32, f32, P, P, P]
            lib.muse_oracle_residual.argtypes = [P, c_int, P, i64, i64, P, f32, f32, P, P, P, P]
            lib.muse_oracle_residual_blend_bwd.argtypes = [P, c_int, P, P, i64, i64, P] + [P] * 11
            lib.muse_oracle_residual_bwd.argtypes = [P, c_int, P, P, i64, i64, P, f32, f32] + [P] * 11
            for name in ("muse_oracle_residual_blend", "muse_oracle_residual_gate_coefficients",
                         "muse_oracle_residual", "muse_oracle_residual_blend_bwd",
                         "muse_oracle_residual_bwd"):
                getattr(lib, name).restype = c_int
            lib.muse_oracle_vision_rope_frequencies.argtypes = [i32, i32, i32, f32, P]
            lib.muse_oracle_vision_rope.argtypes = [c_int, P, P, i64, i32, i32, i32, P,
                                                    P, P, P, P, P, P, P, P]
            for name in ("muse_oracle_vision_rope_frequencies", "muse_oracle_vision_rope"):
                getattr(lib, name).restype = c_int
            for name in ("muse_oracle_inv_freq", "muse_oracle_positions", "muse_oracle_rms_norm",
                         "muse_oracle_input_scale_norm", "muse_oracle_qk_norm_rope",
                         "muse_oracle_output_norm_gate", "muse_oracle_norm_residual",
                         "muse_oracle_rms_norm_bwd", "muse_oracle_input_scale_norm_bwd",
                         "muse_oracle_qk_norm_rope_bwd", "muse_oracle_output_norm_gate_bwd",
                         "muse_oracle_norm_residual_bwd"):
                getattr(lib, name).restype = c_int
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dt(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return F32
    raise TypeError(f"oracle takes uint16 (bf16 bits) or float32 arrays, got {a.dtype}")


def _c(a):
    return None if a is None else np.ascontiguousarray(a)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid argument")


def version() -> int:
    return _load().muse_oracle_version()


def round_bf16(v) -> np.ndarray:
    """Nearest bf16 (ties to even) of each double, as uint16 bit patterns."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    _load().muse_oracle_round_bf16(_ptr(v), _ptr(out), v.size)
    return out


def inv_freq(head_dim: int, base: float) -> np.ndarray:
    out = np.empty(head_dim // 2, dtype=np.float32)
    _check(_load().muse_oracle_inv_freq(head_dim, base, _ptr(out)), "inv_freq")
    return out


def positions(layout: int, batch: int = 0, seqlen: int = 0, cu_seqlens=None,
              total_tokens: int = 0) -> np.ndarray:
    """Default positions: BSHD (layout 0) t mod seqlen; THD (layout 1) t - cu_seqlens[d]."""
    if layout == 0:
        n = batch * seqlen
        cu = None
        ns = 0
    else:
        cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
        ns = cu.size - 1
        n = total_tokens
    out = np.empty(n, dtype=np.int32)
    _check(_load().muse_oracle_positions(layout, batch, seqlen, _ptr(cu), ns, total_tokens,
                                         _ptr(out)), "positions")
    return out


def _checks(shape):
    return (np.empty(shape, np.float64), np.empty(shape, np.float64), np.empty(shape, np.float64))


def rms_norm(x, gain=None, gain_offset=0.0, eps=1e-6):
    x = _c(x)
    gain = _c(gain)
    out = np.empty_like(x)
    lo, hi, mag = _checks(x.shape)
    hidden = x.shape[-1]
    rows = x.size // hidden
    _check(_load().muse_oracle_rms_norm(_dt(x), _ptr(x), rows, hidden, _ptr(gain), gain_offset,
                                        eps, _ptr(out), _ptr(lo), _ptr(hi), _ptr(mag)), "rms_norm")
    return out, lo, hi, mag


def rms_norm_to(x, out_dtype, gain=None, gain_offset=0.0, eps=1e-6):
    """Core 1 with the output in out_dtype (BF16 or F32) whatever x's dtype."""
    x = _c(x)
    gain = _c(gain)
    out = np.empty(x.shape, dtype=np.uint16 if out_dtype == BF16 else np.float32)
    lo, hi, mag = _checks(x.shape)
    hidden = x.shape[-1]
    rows = x.size // hidden
    _check(_load().muse_oracle_rms_norm_to(_dt(x), out_dtype, _ptr(x), rows, hidden, _ptr(gain),
                                           gain_offset, eps, _ptr(out), _ptr(lo), _ptr(hi),
                                           _ptr(mag)), "rms_norm_to")
    return out, lo, hi, mag


def rms_norm_grouped(x, gains, offsets, gain_offset=0.0, eps=1e-6):
    """Per-expert core 1: rows offsets[g]..offsets[g+1]-1 use gains[g]."""
    x = _c(x)
    gains = np.ascontiguousarray(gains, dtype=np.float32)
    offsets = np.ascontiguousarray(offsets, dtype=np.int32)
    out = np.empty_like(x)
    lo, hi, mag = _checks(x.shape)
    hidden = x.shape[-1]
    rows = x.size // hidden
    _check(_load().muse_oracle_rms_norm_grouped(_dt(x), _ptr(x), rows, hidden, _ptr(gains),
                                                gain_offset, _ptr(offsets), offsets.size - 1, eps,
                                                _ptr(out), _ptr(lo), _ptr(hi), _ptr(mag)),
           "rms_norm_grouped")
    return out, lo, hi, mag


def input_scale_norm(x, gain=None, gain_offset=0.0, eps=1e-6):
    x = _c(x)
    gain = _c(gain)
    out = np.empty_like(x)
    lo, hi, mag = _checks(x.shape)
    hidden = x.shape[-1]
    rows = x.size // hidden
    _check(_load().muse_oracle_input_scale_norm(_dt(x), _ptr(x), rows, hidden, _ptr(gain),
                                                gain_offset, eps, _ptr(out), _ptr(lo), _ptr(hi),
                                                _ptr(mag)), "input_scale_norm")
    return out, lo, hi, mag


def qk_norm_rope(q, k, pos, eps=1e-6, query_scale=1.0, use_rope=True, upcast_rope=True,
                 rope_base=10000.0):
    """q [T, Hq, D], k [T, Hkv, D], pos int32 [T].  Returns (q_res, k_res), each (out, lo, hi, mag)."""
    q = _c(q)
    k = _c(k)
    pos = None if pos is None else np.ascontiguousarray(pos, dtype=np.int32)
    T, hq, d = q.shape
    hkv = k.shape[1]
    assert k.shape == (T, hkv, d) and k.dtype == q.dtype
    qo = np.empty_like(q)
    ko = np.empty_like(k)
    ql, qh, qm = _checks(q.shape)
    kl, kh, km = _checks(k.shape)
    _check(_load().muse_oracle_qk_norm_rope(
        _dt(q), _ptr(q), _ptr(k), T, hq, hkv, d, _ptr(pos), eps, query_scale, int(use_rope),
        int(upcast_rope), rope_base, _ptr(qo), _ptr(ql), _ptr(qh), _ptr(qm), _ptr(ko), _ptr(kl),
        _ptr(kh), _ptr(km)), "qk_norm_rope")
    return (qo, ql, qh, qm), (ko, kl, kh, km)


def output_norm_gate(o, g, norm_group=None, eps=1e-6):
    """o, g [T, H, D]; norm_group = D (per head, default) or H*D (whole token)."""
    o = _c(o)
    g = _c(g)
    T, heads, d = o.shape
    assert g.shape == o.shape and g.dtype == o.dtype
    ng = d if norm_group is None else norm_group
    out = np.empty_like(o)
    lo, hi, mag = _checks(o.shape)
    _check(_load().muse_oracle_output_norm_gate(_dt(o), _ptr(o), _ptr(g), T, heads, d, ng, eps,
                                                _ptr(out), _ptr(lo), _ptr(hi), _ptr(mag)),
           "output_norm_gate")
    return out, lo, hi, mag


def norm_residual(stream, branch, theta, gain=None, gain_offset=0.0, input_scale=False,
                  norm_eps=1e-6):
    stream = np.ascontiguousarray(stream, dtype=np.float32)
    branch = _c(branch)
    theta = np.ascontiguousarray(theta, dtype=np.float32)
    gain = _c(gain)
    assert stream.shape == branch.shape
    hidden = stream.shape[-1]
    rows = stream.size // hidden
    out = np.empty_like(stream)
    lo, hi, mag = _checks(stream.shape)
    _check(_load().muse_oracle_norm_residual(
        _ptr(stream), _dt(branch), _ptr(branch), rows, hidden, _ptr(gain), gain_offset,
        _ptr(theta), int(input_scale), norm_eps, _ptr(out), _ptr(lo), _ptr(hi), _ptr(mag)),
        "norm_residual")
    return out, lo, hi, mag


def residual_blend(stream, branch, theta):
    """_residual_core without a branch norm, core 5's declared blend:
    cos(theta) h + sin(theta) branch per channel."""
    stream = np.ascontiguousarray(stream, dtype=np.float32)
    branch = _c(branch)
    theta = np.ascontiguousarray(theta, dtype=np.float32)
    assert stream.shape == branch.shape
    hidden = stream.shape[-1]
    rows = stream.size // hidden
    out = np.empty_like(stream)
    lo, hi, mag = _checks(stream.shape)
    _check(_load().muse_oracle_residual_blend(_ptr(stream), _dt(branch), _ptr(branch), rows, hidden,
                                              _ptr(theta), _ptr(out), _ptr(lo), _ptr(hi), _ptr(mag)),
           "residual_blend")
    return out, lo, hi, mag


def residual_gate_coefficients(gate, temperature=0.3, eps=1e-3):
    """Declared reading of the learned gate: (c, s, theta) in double, with
    c^2 = max(sigmoid(gate/temperature), eps), s^2 = 1 - c^2, theta = atan2(s, c)."""
    gate = np.ascontiguousarray(gate, dtype=np.float32)
    c, s, th = (np.empty(gate.shape, np.float64) for _ in range(3))
    _check(_load().muse_oracle_residual_gate_coefficients(_ptr(gate), gate.size, temperature, eps,
                                                          _ptr(c), _ptr(s), _ptr(th)),
           "residual_gate_coefficients")
    return c, s, th


def residual(stream, branch, gate, temperature=0.3, eps=1e-3):
    """_residual_core(stream, branch, gate, temperature, eps): c h + s branch."""
    stream = np.ascontiguousarray(stream, dtype=np.float32)
    branch = _c(branch)
    gate = np.ascontiguousarray(gate, dtype=np.float32)
    assert stream.shape == branch.shape
    hidden = stream.shape[-1]
    rows = stream.size // hidden
    out = np.empty_like(stream)
    lo, hi, mag = _checks(stream.shape)
    _check(_load().muse_oracle_residual(_ptr(stream), _dt(branch), _ptr(branch), rows, hidden,
                                        _ptr(gate), temperature, eps, _ptr(out), _ptr(lo), _ptr(hi),
                                        _ptr(mag)), "residual")
    return out, lo, hi, mag


def _residual_bwd_call(fn, what, stream, branch, dy, *params):
    stream = np.ascontiguousarray(stream, dtype=np.float32)
    dy = np.ascontiguousarray(dy, dtype=np.float32)
    branch = _c(branch)
    assert stream.shape == branch.shape == dy.shape
    hidden = stream.shape[-1]
    rows = stream.size // hidden
    ds = np.empty_like(stream)
    db = np.empty_like(branch)
    sl, sh, sm = _checks(stream.shape)
    bl, bh, bm = _checks(stream.shape)
    pl, ph, pm = _checks((hidden,))
    _check(fn(_ptr(stream), _dt(branch), _ptr(branch), _ptr(dy), rows, hidden, *params, _ptr(ds), _ptr(sl),
              _ptr(sh), _ptr(sm), _ptr(db), _ptr(bl), _ptr(bh), _ptr(bm), _ptr(pl), _ptr(ph), _ptr(pm)), what)
    return (ds, sl, sh, sm), (db, bl, bh, bm), (pl, ph, pm)


def residual_blend_bwd(stream, branch, dy, theta):
    """Backward of the angle form: (dstream, dbranch, dtheta)."""
    theta = np.ascontiguousarray(theta, dtype=np.float32)
    return _residual_bwd_call(_load().muse_oracle_residual_blend_bwd, "residual_blend_bwd", stream, branch,
                              dy, _ptr(theta))


def residual_bwd(stream, branch, dy, gate, temperature=0.3, eps=1e-3):
    """Backward of the gate form: (dstream, dbranch, dgate)."""
    gate = np.ascontiguousarray(gate, dtype=np.float32)
    return _residual_bwd_call(_load().muse_oracle_residual_bwd, "residual_bwd", stream, branch, dy,
                              _ptr(gate), temperature, eps)


# ------------------------------------------------------------------ backward
# Each returns the input gradients as (out, lo, hi, mag) tuples and the
# parameter gradients as (lo, hi, mag) double triples (None without a gain).


def _rows_bwd(fn, what, x, dy, gain, gain_offset, eps):
    x = _c(x)
    dy = _c(dy)
    gain = _c(gain)
    assert dy.shape == x.shape and dy.dtype == x.dtype
    hidden = x.shape[-1]
    rows = x.size // hidden
    dx = np.empty_like(x)
    lo, hi, mag = _checks(x.shape)
    glo, ghi, gmag = _checks((hidden,)) if gain is not None else (None, None, None)
    _check(fn(_dt(x), _ptr(x), _ptr(dy), rows, hidden, _ptr(gain), gain_offset, eps, _ptr(dx),
              _ptr(lo), _ptr(hi), _ptr(mag), _ptr(glo), _ptr(ghi), _ptr(gmag)), what)
    return (dx, lo, hi, mag), (None if gain is None else (glo, ghi, gmag))


def rms_norm_bwd(x, dy, gain=None, gain_offset=0.0, eps=1e-6):
    """Core 1 backward: (dx, dgain)."""
    return _rows_bwd(_load().muse_oracle_rms_norm_bwd, "rms_norm_bwd", x, dy, gain, gain_offset,
                     eps)


def input_scale_norm_bwd(x, dy, gain=None, gain_offset=0.0, eps=1e-6):
    """Core 2 backward: (dx, dgain)."""
    return _rows_bwd(_load().muse_oracle_input_scale_norm_bwd, "input_scale_norm_bwd", x, dy,
                     gain, gain_offset, eps)


def qk_norm_rope_bwd(q, k, dq_out, dk_out, pos, eps=1e-6, query_scale=1.0, use_rope=True,
                     rope_base=10000.0, round_grads=True, upcast_rope=True):
    """Core 3 backward, FP32 (legacy) or, upcast_rope=False on bf16, v2 rotation: (dq, dk)."""
    q, k, dq_out, dk_out = _c(q), _c(k), _c(dq_out), _c(dk_out)
    pos = None if pos is None else np.ascontiguousarray(pos, dtype=np.int32)
    T, hq, d = q.shape
    hkv = k.shape[1]
    assert dq_out.shape == q.shape and dk_out.shape == k.shape
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    ql, qh, qm = _checks(q.shape)
    kl, kh, km = _checks(k.shape)
    _check(_load().muse_oracle_qk_norm_rope_bwd(
        _dt(q), _ptr(q), _ptr(k), _ptr(dq_out), _ptr(dk_out), T, hq, hkv, d, _ptr(pos), eps,
        query_scale, int(use_rope), int(upcast_rope), rope_base, int(round_grads), _ptr(dq), _ptr(ql), _ptr(qh),
        _ptr(qm), _ptr(dk), _ptr(kl), _ptr(kh), _ptr(km)), "qk_norm_rope_bwd")
    return (dq, ql, qh, qm), (dk, kl, kh, km)


def output_norm_gate_bwd(o, g, dy, norm_group=None, eps=1e-6):
    """Core 4 backward: (do, dg)."""
    o, g, dy = _c(o), _c(g), _c(dy)
    T, heads, d = o.shape
    ng = d if norm_group is None else norm_group
    d_o = np.empty_like(o)
    dg = np.empty_like(o)
    ol, oh, om = _checks(o.shape)
    gl, gh, gm = _checks(o.shape)
    _check(_load().muse_oracle_output_norm_gate_bwd(
        _dt(o), _ptr(o), _ptr(g), _ptr(dy), T, heads, d, ng, eps, _ptr(d_o), _ptr(ol), _ptr(oh),
        _ptr(om), _ptr(dg), _ptr(gl), _ptr(gh), _ptr(gm)), "output_norm_gate_bwd")
    return (d_o, ol, oh, om), (dg, gl, gh, gm)


def norm_residual_bwd(stream, branch, dstream_out, theta, gain=None, gain_offset=0.0,
                      input_scale=False, norm_eps=1e-6, round_grads=True):
    """Core 5 backward: (dstream, dbranch, dgain, dtheta)."""
    stream = np.ascontiguousarray(stream, dtype=np.float32)
    dstream_out = np.ascontiguousarray(dstream_out, dtype=np.float32)
    branch = _c(branch)
    theta = np.ascontiguousarray(theta, dtype=np.float32)
    gain = _c(gain)
    hidden = stream.shape[-1]
    rows = stream.size // hidden
    ds = np.empty_like(stream)
    db = np.empty_like(branch)
    sl, sh, sm = _checks(stream.shape)
    bl, bh, bm = _checks(stream.shape)
    glo, ghi, gmag = _checks((hidden,)) if gain is not None else (None, None, None)
    tlo, thi, tmag = _checks((hidden,))
    _check(_load().muse_oracle_norm_residual_bwd(
        _ptr(stream), _dt(branch), _ptr(branch), _ptr(dstream_out), rows, hidden, _ptr(gain),
        gain_offset, _ptr(theta), int(input_scale), norm_eps, int(round_grads), _ptr(ds),
        _ptr(sl), _ptr(sh), _ptr(sm), _ptr(db), _ptr(bl), _ptr(bh), _ptr(bm), _ptr(glo),
        _ptr(ghi), _ptr(gmag), _ptr(tlo), _ptr(thi), _ptr(tmag)), "norm_residual_bwd")
    return ((ds, sl, sh, sm), (db, bl, bh, bm), None if gain is None else (glo, ghi, gmag),
            (tlo, thi, tmag))


def vision_rope_frequencies(head_dim, grid_h, grid_w, theta=10000.0) -> np.ndarray:
    """Vision 2-D RoPE table of one row-major grid: float32 [grid_h*grid_w, head_dim/2, 2]."""
    out = np.empty((grid_h * grid_w, head_dim // 2, 2), np.float32)
    _check(_load().muse_oracle_vision_rope_frequencies(head_dim, grid_h, grid_w, theta, _ptr(out)),
           "vision_rope_frequencies")
    return out


def vision_rope(q, k, freqs):
    """Vision 2-D RoPE of q [T, hq, D], k [T, hk, D] with freqs [T, D/2, 2]: (q', k')."""
    q, k = _c(q), _c(k)
    freqs = np.ascontiguousarray(freqs, dtype=np.float32)
    T, hq, d = q.shape
    hk = k.shape[1]
    assert k.shape[0] == T and k.shape[2] == d and freqs.shape == (T, d // 2, 2)
    qo, ko = np.empty_like(q), np.empty_like(k)
    ql, qh, qm = _checks(q.shape)
    kl, kh, km = _checks(k.shape)
    _check(_load().muse_oracle_vision_rope(_dt(q), _ptr(q), _ptr(k), T, hq, hk, d, _ptr(freqs),
                                           _ptr(qo), _ptr(ql), _ptr(qh), _ptr(qm), _ptr(ko),
                                           _ptr(kl), _ptr(kh), _ptr(km)), "vision_rope")
    return (qo, ql, qh, qm), (ko, kl, kh, km)
