"""Host-side checks of the C ABI library, no GPU needed: the library loads,
exports every entry point include/muse_cores.h declares, and rejects invalid
arguments before anything is launched.  The pointers below are never
dereferenced: each call fails validation on the host first."""
import ctypes
import os
import re

import pytest

from gate_cores_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muse_cores.h")
INV, UNS = _lib.MUSE_ERR_INVALID_ARGUMENT, _lib.MUSE_ERR_UNSUPPORTED
BF16, F32 = _lib.MUSE_DTYPE_BF16, _lib.MUSE_DTYPE_F32
A = 0x7F0000000000  # a 256-byte aligned fake device address (never touched)


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(muse_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(_lib.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_version_and_status_strings(lib):
    assert _lib.muse_version() == 1
    assert _lib.muse_status_string(0) == "MUSE_OK"
    assert _lib.muse_status_string(2) == "MUSE_ERR_UNSUPPORTED"


def rms(lib, x=A, y=A + (1 << 24), dt=BF16, rows=4, hidden=256, xs=None, ys=None, gain=None,
        off=0.0, eps=1e-6):
    xs = hidden if xs is None else xs
    ys = hidden if ys is None else ys
    return lib.muse_rms_norm(x, y, dt, rows, hidden, xs, ys, gain, off, eps, None)


def test_row_validation(lib):
    assert rms(lib, rows=0) == 0  # empty: OK without a launch
    assert rms(lib, dt=7) == INV
    assert rms(lib, rows=-1) == INV
    assert rms(lib, hidden=0) == INV
    assert rms(lib, x=None) == INV
    assert rms(lib, xs=100) == INV                      # stride < hidden
    assert rms(lib, eps=float("nan")) == INV
    assert rms(lib, eps=-1.0) == INV
    assert rms(lib, x=A + 8) == UNS                     # misaligned pointer
    assert rms(lib, hidden=260) == UNS                  # not a 16-byte row
    assert rms(lib, hidden=256, xs=260) == UNS          # stride not 16-byte
    assert rms(lib, hidden=65536) == UNS                # wider than one CTA row
    assert rms(lib, gain=A + 2) == UNS
    assert rms(lib, gain=A + 8) == UNS                  # gains load as 16-byte vectors
    assert b"muse_rms_norm" in lib.muse_last_error()


def test_row_partial_overlap_rejected(lib):
    # y starts half a row into x: overlapping but not the same tensor
    assert rms(lib, x=A, y=A + 256) == INV
    # y overlaps the gain vector
    assert rms(lib, x=A, y=A + (1 << 20), gain=A + (1 << 20) + 64) == INV
    # input-scale variant shares the checks
    assert lib.muse_input_scale_norm(A, A + 256, BF16, 4, 256, 256, 256, None, 0.0, 1e-6, None) == INV


def qk(lib, q=A, k=A + (1 << 26), qo=A + (2 << 26), ko=A + (3 << 26), dt=BF16, layout=0, batch=2,
       seqlen=8, cu=None, ns=0, total=0, pos=None, hq=4, hkv=2, d=64, qs=None, ks=None, qos=None,
       kos=None, eps=1e-6, scale=1.0, rope=1, upcast=1, base=1e4):
    qs = hq * d if qs is None else qs
    ks = hkv * d if ks is None else ks
    qos = hq * d if qos is None else qos
    kos = hkv * d if kos is None else kos
    return lib.muse_qk_norm_rope(q, k, qo, ko, dt, layout, batch, seqlen, cu, ns, total, pos, hq,
                                 hkv, d, qs, ks, qos, kos, eps, scale, rope, upcast, base, None)


def test_qk_validation(lib):
    assert qk(lib, batch=0) == 0
    assert qk(lib, layout=5) == INV
    assert qk(lib, hq=6, hkv=4) == INV                  # GQA needs hq % hkv == 0
    assert qk(lib, d=63) == INV                         # odd head_dim
    assert qk(lib, base=0.0) == INV
    assert qk(lib, base=float("inf")) == INV
    assert qk(lib, qs=100) == INV                       # stride below the heads' width
    assert qk(lib, layout=1, total=16, cu=None) == INV  # THD with derived positions needs cu_seqlens
    assert qk(lib, layout=1, total=16, cu=A + (5 << 26), ns=0) == INV
    assert qk(lib, layout=1, total=-1) == INV
    assert qk(lib, d=36) == UNS                         # 72-byte heads: not 16-byte multiples
    assert qk(lib, d=512) == UNS                        # above 512 bytes per head
    assert qk(lib, dt=F32, d=256) == UNS
    assert qk(lib, q=A + 4) == UNS
    assert qk(lib, pos=A + (5 << 26) + 2) == UNS


def test_qk_aliasing_rules(lib):
    # q_out half a head into q: partial overlap
    assert qk(lib, qo=A + 64) == INV
    # k_out overlapping q
    assert qk(lib, ko=A + 128) == INV
    # outputs overlapping the positions array
    assert qk(lib, pos=A + (2 << 26) + 64) == INV
    # fused QKV with q_out and k_out landing on each other's columns
    W = (4 + 2 * 2) * 64
    assert qk(lib, q=A, k=A + 4 * 64 * 2, qo=A + 4 * 64 * 2, ko=A, qs=W, ks=W, qos=W, kos=W) == INV


def test_gate_and_residual_validation(lib):
    g = lib.muse_output_norm_gate
    assert g(A, A + (1 << 24), A + (2 << 24), BF16, 4, 4, 64, 32, 1e-6, None) == INV  # norm_group
    assert g(A, A + (1 << 24), A + (2 << 24), BF16, 0, 4, 64, 64, 1e-6, None) == 0
    assert g(A, A + (1 << 24), A + 64, BF16, 4, 4, 64, 64, 1e-6, None) == INV
    assert g(A, A + (1 << 24), A + (2 << 24), BF16, 4, 4, 60, 60, 1e-6, None) == UNS
    r = lib.muse_norm_residual
    assert r(A, A + (1 << 24), A + (2 << 24), BF16, 0, 256, None, 0.0, A + (3 << 24), 0, 1e-6, None) == 0
    assert r(A, A + (1 << 24), A + (2 << 24), BF16, 4, 256, None, 0.0, None, 0, 1e-6, None) == INV
    assert r(A, A + (1 << 24), A + 512, BF16, 4, 256, None, 0.0, A + (3 << 24), 0, 1e-6, None) == INV
    # stream_out overlapping the branch
    assert r(A, A + (1 << 24), A + (1 << 24) + 1024, BF16, 4, 256, None, 0.0, A + (3 << 24), 0,
             1e-6, None) == INV
    assert r(A, A + (1 << 24), A + (2 << 24), BF16, 4, 252, None, 0.0, A + (3 << 24), 0, 1e-6,
             None) == UNS
    assert lib.muse_device_error(None, 0) == INV
    c = lib.muse_stream_copy
    assert c(A, A + 4096, 0, None) == 0
    assert c(A, A + 4096, 8192, None) == INV            # overlapping ranges
    assert c(A, A + (1 << 20), 100, None) == UNS


def test_grouped_and_fused_validation(lib):
    gr = lib.muse_rms_norm_grouped
    G, O = A + (1 << 26), A + (2 << 26)  # gains, offsets
    assert gr(A, A + (1 << 24), BF16, 0, 256, 256, 256, G, 0.0, O, 4, 1e-6, None) == 0
    assert gr(A, A + (1 << 24), BF16, 8, 256, 256, 256, G, 0.0, O, 0, 1e-6, None) == INV  # no groups
    assert gr(A, A + (1 << 24), BF16, 8, 256, 256, 256, G, 0.0, None, 4, 1e-6, None) == INV
    assert gr(A, A + (1 << 24), BF16, 8, 256, 256, 256, G, 0.0, O + 2, 4, 1e-6, None) == UNS
    assert gr(A, A + (1 << 26), BF16, 8, 16384, 16384, 16384, G + (1 << 20), 0.0, O, 4, 1e-6,
              None) == UNS                                   # above 1024 vectors per row
    assert gr(A, G + 64, BF16, 8, 256, 256, 256, G, 0.0, O, 4, 1e-6, None) == INV  # y over the gains
    fz = lib.muse_norm_residual_rms_norm
    T = A + (3 << 26)
    assert fz(A, A + (1 << 24), A + (2 << 24), A + (4 << 24), F32, BF16, 4, 256, None, 0.0, T, 0,
              1e-6, None, 0.0, 1e-6, None) == UNS            # FP32 branch, bf16 y
    assert fz(A, A + (1 << 24), A + (2 << 24), A + (4 << 24), BF16, F32, 0, 256, None, 0.0, T, 0,
              1e-6, None, 0.0, 1e-6, None) == 0
    assert fz(A, A + (1 << 24), A + (2 << 24), A + (2 << 24) + 512, BF16, F32, 4, 256, None, 0.0, T,
              0, 1e-6, None, 0.0, 1e-6, None) == INV         # y inside stream_out


def test_backward_validation(lib):
    ws = lib.muse_norm_backward_workspace_bytes(64, 256)
    assert ws >= 256 * 4
    rb = lib.muse_rms_norm_backward
    assert rb(A, A + (1 << 24), A + (2 << 24), BF16, 0, 256, 256, 256, 256, None, 0.0, 1e-6, None,
              None, 0, None) == 0
    assert rb(A, A + (1 << 24), A + (2 << 24), BF16, 64, 256, 256, 256, 256, A + (3 << 24), 0.0,
              1e-6, A + (4 << 24), A + (5 << 24), 16, None) == INV  # workspace too small
    qb = lib.muse_qk_norm_rope_backward
    args = [A, A + (1 << 26), A + (2 << 26), A + (3 << 26), A + (4 << 26), A + (5 << 26), BF16, 0, 2,
            8, None, 0, 0, None, 4, 2, 64, 256, 128, 256, 128, 256, 128, 1e-6, 1.0, 1, 0, 1e4, None]
    # (args itself is valid and would launch: only its invalid variants are called)
    bad = list(args)
    bad[7] = 5                                               # unknown layout
    assert qb(*bad) == INV
    bad = list(args)
    bad[16] = 63                                             # odd head_dim
    assert qb(*bad) == INV
    bad = list(args)
    bad[4] = A + 64                                          # dq half a head into q
    assert qb(*bad) == INV


def test_vision_validation(lib):
    v = lib.muse_vision_rope
    F = A + (4 << 26)

    def call(q=A, k=A + (1 << 26), qo=A + (2 << 26), ko=A + (3 << 26), dt=BF16, T=16, hq=4, hk=4,
             d=64, qs=None, ks=None, qos=None, kos=None, f=F):
        qs = hq * d if qs is None else qs
        ks = hk * d if ks is None else ks
        qos = hq * d if qos is None else qos
        kos = hk * d if kos is None else kos
        return v(q, k, qo, ko, dt, T, hq, hk, d, qs, ks, qos, kos, f, None)

    assert call(T=0) == 0
    assert call(hq=0) == INV
    assert call(d=63) == INV
    assert call(qs=100) == INV                               # stride below the heads
    assert call(f=None) == INV
    assert call(d=12) == UNS                                 # 24-byte bf16 heads
    assert call(d=264) == UNS                                # 528-byte heads: above 32 vectors
    assert call(d=136, dt=F32) == UNS
    assert call(f=F + 8) == UNS                              # table not 16-byte aligned
    assert call(qo=A + 64) == INV                            # q_out partially over q
    assert call(ko=F + 256) == INV                           # k_out over the table
    assert call(dt=7) == INV
    fr = lib.muse_vision_rope_frequencies
    assert fr(A, 64, 0, 32, 1e4, None) == 0
    assert fr(A, 66, 4, 4, 1e4, None) == INV                 # head_dim not a multiple of 4
    assert fr(A, 64, 4, 4, 0.0, None) == INV
    assert fr(A, 1024, 4, 4, 1e4, None) == UNS
    assert fr(A + 4, 64, 4, 4, 1e4, None) == UNS
    assert fr(None, 64, 4, 4, 1e4, None) == INV


def test_residual_validation(lib):
    S, B, O, P = A, A + (1 << 24), A + (2 << 24), A + (3 << 24)
    blend = lambda **k: lib.muse_residual_blend(k.get("s", S), k.get("b", B), k.get("o", O), k.get("dt", BF16),  # noqa: E731
                                                 k.get("rows", 4), k.get("hidden", 256), k.get("p", P), None)
    gate = lambda **k: lib.muse_residual(k.get("s", S), k.get("b", B), k.get("o", O), k.get("dt", BF16),  # noqa: E731
                                         k.get("rows", 4), k.get("hidden", 256), k.get("p", P),
                                         k.get("t", 0.3), k.get("eps", 1e-3), None)
    for fn in (blend, gate):
        assert fn(rows=0) == 0
        assert fn(dt=5) == INV
        assert fn(rows=-1) == INV and fn(hidden=0) == INV
        assert fn(p=None) == INV and fn(b=None) == INV
        assert fn(s=S + 4) == UNS and fn(p=P + 4) == UNS
        assert fn(hidden=260) == UNS                       # not a 16-byte branch row
        assert fn(o=S + 16) == INV                         # partial overlap with the stream
        assert fn(o=B) == INV                              # output over the branch
    assert gate(t=0.0) == INV and gate(t=float("inf")) == INV and gate(t=-1.0) == INV
    assert gate(eps=-0.1) == INV and gate(eps=1.5) == INV and gate(eps=float("nan")) == INV
    ang = lambda **k: lib.muse_residual_gate_angles(k.get("g", P), k.get("th", O), k.get("hidden", 256),  # noqa: E731
                                                    k.get("t", 0.3), k.get("eps", 1e-3), None)
    assert ang(hidden=0) == INV and ang(g=None) == INV and ang(th=None) == INV
    assert ang(t=0.0) == INV and ang(eps=2.0) == INV
    assert ang(th=P + 8) == INV                            # partial overlap with the gate
    assert ang(g=P + 2) == UNS
    assert b"muse_residual_gate_angles" in lib.muse_last_error()
