"""Memory layouts the C ABI accepts beyond dense tensors: strided rows, Q/K
views into a fused QKV projection buffer, and exact in-place operation.

Each case runs the same values once through dense, separate buffers and once
through the layout under test; the results must be bit-identical (the
kernels' arithmetic does not depend on where the data lives), and bytes of
the surrounding buffers that are not outputs must be left untouched.  The
dense runs themselves are checked against the oracle by test_gpu_parity.
"""
import pytest
import torch

from gate_cores_b200 import cores
from gate_cores_b200._lib import MuseError

pytestmark = pytest.mark.gpu

SHAPES = [  # (tokens, hidden, hq, hkv, head_dim)
    (4096, 4096, 32, 8, 128),
    (37, 264, 6, 2, 80),
]


def _g(seed):
    return torch.Generator(device="cuda").manual_seed(seed)


def _bits(t):
    return t.view(torch.int32) if t.dtype == torch.float32 else t.view(torch.int16)


def _same(a, b):
    return torch.equal(_bits(a.contiguous()), _bits(b.contiguous()))


SENTINEL = -12288.0  # exact in bf16


@pytest.mark.parametrize("T,H,hq,hkv,D", SHAPES)
def test_strided_rows_rms_and_input_scale(cuda_ok, T, H, hq, hkv, D):
    g = _g(1)
    pad = 72  # extra elements per row (144 bytes: keeps 16-byte row strides)
    src = torch.randn(T, H + pad, device="cuda", generator=g).to(torch.bfloat16)
    x = src[:, 8:8 + H]  # rows start 16 bytes in; row stride H + pad
    gain = (1 + 0.1 * torch.randn(H, device="cuda", generator=g)).float()
    for fn in (cores.rms_norm, cores.input_scale_norm):
        dense = fn(x.contiguous(), gain, 0.0, 1e-6)
        dst = torch.full((T, H + 2 * pad), SENTINEL, device="cuda").to(torch.bfloat16)
        y = dst[:, pad:pad + H]
        fn(x, gain, 0.0, 1e-6, out=y)
        torch.cuda.synchronize()
        assert _same(y, dense)
        assert bool((dst[:, :pad] == SENTINEL).all()) and bool((dst[:, pad + H:] == SENTINEL).all())


@pytest.mark.parametrize("T,H,hq,hkv,D", SHAPES)
@pytest.mark.parametrize("upcast", [True, False])
def test_qk_views_into_fused_qkv(cuda_ok, T, H, hq, hkv, D, upcast):
    g = _g(2)
    W = (hq + 2 * hkv) * D
    qkv = torch.randn(T, W, device="cuda", generator=g).to(torch.bfloat16)
    q = qkv[:, :hq * D].view(T, hq, D)
    k = qkv[:, hq * D:(hq + hkv) * D].view(T, hkv, D)
    dq, dk = cores.qk_norm_rope(q.contiguous(), k.contiguous(), eps=1e-6, rope_base=5e5,
                                upcast_rope=upcast, query_scale=0.125)
    out = torch.full((T, W), SENTINEL, device="cuda").to(torch.bfloat16)
    qo = out[:, :hq * D].view(T, hq, D)
    ko = out[:, hq * D:(hq + hkv) * D].view(T, hkv, D)
    cores.qk_norm_rope(q, k, eps=1e-6, rope_base=5e5, upcast_rope=upcast, query_scale=0.125,
                       q_out=qo, k_out=ko)
    torch.cuda.synchronize()
    assert _same(qo, dq) and _same(ko, dk)
    assert bool((out[:, (hq + hkv) * D:] == SENTINEL).all())  # the V part is untouched


@pytest.mark.parametrize("T,H,hq,hkv,D", SHAPES)
def test_exact_in_place(cuda_ok, T, H, hq, hkv, D):
    g = _g(3)
    x = torch.randn(T, H, device="cuda", generator=g).to(torch.bfloat16)
    gain = (1 + 0.1 * torch.randn(H, device="cuda", generator=g)).float()
    theta = (0.5 * torch.rand(H, device="cuda", generator=g)).float()
    stream = torch.randn(T, H, device="cuda", generator=g)

    ref = cores.rms_norm(x, gain, 0.0, 1e-6)
    xi = x.clone()
    cores.rms_norm(xi, gain, 0.0, 1e-6, out=xi)
    torch.cuda.synchronize()
    assert _same(xi, ref)

    ref = cores.norm_residual(stream, x, theta, gain, 0.0)
    si = stream.clone()
    cores.norm_residual(si, x, theta, gain, 0.0, out=si)
    torch.cuda.synchronize()
    assert _same(si, ref)

    q = torch.randn(T, hq, D, device="cuda", generator=g).to(torch.bfloat16)
    k = torch.randn(T, hkv, D, device="cuda", generator=g).to(torch.bfloat16)
    rq, rk = cores.qk_norm_rope(q, k, eps=1e-6, rope_base=5e5)
    qi, ki = q.clone(), k.clone()
    cores.qk_norm_rope(qi, ki, eps=1e-6, rope_base=5e5, q_out=qi, k_out=ki)
    torch.cuda.synchronize()
    assert _same(qi, rq) and _same(ki, rk)

    o = torch.randn(T, hq, D, device="cuda", generator=g).to(torch.bfloat16)
    gate = (2 * torch.randn(T, hq, D, device="cuda", generator=g)).to(torch.bfloat16)
    for ng in (None, hq * D):
        ref = cores.output_norm_gate(o, gate, ng, 1e-6)
        oi = o.clone()
        cores.output_norm_gate(oi, gate, ng, 1e-6, out=oi)
        torch.cuda.synchronize()
        assert _same(oi, ref)


def test_partial_overlap_rejected_before_launch(cuda_ok):
    x = torch.randn(64, 256, device="cuda").to(torch.bfloat16)
    with pytest.raises(MuseError):
        cores.rms_norm(x[1:], None, 0.0, 1e-6, out=x[:-1])
