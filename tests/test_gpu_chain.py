"""Back-to-back calls on one stream, each reading what the previous call wrote.

Every kernel is launched with programmatic stream serialization and starts
by waiting for the previous grid (griddepcontrol.wait), so a consumer kernel
may already be resident while its producer drains.  These tests run chains
shaped like one decoder layer at the prefill size (8192 tokens, hidden 4096,
32 + 8 heads of 128) twice - once launched back to back, once with a device
synchronisation after every call - and require bit-identical results.  A
kernel that read its input before the producer's writes were visible would
differ.
"""
import pytest
import torch

from gate_cores_b200 import cores

pytestmark = pytest.mark.gpu

T, H, HQ, HKV, D = 8192, 4096, 32, 8, 128


def _inputs(seed=0):
    g = torch.Generator(device="cuda").manual_seed(seed)

    def randn(*shape, dtype=torch.bfloat16):
        return torch.randn(*shape, device="cuda", generator=g).to(dtype)

    return dict(
        x=randn(T, H),
        k=randn(T, HKV, D),
        gate=randn(T, HQ, D),
        stream=randn(T, H, dtype=torch.float32),
        gain=(1.0 + 0.1 * torch.randn(H, device="cuda", generator=g)).float(),
        theta=(0.3 * torch.rand(H, device="cuda", generator=g)).float(),
    )


def _layer(inp, sync: bool):
    """rms -> Q/K norm + RoPE (on the normed activations viewed as heads) ->
    output norm + gate -> norm + residual -> input-scale norm -> norm +
    residual again, each call consuming the previous one's output."""
    step = torch.cuda.synchronize if sync else (lambda: None)
    outs = {}
    a = cores.rms_norm(inp["x"], inp["gain"], 0.0, 1e-6)
    step()
    q, k = cores.qk_norm_rope(a.view(2, T // 2, HQ, D), inp["k"].view(2, T // 2, HKV, D), eps=1e-6,
                              rope_base=5e5)
    step()
    o = cores.output_norm_gate(q.view(T, HQ, D), inp["gate"], eps=1e-6)
    step()
    s1 = cores.norm_residual(inp["stream"], o.view(T, H), inp["theta"], inp["gain"], 0.0)
    step()
    b = cores.input_scale_norm(o.view(T, H), inp["gain"], 0.0, 1e-6)
    step()
    s2 = cores.norm_residual(s1, b, inp["theta"], inp["gain"], 0.0, input_scale=True)
    step()
    o2 = cores.output_norm_gate(b.view(T, HQ, D), q.view(T, HQ, D), norm_group=H, eps=1e-6)
    step()
    outs.update(a=a, q=q, k=k, o=o, s1=s1, b=b, s2=s2, o2=o2)
    torch.cuda.synchronize()
    return outs


def _same(x, y):
    return torch.equal(x.view(torch.int32) if x.dtype == torch.float32 else x.view(torch.int16),
                       y.view(torch.int32) if y.dtype == torch.float32 else y.view(torch.int16))


def test_decoder_chain_back_to_back_equals_synchronised(cuda_ok):
    inp = _inputs(0)
    ref = _layer(inp, sync=True)
    for _ in range(3):
        got = _layer(inp, sync=False)
        for name in ref:
            assert _same(got[name], ref[name]), name


def test_residual_stream_chain(cuda_ok):
    # the FP32 stream threaded through eight residual updates in a row
    inp = _inputs(1)
    branch = inp["x"]
    s_ref = inp["stream"]
    for _ in range(8):
        s_ref = cores.norm_residual(s_ref, branch, inp["theta"], inp["gain"], 0.0)
        torch.cuda.synchronize()
    s = inp["stream"]
    for _ in range(8):
        s = cores.norm_residual(s, branch, inp["theta"], inp["gain"], 0.0)
    torch.cuda.synchronize()
    assert _same(s, s_ref)


def test_qk_chain(cuda_ok):
    # Q/K outputs fed straight back as the next call's inputs
    inp = _inputs(2)
    q0 = inp["x"].view(T, HQ, D)
    k0 = inp["k"]
    q, k = q0, k0
    for _ in range(4):
        q, k = cores.qk_norm_rope(q, k, eps=1e-6, rope_base=5e5)
        torch.cuda.synchronize()
    q_ref, k_ref = q, k
    q, k = q0, k0
    for _ in range(4):
        q, k = cores.qk_norm_rope(q, k, eps=1e-6, rope_base=5e5)
    torch.cuda.synchronize()
    assert _same(q, q_ref) and _same(k, k_ref)
