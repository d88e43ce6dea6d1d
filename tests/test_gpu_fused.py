"""GPU parity of core 5 fused with the next sublayer's pre-norm
(muse_norm_residual_rms_norm), and of _residual_core fused with it
(muse_residual_blend_rms_norm).

The new stream must be bit-identical to muse_norm_residual's (same
arithmetic) and within the core 5 rule of the oracle; the pre-norm output is
checked against the oracle's core 1 applied to the stream values the call
wrote (FP32 in, y dtype out), so the check does not depend on FP32 rounding
differences upstream.
"""
import pytest
import torch

import oracle
from gate_cores_b200 import cores, inputs
from gate_cores_b200.inputs import Workload, to_numpy

from . import harness
from .parity import check

pytestmark = pytest.mark.gpu

WLS = [
    inputs.WORKLOADS["tiny_t64_h256"],
    Workload("ragged_t37_h264", hidden=264, hq=6, hkv=2, head_dim=80, rope_base=1.0e4, batch=1, seqlen=37),
    Workload("ragged_b3s5_h40", hidden=40, hq=3, hkv=1, head_dim=16, rope_base=1.0e4, batch=3, seqlen=5),
    Workload("ragged_t1_h4096", hidden=4096, hq=32, hkv=8, head_dim=128, rope_base=5.0e5, batch=1, seqlen=1),
    Workload("ragged_t300_h8192", hidden=8192, hq=64, hkv=8, head_dim=128, rope_base=5.0e5, batch=3,
             seqlen=100, outlier_frac=0.01),
    inputs.WORKLOADS["prefill_t8192_h4096"],
]
CASES = [(v, yd, ng) for v in ("gain_after", "gain_before", "no_gain", "f32_branch")
         for yd in ("f32", "bf16") for ng in ("zc", "none")]


def _np(t):
    return None if t is None else to_numpy(t.cpu())


@pytest.mark.parametrize("wl", WLS, ids=lambda w: w.name)
@pytest.mark.parametrize("variant,ydt,next_gain", CASES, ids=lambda x: str(x))
def test_fused_residual_prenorm(cuda_ok, wl, variant, ydt, next_gain):
    ci = harness.make(wl, "norm_residual", variant)
    t, s = ci.tensors, ci.scalars
    br = t["branch"]
    if br.dtype == torch.float32 and wl.hidden // 4 > 1024:
        pytest.skip("rows above the fused call's documented limit")
    g2, off2 = (inputs.gain(wl, 0, "gain_next", True) if next_gain == "zc" else (None, 0.0))
    y_dtype = torch.float32 if ydt == "f32" else torch.bfloat16
    if br.dtype == torch.float32 and y_dtype != torch.float32:
        pytest.skip("y is FP32 or in the branch dtype (test_fused_rejects_other_y_dtype)")
    dev = lambda x: None if x is None else x.cuda()
    args = (dev(t["stream"]), dev(br), dev(t["theta"]), dev(t["gain"]), s["gain_offset"],
            s.get("input_scale", False), s["norm_eps"])
    h, y = cores.norm_residual_rms_norm(*args, next_gain=dev(g2), next_gain_offset=off2,
                                        next_eps=1e-6, y_dtype=y_dtype)
    ref_h = cores.norm_residual(*args)
    torch.cuda.synchronize()
    assert torch.equal(h.view(torch.int32), ref_h.view(torch.int32))
    what = f"{wl.name}/{variant}/{ydt}/{next_gain}"
    rh = oracle.norm_residual(_np(t["stream"]), _np(br), _np(t["theta"]), _np(t["gain"]),
                              s["gain_offset"], s.get("input_scale", False), s["norm_eps"])
    check(_np(h), rh, what + "/stream")
    ry = oracle.rms_norm_to(_np(h), oracle.F32 if ydt == "f32" else oracle.BF16, _np(g2), off2, 1e-6)
    check(_np(y), ry, what + "/y")


def test_fused_rejects_wide_rows(cuda_ok):
    from gate_cores_b200._lib import MuseError, MUSE_ERR_UNSUPPORTED
    H = 16384
    x = torch.zeros(4, H, device="cuda")
    b = torch.zeros(4, H, device="cuda", dtype=torch.bfloat16)
    th = torch.zeros(H, device="cuda")
    with pytest.raises(MuseError) as e:
        cores.norm_residual_rms_norm(x, b, th)
    assert e.value.status == MUSE_ERR_UNSUPPORTED


def test_fused_rejects_other_y_dtype(cuda_ok):
    from gate_cores_b200._lib import MuseError, MUSE_ERR_UNSUPPORTED
    x = torch.zeros(4, 256, device="cuda")
    th = torch.zeros(256, device="cuda")
    with pytest.raises(MuseError) as e:
        cores.norm_residual_rms_norm(x, x.clone(), th, y_dtype=torch.bfloat16)
    assert e.value.status == MUSE_ERR_UNSUPPORTED


BLEND_CASES = [(v, yd, ng) for v in ("bf16_branch", "f32_branch") for yd in ("f32", "bf16") for ng in ("zc", "none")]


@pytest.mark.parametrize("wl", WLS + [Workload("wrap_t65536_h256", hidden=256, hq=2, hkv=1, head_dim=128,
                                               rope_base=1.0e4, batch=16, seqlen=4096)], ids=lambda w: w.name)
@pytest.mark.parametrize("variant,ydt,next_gain", BLEND_CASES, ids=lambda x: str(x))
def test_fused_residual_blend_prenorm(cuda_ok, wl, variant, ydt, next_gain):
    # _residual_core (angle form) fused with the next pre-norm: the stream is
    # bit-identical to muse_residual_blend's and within the oracle's blend;
    # y is the oracle's core 1 of the stream the call wrote
    ci = harness.make(wl, "residual_blend", variant)
    t = ci.tensors
    br = t["branch"]
    if br.dtype == torch.float32 and wl.hidden // 4 > 1024:
        pytest.skip("rows above the fused call's documented limit")
    y_dtype = torch.float32 if ydt == "f32" else torch.bfloat16
    if br.dtype == torch.float32 and y_dtype != torch.float32:
        pytest.skip("y is FP32 or in the branch dtype")
    g2, off2 = (inputs.gain(wl, 0, "gain_next", True) if next_gain == "zc" else (None, 0.0))
    dev = lambda x: None if x is None else x.cuda()  # noqa: E731
    h, y = cores.residual_blend_rms_norm(dev(t["stream"]), dev(br), dev(t["theta"]), next_gain=dev(g2),
                                         next_gain_offset=off2, next_eps=1e-6, y_dtype=y_dtype)
    ref_h = cores.residual_blend(dev(t["stream"]), dev(br), dev(t["theta"]))
    torch.cuda.synchronize()
    assert torch.equal(h.view(torch.int32), ref_h.view(torch.int32))
    what = f"{wl.name}/blend/{variant}/{ydt}/{next_gain}"
    check(_np(h), oracle.residual_blend(_np(t["stream"]), _np(br), _np(t["theta"])), what + "/stream")
    ry = oracle.rms_norm_to(_np(h), oracle.F32 if ydt == "f32" else oracle.BF16, _np(g2), off2, 1e-6)
    check(_np(y), ry, what + "/y")


def test_fused_blend_in_place_and_rejections(cuda_ok):
    from gate_cores_b200._lib import MuseError, MUSE_ERR_UNSUPPORTED
    wl = inputs.WORKLOADS["prefill_t8192_h4096"]
    ci = harness.make(wl, "residual_blend", "bf16_branch")
    t = {k: v.cuda() for k, v in ci.tensors.items()}
    ref_h, ref_y = cores.residual_blend_rms_norm(t["stream"], t["branch"], t["theta"], y_dtype=torch.bfloat16)
    h = t["stream"].clone()
    yb = t["branch"].clone()  # y over the branch, the stream in place
    cores.residual_blend_rms_norm(h, yb, t["theta"], y_dtype=torch.bfloat16, out=h, y=yb)
    torch.cuda.synchronize()
    assert torch.equal(h.view(torch.int32), ref_h.view(torch.int32))
    assert torch.equal(yb.view(torch.int16), ref_y.view(torch.int16))
    with pytest.raises(MuseError) as e:
        H = 16384
        cores.residual_blend_rms_norm(torch.zeros(4, H, device="cuda"),
                                      torch.zeros(4, H, device="cuda", dtype=torch.bfloat16),
                                      torch.zeros(H, device="cuda"))
    assert e.value.status == MUSE_ERR_UNSUPPORTED
