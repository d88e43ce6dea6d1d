"""GPU parity of the backward calls (cores 1, 2, 5) against the oracle.

Forward inputs come from the same seeded generators as the forward parity
tests, the incoming gradient from inputs.upstream_grad.  Every output is
compared element by element: input gradients with the backward allowances of
tests/parity.py, parameter gradients (FP32 row sums) with check_param.  The
prefill-size cases run in the launch configuration the benchmark uses.
"""
import pytest
import torch

import oracle
from gate_cores_b200 import _lib, cores, inputs
from gate_cores_b200.inputs import Workload, to_numpy

from . import harness
from .parity import check, check_param

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
ROW_CASES = [("rms_norm", v) for v in ("zc_gain", "plain_gain", "no_gain", "f32_io")] + \
    [("input_scale_norm", v) for v in ("plain_gain", "zc_gain", "f32_io")]
RES_CASES = ["gain_after", "gain_before", "no_gain", "f32_branch"]


def _np(t):
    return None if t is None else to_numpy(t.cpu())


def _skip_wide(width, dtype):
    vec = 8 if dtype == torch.bfloat16 else 4
    if width // vec > 1024:
        pytest.skip("rows above the backward's documented limit of 1024 16-byte vectors")


@pytest.mark.parametrize("wl", WLS, ids=lambda w: w.name)
@pytest.mark.parametrize("core,variant", ROW_CASES, ids=lambda x: str(x))
def test_row_backward(cuda_ok, wl, core, variant):
    ci = harness.make(wl, core, variant)
    t, s = ci.tensors, ci.scalars
    x = t["x"]
    _skip_wide(x.shape[-1], x.dtype)
    dy = inputs.upstream_grad(wl, 0, core, tuple(x.shape), x.dtype)
    fn = cores.rms_norm_backward if core == "rms_norm" else cores.input_scale_norm_backward
    g = None if t["gain"] is None else t["gain"].cuda()
    dx, dgain = fn(x.cuda(), dy.cuda(), g, s["gain_offset"], s["eps"])
    torch.cuda.synchronize()
    ofn = oracle.rms_norm_bwd if core == "rms_norm" else oracle.input_scale_norm_bwd
    (rdx, rgain) = ofn(_np(x), _np(dy), _np(t["gain"]), s["gain_offset"], s["eps"])
    check(_np(dx), rdx, f"{wl.name}/{core}/{variant}/dx", backward=True)
    if g is None:
        assert dgain is None
    else:
        check_param(dgain.cpu().numpy(), rgain, f"{wl.name}/{core}/{variant}/dgain")


@pytest.mark.parametrize("wl", WLS, ids=lambda w: w.name)
@pytest.mark.parametrize("variant", RES_CASES)
def test_norm_residual_backward(cuda_ok, wl, variant):
    ci = harness.make(wl, "norm_residual", variant)
    t, s = ci.tensors, ci.scalars
    _skip_wide(t["branch"].shape[-1], t["branch"].dtype)
    dout = inputs.upstream_grad(wl, 0, "norm_residual", tuple(t["stream"].shape), torch.float32)
    g = None if t["gain"] is None else t["gain"].cuda()
    dsi, db, dgain, dtheta = cores.norm_residual_backward(
        t["stream"].cuda(), t["branch"].cuda(), dout.cuda(), t["theta"].cuda(), g, s["gain_offset"],
        s.get("input_scale", False), s["norm_eps"])
    torch.cuda.synchronize()
    rds, rdb, rg, rt = oracle.norm_residual_bwd(
        _np(t["stream"]), _np(t["branch"]), _np(dout), _np(t["theta"]), _np(t["gain"]),
        s["gain_offset"], s.get("input_scale", False), s["norm_eps"])
    what = f"{wl.name}/norm_residual/{variant}"
    check(_np(dsi), rds, what + "/dstream", backward=True)
    check(_np(db), rdb, what + "/dbranch", backward=True)
    check_param(dtheta.cpu().numpy(), rt, what + "/dtheta")
    if g is None:
        assert dgain is None
    else:
        check_param(dgain.cpu().numpy(), rg, what + "/dgain")


def test_backward_is_deterministic(cuda_ok):
    wl = inputs.WORKLOADS["prefill_t8192_h4096"]
    ci = harness.make(wl, "norm_residual", "gain_after")
    t, s = ci.tensors, ci.scalars
    dout = inputs.upstream_grad(wl, 0, "norm_residual", tuple(t["stream"].shape), torch.float32).cuda()
    args = (t["stream"].cuda(), t["branch"].cuda(), dout, t["theta"].cuda(), t["gain"].cuda(),
            s["gain_offset"], False, s["norm_eps"])
    a = cores.norm_residual_backward(*args)
    b = cores.norm_residual_backward(*args)
    for u, v in zip(a, b):
        assert torch.equal(u.view(torch.int32) if u.dtype == torch.float32 else u.view(torch.int16),
                           v.view(torch.int32) if v.dtype == torch.float32 else v.view(torch.int16))


def test_backward_without_parameter_gradients(cuda_ok):
    # dgain / dtheta skipped: no workspace needed, input gradients unchanged
    wl = inputs.WORKLOADS["tiny_t64_h256"]
    ci = harness.make(wl, "rms_norm", "zc_gain")
    x, g = ci.tensors["x"].cuda(), ci.tensors["gain"].cuda()
    dy = inputs.upstream_grad(wl, 0, "rms_norm", tuple(x.shape), x.dtype).cuda()
    a, da = cores.rms_norm_backward(x, dy, g, 1.0, 1e-6)
    b, db = cores.rms_norm_backward(x, dy, g, 1.0, 1e-6, want_dgain=False)
    assert db is None and torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_backward_workspace_checked(cuda_ok):
    x = torch.zeros(64, 256, device="cuda", dtype=torch.bfloat16)
    g = torch.ones(256, device="cuda")
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises((_lib.MuseError, ValueError)):
        cores.rms_norm_backward(x, x, g, 0.0, 1e-6, workspace=small)
    assert _lib.muse_norm_backward_workspace_bytes(64, 256) >= 256 * 4
    assert _lib.muse_device_error() == 0
