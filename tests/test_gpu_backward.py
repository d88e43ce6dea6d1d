"""GPU parity of the backward calls (all five cores) against the oracle.

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
    # core 5 rows of 514 / 640 / 1024 vectors run on CTA pairs (idle consumers
    # in each half at 514); 513 vectors (odd) on one CTA with two slots
    Workload("ragged_t97_h4112", hidden=4112, hq=32, hkv=8, head_dim=128, rope_base=5.0e5, batch=1, seqlen=97),
    Workload("ragged_t61_h4104", hidden=4104, hq=32, hkv=8, head_dim=128, rope_base=5.0e5, batch=1, seqlen=61),
    Workload("ragged_t203_h5120", hidden=5120, hq=40, hkv=8, head_dim=128, rope_base=5.0e5, batch=1, seqlen=203),
    Workload("mid_t2048_h8192", hidden=8192, hq=64, hkv=8, head_dim=128, rope_base=5.0e5, batch=1,
             seqlen=2048, outlier_frac=0.01),
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


HEAD_WLS = [
    inputs.WORKLOADS["tiny_t64_h256"],
    Workload("ragged_t37_h264", hidden=264, hq=6, hkv=2, head_dim=80, rope_base=1.0e4, batch=1, seqlen=37),
    Workload("ragged_b3s5_h40", hidden=40, hq=3, hkv=1, head_dim=16, rope_base=1.0e4, batch=3, seqlen=5),
    Workload("ragged_thd_h512", hidden=512, hq=8, hkv=4, head_dim=64, rope_base=5.0e5, layout="thd",
             positions="restart", num_seqs=7, seq_len_range=(0, 40)),
    Workload("ragged_t1_h4096", hidden=4096, hq=32, hkv=8, head_dim=128, rope_base=5.0e5, batch=1, seqlen=1),
    Workload("ragged_t300_h8192", hidden=8192, hq=64, hkv=8, head_dim=256, rope_base=5.0e5, batch=3,
             seqlen=100, outlier_frac=0.01),
    inputs.WORKLOADS["decode_t128_h4096"],
    inputs.WORKLOADS["prefill_t8192_h4096"],
]
GATE_CASES = ["per_head", "per_token", "f32"]
QK_CASES = ["upcast", "qscale", "no_rope", "explicit_pos", "f32", "v2", "v2_qscale"]


@pytest.mark.parametrize("wl", HEAD_WLS, ids=lambda w: w.name)
@pytest.mark.parametrize("variant", GATE_CASES)
def test_output_norm_gate_backward(cuda_ok, wl, variant):
    ci = harness.make(wl, "output_norm_gate", variant)
    t, s = ci.tensors, ci.scalars
    o, g = t["o"], t["g"]
    dy = inputs.upstream_grad(wl, 0, "output_norm_gate", tuple(o.shape), o.dtype)
    ng = o.shape[-2] * o.shape[-1] if s.get("per_token") else None
    if ng is not None and ng * o.element_size() > 65536:
        pytest.skip("norm group above the documented 64 KB")
    d_o, dg = cores.output_norm_gate_backward(o.cuda(), g.cuda(), dy.cuda(), ng, s["eps"])
    torch.cuda.synchronize()
    r_o, r_g = oracle.output_norm_gate_bwd(_np(o), _np(g), _np(dy), ng, s["eps"])
    what = f"{wl.name}/output_norm_gate/{variant}"
    check(_np(d_o), r_o, what + "/do", backward=True)
    check(_np(dg), r_g, what + "/dgate", backward=True)


@pytest.mark.parametrize("wl", HEAD_WLS, ids=lambda w: w.name)
@pytest.mark.parametrize("variant", QK_CASES)
def test_qk_norm_rope_backward(cuda_ok, wl, variant):
    ci = harness.make(wl, "qk_norm_rope", variant)
    t, s = ci.tensors, ci.scalars
    q, k = t["q"], t["k"]
    if q.dtype == torch.float32 and wl.head_dim * 4 > 512:
        pytest.skip("f32 heads above 512 bytes are outside the documented limit")
    gq = inputs.upstream_grad(wl, 0, "qk_q", tuple(q.shape), q.dtype)
    gk = inputs.upstream_grad(wl, 0, "qk_k", tuple(k.shape), k.dtype)
    qd, kd, gqd, gkd = q.cuda(), k.cuda(), gq.cuda(), gk.cuda()
    if s["layout"] == "bshd":
        B, S = s["batch"], s["seqlen"]
        qd, kd, gqd, gkd = (x.view(B, S, *x.shape[1:]) for x in (qd, kd, gqd, gkd))
    pos = t["positions"]
    dq, dk = cores.qk_norm_rope_backward(
        qd, kd, gqd, gkd, positions=None if pos is None else pos.cuda(),
        cu_seqlens=t["cu_seqlens"].cuda() if s["layout"] == "thd" else None, eps=s["eps"],
        query_scale=s.get("query_scale", 1.0), use_rope=s.get("use_rope", True), rope_base=s["rope_base"],
        upcast_rope=s.get("upcast_rope", True))
    torch.cuda.synchronize()
    rq, rk = oracle.qk_norm_rope_bwd(_np(q), _np(k), _np(gq), _np(gk), harness.all_positions(wl, ci),
                                     s["eps"], s.get("query_scale", 1.0), s.get("use_rope", True),
                                     s["rope_base"], upcast_rope=s.get("upcast_rope", True))
    what = f"{wl.name}/qk_norm_rope/{variant}"
    check(_np(dq.reshape(q.shape)), rq, what + "/dq", backward=True)
    check(_np(dk.reshape(k.shape)), rk, what + "/dk", backward=True)


def test_no_device_error_after_backward_runs(cuda_ok):
    assert _lib.muse_device_error() == 0


def test_backward_graph_replay_matches_eager(cuda_ok):
    # captured backward calls (the row kernel and its fixed-order reduction of
    # the parameter partials, programmatic launches and, for core 5, both
    # parameter gradients) replay to the eager calls' bits
    wl = inputs.WORKLOADS["prefill_t8192_h4096"]
    ci = harness.make(wl, "rms_norm", "zc_gain")
    x, g = ci.tensors["x"].cuda(), ci.tensors["gain"].cuda()
    dy = inputs.upstream_grad(wl, 0, "rms_norm", tuple(x.shape), x.dtype).cuda()
    ws = torch.empty(_lib.muse_norm_backward_workspace_bytes(x.shape[0], x.shape[1]), dtype=torch.uint8,
                     device="cuda")
    ref_dx, ref_dg = cores.rms_norm_backward(x, dy, g, 1.0, 1e-6, workspace=ws)
    cr = harness.make(wl, "norm_residual", "gain_after")
    t, s = cr.tensors, cr.scalars
    h, b, th, gr = (t[k].cuda() for k in ("stream", "branch", "theta", "gain"))
    dout = inputs.upstream_grad(wl, 0, "norm_residual", tuple(h.shape), torch.float32).cuda()
    ws5 = torch.empty(_lib.muse_norm_backward_workspace_bytes(h.shape[0], h.shape[1]), dtype=torch.uint8,
                      device="cuda")
    res = (h, b, dout, th, gr, s["gain_offset"], False, s["norm_eps"])
    ref5 = cores.norm_residual_backward(*res, workspace=ws5)
    dx = torch.empty_like(x)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up outside the capture
        cores.rms_norm_backward(x, dy, g, 1.0, 1e-6, dx=dx, workspace=ws)
        cores.norm_residual_backward(*res, workspace=ws5)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out = cores.rms_norm_backward(x, dy, g, 1.0, 1e-6, dx=dx, workspace=ws)
        out5 = cores.norm_residual_backward(*res, workspace=ws5)
    for _ in range(3):
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out[0].view(torch.int16), ref_dx.view(torch.int16))
        assert torch.equal(out[1].view(torch.int32), ref_dg.view(torch.int32))
        for u, v in zip(out5, ref5):
            assert torch.equal(u.view(torch.int32) if u.dtype == torch.float32 else u.view(torch.int16),
                               v.view(torch.int32) if v.dtype == torch.float32 else v.view(torch.int16))
    del graph
    assert _lib.muse_device_error() == 0
