"""GPU parity of the _residual_core forms (muse_residual_blend, muse_residual,
muse_residual_gate_angles) and of their backward (muse_residual_blend_backward,
muse_residual_backward) through the C ABI against the oracle, element by
element over the whole output: small and ragged shapes, a case with many rows
per CTA, and the full-size workloads (every token)."""
import numpy as np
import pytest
import torch

import oracle
from gate_cores_b200 import cores, inputs

from . import harness
from .test_gpu_parity import RAGGED, WRAP

pytestmark = pytest.mark.gpu

SMALL = [inputs.WORKLOADS["tiny_t64_h256"]] + RAGGED + [WRAP]
CASES = [(c, v) for c in harness.RESIDUAL_CORES for v in harness.VARIANTS[c]]
FULL = ["prefill_t8192_h4096", "decode_t128_h4096", "thd16_h5120", "large_t32768_h8192"]


def _compare(wl, core, variant):
    ci = harness.make(wl, core, variant)
    outs = harness.run_gpu(wl, core, ci)
    torch.cuda.synchronize()
    return harness.compare_full(wl, core, ci, outs, f"{wl.name}/{core}/{variant}")


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("core,variant", CASES, ids=lambda x: str(x))
def test_small_full_outputs(cuda_ok, wl, core, variant):
    _compare(wl, core, variant)


@pytest.mark.parametrize("name", FULL)
@pytest.mark.parametrize("core,variant", CASES, ids=lambda x: str(x))
def test_full_size_all_tokens(cuda_ok, name, core, variant):
    _compare(inputs.WORKLOADS[name], core, variant)


@pytest.mark.parametrize("core", harness.RESIDUAL_CORES)
def test_in_place_equals_out_of_place(cuda_ok, core):
    wl = inputs.WORKLOADS["prefill_t8192_h4096"]
    ci = harness.make(wl, core, harness.DEFAULT_VARIANT[core])
    t = {k: (None if v is None else v.cuda()) for k, v in ci.tensors.items()}
    p = t["theta"] if core == "residual_blend" else t["gate"]
    ref = (cores.residual_blend(t["stream"], t["branch"], p) if core == "residual_blend"
           else cores.residual(t["stream"], t["branch"], p))
    h = t["stream"].clone()
    if core == "residual_blend":
        cores.residual_blend(h, t["branch"], p, out=h)
    else:
        cores.residual(h, t["branch"], p, out=h)
    torch.cuda.synchronize()
    assert torch.equal(h.view(torch.int32), ref.view(torch.int32))


@pytest.mark.parametrize("temperature,eps", [(0.3, 1e-3), (0.05, 0.01), (2.0, 0.0), (0.3, 1.0)])
def test_gate_angles_against_oracle(cuda_ok, temperature, eps):
    r = np.random.default_rng(7)
    g = np.concatenate([r.standard_normal(4093) * 3, [0.0, -1e4, 1e4, 60.0]]).astype(np.float32)
    th = cores.residual_gate_angles(torch.from_numpy(g).cuda(), temperature, eps).cpu().numpy()
    _, _, want = oracle.residual_gate_coefficients(g, temperature, float(np.float32(eps)))
    err = np.abs(th.astype(np.float64) - want)
    assert np.all(err <= 2e-6 * np.abs(want) + 16 * 2.0 ** -149), (err.max(), g[np.argmax(err)])


def test_gate_form_equals_blend_of_its_angles(cuda_ok):
    # muse_residual and muse_residual_blend with theta = muse_residual_gate_angles
    # agree within FP32 evaluation of the coefficients
    wl = inputs.WORKLOADS["tiny_t64_h256"]
    ci = harness.make(wl, "residual", "bf16_branch")
    h, b, g = (ci.tensors[k].cuda() for k in ("stream", "branch", "gate"))
    th = cores.residual_gate_angles(g)
    y1 = cores.residual(h, b, g)
    y2 = cores.residual_blend(h, b, th)
    torch.cuda.synchronize()
    d = (y1.double() - y2.double()).abs()
    mag = h.double().abs() + b.double().abs()
    assert bool((d <= 1e-6 * mag + 1e-30).all())


# ------------------------------------------------------------------ backward

# up to the prefill size: the parameter gradients are whole-tensor row sums, so
# the oracle runs in one call (its per-element check arrays at the large
# workload would take 13 GB of host memory)
BWD_WLS = [inputs.WORKLOADS["tiny_t64_h256"]] + RAGGED + [WRAP, inputs.WORKLOADS["prefill_t8192_h4096"]]


@pytest.mark.parametrize("wl", BWD_WLS, ids=lambda w: w.name)
@pytest.mark.parametrize("core,variant", CASES, ids=lambda x: str(x))
def test_backward_against_oracle(cuda_ok, wl, core, variant):
    from gate_cores_b200.inputs import to_numpy

    from .parity import check, check_param

    ci = harness.make(wl, core, variant)
    t, s = ci.tensors, ci.scalars
    dy = inputs.upstream_grad(wl, 0, core, tuple(t["stream"].shape), torch.float32)
    h, b = t["stream"].cuda(), t["branch"].cuda()
    if core == "residual_blend":
        dsi, db, dp = cores.residual_backward(h, b, dy.cuda(), theta=t["theta"].cuda())
    else:
        dsi, db, dp = cores.residual_backward(h, b, dy.cuda(), gate=t["gate"].cuda(),
                                              temperature=s["temperature"], eps=s["eps"])
    torch.cuda.synchronize()
    np_ = lambda x: to_numpy(x.cpu())  # noqa: E731
    if core == "residual_blend":
        rs, rb, rp = oracle.residual_blend_bwd(np_(t["stream"]), np_(t["branch"]), np_(dy), np_(t["theta"]))
    else:
        rs, rb, rp = oracle.residual_bwd(np_(t["stream"]), np_(t["branch"]), np_(dy), np_(t["gate"]),
                                         s["temperature"], float(np.float32(s["eps"])))
    what = f"{wl.name}/{core}/{variant}"
    check(np_(dsi), rs, what + "/dstream", backward=True)
    check(np_(db), rb, what + "/dbranch", backward=True)
    check_param(dp.cpu().numpy(), rp, what + "/dparam")


def test_backward_in_place_deterministic_and_optional_param(cuda_ok):
    wl = inputs.WORKLOADS["prefill_t8192_h4096"]
    ci = harness.make(wl, "residual", "bf16_branch")
    t = {k: v.cuda() for k, v in ci.tensors.items()}
    dy = inputs.upstream_grad(wl, 0, "residual", tuple(t["stream"].shape), torch.float32).cuda()
    a = cores.residual_backward(t["stream"], t["branch"], dy, gate=t["gate"])
    b2 = cores.residual_backward(t["stream"], t["branch"], dy, gate=t["gate"])
    c = cores.residual_backward(t["stream"], t["branch"], dy, gate=t["gate"], want_param=False)
    torch.cuda.synchronize()
    for x, y in zip(a, b2):  # bit-reproducible, parameter gradient included
        assert torch.equal(x.view(torch.int16) if x.dtype == torch.bfloat16 else x.view(torch.int32),
                           y.view(torch.int16) if y.dtype == torch.bfloat16 else y.view(torch.int32))
    assert c[2] is None and torch.equal(c[0].view(torch.int32), a[0].view(torch.int32))
    # dstream_in in place of dstream_out
    from gate_cores_b200 import _lib
    d = dy.clone()
    db = torch.empty_like(t["branch"])
    H = t["stream"].shape[-1]
    T = t["stream"].numel() // H
    _lib.muse_residual_backward(t["stream"].data_ptr(), t["branch"].data_ptr(), d.data_ptr(), d.data_ptr(),
                                db.data_ptr(), _lib.MUSE_DTYPE_BF16, T, H, t["gate"].data_ptr(), 0.3, 1e-3, None,
                                None, 0, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert torch.equal(d.view(torch.int32), a[0].view(torch.int32))
    assert torch.equal(db.view(torch.int16), a[1].view(torch.int16))


def test_backward_zero_rows_zeroes_param(cuda_ok):
    h = torch.zeros(0, 64, device="cuda")
    b = torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda")
    _, _, dp = cores.residual_backward(h, b, h, theta=torch.ones(64, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(dp, torch.zeros(64, device="cuda"))
