"""The allocation-free core 1 backward (muse_rms_norm_backward_noalloc)
against muse_rms_norm_backward with a caller workspace: two calls of each on
the same inputs give bit-identical input and gain gradients; an oversize call
is rejected before any launch; a call without a gain gradient needs no
scratch.  (Named to be collected last.)"""
import pytest
import torch

from gate_cores_b200 import _lib, cores, inputs

from . import harness

pytestmark = pytest.mark.gpu


def _noalloc(x, dy, gain, offset, eps, want_dgain=True):
    dx = torch.empty_like(x)
    dgain = torch.empty(x.shape[-1], dtype=torch.float32, device=x.device) if want_dgain else None
    H = x.shape[-1]
    _lib.muse_rms_norm_backward_noalloc(
        x.data_ptr(), dy.data_ptr(), dx.data_ptr(), _lib.MUSE_DTYPE_BF16, x.shape[0], H, H, H, H,
        gain.data_ptr(), offset, eps, None if dgain is None else dgain.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    return dx, dgain


def test_noalloc_matches_workspace_call_twice(cuda_ok):
    wl = inputs.WORKLOADS["prefill_t8192_h4096"]
    ci = harness.make(wl, "rms_norm", "zc_gain")
    x, g = ci.tensors["x"].cuda(), ci.tensors["gain"].cuda()
    off, eps = ci.scalars["gain_offset"], ci.scalars["eps"]
    dy = inputs.upstream_grad(wl, 0, "rms_norm", tuple(x.shape), x.dtype).cuda()
    for _ in range(2):
        ref_dx, ref_dg = cores.rms_norm_backward(x, dy, g, off, eps)
        dx, dg = _noalloc(x, dy, g, off, eps)
        torch.cuda.synchronize()
        assert torch.equal(dx.view(torch.int16), ref_dx.view(torch.int16))
        assert torch.equal(dg.view(torch.int32), ref_dg.view(torch.int32))
    assert _lib.muse_device_error() == 0


def test_noalloc_without_gain_gradient(cuda_ok):
    wl = inputs.WORKLOADS["tiny_t64_h256"]
    ci = harness.make(wl, "rms_norm", "plain_gain")
    x, g = ci.tensors["x"].cuda(), ci.tensors["gain"].cuda()
    dy = inputs.upstream_grad(wl, 0, "rms_norm", tuple(x.shape), x.dtype).cuda()
    ref_dx, _ = cores.rms_norm_backward(x, dy, g, 0.0, 1e-6, want_dgain=False)
    dx, _ = _noalloc(x, dy, g, 0.0, 1e-6, want_dgain=False)
    torch.cuda.synchronize()
    assert torch.equal(dx.view(torch.int16), ref_dx.view(torch.int16))


def test_noalloc_rejects_oversize(cuda_ok):
    # 8192-wide rows: one 32 KB partial row per CTA exceeds the fixed 16 MiB
    # once the grid passes 512 CTAs
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rows = 4 * sms
    if rows * 8192 * 4 <= 16 << 20:
        pytest.skip("this GPU's backward grid fits the fixed scratch at 8192 columns")
    x = torch.zeros(rows, 8192, dtype=torch.bfloat16, device="cuda")
    g = torch.ones(8192, device="cuda")
    with pytest.raises(_lib.MuseError) as e:
        _noalloc(x, x, g, 0.0, 1e-6)
    assert e.value.status == _lib.MUSE_ERR_UNSUPPORTED
