"""The allocation-free core 1 backward (muse_rms_norm_backward_noalloc)
against muse_rms_norm_backward with a caller workspace: two calls of each on
the same inputs give bit-identical input and gain gradients; wide rows either
fit the fixed scratch (and match) or are rejected before any launch; an
invalid call reports its argument error; a call without a gain gradient needs
no scratch.  (Named to be collected last.)"""
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


def test_noalloc_wide_rows_fit_or_are_rejected(cuda_ok):
    # 8192-wide rows at 4 rows per SM: one 32 KB partial row per CTA of the
    # grid the launch uses.  The call either reports that the partials exceed
    # the fixed 16 MiB (MUSE_ERR_UNSUPPORTED, nothing launched) or gives the
    # workspace call's results bit for bit.
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rows, H = 4 * sms, 8192
    wl = inputs.Workload("noalloc_h8192", hidden=H, hq=64, hkv=8, head_dim=128, rope_base=5e5,
                         batch=1, seqlen=rows)
    ci = harness.make(wl, "rms_norm", "zc_gain")
    x, g = ci.tensors["x"].cuda(), ci.tensors["gain"].cuda()
    dy = inputs.upstream_grad(wl, 0, "rms_norm", tuple(x.shape), x.dtype).cuda()
    try:
        dx, dg = _noalloc(x, dy, g, 1.0, 1e-6)
    except _lib.MuseError as e:
        assert e.status == _lib.MUSE_ERR_UNSUPPORTED, e
        return
    ref_dx, ref_dg = cores.rms_norm_backward(x, dy, g, 1.0, 1e-6)
    torch.cuda.synchronize()
    assert torch.equal(dx.view(torch.int16), ref_dx.view(torch.int16))
    assert torch.equal(dg.view(torch.int32), ref_dg.view(torch.int32))


def test_noalloc_invalid_call_fails_before_any_lookup(cuda_ok):
    # argument errors are reported as such, ahead of the scratch size check
    x = torch.zeros(16, 4096, dtype=torch.bfloat16, device="cuda")
    g = torch.ones(4096, device="cuda")
    dg = torch.empty(4096, device="cuda")
    with pytest.raises(_lib.MuseError) as e:
        _lib.muse_rms_norm_backward_noalloc(
            x.data_ptr(), x.data_ptr(), None, _lib.MUSE_DTYPE_BF16, 16, 4096, 4096, 4096, 4096,
            g.data_ptr(), 0.0, 1e-6, dg.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert e.value.status == _lib.MUSE_ERR_INVALID_ARGUMENT
