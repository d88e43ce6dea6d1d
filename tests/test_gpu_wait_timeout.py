"""The give-up path of the bounded mbarrier waits, driven without a fault.

muse_rms_norm_stall_probe runs core 1's bulk-copy kernel with one stage that
its producer never signals (a flag that nothing sets) and a short poll limit.
The consumers of that CTA give up on it; the test checks that the device
error word reports it, that exactly the stalled CTA's rows from the stalled
one on are left unwritten while every written row matches the oracle, that
the context stays usable (the next ordinary call on the same inputs is
oracle-exact), and that clearing the word works.  Every copy the probe issues
is a normal in-bounds copy that completes.
"""
import numpy as np
import pytest
import torch

from gate_cores_b200 import _lib, inputs

from . import harness

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FC1  # a bf16 NaN pattern no normalised row produces


def _probe(x, gain, offset, eps, spin_limit, stall_row):
    y = torch.full(x.shape, SENTINEL, dtype=torch.int16, device=x.device).view(torch.bfloat16)
    H = x.shape[-1]
    _lib.muse_rms_norm_stall_probe(x.data_ptr(), y.data_ptr(), _lib.MUSE_DTYPE_BF16, x.shape[0], H, H, H,
                                   gain.data_ptr(), offset, eps, spin_limit, stall_row,
                                   torch.cuda.current_stream().cuda_stream)
    return y


def _unwritten_rows(y):
    bits = y.view(torch.int16).cpu().numpy().view(np.uint16)
    return np.flatnonzero((bits == SENTINEL).all(axis=1)), bits


@pytest.mark.parametrize("T,stall", [(1, 0), (8192, 5 * 592 + 17)], ids=["one_row", "mid_ring"])
def test_wait_gives_up_and_context_recovers(cuda_ok, T, stall):
    from gate_cores_b200 import cores

    assert _lib.muse_device_error(clear=True) == 0
    wl = inputs.Workload("stall_h4096", hidden=4096, hq=32, hkv=8, head_dim=128, rope_base=5e5,
                         batch=1, seqlen=T)
    ci = harness.make(wl, "rms_norm", "zc_gain")
    x, g = ci.tensors["x"].cuda(), ci.tensors["gain"].cuda()
    off, eps = ci.scalars["gain_offset"], ci.scalars["eps"]

    y = _probe(x, g, off, eps, spin_limit=1 << 10, stall_row=stall)
    torch.cuda.synchronize()  # the kernel ended: no wait is left spinning
    flags = _lib.muse_device_error()
    assert flags & 1, flags

    # the unwritten rows are the stalled CTA's rows from stall_row on: stall_row,
    # stall_row + grid, ... (rows are dealt round-robin)
    bad, _ = _unwritten_rows(y)
    assert bad.size >= 1 and bad[0] == stall, bad[:4]
    if bad.size > 1:
        step = int(bad[1] - bad[0])
        assert step > 0 and np.array_equal(bad, np.arange(stall, T, step)), bad[:8]

    # every written row matches the oracle; then the ordinary call is exact
    good = np.setdiff1d(np.arange(T), bad)
    if good.size:
        ref = harness.run_oracle(wl, "rms_norm", ci, good)[0]
        from .parity import check
        check(harness.to_host(y, good), ref, "probe written rows")
    y2 = cores.rms_norm(x, g, off, eps)
    torch.cuda.synchronize()
    harness.compare_full(wl, "rms_norm", ci, [y2], "after probe")

    # the word keeps the timeout until cleared
    assert _lib.muse_device_error(clear=True) & 1
    assert _lib.muse_device_error() == 0


def test_probe_rejects_bad_arguments(cuda_ok):
    x = torch.zeros(4, 4096, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(4096, device="cuda")
    for limit, row in ((0, 0), (1 << 25, 0), (16, 4), (16, -1)):
        with pytest.raises(_lib.MuseError) as e:
            _probe(x, g, 1.0, 1e-6, limit, row)
        assert e.value.status == _lib.MUSE_ERR_INVALID_ARGUMENT
    wide = torch.zeros(4, 16384, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.MuseError) as e:
        _probe(wide, torch.zeros(16384, device="cuda"), 1.0, 1e-6, 16, 0)
    assert e.value.status == _lib.MUSE_ERR_UNSUPPORTED
    assert _lib.muse_device_error() == 0
