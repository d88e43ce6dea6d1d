"""GPU parity of the per-expert core 1 (muse_rms_norm_grouped) against the
oracle: routed-token groups of skewed sizes (some empty), bf16 and FP32,
zero-centered and plain gains, tiny, ragged and prefill-size batches."""
import pytest
import torch

import oracle
from gate_cores_b200 import cores, inputs
from gate_cores_b200.inputs import Workload, to_numpy

from .parity import check

pytestmark = pytest.mark.gpu

WLS = [
    (inputs.WORKLOADS["tiny_t64_h256"], 8),
    (Workload("ragged_t37_h264", hidden=264, hq=6, hkv=2, head_dim=80, rope_base=1.0e4, batch=1, seqlen=37), 5),
    (Workload("ragged_b3s5_h40", hidden=40, hq=3, hkv=1, head_dim=16, rope_base=1.0e4, batch=3, seqlen=5), 3),
    (Workload("ragged_t300_h8192", hidden=8192, hq=64, hkv=8, head_dim=128, rope_base=5.0e5, batch=3,
              seqlen=100), 16),
    (inputs.WORKLOADS["prefill_t8192_h4096"], 64),
]


@pytest.mark.parametrize("wl,E", WLS, ids=lambda x: getattr(x, "name", str(x)))
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("zc", [True, False], ids=["zc_gain", "plain_gain"])
def test_rms_norm_grouped(cuda_ok, wl, E, dtype, zc):
    T = inputs.num_tokens(wl)
    if dtype == torch.float32 and wl.hidden // 4 > 1024:
        pytest.skip("rows above the documented 1024 16-byte vectors")
    x = inputs.activation(wl, 0, "x_moe", (T, wl.hidden), dtype)
    gains, off = inputs.expert_gains(wl, 0, E, zc)
    offs = inputs.expert_groups(wl, 0, E)
    y = cores.rms_norm_grouped(x.cuda(), gains.cuda(), offs.cuda(), off, 1e-6)
    torch.cuda.synchronize()
    ref = oracle.rms_norm_grouped(to_numpy(x), gains.numpy(), offs.numpy(), off, 1e-6)
    check(to_numpy(y.cpu()), ref, f"{wl.name}/grouped/E{E}")


def test_rms_norm_grouped_one_group_is_core1(cuda_ok):
    wl = inputs.WORKLOADS["tiny_t64_h256"]
    x = inputs.activation(wl, 0, "x_moe", (64, 256)).cuda()
    g, off = inputs.gain(wl, 0, "gain_one", True)
    y1 = cores.rms_norm_grouped(x, g[None].cuda(), torch.tensor([0, 64], dtype=torch.int32, device="cuda"), off)
    y2 = cores.rms_norm(x, g.cuda(), off)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("T,H,E,single", [(8192, 1024, 8192, True), (8192, 4096, 2000, False),
                                          (1000, 8192, 997, False)],
                         ids=["one_row_per_expert", "t8192_h4096_e2000", "t1000_h8192_e997"])
def test_rms_norm_grouped_many_runs_per_cta(cuda_ok, T, H, E, single):
    # each CTA's contiguous rows cross many expert boundaries, so the two
    # gain slots are refilled again and again within one CTA
    g = torch.Generator().manual_seed(1234 + E)
    x = (torch.randn(T, H, generator=g) * 2.0).to(torch.bfloat16)
    gains = torch.rand(E, H, generator=g) * 0.4 - 0.2
    if single:
        offs = torch.arange(E + 1, dtype=torch.int32)
    else:
        w = torch.rand(E, generator=g, dtype=torch.float64) ** 3
        w[torch.randperm(E, generator=g)[: E // 8]] = 0.0
        cuts = torch.floor(torch.cumsum(w, 0) / w.sum() * T).to(torch.int64)
        cuts[-1] = T
        offs = torch.cat([torch.zeros(1, dtype=torch.int64), cuts]).to(torch.int32)
    y = cores.rms_norm_grouped(x.cuda(), gains.cuda(), offs.cuda(), 1.0, 1e-6)
    torch.cuda.synchronize()
    ref = oracle.rms_norm_grouped(to_numpy(x), gains.numpy(), offs.numpy(), 1.0, 1e-6)
    check(to_numpy(y.cpu()), ref, f"grouped/T{T}/H{H}/E{E}")
    from gate_cores_b200 import _lib
    assert _lib.muse_device_error() == 0
