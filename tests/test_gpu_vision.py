"""GPU parity of the vision 2-D RoPE (muse_vision_rope, muse_vision_rope_frequencies)
against the oracle.

Tables come from the oracle's grid generator (one table per image, packed in
patch order) or from arbitrary angles; the rotation is checked element by
element (bf16 within the 1-ulp rule, FP32 within 2e-6 of the terms'
magnitudes), the GPU's own tables against the oracle's within 2e-6.
"""
import numpy as np
import pytest
import torch

import oracle
from gate_cores_b200 import _lib, cores, inputs
from gate_cores_b200.inputs import VISION_WORKLOADS, VisionWorkload, to_numpy

from .parity import check

pytestmark = pytest.mark.gpu

WLS = [VISION_WORKLOADS["vision_i2_g5x7_h3x16"],
       VisionWorkload("vision_i3_g9x4_h12x72", 3, 9, 4, 12, 72),
       VisionWorkload("vision_i1_g1x1_h1x8", 1, 1, 1, 1, 8),
       VisionWorkload("vision_i4_g16x16_h8x128", 4, 16, 16, 8, 128, 5e5),
       VISION_WORKLOADS["vision_i16_g32x32_h16x80"]]


def oracle_table(vw: VisionWorkload) -> np.ndarray:
    t = oracle.vision_rope_frequencies(vw.head_dim, vw.grid_h, vw.grid_w, vw.theta)
    return np.concatenate([t] * vw.images, axis=0)


def angle_table(vw: VisionWorkload) -> np.ndarray:
    a = inputs.vision_angles(vw, 0).numpy()
    return np.stack([np.cos(a), np.sin(a)], -1).astype(np.float32)


@pytest.mark.parametrize("vw", WLS, ids=lambda w: w.name)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
@pytest.mark.parametrize("table", ["grid", "angles"])
def test_vision_rope(cuda_ok, vw, dtype, table):
    if dtype == torch.bfloat16 and vw.head_dim % 8:
        pytest.skip("bf16 heads must be 16-byte multiples")
    q, k = inputs.vision_qk(vw, 0, dtype)
    f = oracle_table(vw) if table == "grid" else angle_table(vw)
    qo, ko = cores.vision_rope(q.cuda(), k.cuda(), torch.from_numpy(f).cuda())
    torch.cuda.synchronize()
    rq, rk = oracle.vision_rope(to_numpy(q), to_numpy(k), f)
    check(to_numpy(qo.cpu()), rq, f"{vw.name}/{table}/q")
    check(to_numpy(ko.cpu()), rk, f"{vw.name}/{table}/k")


@pytest.mark.parametrize("vw", WLS, ids=lambda w: w.name)
def test_vision_rope_frequencies(cuda_ok, vw):
    g = cores.vision_rope_frequencies(vw.head_dim, vw.grid_h, vw.grid_w, vw.theta)
    torch.cuda.synchronize()
    ref = oracle.vision_rope_frequencies(vw.head_dim, vw.grid_h, vw.grid_w, vw.theta).astype(np.float64)
    err = np.abs(g.cpu().numpy().astype(np.float64) - ref)
    assert err.max() <= 2e-6, float(err.max())


def test_vision_rope_in_place_and_strided(cuda_ok):
    # Q and K as views into one fused [T, (hq + hk) * D] projection, rotated in place
    vw = VisionWorkload("vision_i2_g6x6_h4x64", 2, 6, 6, 4, 64)
    q, k = inputs.vision_qk(vw, 1)
    fused = torch.cat([q.reshape(vw.tokens, -1), k.reshape(vw.tokens, -1)], 1).cuda()
    qv = fused[:, : 4 * 64].view(vw.tokens, 4, 64)
    kv = fused[:, 4 * 64:].view(vw.tokens, 4, 64)
    f = oracle_table(vw)
    ref_q, ref_k = cores.vision_rope(q.cuda(), k.cuda(), torch.from_numpy(f).cuda())
    cores.vision_rope(qv, kv, torch.from_numpy(f).cuda(), q_out=qv, k_out=kv)
    torch.cuda.synchronize()
    assert torch.equal(qv.reshape(-1).view(torch.int16), ref_q.reshape(-1).view(torch.int16))
    assert torch.equal(kv.reshape(-1).view(torch.int16), ref_k.reshape(-1).view(torch.int16))


def test_vision_rope_rejects(cuda_ok):
    f = torch.zeros(4, 6, 2, device="cuda")
    q = torch.zeros(4, 2, 12, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.MuseError) as e:  # 24-byte heads: not a 16-byte multiple
        cores.vision_rope(q, q.clone(), f)
    assert e.value.status == _lib.MUSE_ERR_UNSUPPORTED
    q = torch.zeros(4, 2, 16, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(4, 8, 2, device="cuda")
    buf = torch.zeros(4 * 32 + 8, dtype=torch.bfloat16, device="cuda")
    out = buf[8:].view(4, 2, 16)  # overlaps q = buf[:128] partially
    with pytest.raises(_lib.MuseError) as e:
        cores.vision_rope(buf[:128].view(4, 2, 16), q, f, q_out=out)
    assert e.value.status == _lib.MUSE_ERR_INVALID_ARGUMENT
    empty = torch.zeros(0, 2, 16, dtype=torch.bfloat16, device="cuda")
    cores.vision_rope(empty, empty, torch.zeros(0, 8, 2, device="cuda"))
    assert _lib.muse_device_error() == 0
