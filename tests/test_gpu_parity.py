"""GPU parity: every core, every variant, through the C ABI, against the oracle.

Every comparison covers the whole output, element by element: the oracle runs
over row chunks on all host threads (harness.compare_full).

  * Small workloads: the tiny decoder-layer pass and ragged shapes that leave
    idle lanes, idle threads and odd tails; plus a ring-wrap case with many
    times more rows than the row kernels' grid, so every CTA reuses each stage
    of its ring several times (stage reuse, phase parity, round-robin rows).
  * Full-size workloads (prefill, decode, packed THD, large-hidden with
    outliers) in the launch configuration the benchmark times: the default
    variant of each core and the other precision / layout modes, every token.
"""
import pytest
import torch

from gate_cores_b200 import inputs
from gate_cores_b200.inputs import Workload

from . import harness

pytestmark = pytest.mark.gpu

RAGGED = [
    Workload("ragged_t37_h264", hidden=264, hq=6, hkv=2, head_dim=80, rope_base=1.0e4,
             batch=1, seqlen=37),
    Workload("ragged_b3s5_h40", hidden=40, hq=3, hkv=1, head_dim=16, rope_base=1.0e4,
             batch=3, seqlen=5),
    Workload("ragged_thd_h512", hidden=512, hq=8, hkv=4, head_dim=64, rope_base=5.0e5,
             layout="thd", positions="restart", num_seqs=7, seq_len_range=(0, 40)),
    Workload("ragged_t1_h4096", hidden=4096, hq=32, hkv=8, head_dim=128, rope_base=5.0e5,
             batch=1, seqlen=1),
    Workload("ragged_t300_h8192", hidden=8192, hq=64, hkv=8, head_dim=256, rope_base=5.0e5,
             batch=3, seqlen=100, outlier_frac=0.01),
]
# 65536 rows of 256 elements: the row kernels' grid (resident CTAs x SMs) is
# a few thousand CTAs, so each CTA streams 14-21 rows through a 3-stage ring.
WRAP = Workload("wrap_t65536_h256", hidden=256, hq=2, hkv=1, head_dim=128, rope_base=1.0e4,
                batch=16, seqlen=4096)

SMALL = [inputs.WORKLOADS["tiny_t64_h256"]] + RAGGED + [WRAP]
CASES = [(core, var) for core in inputs.CORES for var in harness.VARIANTS[core]]


def _compare(wl, core, ci, tag=""):
    outs = harness.run_gpu(wl, core, ci)
    torch.cuda.synchronize()
    return harness.compare_full(wl, core, ci, outs, f"{wl.name}/{core}/{tag}")


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("core,variant", CASES, ids=lambda x: str(x))
def test_small_full_outputs(cuda_ok, wl, core, variant):
    if core == "qk_norm_rope" and variant == "f32" and wl.head_dim // 4 > 32:
        pytest.skip("f32 heads above 512 bytes are outside the documented limit")
    ci = harness.make(wl, core, variant)
    _compare(wl, core, ci, variant)


FULL = ["prefill_t8192_h4096", "decode_t128_h4096", "thd16_h5120", "large_t32768_h8192"]
FULL_CASES = [(c, harness.DEFAULT_VARIANT[c]) for c in inputs.CORES] + [
    ("qk_norm_rope", "v2"), ("norm_residual", "gain_before"), ("output_norm_gate", "per_token"),
    ("rms_norm", "f32_io")]
OTHER_CASES = [c for c in CASES if c not in FULL_CASES]


def _full(name, core, variant):
    wl = inputs.WORKLOADS[name]
    ci = harness.make(name, core, variant)
    for st in _compare(wl, core, ci, variant):
        # the two-candidate rule for in-doubt intermediate casts stays a
        # corner case, not a loophole
        assert st["ambiguous"] <= max(10, 2e-3 * st["n"]), st


@pytest.mark.parametrize("name", FULL)
@pytest.mark.parametrize("core,variant", FULL_CASES, ids=lambda x: str(x))
def test_full_size_all_tokens(cuda_ok, name, core, variant):
    _full(name, core, variant)


@pytest.mark.parametrize("core,variant", OTHER_CASES, ids=lambda x: str(x))
def test_prefill_other_variants_all_tokens(cuda_ok, core, variant):
    _full("prefill_t8192_h4096", core, variant)


@pytest.mark.parametrize("name", ["decode_t128_h4096", "thd16_h5120", "large_t32768_h8192"])
@pytest.mark.parametrize("core,variant", OTHER_CASES, ids=lambda x: str(x))
def test_full_size_other_variants_sampled(cuda_ok, name, core, variant):
    # the remaining variants at the other full sizes, on sampled tokens
    from .parity import check

    wl = inputs.WORKLOADS[name]
    ci = harness.make(name, core, variant)
    rows = harness.sample_rows(inputs.num_tokens(wl), 40, seed=hash(core) & 0xFFFF)
    outs = harness.run_gpu(wl, core, ci)
    torch.cuda.synchronize()
    for o, r in zip(outs, harness.run_oracle(wl, core, ci, rows)):
        check(harness.to_host(o, rows), r, f"{name}/{core}/{variant}")


def test_positions_explicit_equal_derived_bitwise(cuda_ok):
    for name in ("prefill_t8192_h4096", "thd16_h5120"):
        wl = inputs.WORKLOADS[name]
        a = harness.run_gpu(wl, "qk_norm_rope", harness.make(name, "qk_norm_rope", "upcast"))
        b = harness.run_gpu(wl, "qk_norm_rope", harness.make(name, "qk_norm_rope", "explicit_pos"))
        for x, y in zip(a, b):
            assert torch.equal(x.view(torch.int16), y.view(torch.int16))


def test_no_device_error_after_parity_runs(cuda_ok):
    # every bounded mbarrier wait in the row kernels completed
    from gate_cores_b200 import _lib
    assert _lib.muse_device_error() == 0


def test_wrap_case_has_rows_beyond_the_grid():
    # host-side check of the premise of the ring-wrap case: more than three
    # rows per CTA even at the largest resident grid on a 148-SM part (32
    # CTAs per SM for 64-thread CTAs)
    assert inputs.num_tokens(WRAP) >= 3 * 32 * 148 * 4
