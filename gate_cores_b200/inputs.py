"""Seeded synthetic inputs shaped like Muse Spark Open decoder-layer activations.

This module holds random draws, shapes and the workload table only - none of
the normalisation arithmetic.  The same host tensors feed the CUDA library
(uploaded by the caller) and the CPU oracle, so both sides see bit-identical
inputs.

Distributions (per tensor, each from its own seeded ``torch.Generator``):
  * activations x, q, k, o, branch: N(0, 1) drawn in FP32, rounded to the
    activation dtype (bf16 by default);
  * FP32 residual stream: N(0, 1);
  * gains: U(0.5, 1.5) with offset 0, or zero-centered U(-0.5, 0.5) with offset 1;
  * gate logits: N(0, 1) * 2 (standard deviation 2);
  * blend angles theta: U(0, pi/2) in FP32;
  * outliers (large-hidden stress workload): 1% of the channel indices of each
    activation row, chosen by the seed and the same for every row, scaled by
    1000 in FP32 before the rounding to the activation dtype;
  * positions: 0..S-1 per batch row (BSHD), U[0, 32768) (decode), or
    restarting at 0 for each packed document (THD).
"""
from __future__ import annotations

import math
import zlib
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    hidden: int
    hq: int
    hkv: int
    head_dim: int
    rope_base: float
    batch: int = 1
    seqlen: int = 1
    layout: str = "bshd"          # "bshd" or "thd"
    positions: str = "seq"        # "seq": t mod S; "uniform": U[0, pos_max); "restart": per document
    pos_max: int = 0
    num_seqs: int = 0
    seq_len_range: tuple = (0, 0)
    outlier_frac: float = 0.0
    note: str = ""


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_t64_h256", hidden=256, hq=4, hkv=2, head_dim=64, rope_base=1.0e4,
                 batch=1, seqlen=64, note="tiny decoder-layer pass"),
        Workload("prefill_t8192_h4096", hidden=4096, hq=32, hkv=8, head_dim=128, rope_base=5.0e5,
                 batch=2, seqlen=4096, note="prefill layer, B=2 S=4096"),
        Workload("decode_t128_h4096", hidden=4096, hq=32, hkv=8, head_dim=128, rope_base=5.0e5,
                 batch=128, seqlen=1, positions="uniform", pos_max=32768,
                 note="decode step, B=128 S=1"),
        Workload("thd16_h5120", hidden=5120, hq=40, hkv=8, head_dim=128, rope_base=5.0e5,
                 layout="thd", positions="restart", num_seqs=16, seq_len_range=(512, 8192),
                 note="packed THD varlen, 16 documents"),
        Workload("large_t32768_h8192", hidden=8192, hq=64, hkv=8, head_dim=128, rope_base=5.0e5,
                 batch=4, seqlen=8192, outlier_frac=0.01, note="large-hidden stress, 1% outliers"),
    ]
}

# Workload order used by the tests (index 0 is the tiny case, 1 the prefill case).
ORDER = ["tiny_t64_h256", "prefill_t8192_h4096", "decode_t128_h4096", "thd16_h5120",
         "large_t32768_h8192"]


def _gen(seed: int, *tags) -> torch.Generator:
    key = "/".join(str(t) for t in tags).encode()
    g = torch.Generator(device="cpu")
    g.manual_seed((int(seed) * 0x9E3779B1 + zlib.crc32(key)) & 0x7FFFFFFFFFFFFFFF)
    return g


def cu_seqlens(wl: Workload, seed: int = 0) -> torch.Tensor | None:
    """int32 document boundaries [num_seqs + 1] for THD workloads, else None."""
    if wl.layout != "thd":
        return None
    lo, hi = wl.seq_len_range
    lens = torch.randint(lo, hi + 1, (wl.num_seqs,), generator=_gen(seed, wl.name, "seqlens"),
                         dtype=torch.int64)
    cu = torch.zeros(wl.num_seqs + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lens, 0)
    return cu.to(torch.int32)


def num_tokens(wl: Workload, seed: int = 0) -> int:
    if wl.layout == "thd":
        return int(cu_seqlens(wl, seed)[-1])
    return wl.batch * wl.seqlen


def explicit_positions(wl: Workload, seed: int = 0) -> torch.Tensor | None:
    """Caller-supplied positions (int32 [T]) for workloads whose positions are
    not derivable from the layout; None when the layout default applies."""
    if wl.positions == "uniform":
        T = num_tokens(wl, seed)
        return torch.randint(0, wl.pos_max, (T,), generator=_gen(seed, wl.name, "positions"),
                             dtype=torch.int64).to(torch.int32)
    return None


def _outlier_channels(wl: Workload, seed: int, tag: str, width: int) -> torch.Tensor | None:
    if wl.outlier_frac <= 0:
        return None
    n = max(1, int(round(wl.outlier_frac * width)))
    return torch.randperm(width, generator=_gen(seed, wl.name, tag, "outliers"))[:n]


def activation(wl: Workload, seed: int, tag: str, shape, dtype=torch.bfloat16,
               scale: float = 1.0) -> torch.Tensor:
    """N(0, scale^2) activation with the workload's outlier channels, rounded to dtype.
    The last len(shape)-1 dims form one channel row of width prod(shape[1:])."""
    x = torch.randn(shape, generator=_gen(seed, wl.name, tag), dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    width = int(math.prod(shape[1:]))
    idx = _outlier_channels(wl, seed, tag, width)
    if idx is not None:
        flat = x.view(shape[0], width)
        flat[:, idx] *= 1000.0
    return x.to(dtype)


def gain(wl: Workload, seed: int, tag: str, zero_centered: bool) -> tuple[torch.Tensor, float]:
    """(gain [H] f32, offset): U(-0.5, 0.5) with offset 1 or U(0.5, 1.5) with offset 0."""
    u = torch.rand(wl.hidden, generator=_gen(seed, wl.name, tag), dtype=torch.float32)
    if zero_centered:
        return (u - 0.5), 1.0
    return (u + 0.5), 0.0


def theta(wl: Workload, seed: int, tag: str = "theta") -> torch.Tensor:
    u = torch.rand(wl.hidden, generator=_gen(seed, wl.name, tag), dtype=torch.float32)
    return u * float(math.pi / 2)


def residual_gate(wl: Workload, seed: int, tag: str = "residual_gate") -> torch.Tensor:
    """Learned residual gate [H] FP32 for _residual_core: N(0, 1) (the pages
    give no distribution; at temperature 0.3 this spans the sigmoid from its
    lower bound to saturation)."""
    return torch.randn(wl.hidden, generator=_gen(seed, wl.name, tag), dtype=torch.float32)


def expert_groups(wl: Workload, seed: int, num_groups: int, tokens: int | None = None) -> torch.Tensor:
    """Routed-token group boundaries for per-expert norms: int32 [num_groups + 1],
    0 .. tokens, group sizes drawn from a seeded Dirichlet-like split (some
    groups empty)."""
    T = num_tokens(wl, seed) if tokens is None else tokens
    g = _gen(seed, wl.name, "expert_groups", num_groups)
    w = torch.rand(num_groups, generator=g, dtype=torch.float64) ** 3  # skewed loads
    w[torch.randperm(num_groups, generator=g)[: max(1, num_groups // 8)]] = 0.0  # idle experts
    if float(w.sum()) == 0.0:
        w[0] = 1.0
    cuts = torch.floor(torch.cumsum(w, 0) / w.sum() * T).to(torch.int64)
    cuts[-1] = T
    off = torch.zeros(num_groups + 1, dtype=torch.int64)
    off[1:] = cuts
    return off.to(torch.int32)


def expert_gains(wl: Workload, seed: int, num_groups: int, zero_centered: bool) -> tuple[torch.Tensor, float]:
    """(gains [num_groups, H] f32, offset), each row drawn like gain()."""
    rows, off = [], 0.0
    for e in range(num_groups):
        gr, off = gain(wl, seed, f"gain_expert_{e}", zero_centered)
        rows.append(gr)
    return torch.stack(rows), off


@dataclass(frozen=True)
class VisionWorkload:
    """Packed patches of the vision tower: `images` row-major grids of
    grid_h x grid_w patches (448-pixel images at patch 14 give 32 x 32),
    `heads` x `head_dim` per token for Q and K; the RoPE base."""
    name: str
    images: int
    grid_h: int
    grid_w: int
    heads: int
    head_dim: int
    theta: float = 10000.0

    @property
    def tokens(self) -> int:
        return self.images * self.grid_h * self.grid_w


VISION_WORKLOADS = {
    "vision_i16_g32x32_h16x80": VisionWorkload("vision_i16_g32x32_h16x80", 16, 32, 32, 16, 80),
    "vision_i2_g5x7_h3x16": VisionWorkload("vision_i2_g5x7_h3x16", 2, 5, 7, 3, 16, 100.0),
}


def vision_qk(vw: VisionWorkload, seed: int, dtype=torch.bfloat16) -> tuple[torch.Tensor, torch.Tensor]:
    """(q, k) [tokens, heads, head_dim]: N(0, 1) projections rounded to dtype."""
    shape = (vw.tokens, vw.heads, vw.head_dim)
    q = torch.randn(shape, generator=_gen(seed, vw.name, "vision_q"), dtype=torch.float32)
    k = torch.randn(shape, generator=_gen(seed, vw.name, "vision_k"), dtype=torch.float32)
    return q.to(dtype), k.to(dtype)


def vision_angles(vw: VisionWorkload, seed: int) -> torch.Tensor:
    """Arbitrary per-token pair angles U(-100, 100) rad [tokens, head_dim/2] for
    tables not drawn from a grid."""
    g = _gen(seed, vw.name, "vision_angles")
    return torch.rand((vw.tokens, vw.head_dim // 2), generator=g, dtype=torch.float64) * 200.0 - 100.0


def upstream_grad(wl: Workload, seed: int, tag: str, shape, dtype=torch.bfloat16) -> torch.Tensor:
    """Incoming gradient dL/d(output) for the backward calls: N(0, 1) drawn in
    FP32 and rounded to dtype (no outlier channels)."""
    x = torch.randn(shape, generator=_gen(seed, wl.name, "grad", tag), dtype=torch.float32)
    return x.to(dtype)


@dataclass
class CoreInputs:
    """Host tensors for one core on one workload."""
    core: str
    tensors: dict = field(default_factory=dict)
    scalars: dict = field(default_factory=dict)


def make_inputs(wl: Workload | str, core: str, seed: int = 0, act_dtype=torch.bfloat16,
                zero_centered: bool = True) -> CoreInputs:
    """Inputs of one core.  core in {rms_norm, input_scale_norm, qk_norm_rope,
    output_norm_gate, norm_residual, residual_blend, residual}."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    T = num_tokens(wl, seed)
    H = wl.hidden
    ci = CoreInputs(core)
    if core == "rms_norm":
        ci.tensors["x"] = activation(wl, seed, "x_rms", (T, H), act_dtype)
        g, off = gain(wl, seed, "gain_rms", zero_centered)
        ci.tensors["gain"] = g
        ci.scalars.update(gain_offset=off, eps=1e-6)
    elif core == "input_scale_norm":
        ci.tensors["x"] = activation(wl, seed, "x_isn", (T, H), act_dtype)
        g, off = gain(wl, seed, "gain_isn", zero_centered)
        ci.tensors["gain"] = g
        ci.scalars.update(gain_offset=off, eps=1e-6)
    elif core == "qk_norm_rope":
        ci.tensors["q"] = activation(wl, seed, "q", (T, wl.hq, wl.head_dim), act_dtype)
        ci.tensors["k"] = activation(wl, seed, "k", (T, wl.hkv, wl.head_dim), act_dtype)
        ci.tensors["positions"] = explicit_positions(wl, seed)
        ci.tensors["cu_seqlens"] = cu_seqlens(wl, seed)
        ci.scalars.update(eps=1e-6, query_scale=1.0, rope_base=wl.rope_base,
                          layout=wl.layout, batch=wl.batch, seqlen=wl.seqlen)
    elif core == "output_norm_gate":
        ci.tensors["o"] = activation(wl, seed, "o", (T, wl.hq, wl.head_dim), act_dtype)
        ci.tensors["g"] = activation(wl, seed, "g", (T, wl.hq, wl.head_dim), act_dtype, scale=2.0)
        ci.scalars.update(eps=1e-6)
    elif core == "norm_residual":
        ci.tensors["stream"] = activation(wl, seed, "stream", (T, H), torch.float32)
        ci.tensors["branch"] = activation(wl, seed, "branch", (T, H), act_dtype)
        g, off = gain(wl, seed, "gain_res", zero_centered)
        ci.tensors["gain"] = g
        ci.tensors["theta"] = theta(wl, seed)
        ci.scalars.update(gain_offset=off, norm_eps=1e-6)
    elif core in ("residual_blend", "residual"):
        ci.tensors["stream"] = activation(wl, seed, "stream", (T, H), torch.float32)
        ci.tensors["branch"] = activation(wl, seed, "branch", (T, H), act_dtype)
        if core == "residual_blend":
            ci.tensors["theta"] = theta(wl, seed)
        else:
            ci.tensors["gate"] = residual_gate(wl, seed)
            ci.scalars.update(temperature=0.3, eps=1e-3)
    else:
        raise ValueError(f"unknown core {core!r}")
    return ci


CORES = ["rms_norm", "input_scale_norm", "qk_norm_rope", "output_norm_gate", "norm_residual"]


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> NumPy uint16 bit patterns (a view-cast, no arithmetic)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view("uint16")


def to_numpy(t: torch.Tensor):
    """Host tensor -> NumPy array in the oracle's convention (bf16 as uint16 bits)."""
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        return bf16_bits(t)
    return t.contiguous().numpy()
