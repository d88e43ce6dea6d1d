"""Run one core on the GPU (through the C ABI) and the oracle on the same
seeded host inputs; shared by the GPU parity tests, the smoke check and the
benchmark's parity spot check."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from gate_cores_b200 import cores, inputs
from gate_cores_b200.inputs import to_numpy

# Variants exercised per core: name -> keyword overrides.
VARIANTS = {
    "rms_norm": {
        "zc_gain": dict(zero_centered=True),
        "plain_gain": dict(zero_centered=False),
        "no_gain": dict(no_gain=True),
        "f32_io": dict(act_dtype=torch.float32),
    },
    "input_scale_norm": {
        "plain_gain": dict(zero_centered=False),
        "zc_gain": dict(zero_centered=True),
        "f32_io": dict(act_dtype=torch.float32, zero_centered=False),
    },
    "qk_norm_rope": {
        "upcast": dict(),
        "v2": dict(upcast_rope=False),
        "qscale": dict(query_scale=float(np.float32(128 ** -0.5))),
        "v2_qscale": dict(upcast_rope=False, query_scale=float(np.float32(128 ** -0.5))),
        "no_rope": dict(use_rope=False),
        "explicit_pos": dict(explicit_positions=True),
        "f32": dict(act_dtype=torch.float32),
    },
    "output_norm_gate": {
        "per_head": dict(),
        "per_token": dict(per_token=True),
        "f32": dict(act_dtype=torch.float32),
    },
    "norm_residual": {
        "gain_after": dict(),
        "gain_before": dict(input_scale=True),
        "no_gain": dict(no_gain=True),
        "f32_branch": dict(act_dtype=torch.float32),
    },
    "residual_blend": {
        "bf16_branch": dict(),
        "f32_branch": dict(act_dtype=torch.float32),
    },
    "residual": {
        "bf16_branch": dict(),
        "f32_branch": dict(act_dtype=torch.float32),
        "sharp_gate": dict(temperature=0.05, eps=0.01),
    },
}
# _residual_core forms (not among the five cores of the benchmark step)
RESIDUAL_CORES = ("residual_blend", "residual")

DEFAULT_VARIANT = {"rms_norm": "zc_gain", "input_scale_norm": "plain_gain",
                   "qk_norm_rope": "upcast", "output_norm_gate": "per_head",
                   "norm_residual": "gain_after", "residual_blend": "bf16_branch",
                   "residual": "bf16_branch"}


def make(wl, core, variant, seed=0):
    v = dict(VARIANTS[core][variant])
    ci = inputs.make_inputs(wl, core, seed=seed, act_dtype=v.pop("act_dtype", torch.bfloat16),
                            zero_centered=v.pop("zero_centered", True))
    if v.pop("no_gain", False):
        ci.tensors["gain"] = None
        ci.scalars["gain_offset"] = 0.0
    if core == "qk_norm_rope":
        wlo = inputs.WORKLOADS[wl] if isinstance(wl, str) else wl
        if v.pop("explicit_positions", False) and ci.tensors["positions"] is None:
            ci.tensors["positions"] = torch.from_numpy(all_positions(wlo, ci))
    ci.scalars.update(v)
    return ci


def all_positions(wl, ci) -> np.ndarray:
    """Every token's position: explicit ones, else the layout rule (oracle)."""
    if ci.tensors.get("positions") is not None:
        return ci.tensors["positions"].numpy().astype(np.int32)
    if ci.scalars["layout"] == "thd":
        cu = ci.tensors["cu_seqlens"].numpy()
        return oracle.positions(1, cu_seqlens=cu, total_tokens=int(cu[-1]))
    return oracle.positions(0, batch=ci.scalars["batch"], seqlen=ci.scalars["seqlen"])


def _d(t):
    return None if t is None else t.cuda()


def run_gpu(wl, core, ci, stream=None):
    """Upload, run the core through the C ABI, return device outputs."""
    t, s = ci.tensors, ci.scalars
    if core == "rms_norm":
        return (cores.rms_norm(_d(t["x"]), _d(t["gain"]), s["gain_offset"], s["eps"], stream=stream),)
    if core == "input_scale_norm":
        return (cores.input_scale_norm(_d(t["x"]), _d(t["gain"]), s["gain_offset"], s["eps"],
                                       stream=stream),)
    if core == "qk_norm_rope":
        q, k = _d(t["q"]), _d(t["k"])
        if s["layout"] == "bshd":
            B, S = s["batch"], s["seqlen"]
            q = q.view(B, S, *q.shape[1:])
            k = k.view(B, S, *k.shape[1:])
        qo, ko = cores.qk_norm_rope(
            q, k, positions=_d(t["positions"]),
            cu_seqlens=_d(t["cu_seqlens"]) if s["layout"] == "thd" else None, eps=s["eps"],
            query_scale=s.get("query_scale", 1.0), use_rope=s.get("use_rope", True),
            upcast_rope=s.get("upcast_rope", True), rope_base=s["rope_base"], stream=stream)
        return qo.reshape(-1, *qo.shape[-2:]), ko.reshape(-1, *ko.shape[-2:])
    if core == "output_norm_gate":
        o = _d(t["o"])
        ng = o.shape[-2] * o.shape[-1] if s.get("per_token") else None
        return (cores.output_norm_gate(o, _d(t["g"]), ng, s["eps"], stream=stream),)
    if core == "norm_residual":
        return (cores.norm_residual(_d(t["stream"]), _d(t["branch"]), _d(t["theta"]), _d(t["gain"]),
                                    s["gain_offset"], s.get("input_scale", False), s["norm_eps"],
                                    stream=stream),)
    if core == "residual_blend":
        return (cores.residual_blend(_d(t["stream"]), _d(t["branch"]), _d(t["theta"]), stream=stream),)
    if core == "residual":
        return (cores.residual(_d(t["stream"]), _d(t["branch"]), _d(t["gate"]), s["temperature"], s["eps"],
                               stream=stream),)
    raise ValueError(core)


def run_oracle(wl, core, ci, rows=None):
    """Oracle outputs for the selected rows (tokens); all rows when None.
    Returns a list of (out, lo, hi, mag) tuples matching run_gpu's outputs."""
    t, s = ci.tensors, ci.scalars
    sel = (lambda a: a) if rows is None else (lambda a: a[rows])
    np_ = lambda x: None if x is None else to_numpy(x)
    if core in ("rms_norm", "input_scale_norm"):
        fn = getattr(oracle, core)
        return [fn(sel(np_(t["x"])), np_(t["gain"]), s["gain_offset"], s["eps"])]
    if core == "qk_norm_rope":
        pos = all_positions(wl, ci)
        rq, rk = oracle.qk_norm_rope(
            sel(np_(t["q"])), sel(np_(t["k"])), sel(pos), s["eps"], s.get("query_scale", 1.0),
            s.get("use_rope", True), s.get("upcast_rope", True), s["rope_base"])
        return [rq, rk]
    if core == "output_norm_gate":
        o = sel(np_(t["o"]))
        ng = o.shape[-2] * o.shape[-1] if s.get("per_token") else None
        return [oracle.output_norm_gate(o, sel(np_(t["g"])), ng, s["eps"])]
    if core == "norm_residual":
        return [oracle.norm_residual(sel(np_(t["stream"])), sel(np_(t["branch"])), np_(t["theta"]),
                                     np_(t["gain"]), s["gain_offset"], s.get("input_scale", False),
                                     s["norm_eps"])]
    if core == "residual_blend":
        return [oracle.residual_blend(sel(np_(t["stream"])), sel(np_(t["branch"])), np_(t["theta"]))]
    if core == "residual":
        return [oracle.residual(sel(np_(t["stream"])), sel(np_(t["branch"])), np_(t["gate"]),
                                s["temperature"], float(np.float32(s["eps"])))]
    raise ValueError(core)


def compare_full(wl, core, ci, outs, what="", chunk_elems=1 << 21, threads=None):
    """Every output element of the GPU against the oracle on the same inputs.

    The oracle runs over consecutive row (token) chunks of about chunk_elems
    output elements on all host threads (its C routines release the
    interpreter lock); each chunk is checked element by element with
    parity.check.  Returns per output the combined statistics (n, ambiguous,
    and max_ulp_vs_oracle_out or max_rel_vs_mag).  Raises AssertionError with
    the first failing chunk."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    from .parity import check

    host = [to_host(o) for o in outs]
    T = host[0].shape[0]
    width = max(int(np.prod(h.shape[1:])) for h in host)
    step = max(1, chunk_elems // max(1, width))
    spans = [(lo, min(T, lo + step)) for lo in range(0, T, step)]

    def one(span):
        lo, hi = span
        refs = run_oracle(wl, core, ci, slice(lo, hi))
        return [check(h[lo:hi], r, f"{what} rows {lo}..{hi - 1}") for h, r in zip(host, refs)]

    n = threads or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=n) as ex:
        parts = list(ex.map(one, spans))
    total = []
    for k in range(len(host)):
        st = [p[k] for p in parts]
        agg = {"n": sum(s["n"] for s in st), "ambiguous": sum(s["ambiguous"] for s in st)}
        if "max_ulp_vs_oracle_out" in st[0]:
            agg["max_ulp_vs_oracle_out"] = max(s["max_ulp_vs_oracle_out"] for s in st)
            agg["exact_frac"] = sum(s["exact_frac"] * s["n"] for s in st) / max(1, agg["n"])
        else:
            agg["max_rel_vs_mag"] = max(s["max_rel_vs_mag"] for s in st)
        total.append(agg)
    return total


def to_host(x: torch.Tensor, rows=None) -> np.ndarray:
    if rows is not None:
        x = x[torch.as_tensor(rows, device=x.device)]
    return to_numpy(x.cpu())


def sample_rows(T: int, n: int = 48, seed: int = 0) -> np.ndarray:
    r = np.random.default_rng(seed)
    base = {0, 1, T - 1, T - 2, T // 2}
    extra = r.choice(T, size=min(n, T), replace=False)
    return np.array(sorted({int(i) for i in base | set(extra.tolist()) if 0 <= i < T}), dtype=np.int64)


__all__ = ["VARIANTS", "DEFAULT_VARIANT", "make", "run_gpu", "run_oracle", "to_host",
           "sample_rows", "all_positions", "compare_full"]
