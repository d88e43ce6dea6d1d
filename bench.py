#!/usr/bin/env python
"""Benchmark of the five fused normalisation cores on B200.

One step = one pass of the whole hot path over one batch of synthetic
decoder-layer activations: rms_norm, input_scale_norm, qk_norm_rope,
output_norm_gate and norm_residual, each a single CUDA kernel launched through
the C ABI.  Default workload: prefill, B=2 x S=4096 tokens, H=4096, 32 Q / 8 KV
heads of 128.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (weak scaling, no collective on the data path): each rank runs the
same step on its own batch; launch with torch.distributed.run.  Prints one
JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gate_cores_b200 import cores, inputs  # noqa: E402
from gate_cores_b200.inputs import WORKLOADS, num_tokens  # noqa: E402

CORE_ORDER = inputs.CORES
METRIC = "tokens/s and effective HBM GB/s per fused core vs measured ~8 TB/s peak"
DOMINANT = "norm_residual"  # largest algorithmic byte count of the five
# sources whose change invalidates the committed dram-traffic figure of the dominant kernel
DOMINANT_SOURCES = ("row_tma.cu", "tma_pipe.cuh", "common.cuh", "kernels.h")
KERNEL_NAMES = {c: c + "_kernel" for c in inputs.CORES}
VARIANT = {"rms_norm": "zero-centered gain (offset 1)", "input_scale_norm": "gain U(0.5,1.5)",
           "qk_norm_rope": "RoPE in FP32 (legacy), query_scale 1, BSHD-derived positions",
           "output_norm_gate": "one norm per head", "norm_residual": "gain after the norm"}


def algo_bytes(wl, core: str, tokens: int) -> int:
    """Minimum HBM bytes of one launch: every input read once, every output written once."""
    H, D = wl.hidden, wl.head_dim
    per_tok = {"rms_norm": 4 * H, "input_scale_norm": 4 * H,
               "qk_norm_rope": 4 * (wl.hq + wl.hkv) * D + (4 if wl.positions == "uniform" else 0),
               "output_norm_gate": 6 * wl.hq * D, "norm_residual": 10 * H}[core]
    fixed = {"rms_norm": 4 * H, "input_scale_norm": 4 * H, "qk_norm_rope": 0,
             "output_norm_gate": 0, "norm_residual": 8 * H}[core]
    return per_tok * tokens + fixed


def algo_bytes_bwd(wl, core: str, tokens: int) -> int:
    """Minimum HBM bytes of one backward launch (bf16 activations, FP32 stream):
    the forward inputs and the incoming gradient read once, every gradient
    written once; gains / angles and their gradients once per launch."""
    H, D = wl.hidden, wl.head_dim
    per_tok = {"rms_norm": 6 * H, "input_scale_norm": 6 * H,
               "qk_norm_rope": 6 * (wl.hq + wl.hkv) * D + (4 if wl.positions == "uniform" else 0),
               "output_norm_gate": 10 * wl.hq * D, "norm_residual": 16 * H}[core]
    fixed = {"rms_norm": 8 * H, "input_scale_norm": 8 * H, "qk_norm_rope": 0,
             "output_norm_gate": 0, "norm_residual": 16 * H}[core]
    return per_tok * tokens + fixed


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ------------------------------------------------------------------ distributed

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def allreduce_max(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU is under load.

    The GPU is named by its UUID (the process may see it under another index
    than nvidia-smi does); start() returns once the first sample has arrived,
    so a short timed region is still covered."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, period_ms: int = 20):
        self.proc = None
        self.error = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        gid = str(index)
        try:
            u = str(torch.cuda.get_device_properties(index).uuid)
            gid = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:  # noqa: BLE001 - fall back to the index
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gid}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 f"-lms={period_ms}"], stdout=self.f, stderr=subprocess.PIPE)
        except (FileNotFoundError, OSError) as e:
            self.proc, self.error = None, str(e)
            return
        t0 = time.time()
        while time.time() - t0 < 10.0 and self.proc.poll() is None:
            if os.path.getsize(self.f.name) > 0:
                break
            time.sleep(0.05)
        if self.proc.poll() is not None:
            self.error = (self.proc.stderr.read() or b"").decode(errors="replace").strip()[:200]

    def stop(self):
        if self.proc is None:
            return {"error": self.error or "nvidia-smi not available", "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r for r in csv.reader(io.StringIO(self.f.read())) if len(r) >= 9]
        os.unlink(self.f.name)
        if not rows:
            return {"error": self.error or "no samples", "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ our arm

class Step:
    """Device-resident inputs and outputs of the five cores for one batch."""

    def __init__(self, wl, seed: int):
        self.wl = wl
        self.T = num_tokens(wl, seed)
        self.host = {c: inputs.make_inputs(wl, c, seed=seed, zero_centered=(c != "input_scale_norm"))
                     for c in CORE_ORDER}
        self.dev = {c: {k: (None if v is None else v.cuda()) for k, v in ci.tensors.items()}
                    for c, ci in self.host.items()}
        d = self.dev
        self.out = {
            "rms_norm": torch.empty_like(d["rms_norm"]["x"]),
            "input_scale_norm": torch.empty_like(d["input_scale_norm"]["x"]),
            "qk_q": torch.empty_like(d["qk_norm_rope"]["q"]),
            "qk_k": torch.empty_like(d["qk_norm_rope"]["k"]),
            "output_norm_gate": torch.empty_like(d["output_norm_gate"]["o"]),
            "norm_residual": torch.empty_like(d["norm_residual"]["stream"]),
        }
        B, S = wl.batch, wl.seqlen
        q, k = d["qk_norm_rope"]["q"], d["qk_norm_rope"]["k"]
        self.thd = wl.layout == "thd"
        if not self.thd:
            self.q4 = q.view(B, S, wl.hq, wl.head_dim)
            self.k4 = k.view(B, S, wl.hkv, wl.head_dim)
            self.qo4 = self.out["qk_q"].view(B, S, wl.hq, wl.head_dim)
            self.ko4 = self.out["qk_k"].view(B, S, wl.hkv, wl.head_dim)

    def launch(self, core: str):
        d, s, o = self.dev[core], self.host[core].scalars, self.out
        if core == "rms_norm":
            cores.rms_norm(d["x"], d["gain"], s["gain_offset"], s["eps"], out=o["rms_norm"])
        elif core == "input_scale_norm":
            cores.input_scale_norm(d["x"], d["gain"], s["gain_offset"], s["eps"], out=o["input_scale_norm"])
        elif core == "qk_norm_rope":
            if self.thd:
                cores.qk_norm_rope(d["q"], d["k"], d["positions"], d["cu_seqlens"], s["eps"], 1.0, True,
                                   True, s["rope_base"], q_out=o["qk_q"], k_out=o["qk_k"])
            else:
                cores.qk_norm_rope(self.q4, self.k4, d["positions"], None, s["eps"], 1.0, True, True,
                                   s["rope_base"], q_out=self.qo4, k_out=self.ko4)
        elif core == "output_norm_gate":
            cores.output_norm_gate(d["o"], d["g"], None, s["eps"], out=o["output_norm_gate"])
        elif core == "norm_residual":
            cores.norm_residual(d["stream"], d["branch"], d["theta"], d["gain"], s["gain_offset"],
                                False, s["norm_eps"], out=o["norm_residual"])

    def input_tensors(self):
        for c in CORE_ORDER:
            for k, v in self.dev[c].items():
                if v is not None:
                    yield (c, k), v

    def output_tensors(self):
        return list(self.out.values())


class BwdStep:
    """Device-resident inputs, incoming gradients, gradient outputs and the
    parameter-gradient workspace of the five backward calls for one batch;
    launch() calls the C ABI directly on preallocated buffers."""

    def __init__(self, st: "Step", seed: int):
        from gate_cores_b200 import _lib
        self.lib = _lib
        self.wl, self.T, self.st = st.wl, st.T, st
        wl, d = st.wl, st.dev
        g = lambda tag, like: inputs.upstream_grad(wl, seed, tag, tuple(like.shape), like.dtype).cuda()
        self.dy = {
            "rms_norm": g("rms_norm", d["rms_norm"]["x"]),
            "input_scale_norm": g("input_scale_norm", d["input_scale_norm"]["x"]),
            "qk_q": g("qk_q", d["qk_norm_rope"]["q"]),
            "qk_k": g("qk_k", d["qk_norm_rope"]["k"]),
            "output_norm_gate": g("output_norm_gate", d["output_norm_gate"]["o"]),
            "norm_residual": g("norm_residual", d["norm_residual"]["stream"]),
        }
        self.out = {
            "rms_norm": torch.empty_like(d["rms_norm"]["x"]),
            "input_scale_norm": torch.empty_like(d["input_scale_norm"]["x"]),
            "dq": torch.empty_like(d["qk_norm_rope"]["q"]),
            "dk": torch.empty_like(d["qk_norm_rope"]["k"]),
            "do": torch.empty_like(d["output_norm_gate"]["o"]),
            "dg": torch.empty_like(d["output_norm_gate"]["o"]),
            "dstream": torch.empty_like(d["norm_residual"]["stream"]),
            "dbranch": torch.empty_like(d["norm_residual"]["branch"]),
        }
        H = wl.hidden
        self.dparam = {c: torch.empty(H, dtype=torch.float32, device="cuda")
                       for c in ("rms_norm", "input_scale_norm", "gain_res", "theta_res")}
        self.ws_bytes = _lib.muse_norm_backward_workspace_bytes(self.T, H)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
        self.qk_upcast = True  # the Q/K backward's rotation: FP32 (legacy) or v2

    def launch(self, core: str):
        L, wl, T, H = self.lib, self.wl, self.T, self.wl.hidden
        d, sc = self.st.dev[core], self.st.host[core].scalars
        stream = torch.cuda.current_stream().cuda_stream
        bf = L.MUSE_DTYPE_BF16
        if core in ("rms_norm", "input_scale_norm"):
            fn = L.muse_rms_norm_backward if core == "rms_norm" else L.muse_input_scale_norm_backward
            fn(d["x"].data_ptr(), self.dy[core].data_ptr(), self.out[core].data_ptr(), bf, T, H, H, H, H,
               d["gain"].data_ptr(), sc["gain_offset"], sc["eps"], self.dparam[core].data_ptr(),
               self.ws.data_ptr(), self.ws_bytes, stream)
        elif core == "qk_norm_rope":
            qw, kw = wl.hq * wl.head_dim, wl.hkv * wl.head_dim
            pos = d["positions"]
            if self.st.thd:
                cu = d["cu_seqlens"]
                layout, bsz, sl, cup, nseq = L.MUSE_LAYOUT_THD, 0, 0, cu.data_ptr(), cu.numel() - 1
            else:
                layout, bsz, sl, cup, nseq = L.MUSE_LAYOUT_BSHD, wl.batch, wl.seqlen, None, 0
            L.muse_qk_norm_rope_backward(
                d["q"].data_ptr(), d["k"].data_ptr(), self.dy["qk_q"].data_ptr(), self.dy["qk_k"].data_ptr(),
                self.out["dq"].data_ptr(), self.out["dk"].data_ptr(), bf, layout, bsz, sl, cup, nseq, T,
                None if pos is None else pos.data_ptr(), wl.hq, wl.hkv,
                wl.head_dim, qw, kw, qw, kw, qw, kw, sc["eps"], 1.0, True, self.qk_upcast, sc["rope_base"],
                stream)
        elif core == "output_norm_gate":
            L.muse_output_norm_gate_backward(
                d["o"].data_ptr(), d["g"].data_ptr(), self.dy[core].data_ptr(), self.out["do"].data_ptr(),
                self.out["dg"].data_ptr(), bf, T, wl.hq, wl.head_dim, wl.head_dim, sc["eps"], stream)
        else:
            L.muse_norm_residual_backward(
                d["stream"].data_ptr(), d["branch"].data_ptr(), self.dy[core].data_ptr(),
                self.out["dstream"].data_ptr(), self.out["dbranch"].data_ptr(), bf, T, H,
                d["gain"].data_ptr(), sc["gain_offset"], d["theta"].data_ptr(), False, sc["norm_eps"],
                self.dparam["gain_res"].data_ptr(), self.dparam["theta_res"].data_ptr(),
                self.ws.data_ptr(), self.ws_bytes, stream)


def fused_calls(st: "Step"):
    """(fused, unfused): core 5 with the next sublayer's pre-norm in one call,
    and core 5 then core 1 on its output, on the batch's core 5 inputs."""
    wl = st.wl
    d, sc = st.dev["norm_residual"], st.host["norm_residual"].scalars
    g2, off2 = inputs.gain(wl, 0, "gain_next", True)
    g2 = g2.cuda()
    h = torch.empty_like(d["stream"])
    y = torch.empty_like(d["stream"])
    res = (d["stream"], d["branch"], d["theta"], d["gain"], sc["gain_offset"], False, sc["norm_eps"])

    def fused():
        cores.norm_residual_rms_norm(*res, next_gain=g2, next_gain_offset=off2, next_eps=1e-6,
                                     out=h, y=y)

    def unfused():
        cores.norm_residual(*res, out=h)
        cores.rms_norm(h, g2, off2, 1e-6, out=y)

    return fused, unfused


def blend_fused_calls(st: "Step", seed: int = 0):
    """(fused, unfused): _residual_core (angle form) with the next sublayer's
    pre-norm in one call, and the blend then core 1 on its output."""
    wl = st.wl
    ci = inputs.make_inputs(wl, "residual_blend", seed=seed)
    h_in, b, th = (ci.tensors[k].cuda() for k in ("stream", "branch", "theta"))
    g2, off2 = inputs.gain(wl, 0, "gain_next", True)
    g2 = g2.cuda()
    h, y = torch.empty_like(h_in), torch.empty_like(h_in)

    def fused():
        cores.residual_blend_rms_norm(h_in, b, th, next_gain=g2, next_gain_offset=off2, next_eps=1e-6,
                                      out=h, y=y)

    def unfused():
        cores.residual_blend(h_in, b, th, out=h)
        cores.rms_norm(h, g2, off2, 1e-6, out=y)

    return fused, unfused


def fused_vs_unfused(st: "Step", peak: float, flush: torch.Tensor, warmup: int = 10, reps: int = 50,
                     calls=None, note=None):
    """Core 5 fused with the next sublayer's pre-norm (FP32 y) against core 5
    followed by core 1 on the new FP32 stream: median of `reps`, each call
    pair timed with events around both launches, L2 read-flushed before each."""
    T, H = st.T, st.wl.hidden
    fused, unfused = calls if calls is not None else fused_calls(st)
    stream = torch.cuda.current_stream()
    out = {}
    for name, fn in (("fused", fused), ("unfused", unfused)):
        torch.cuda.synchronize()
        torch.cuda._sleep(20_000_000)
        ev = []
        for i in range(warmup + reps):
            flush.amax()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            if i >= warmup:
                ev.append((e0, e1))
        torch.cuda.synchronize()
        out[name + "_us"] = round(statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3, 3)
    nb = 14 * H * T + 12 * H  # branch + stream in, stream + FP32 y out; gains and angles once
    out["fused_gbs"] = round(nb / (out["fused_us"] * 1e-6) / 1e9, 1)
    out["fused_frac"] = round(out["fused_gbs"] / peak, 4)
    out["algo_bytes_fused"] = nb
    out["algo_bytes_unfused"] = 18 * H * T + 16 * H
    out["note"] = note or ("core 5 + the next sublayer's RMS pre-norm of the new FP32 stream (FP32 y) in one "
                           "pass, against muse_norm_residual then muse_rms_norm on its output")
    return out


def grouped_call(st: "Step", experts: int = 64):
    """Per-expert core 1 on the batch's core 1 activations routed to `experts`
    groups of skewed sizes."""
    wl, T = st.wl, st.T
    x = st.dev["rms_norm"]["x"]
    gains, off = inputs.expert_gains(wl, 0, experts, True)
    gains = gains.cuda()
    offs = inputs.expert_groups(wl, 0, experts, T).cuda()
    y = torch.empty_like(x)

    def call():
        cores.rms_norm_grouped(x, gains, offs, off, 1e-6, out=y)

    return call


def vision_call(name: str = "vision_i16_g32x32_h16x80"):
    """Vision 2-D RoPE on a packed batch of patch grids: the table built by
    muse_vision_rope_frequencies (one launch per image, written in patch
    order), then a callable rotating Q and K into fresh outputs."""
    vw = inputs.VISION_WORKLOADS[name]
    q, k = (t.cuda() for t in inputs.vision_qk(vw, 0))
    per = vw.grid_h * vw.grid_w
    table = torch.empty((vw.tokens, vw.head_dim // 2, 2), dtype=torch.float32, device="cuda")
    for i in range(vw.images):
        cores.vision_rope_frequencies(vw.head_dim, vw.grid_h, vw.grid_w, vw.theta, out=table[i * per:(i + 1) * per])
    qo, ko = torch.empty_like(q), torch.empty_like(k)

    def call():
        cores.vision_rope(q, k, table, q_out=qo, k_out=ko)

    return vw, call


def vision_rope_timing(peak: float, flush: torch.Tensor, warmup: int = 10, reps: int = 50):
    """The vision rotation alone: median of `reps` launches, L2 read-flushed before each."""
    vw, call = vision_call()
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    torch.cuda._sleep(20_000_000)
    ev = []
    for i in range(warmup + reps):
        flush.amax()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        if i >= warmup:
            ev.append((e0, e1))
    torch.cuda.synchronize()
    us = statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3
    nb = vw.tokens * (2 * 2 * 2 * vw.heads * vw.head_dim + 4 * vw.head_dim)  # Q, K in and out (bf16); table
    return {"workload": vw.name, "tokens": vw.tokens, "us": round(us, 3),
            "tokens_per_s": round(vw.tokens / (us * 1e-6), 1), "gbs": round(nb / (us * 1e-6) / 1e9, 1),
            "frac": round(nb / (us * 1e-6) / 1e9 / peak, 4), "algo_bytes": nb,
            "note": "muse_vision_rope: Q and K (16 heads x 80) of 16 images of 32x32 patches, bf16"}


def grouped_norm(st: "Step", peak: float, flush: torch.Tensor, experts: int = 64, warmup: int = 10,
                 reps: int = 50):
    """Per-expert core 1 (MoE pre/post expert norm) on the batch's activations
    routed to `experts` groups of skewed sizes: median of `reps` launches,
    L2 read-flushed before each."""
    T, H = st.T, st.wl.hidden
    call = grouped_call(st, experts)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    torch.cuda._sleep(20_000_000)
    ev = []
    for i in range(warmup + reps):
        flush.amax()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        if i >= warmup:
            ev.append((e0, e1))
    torch.cuda.synchronize()
    us = statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3
    nb = 4 * H * T + 4 * H * experts + 4 * (experts + 1)
    # launched back to back (steady state), as per_core_steady
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    torch.cuda._sleep(20_000_000)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    us_st = e0.elapsed_time(e1) * 1e3 / reps
    return {"us": round(us, 3), "gbs": round(nb / (us * 1e-6) / 1e9, 1),
            "frac": round(nb / (us * 1e-6) / 1e9 / peak, 4),
            "steady_us": round(us_st, 3), "steady_frac": round(nb / (us_st * 1e-6) / 1e9 / peak, 4),
            "experts": experts, "algo_bytes": nb,
            "note": "muse_rms_norm_grouped: rows grouped by expert, each group with its own FP32 gain row; "
                    "us alone with a read-flushed L2, steady_us launched back to back"}


def per_core_isolated(st, peak: float, flush: torch.Tensor | None, warmup: int = 10,
                      reps: int = 50, nbytes=None, which=CORE_ORDER):
    """Each core launched alone: `warmup` launches, then the median of `reps`
    launches timed with CUDA events around each one on the launching stream.
    With `flush`, a read pass over that buffer (> L2, reading leaves no dirty
    lines) precedes every launch, so each launch starts from a clean, cold L2;
    without it, L2 stays warm (the decode latency figures)."""
    stream = torch.cuda.current_stream()
    out = {}
    for c in which:
        ev = []
        torch.cuda.synchronize()
        # hold the GPU for a few ms so that the host queues every launch ahead
        # of the device: the events then time the kernels, not the host
        torch.cuda._sleep(20_000_000)
        for i in range(warmup + reps):
            if flush is not None:
                flush.amax()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            st.launch(c)
            e1.record(stream)
            if i >= warmup:
                ev.append((e0, e1))
        torch.cuda.synchronize()
        us = statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3
        nb = (nbytes or algo_bytes)(st.wl, c, st.T)
        gbs = nb / (us * 1e-6) / 1e9
        out[c] = {"us": round(us, 3), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}
    return out


def per_core_steady(st, peak: float, reps: int, warmup: int = 3, nbytes=None, which=CORE_ORDER):
    """Each core launched alone `reps` times back to back on the same batch,
    with two CUDA events around the loop on the launching stream and no flush.
    Every launch streams more than the 126 MB L2, so each one starts with its
    predecessor's dirty output lines still to be written back and keeps the
    programmatic-launch overlap with it, as inside the five-core step: a
    steady-state per-core figure that neither credits writes left in L2 nor
    charges the idle gap an event between two kernels adds."""
    stream = torch.cuda.current_stream()
    out = {}
    for c in which:
        for _ in range(warmup):
            st.launch(c)
        torch.cuda.synchronize()
        torch.cuda._sleep(20_000_000)  # the host queues every launch ahead of the device
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            st.launch(c)
        e1.record(stream)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / reps
        nb = (nbytes or algo_bytes)(st.wl, c, st.T)
        gbs = nb / (us * 1e-6) / 1e9
        out[c] = {"us": round(us, 3), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}
    return out


class LaunchFloor:
    """A 16-byte copy through the library's copy entry point: one CTA, launched
    with programmatic dependent launch like every core, doing no real work -
    the floor under the decode-batch latencies."""

    def __init__(self):
        self.src = torch.zeros(16, dtype=torch.uint8, device="cuda")
        self.dst = torch.empty_like(self.src)
        self.wl, self.T = None, 0

    def launch(self, _core=None):
        cores.stream_copy(self.src, self.dst)


def per_config(args, peak: float, rank: int, world: int,
               names=("thd16_h5120", "large_t32768_h8192")):
    """The five cores on the other full-size workloads: per-core steady-state
    figures (per_core_steady) of the forward and of the backward calls, the
    five-core step (K steps back to back, two events), and the oracle on all
    host cores on a bounded sample of the same batch (rank 0, one GPU)."""
    stream = torch.cuda.current_stream()
    reps = max(10, min(args.steps, 50))
    out = {}
    for name in names:
        wl = WORKLOADS[name]
        st = Step(wl, seed=rank)
        steady = per_core_steady(st, peak, reps)
        for _ in range(3):
            for c in CORE_ORDER:
                st.launch(c)
        torch.cuda.synchronize()
        torch.cuda._sleep(20_000_000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            for c in CORE_ORDER:
                st.launch(c)
        e1.record(stream)
        torch.cuda.synchronize()
        el = allreduce_max(e0.elapsed_time(e1) / 1e3, world)
        nb = sum(algo_bytes(wl, c, st.T) for c in CORE_ORDER)
        rec = {"tokens": st.T, "hidden": wl.hidden, "q_heads": wl.hq, "kv_heads": wl.hkv,
               "per_core_steady": steady,
               "step": {"ms": round(el / reps * 1e3, 4), "tokens_per_s": round(world * st.T * reps / el, 1),
                        "gbs": round(nb * reps / el / 1e9, 1), "frac": round(nb * reps / el / 1e9 / peak, 4),
                        "algo_bytes": nb, "steps": reps}}
        bst = BwdStep(st, seed=rank)
        rec["backward_steady"] = per_core_steady(bst, peak, reps, nbytes=algo_bytes_bwd)
        del bst
        if rank == 0 and world == 1 and args.cpu_baseline:
            rec["cpu_oracle_all_cores"] = cpu_baseline_threads(wl, seconds=4.0, host=st.host)
        out[name] = rec
        del st
        torch.cuda.empty_cache()
    return out


class ResidualStep:
    """_residual_core on the batch's shape: the FP32 stream blended with the
    bf16 branch, in the gate form (muse_residual, temperature 0.3, eps 1e-3)
    and the angle form (muse_residual_blend)."""

    def __init__(self, wl, seed: int):
        self.wl = wl
        self.T = num_tokens(wl, seed)
        dev = lambda ci: {k: v.cuda() for k, v in ci.tensors.items()}  # noqa: E731
        self.g = dev(inputs.make_inputs(wl, "residual", seed=seed))
        self.b = dev(inputs.make_inputs(wl, "residual_blend", seed=seed))
        self.out = torch.empty_like(self.g["stream"])
        self.dy = inputs.upstream_grad(wl, seed, "residual", tuple(self.out.shape), torch.float32).cuda()
        self.dstream = torch.empty_like(self.out)
        self.dbranch = torch.empty_like(self.g["branch"])
        self.dparam = torch.empty(wl.hidden, dtype=torch.float32, device="cuda")
        from gate_cores_b200 import _lib
        self.lib = _lib
        self.ws_bytes = _lib.muse_residual_backward_workspace_bytes(self.T, wl.hidden)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")

    def launch(self, core: str):
        L, T, H = self.lib, self.T, self.wl.hidden
        stream = torch.cuda.current_stream().cuda_stream
        if core == "residual":
            cores.residual(self.g["stream"], self.g["branch"], self.g["gate"], 0.3, 1e-3, out=self.out)
        elif core == "residual_blend":
            cores.residual_blend(self.b["stream"], self.b["branch"], self.b["theta"], out=self.out)
        elif core == "residual_bwd":
            L.muse_residual_backward(self.g["stream"].data_ptr(), self.g["branch"].data_ptr(), self.dy.data_ptr(),
                                     self.dstream.data_ptr(), self.dbranch.data_ptr(), L.MUSE_DTYPE_BF16, T, H,
                                     self.g["gate"].data_ptr(), 0.3, 1e-3, self.dparam.data_ptr(),
                                     self.ws.data_ptr(), self.ws_bytes, stream)
        else:
            L.muse_residual_blend_backward(self.b["stream"].data_ptr(), self.b["branch"].data_ptr(),
                                           self.dy.data_ptr(), self.dstream.data_ptr(), self.dbranch.data_ptr(),
                                           L.MUSE_DTYPE_BF16, T, H, self.b["theta"].data_ptr(),
                                           self.dparam.data_ptr(), self.ws.data_ptr(), self.ws_bytes, stream)


def residual_bytes(wl, core: str, tokens: int) -> int:
    """Forward: FP32 stream in and out, bf16 branch in; the gate or the angles
    once.  Backward: the stream, the bf16 branch and dL/dout (FP32) in, the
    stream and branch gradients out; the gate or angles and their gradient once."""
    if core.endswith("_bwd"):
        return 16 * wl.hidden * tokens + 8 * wl.hidden
    return 10 * wl.hidden * tokens + 4 * wl.hidden


def residual_timing(st, peak: float, flush: torch.Tensor, reps: int, rank: int):
    rs = ResidualStep(st.wl, seed=rank)
    which = ("residual", "residual_blend", "residual_bwd", "residual_blend_bwd")
    out = {"steady": per_core_steady(rs, peak, reps, nbytes=residual_bytes, which=which),
           "isolated": per_core_isolated(rs, peak, flush, nbytes=residual_bytes, which=which),
           "algo_bytes": residual_bytes(st.wl, "residual", st.T),
           "algo_bytes_bwd": residual_bytes(st.wl, "residual_bwd", st.T),
           "kernel": "residual_blend_kernel",
           "note": "_residual_core: FP32 stream blended with the bf16 branch per channel; residual = the "
                   "gate form (temperature 0.3, eps 1e-3), residual_blend = the angle form; *_bwd = their "
                   "backward with the gate / angle gradient (the kernel and the fixed-order reduction)"}
    del rs
    return out


def time_copy_kernel(gib: float = 1.0, reps: int = 10) -> float:
    n = int(gib * (1 << 30)) // 16 * 16
    src = torch.empty(n, dtype=torch.uint8, device="cuda")
    dst = torch.empty_like(src)
    src.fill_(1)
    for _ in range(3):
        cores.stream_copy(src, dst)
    best = math.inf
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(reps):
        torch.cuda.synchronize()
        e0.record()
        cores.stream_copy(src, dst)
        e1.record()
        e1.synchronize()
        best = min(best, e0.elapsed_time(e1) / 1e3)
    del src, dst
    torch.cuda.empty_cache()
    return 2 * n / best / 1e9


def traffic_from_profile(wl_name: str):
    """dram read+write bytes per launch of the dominant kernel from the committed
    ncu figure (profiles/<kernel>__<workload>.json), when the kernel sources are
    unchanged since the capture (their sha256 is stored beside the figure)."""
    import hashlib

    p = os.path.join(ROOT, "profiles", f"{DOMINANT}__{wl_name}.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p))
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gate_cores_b200", "csrc")
    for f in DOMINANT_SOURCES:
        h.update(open(os.path.join(csrc, f), "rb").read())
    if rec.get("csrc_sha256") != h.hexdigest() or "traffic_bytes_per_launch" not in rec:
        return None
    return float(rec["traffic_bytes_per_launch"])


def cpu_baseline(wl, seconds: float = 12.0, chunk: int = 256):
    """The oracle as it stands, single-threaded, on the first tokens of the same
    batch: all five cores per chunk of `chunk` tokens until `seconds` elapse."""
    import numpy as np

    from tests import harness

    host = {c: harness.make(wl.name, c, harness.DEFAULT_VARIANT[c]) for c in CORE_ORDER}
    T = num_tokens(wl)
    done, t0 = 0, time.perf_counter()
    while done < T and time.perf_counter() - t0 < seconds:
        rows = np.arange(done, min(T, done + chunk))
        for c in CORE_ORDER:
            harness.run_oracle(wl.name, c, host[c], rows)
        done += len(rows)
    el = time.perf_counter() - t0
    return {"value": done / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"first {done} of {T} tokens of {wl.name}, all five cores, "
                      f"{el:.1f} s single-threaded double-precision oracle"}


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline_threads(wl, seconds: float = 8.0, chunk: int = 64, threads: int | None = None,
                         host=None):
    """The same oracle over row chunks on all host cores: threads pull chunks
    of `chunk` tokens from a shared counter (the oracle's C routines run
    without the interpreter lock), all five cores per chunk, until `seconds`
    elapse or the batch is done."""
    import threading

    import numpy as np

    from tests import harness

    n = threads or min(os.cpu_count() or 1, 128)
    if host is None:
        host = {c: harness.make(wl.name, c, harness.DEFAULT_VARIANT[c]) for c in CORE_ORDER}
    T = num_tokens(wl)
    lock = threading.Lock()
    state = {"next": 0, "done": 0}
    t0 = time.perf_counter()

    def work():
        while time.perf_counter() - t0 < seconds:
            with lock:
                lo = state["next"]
                if lo >= T:
                    return
                state["next"] = min(T, lo + chunk)
            rows = np.arange(lo, min(T, lo + chunk))
            for c in CORE_ORDER:
                harness.run_oracle(wl.name, c, host[c], rows)
            with lock:
                state["done"] += len(rows)

    ts = [threading.Thread(target=work) for _ in range(n)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    el = time.perf_counter() - t0
    return {"value": state["done"] / el, "unit": "tokens/s", "cores": n, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{state['done']} of {T} tokens of {wl.name}, all five cores, {el:.1f} s, "
                      f"double-precision oracle over {chunk}-token chunks on {n} threads"}


def run_ours(args, world, rank, local):
    wl = WORKLOADS[args.workload]
    torch.manual_seed(0)
    st = Step(wl, seed=rank)
    T = st.T
    stream = torch.cuda.current_stream()
    peak, peak_kind = measured_peaks()
    sampler = ClockSampler(local) if rank == 0 else None
    copy_gbs = time_copy_kernel() if args.copy_ref else None

    for _ in range(args.warmup):
        for c in CORE_ORDER:
            st.launch(c)
    torch.cuda.synchronize()

    # Timed region: K steps launched back to back.  An event recorded between
    # two kernels costs a few microseconds of idle GPU and cancels the
    # programmatic-launch overlap of the pair, so none is recorded inside it.
    barrier(world)
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        for c in CORE_ORDER:
            st.launch(c)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    elapsed = t_start.elapsed_time(t_end) / 1e3
    elapsed = allreduce_max(elapsed, world)
    ms_per_step = elapsed / args.steps * 1e3
    value = world * T * args.steps / elapsed

    # Kernel pass: the same K steps again, each launch bracketed by events on
    # the launching stream; per-kernel durations for the roofline.
    ev = {c: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)] for c in CORE_ORDER}
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        for c in CORE_ORDER:
            ev[c][i][0].record(stream)
            st.launch(c)
            ev[c][i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)

    per_core = {}
    for c in CORE_ORDER:
        us = statistics.mean(a.elapsed_time(b) for a, b in ev[c]) * 1e3
        us = allreduce_max(us, world)
        nb = algo_bytes(wl, c, T)
        per_core[c] = {"us": round(us, 3), "tokens_per_s": round(T / (us * 1e-6), 1),
                       "gbs": round(nb / (us * 1e-6) / 1e9, 1),
                       "frac": round(nb / (us * 1e-6) / 1e9 / peak, 4), "algo_bytes": nb,
                       "kernel": KERNEL_NAMES[c], "variant": VARIANT[c]}
    dom = per_core[DOMINANT]
    traffic = traffic_from_profile(wl.name)
    roofline = {"bound": "hbm", "achieved": dom["gbs"], "peak": peak, "unit": "GB/s",
                "frac": round(dom["gbs"] / peak, 4), "traffic": traffic,
                "kernel": KERNEL_NAMES[DOMINANT], "peak_source": peak_kind,
                "algo_bytes_per_launch": dom["algo_bytes"]}

    # Each core alone on the same batch, L2 read-flushed before every launch;
    # and the decode batch (128 tokens), whose launches are latency-bound.
    flush = torch.empty(64 << 20, dtype=torch.int64, device="cuda").fill_(1)  # 512 MiB
    steady = per_core_steady(st, peak, max(10, min(args.steps, 100)))
    isolated = per_core_isolated(st, peak, flush)
    dec = Step(WORKLOADS["decode_t128_h4096"], seed=rank)
    decode_cold = per_core_isolated(dec, peak, flush)
    decode_warm = per_core_isolated(dec, peak, None)
    decode = {c: {"us_cold_l2": decode_cold[c]["us"], "us_warm_l2": decode_warm[c]["us"]}
              for c in CORE_ORDER}
    fl = LaunchFloor()
    one = lambda wl, c, T: 32  # noqa: E731 - 16 bytes read, 16 written
    decode["launch_floor"] = {"us_cold_l2": per_core_isolated(fl, peak, flush, nbytes=one, which=("floor",))["floor"]["us"],
                              "us_warm_l2": per_core_isolated(fl, peak, None, nbytes=one, which=("floor",))["floor"]["us"],
                              "note": "one-CTA 16-byte copy launched like the cores (programmatic "
                                      "dependent launch), timed the same way"}
    del dec, fl
    # Backward of the five cores on the same batch: each call alone (L2
    # read-flushed, median of 50) and the five back to back (K steps timed
    # with two events, as the forward step).
    bst = BwdStep(st, seed=rank)
    bwd_iso = per_core_isolated(bst, peak, flush, nbytes=algo_bytes_bwd)
    bst.qk_upcast = False  # the v2 (bf16) rotation's backward, alone
    bwd_iso["qk_norm_rope_v2"] = per_core_isolated(bst, peak, flush, nbytes=algo_bytes_bwd,
                                                   which=("qk_norm_rope",))["qk_norm_rope"]
    bst.qk_upcast = True
    for _ in range(3):
        for c in CORE_ORDER:
            bst.launch(c)
    barrier(world)
    torch.cuda.synchronize()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b0.record(stream)
    for _ in range(args.steps):
        for c in CORE_ORDER:
            bst.launch(c)
    b1.record(stream)
    torch.cuda.synchronize()
    bwd_el = allreduce_max(b0.elapsed_time(b1) / 1e3, world)
    bwd_bytes = sum(algo_bytes_bwd(wl, c, T) for c in CORE_ORDER)
    backward = {"tokens_per_s": round(world * T * args.steps / bwd_el, 1),
                "ms_per_step": round(bwd_el / args.steps * 1e3, 5),
                "gbs": round(bwd_bytes * args.steps / bwd_el / 1e9, 1),
                "frac": round(bwd_bytes * args.steps / bwd_el / 1e9 / peak, 4),
                "algo_bytes_per_step": bwd_bytes,
                "gpu_launches_per_step": 9,
                "per_core_isolated": bwd_iso,
                "note": "gradients of the five cores (the Q/K call with the FP32 rotation; "
                        "per_core_isolated.qk_norm_rope_v2 is the v2 rotation's backward alone); gain and "
                        "theta gradients reduced through the caller's workspace"}
    del bst
    fused = fused_vs_unfused(st, peak, flush)
    fused_blend = fused_vs_unfused(st, peak, flush, calls=blend_fused_calls(st, rank),
                                   note="_residual_core (angle form) + the next sublayer's RMS pre-norm (FP32 y) in "
                                        "one pass, against muse_residual_blend then muse_rms_norm on its output")
    grouped = grouped_norm(st, peak, flush)
    vision = vision_rope_timing(peak, flush)
    residual_core = residual_timing(st, peak, flush, max(10, min(args.steps, 100)), rank)
    del flush
    torch.cuda.empty_cache()
    configs = per_config(args, peak, rank, world) if args.per_config else None
    clocks = sampler.stop() if sampler else None

    e2e = run_e2e(st, args, world) if args.e2e else None

    cpu = cpu_par = None
    if rank == 0 and world == 1 and args.cpu_baseline:
        cpu = cpu_baseline(wl)
        cpu_par = cpu_baseline_threads(wl)
    barrier(world)
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 activations, FP32 residual stream)",
            "config": run_config(wl, T, world),
            "per_core": per_core,
            "per_core_steady": steady,
            "per_core_isolated": isolated,
            "decode_t128_h4096_latency": decode,
            "backward": backward,
            "fused_residual_prenorm": fused,
            "fused_residual_blend_prenorm": fused_blend,
            "per_expert_norm": grouped,
            "vision_rope": vision,
            "residual_core": residual_core,
            "per_config": configs,
            "roofline": roofline,
            "copy_kernel_gbs": None if copy_gbs is None else round(copy_gbs, 1),
            "e2e": e2e,
            "cpu_baseline": cpu,
            "cpu_baseline_all_cores": cpu_par,
            "gpu_launches": len(CORE_ORDER) * args.steps,
            "kernel_timing": "per_core and roofline: a second pass of the same K steps with "
                             "CUDA events around each launch (the timed region has none); "
                             "per_core_steady: each core alone, launched back to back with two "
                             "events around the loop, no flush (each launch drains its "
                             "predecessor's dirty L2 lines, as in the step); "
                             "per_core_isolated: each core alone, median of 50 launches, "
                             "a 512 MiB read pass before each (a clean, cold L2 - credits the "
                             "output lines still dirty in L2 when the kernel ends); decode "
                             "latency: median of 50, cold (read-flushed) and warm L2, beside a "
                             "launch floor",
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


def run_e2e(st: Step, args, world):
    """Same metric through the public API with host buffers: every step copies
    its inputs from pinned host memory, runs the five cores and reads every
    output back to pinned host memory.  Two sets of device and host buffers
    and three streams (upload, compute, download) let one step's download
    overlap the next step's upload and compute - PCIe carries both directions
    at once - with events ordering each set's reuse."""
    rank = int(os.environ.get("RANK", "0"))
    sets = [st, Step(st.wl, seed=rank)]
    pin_in = [[(dev, torch.empty(dev.shape, dtype=dev.dtype, pin_memory=True).copy_(dev.cpu()))
               for _, dev in s_.input_tensors()] for s_ in sets]
    pin_out = [[(dev, torch.empty(dev.shape, dtype=dev.dtype, pin_memory=True)) for dev in s_.output_tensors()]
               for s_ in sets]
    h2d = sum(h.numel() * h.element_size() for _, h in pin_in[0])
    d2h = sum(h.numel() * h.element_size() for _, h in pin_out[0])
    steps = max(3, min(args.steps, 20))
    up, comp, down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    up_done, comp_done, down_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for k in range(2):  # every event recorded once before its first wait
        for e in (up_done[k], comp_done[k], down_done[k]):
            e.record(comp)

    def one(k):
        j = k % 2
        with torch.cuda.stream(up):
            up.wait_event(comp_done[j])          # the set's previous inputs are consumed
            for dev, h in pin_in[j]:
                dev.copy_(h, non_blocking=True)
            up_done[j].record(up)
        with torch.cuda.stream(comp):
            comp.wait_event(up_done[j])
            comp.wait_event(down_done[j])        # the set's previous outputs are read back
            for c in CORE_ORDER:
                sets[j].launch(c)
            comp_done[j].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(comp_done[j])
            for dev, h in pin_out[j]:
                h.copy_(dev, non_blocking=True)
            down_done[j].record(down)

    for k in range(2):
        one(k)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(up)
    for k in range(steps):
        one(k)
    up.wait_stream(down)
    e1.record(up)
    torch.cuda.synchronize()
    el = allreduce_max(e0.elapsed_time(e1) / 1e3, world)
    del sets[1]
    return {"value": round(world * st.T * steps / el, 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "overlap": "two buffer sets; upload, compute and download on three streams"}


# ------------------------------------------------------------------ reference arm

def run_config(wl, tokens: int, world: int) -> dict:
    """The `config` of the JSON line (both arms)."""
    return {"workload": wl.name, "tokens_per_gpu": tokens, "batch": wl.batch, "seq_len": wl.seqlen,
            "hidden": wl.hidden, "q_heads": wl.hq, "kv_heads": wl.hkv, "head_dim": wl.head_dim,
            "parallelism": f"token shards x{world} (no collective)",
            "l2": "no flush: each step streams %.2f GB, > 126 MB L2"
                  % (sum(algo_bytes(wl, c, tokens) for c in CORE_ORDER) / 1e9)}


def run_reference(args, world, rank):
    """The oracle (plain double-precision C, single-threaded) on the host cores:
    each step is a bounded sample (64 consecutive tokens, rotating through the
    batch) of the same workload, all five cores."""
    if rank != 0:
        return
    import numpy as np

    from tests import harness

    wl = WORKLOADS[args.workload]
    host = {c: harness.make(wl.name, c, harness.DEFAULT_VARIANT[c]) for c in CORE_ORDER}
    T = num_tokens(wl)
    per_step = 64

    def step(i):
        lo = (i * per_step) % (T - per_step + 1)
        rows = np.arange(lo, lo + per_step)
        for c in CORE_ORDER:
            harness.run_oracle(wl.name, c, host[c], rows)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    el = time.perf_counter() - t0
    value = per_step * args.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, same generator as the GPU arm)",
        "config": run_config(wl, T, world),
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"{per_step} consecutive tokens per step of the {T}-token batch of {wl.name} "
                                   f"(rotating through it), all five cores; value = tokens of the samples / time"},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def profile_pass(args):
    """Each forward core, each backward core, core 5 fused with the next
    pre-norm, the per-expert core 1, the vision RoPE and the two _residual_core
    forms with their backward and the blend fused with the next pre-norm, the
    sequence launched twice on the workload's batch: a short, fixed launch
    sequence for an ncu capture (16 table launches first, then 24 kernel
    launches per pass; skip the table and the first pass to capture warm
    ones)."""
    wl = WORKLOADS[args.workload]
    st = Step(wl, seed=0)
    bst = BwdStep(st, seed=0)
    fused, _ = fused_calls(st)
    fused_blend, _ = blend_fused_calls(st)
    grouped = grouped_call(st)
    rs = ResidualStep(wl, seed=0)
    _, vision = vision_call()  # 16 table launches before the passes
    for _ in range(2):
        for c in CORE_ORDER:
            st.launch(c)
        for c in CORE_ORDER:
            bst.launch(c)
        fused()
        grouped()
        vision()
        for c in ("residual", "residual_blend", "residual_bwd", "residual_blend_bwd"):
            rs.launch(c)
        fused_blend()
    torch.cuda.synchronize()
    print("profile pass: 16 vision-table launches, then 2 x (5 forward + 5 backward calls, fused core 5 + "
          "pre-norm, per-expert core 1, vision RoPE, residual gate and angle forms, their backward and the "
          "fused blend + pre-norm) on "
          + wl.name, file=sys.stderr)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_t8192_h4096", choices=sorted(WORKLOADS))
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-copy-ref", dest="copy_ref", action="store_false")
    ap.add_argument("--no-per-config", dest="per_config", action="store_false",
                    help="skip the packed-THD and large-hidden workloads")
    ap.add_argument("--profile-pass", action="store_true",
                    help="for profilers: launch every forward and backward core twice on the batch "
                         "(no timing, no JSON line) and exit")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            if not torch.cuda.is_available():
                raise SystemExit("bench.py: no CUDA device (the cores run only on the GPU)")
            if args.profile_pass:
                profile_pass(args)
            else:
                run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
