"""Tensor-level front end: PyTorch CUDA tensors in, PyTorch CUDA tensors out.

Marshalling only - pointers, shapes, strides and the current stream go to the
C entry points in ``_lib``; every step of the computation runs in the CUDA
library.  Outputs are fresh tensors unless ``out=`` is given (``out`` may be
the input itself for an in-place call).
"""
from __future__ import annotations

import torch

from . import _lib

_DT = {torch.bfloat16: _lib.MUSE_DTYPE_BF16, torch.float32: _lib.MUSE_DTYPE_F32}


def _dtype(t: torch.Tensor) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32") from None


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")


def _rows(x: torch.Tensor):
    """View x as rows of its last dim: (rows, hidden, row_stride); the last dim must be unit-stride."""
    if x.dim() < 1 or x.stride(-1) != 1:
        raise ValueError("last dimension must be contiguous")
    hidden = x.shape[-1]
    if x.dim() == 1:
        return 1, hidden, hidden
    if x.dim() == 2:
        return x.shape[0], hidden, x.stride(0)
    if not x.is_contiguous():
        raise ValueError("tensors with more than 2 dims must be contiguous")
    return x.numel() // hidden, hidden, hidden


def _out_like(x, out):
    if out is None:
        return torch.empty_like(x, memory_format=torch.contiguous_format)
    if out.shape != x.shape or out.dtype != x.dtype:
        raise ValueError("out must match the input's shape and dtype")
    return out


def _gain(gain):
    if gain is None:
        return None
    if gain.dtype != torch.float32:
        raise TypeError("gain must be float32")
    return gain.contiguous()


def rms_norm(x: torch.Tensor, gain: torch.Tensor | None = None, gain_offset: float = 0.0,
             eps: float = 1e-6, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Core 1 (_rms_norm_core) on the last dim of x."""
    _cuda(x, gain, out)
    y = _out_like(x, out)
    rows, hidden, xs = _rows(x)
    _, _, ys = _rows(y)
    g = _gain(gain)
    _lib.muse_rms_norm(x.data_ptr(), y.data_ptr(), _dtype(x), rows, hidden, xs, ys, _ptr(g),
                       gain_offset, eps, _stream(stream))
    return y


def input_scale_norm(x: torch.Tensor, gain: torch.Tensor | None = None, gain_offset: float = 0.0,
                     eps: float = 1e-6, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Core 2 (_input_scale_norm_core) on the last dim of x."""
    _cuda(x, gain, out)
    y = _out_like(x, out)
    rows, hidden, xs = _rows(x)
    _, _, ys = _rows(y)
    g = _gain(gain)
    _lib.muse_input_scale_norm(x.data_ptr(), y.data_ptr(), _dtype(x), rows, hidden, xs, ys,
                               _ptr(g), gain_offset, eps, _stream(stream))
    return y


def _tok_stride(t: torch.Tensor, heads: int, d: int) -> int:
    # heads and head_dim of one token must be packed: strides (.., d, 1)
    if t.stride(-1) != 1 or t.stride(-2) != d or t.shape[-2] != heads:
        raise ValueError("each token's heads must be contiguous ([.., heads, head_dim])")
    if t.dim() == 4 and t.stride(0) != t.shape[1] * t.stride(1):
        raise ValueError("BSHD tensors need a uniform token stride")
    return t.stride(-3)


def qk_norm_rope(q: torch.Tensor, k: torch.Tensor, positions: torch.Tensor | None = None,
                 cu_seqlens: torch.Tensor | None = None, eps: float = 1e-6,
                 query_scale: float = 1.0, use_rope: bool = True, upcast_rope: bool = True,
                 rope_base: float = 10000.0, q_out: torch.Tensor | None = None,
                 k_out: torch.Tensor | None = None, stream=None):
    """Core 3 (_qk_norm_rope_core).  q [B,S,Hq,D] (BSHD) or [T,Hq,D] (THD with
    cu_seqlens [docs+1] int32, or explicit positions [T]); k with Hkv heads.
    positions: int32, [B,S] or [T]; None derives them from the layout."""
    _cuda(q, k, positions, cu_seqlens, q_out, k_out)
    if q.dim() == 4:
        layout, batch, seqlen, T = _lib.MUSE_LAYOUT_BSHD, q.shape[0], q.shape[1], q.shape[0] * q.shape[1]
    elif q.dim() == 3:
        T = q.shape[0]
        if cu_seqlens is not None:
            layout, batch, seqlen = _lib.MUSE_LAYOUT_THD, 0, 0
        else:
            layout, batch, seqlen = _lib.MUSE_LAYOUT_BSHD, 1, T
    else:
        raise ValueError("q must be [B,S,Hq,D] or [T,Hq,D]")
    hq, d = q.shape[-2], q.shape[-1]
    hkv = k.shape[-2]
    if k.shape[:-2] != q.shape[:-2] or k.shape[-1] != d or k.dtype != q.dtype:
        raise ValueError("k must match q's leading dims, head_dim and dtype")
    qo = _out_like(q, q_out)
    ko = _out_like(k, k_out)
    if positions is not None:
        if positions.dtype != torch.int32 or positions.numel() != T:
            raise ValueError("positions must be int32 with one entry per token")
        positions = positions.contiguous()
    num_seqs = 0
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32:
            raise ValueError("cu_seqlens must be int32")
        cu_seqlens = cu_seqlens.contiguous()
        num_seqs = cu_seqlens.numel() - 1
    _lib.muse_qk_norm_rope(
        q.data_ptr(), k.data_ptr(), qo.data_ptr(), ko.data_ptr(), _dtype(q), layout, batch,
        seqlen, _ptr(cu_seqlens), num_seqs, T, _ptr(positions), hq, hkv, d,
        _tok_stride(q, hq, d), _tok_stride(k, hkv, d), _tok_stride(qo, hq, d),
        _tok_stride(ko, hkv, d), eps, query_scale, use_rope, upcast_rope, rope_base,
        _stream(stream))
    return qo, ko


def output_norm_gate(o: torch.Tensor, gate: torch.Tensor, norm_group: int | None = None,
                     eps: float = 1e-6, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Core 4 (_output_norm_gate_core).  o, gate [B,S,H,D] or [T,H,D], contiguous.
    norm_group None/D: per head; H*D: per token."""
    _cuda(o, gate, out)
    if gate.shape != o.shape or gate.dtype != o.dtype:
        raise ValueError("gate must match o")
    if not (o.is_contiguous() and gate.is_contiguous()):
        raise ValueError("o and gate must be contiguous")
    y = _out_like(o, out)
    heads, d = o.shape[-2], o.shape[-1]
    tokens = o.numel() // (heads * d)
    ng = d if norm_group is None else norm_group
    _lib.muse_output_norm_gate(o.data_ptr(), gate.data_ptr(), y.data_ptr(), _dtype(o), tokens,
                               heads, d, ng, eps, _stream(stream))
    return y


def norm_residual(stream_in: torch.Tensor, branch: torch.Tensor, theta: torch.Tensor,
                  gain: torch.Tensor | None = None, gain_offset: float = 0.0,
                  input_scale: bool = False, norm_eps: float = 1e-6,
                  out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Core 5 (_norm_residual_core) with the per-channel cos/sin blend.
    stream_in FP32 [..., H]; branch [..., H] bf16/f32; theta FP32 [H]."""
    _cuda(stream_in, branch, theta, gain, out)
    if stream_in.dtype != torch.float32 or theta.dtype != torch.float32:
        raise TypeError("stream and theta must be float32")
    if branch.shape != stream_in.shape:
        raise ValueError("branch must match the stream's shape")
    if not (stream_in.is_contiguous() and branch.is_contiguous()):
        raise ValueError("stream and branch must be contiguous")
    h_out = _out_like(stream_in, out)
    hidden = stream_in.shape[-1]
    rows = stream_in.numel() // hidden
    g = _gain(gain)
    _lib.muse_norm_residual(stream_in.data_ptr(), branch.data_ptr(), h_out.data_ptr(),
                            _dtype(branch), rows, hidden, _ptr(g), gain_offset,
                            theta.contiguous().data_ptr(), input_scale, norm_eps, _stream(stream))
    return h_out


def _residual_args(stream_in, branch, p, what):
    _cuda(stream_in, branch, p)
    if stream_in.dtype != torch.float32 or p.dtype != torch.float32:
        raise TypeError(f"stream and {what} must be float32")
    if branch.shape != stream_in.shape:
        raise ValueError("branch must match the stream's shape")
    if not (stream_in.is_contiguous() and branch.is_contiguous()):
        raise ValueError("stream and branch must be contiguous")
    hidden = stream_in.shape[-1]
    return hidden, stream_in.numel() // hidden


def residual_blend(stream_in: torch.Tensor, branch: torch.Tensor, theta: torch.Tensor,
                   out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """_residual_core without a branch norm, in core 5's angle form:
    cos(theta) * stream + sin(theta) * branch per channel (theta FP32 [H])."""
    hidden, rows = _residual_args(stream_in, branch, theta, "theta")
    _cuda(out)
    h_out = _out_like(stream_in, out)
    _lib.muse_residual_blend(stream_in.data_ptr(), branch.data_ptr(), h_out.data_ptr(), _dtype(branch), rows,
                             hidden, theta.contiguous().data_ptr(), _stream(stream))
    return h_out


def residual(stream_in: torch.Tensor, branch: torch.Tensor, gate: torch.Tensor, temperature: float = 0.3,
             eps: float = 1e-3, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """_residual_core(stream, branch, gate, temperature, eps): c * stream +
    s * branch per channel with c^2 = max(sigmoid(gate / temperature), eps),
    s^2 = 1 - c^2 (gate FP32 [H])."""
    hidden, rows = _residual_args(stream_in, branch, gate, "gate")
    _cuda(out)
    h_out = _out_like(stream_in, out)
    _lib.muse_residual(stream_in.data_ptr(), branch.data_ptr(), h_out.data_ptr(), _dtype(branch), rows, hidden,
                       gate.contiguous().data_ptr(), temperature, eps, _stream(stream))
    return h_out


def residual_blend_rms_norm(stream_in: torch.Tensor, branch: torch.Tensor, theta: torch.Tensor,
                            next_gain: torch.Tensor | None = None, next_gain_offset: float = 0.0,
                            next_eps: float = 1e-6, y_dtype=torch.float32, out: torch.Tensor | None = None,
                            y: torch.Tensor | None = None, stream=None):
    """_residual_core (angle form) and the next sublayer's RMS pre-norm of the
    new stream in one pass.  Returns (stream_out, y)."""
    hidden, rows = _residual_args(stream_in, branch, theta, "theta")
    _cuda(next_gain, out, y)
    h_out = _out_like(stream_in, out)
    if y is None:
        y = torch.empty(stream_in.shape, dtype=y_dtype, device=stream_in.device)
    elif y.shape != stream_in.shape or y.dtype != y_dtype or not y.is_contiguous():
        raise ValueError("y must be contiguous, shaped like the stream, in y_dtype")
    g2 = _gain(next_gain)
    _lib.muse_residual_blend_rms_norm(stream_in.data_ptr(), branch.data_ptr(), h_out.data_ptr(), y.data_ptr(),
                                      _dtype(branch), _dtype(y), rows, hidden, theta.contiguous().data_ptr(),
                                      _ptr(g2), next_gain_offset, next_eps, _stream(stream))
    return h_out, y


def residual_gate_angles(gate: torch.Tensor, temperature: float = 0.3, eps: float = 1e-3,
                         out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Blend angle per channel from the learned gate: atan2(s, c) (FP32 [H])."""
    _cuda(gate, out)
    if gate.dtype != torch.float32 or gate.dim() != 1:
        raise TypeError("gate must be a float32 vector")
    theta = _out_like(gate, out)
    _lib.muse_residual_gate_angles(gate.contiguous().data_ptr(), theta.data_ptr(), gate.numel(), temperature,
                                   eps, _stream(stream))
    return theta


def rms_norm_grouped(x: torch.Tensor, gains: torch.Tensor, group_offsets: torch.Tensor,
                     gain_offset: float = 0.0, eps: float = 1e-6, out: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Per-expert core 1: rows group_offsets[g]..group_offsets[g+1]-1 of x use
    gains[g] (gains FP32 [E, H]; group_offsets int32 [E+1] on the device)."""
    _cuda(x, gains, group_offsets, out)
    if gains.dtype != torch.float32 or group_offsets.dtype != torch.int32:
        raise TypeError("gains must be float32 and group_offsets int32")
    y = _out_like(x, out)
    rows, hidden, xs = _rows(x)
    _, _, ys = _rows(y)
    gains = gains.contiguous()
    group_offsets = group_offsets.contiguous()
    if gains.shape[-1] != hidden or gains.numel() != hidden * (group_offsets.numel() - 1):
        raise ValueError("gains must be [num_groups, hidden] with num_groups + 1 offsets")
    _lib.muse_rms_norm_grouped(x.data_ptr(), y.data_ptr(), _dtype(x), rows, hidden, xs, ys,
                               gains.data_ptr(), gain_offset, group_offsets.data_ptr(),
                               group_offsets.numel() - 1, eps, _stream(stream))
    return y


def vision_rope(q: torch.Tensor, k: torch.Tensor, freqs: torch.Tensor, q_out: torch.Tensor | None = None,
                k_out: torch.Tensor | None = None, stream=None):
    """Vision 2-D RoPE: q [T, hq, D], k [T, hk, D] rotated by freqs FP32
    [T, D/2, 2] ((cos, sin) per token and pair); returns (q', k') in q's
    dtype.  q_out / k_out may be q / k (in place)."""
    _cuda(q, k, freqs, q_out, k_out)
    if q.dim() != 3 or k.dim() != 3 or q.shape[0] != k.shape[0] or q.shape[-1] != k.shape[-1]:
        raise ValueError("q, k must be [T, heads, head_dim] with the same T and head_dim")
    if q.dtype != k.dtype:
        raise TypeError("q and k must share a dtype")
    T, hq, d = q.shape
    hk = k.shape[1]
    if freqs.dtype != torch.float32 or tuple(freqs.shape) != (T, d // 2, 2):
        raise ValueError("freqs must be float32 [T, head_dim/2, 2]")
    freqs = freqs.contiguous()
    qo = torch.empty_like(q, memory_format=torch.contiguous_format) if q_out is None else q_out
    ko = torch.empty_like(k, memory_format=torch.contiguous_format) if k_out is None else k_out
    _lib.muse_vision_rope(q.data_ptr(), k.data_ptr(), qo.data_ptr(), ko.data_ptr(), _dtype(q), T, hq, hk, d,
                          _tok_stride(q, hq, d), _tok_stride(k, hk, d), _tok_stride(qo, hq, d),
                          _tok_stride(ko, hk, d), freqs.data_ptr(), _stream(stream))
    return qo, ko


def vision_rope_frequencies(head_dim: int, grid_h: int, grid_w: int, theta: float = 10000.0,
                            out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The vision RoPE table of one row-major grid: FP32 [grid_h*grid_w, head_dim/2, 2]
    on the current CUDA device (or written into `out`)."""
    if out is None:
        out = torch.empty((grid_h * grid_w, head_dim // 2, 2), dtype=torch.float32, device="cuda")
    _cuda(out)
    if out.dtype != torch.float32 or not out.is_contiguous() or out.numel() != grid_h * grid_w * head_dim:
        raise ValueError("out must be contiguous float32 [grid_h*grid_w, head_dim/2, 2]")
    _lib.muse_vision_rope_frequencies(out.data_ptr(), head_dim, grid_h, grid_w, theta, _stream(stream))
    return out


def norm_residual_rms_norm(stream_in: torch.Tensor, branch: torch.Tensor, theta: torch.Tensor,
                           gain: torch.Tensor | None = None, gain_offset: float = 0.0,
                           input_scale: bool = False, norm_eps: float = 1e-6,
                           next_gain: torch.Tensor | None = None, next_gain_offset: float = 0.0,
                           next_eps: float = 1e-6, y_dtype=torch.float32, out=None, y=None,
                           stream=None):
    """Core 5 fused with the next sublayer's RMS pre-norm of the new stream:
    returns (stream_out, y), y = rms_norm(stream_out) in y_dtype."""
    _cuda(stream_in, branch, theta, gain, next_gain, out, y)
    if stream_in.dtype != torch.float32 or theta.dtype != torch.float32:
        raise TypeError("stream and theta must be float32")
    if branch.shape != stream_in.shape or not (stream_in.is_contiguous() and branch.is_contiguous()):
        raise ValueError("stream and branch must be contiguous and of one shape")
    h_out = _out_like(stream_in, out)
    if y is None:
        y = torch.empty(stream_in.shape, dtype=y_dtype, device=stream_in.device)
    hidden = stream_in.shape[-1]
    rows = stream_in.numel() // hidden
    g, g2 = _gain(gain), _gain(next_gain)
    _lib.muse_norm_residual_rms_norm(
        stream_in.data_ptr(), branch.data_ptr(), h_out.data_ptr(), y.data_ptr(), _dtype(branch),
        _dtype(y), rows, hidden, _ptr(g), gain_offset, theta.contiguous().data_ptr(), input_scale,
        norm_eps, _ptr(g2), next_gain_offset, next_eps, _stream(stream))
    return h_out, y


def stream_copy(src: torch.Tensor, dst: torch.Tensor, stream=None) -> torch.Tensor:
    """16-byte vector copy of src into dst (same byte size) - the HBM reference kernel."""
    _cuda(src, dst)
    nbytes = src.numel() * src.element_size()
    if dst.numel() * dst.element_size() != nbytes or not (src.is_contiguous() and dst.is_contiguous()):
        raise ValueError("src and dst must be contiguous and of equal byte size")
    _lib.muse_stream_copy(src.data_ptr(), dst.data_ptr(), nbytes, _stream(stream))
    return dst


# ------------------------------------------------------------------ backward


def _workspace(rows: int, hidden: int, device, workspace):
    need = _lib.muse_norm_backward_workspace_bytes(rows, hidden)
    if workspace is None:
        return torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace needs {need} bytes")
    return workspace


def _row_bwd(fn, x, dy, gain, gain_offset, eps, dx, want_dgain, workspace, stream):
    _cuda(x, dy, gain, dx)
    if dy.shape != x.shape or dy.dtype != x.dtype:
        raise ValueError("dy must match x")
    dx = _out_like(x, dx)
    rows, hidden, xs = _rows(x)
    _, _, dys = _rows(dy)
    _, _, dxs = _rows(dx)
    g = _gain(gain)
    dgain = None
    ws = None
    if want_dgain and g is not None:
        dgain = torch.empty(hidden, dtype=torch.float32, device=x.device)
        ws = _workspace(rows, hidden, x.device, workspace)
    fn(x.data_ptr(), dy.data_ptr(), dx.data_ptr(), _dtype(x), rows, hidden, xs, dys, dxs, _ptr(g),
       gain_offset, eps, _ptr(dgain), _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream))
    return dx, dgain


def rms_norm_backward(x, dy, gain=None, gain_offset: float = 0.0, eps: float = 1e-6, dx=None,
                      want_dgain: bool = True, workspace=None, stream=None):
    """Backward of core 1: returns (dx, dgain); dgain is None without a gain."""
    return _row_bwd(_lib.muse_rms_norm_backward, x, dy, gain, gain_offset, eps, dx, want_dgain,
                    workspace, stream)


def input_scale_norm_backward(x, dy, gain=None, gain_offset: float = 0.0, eps: float = 1e-6,
                              dx=None, want_dgain: bool = True, workspace=None, stream=None):
    """Backward of core 2: returns (dx, dgain); dgain is None without a gain."""
    return _row_bwd(_lib.muse_input_scale_norm_backward, x, dy, gain, gain_offset, eps, dx,
                    want_dgain, workspace, stream)


def norm_residual_backward(stream_in, branch, dstream_out, theta, gain=None,
                           gain_offset: float = 0.0, input_scale: bool = False,
                           norm_eps: float = 1e-6, want_params: bool = True, workspace=None,
                           stream=None):
    """Backward of core 5: returns (dstream_in, dbranch, dgain, dtheta)."""
    _cuda(stream_in, branch, dstream_out, theta, gain)
    if stream_in.dtype != torch.float32 or dstream_out.dtype != torch.float32:
        raise TypeError("stream tensors must be float32")
    if not (stream_in.is_contiguous() and branch.is_contiguous() and dstream_out.is_contiguous()):
        raise ValueError("stream, branch and dstream_out must be contiguous")
    hidden = stream_in.shape[-1]
    rows = stream_in.numel() // hidden
    dsi = torch.empty_like(stream_in)
    db = torch.empty_like(branch)
    g = _gain(gain)
    dgain = dtheta = ws = None
    if want_params:
        dtheta = torch.empty(hidden, dtype=torch.float32, device=stream_in.device)
        if g is not None:
            dgain = torch.empty(hidden, dtype=torch.float32, device=stream_in.device)
        ws = _workspace(rows, hidden, stream_in.device, workspace)
    _lib.muse_norm_residual_backward(
        stream_in.data_ptr(), branch.data_ptr(), dstream_out.data_ptr(), dsi.data_ptr(),
        db.data_ptr(), _dtype(branch), rows, hidden, _ptr(g), gain_offset,
        theta.contiguous().data_ptr(), input_scale, norm_eps, _ptr(dgain), _ptr(dtheta), _ptr(ws),
        0 if ws is None else ws.numel(), _stream(stream))
    return dsi, db, dgain, dtheta


def residual_backward(stream_in, branch, dstream_out, theta=None, gate=None, temperature: float = 0.3,
                      eps: float = 1e-3, want_param: bool = True, workspace=None, stream=None):
    """Backward of _residual_core: the angle form (theta given) or the gate form
    (gate given).  Returns (dstream_in, dbranch, dtheta or dgate)."""
    if (theta is None) == (gate is None):
        raise ValueError("give exactly one of theta and gate")
    p = theta if gate is None else gate
    hidden, rows = _residual_args(stream_in, branch, p, "theta / gate")
    _cuda(dstream_out)
    if dstream_out.dtype != torch.float32 or dstream_out.shape != stream_in.shape or not dstream_out.is_contiguous():
        raise ValueError("dstream_out must be float32, contiguous and shaped like the stream")
    dsi = torch.empty_like(stream_in)
    db = torch.empty_like(branch)
    dp = ws = None
    if want_param:
        dp = torch.empty(hidden, dtype=torch.float32, device=stream_in.device)
        need = _lib.muse_residual_backward_workspace_bytes(rows, hidden)
        ws = workspace if workspace is not None else torch.empty(max(need, 16), dtype=torch.uint8,
                                                                 device=stream_in.device)
    args = (stream_in.data_ptr(), branch.data_ptr(), dstream_out.data_ptr(), dsi.data_ptr(), db.data_ptr(),
            _dtype(branch), rows, hidden, p.contiguous().data_ptr())
    tail = (_ptr(dp), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    if gate is None:
        _lib.muse_residual_blend_backward(*args, *tail)
    else:
        _lib.muse_residual_backward(*args, temperature, eps, *tail)
    return dsi, db, dp


def output_norm_gate_backward(o, gate, dy, norm_group=None, eps: float = 1e-6, stream=None):
    """Backward of core 4: returns (d_o, dgate)."""
    _cuda(o, gate, dy)
    if gate.shape != o.shape or dy.shape != o.shape or gate.dtype != o.dtype or dy.dtype != o.dtype:
        raise ValueError("gate and dy must match o")
    if not (o.is_contiguous() and gate.is_contiguous() and dy.is_contiguous()):
        raise ValueError("o, gate and dy must be contiguous")
    heads, d = o.shape[-2], o.shape[-1]
    tokens = o.numel() // (heads * d)
    d_o = torch.empty_like(o)
    dg = torch.empty_like(o)
    ng = d if norm_group is None else norm_group
    _lib.muse_output_norm_gate_backward(o.data_ptr(), gate.data_ptr(), dy.data_ptr(), d_o.data_ptr(),
                                        dg.data_ptr(), _dtype(o), tokens, heads, d, ng, eps,
                                        _stream(stream))
    return d_o, dg


def qk_norm_rope_backward(q, k, dq_out, dk_out, positions=None, cu_seqlens=None, eps: float = 1e-6,
                          query_scale: float = 1.0, use_rope: bool = True,
                          rope_base: float = 10000.0, upcast_rope: bool = True, stream=None):
    """Backward of core 3 (FP32 rotation, or the v2 bf16 rotation with
    upcast_rope=False): returns (dq, dk) shaped like q, k.  Layout and
    positions as in qk_norm_rope."""
    _cuda(q, k, dq_out, dk_out, positions, cu_seqlens)
    if q.dim() == 4:
        layout, batch, seqlen, T = _lib.MUSE_LAYOUT_BSHD, q.shape[0], q.shape[1], q.shape[0] * q.shape[1]
    elif q.dim() == 3:
        T = q.shape[0]
        if cu_seqlens is not None:
            layout, batch, seqlen = _lib.MUSE_LAYOUT_THD, 0, 0
        else:
            layout, batch, seqlen = _lib.MUSE_LAYOUT_BSHD, 1, T
    else:
        raise ValueError("q must be [B,S,Hq,D] or [T,Hq,D]")
    hq, d = q.shape[-2], q.shape[-1]
    hkv = k.shape[-2]
    if dq_out.shape != q.shape or dk_out.shape != k.shape:
        raise ValueError("incoming gradients must match q and k")
    dq = torch.empty_like(q, memory_format=torch.contiguous_format)
    dk = torch.empty_like(k, memory_format=torch.contiguous_format)
    if positions is not None:
        positions = positions.contiguous()
    num_seqs = 0
    if cu_seqlens is not None:
        cu_seqlens = cu_seqlens.contiguous()
        num_seqs = cu_seqlens.numel() - 1
    _lib.muse_qk_norm_rope_backward(
        q.data_ptr(), k.data_ptr(), dq_out.data_ptr(), dk_out.data_ptr(), dq.data_ptr(), dk.data_ptr(),
        _dtype(q), layout, batch, seqlen, _ptr(cu_seqlens), num_seqs, T, _ptr(positions), hq, hkv, d,
        _tok_stride(q, hq, d), _tok_stride(k, hkv, d), _tok_stride(dq_out, hq, d),
        _tok_stride(dk_out, hkv, d), _tok_stride(dq, hq, d), _tok_stride(dk, hkv, d), eps,
        query_scale, use_rope, upcast_rope, rope_base, _stream(stream))
    return dq, dk
