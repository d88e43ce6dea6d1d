"""ctypes binding of libmuse_cores.so: the C entry points under their own names.

Argument marshalling only.  Pointers are plain integers (device addresses),
streams are integer cudaStream_t handles.  Each wrapper raises MuseError on a
non-OK status.  There is no fallback: if the library is missing, the first
call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmuse_cores.so")

MUSE_OK = 0
MUSE_ERR_INVALID_ARGUMENT = 1
MUSE_ERR_UNSUPPORTED = 2
MUSE_ERR_CUDA = 3

MUSE_DTYPE_BF16 = 0
MUSE_DTYPE_F32 = 1
MUSE_LAYOUT_BSHD = 0
MUSE_LAYOUT_THD = 1

# Every symbol include/muse_cores.h declares.
EXPORTS = (
    "muse_version", "muse_status_string", "muse_last_error", "muse_rms_norm",
    "muse_input_scale_norm", "muse_qk_norm_rope", "muse_output_norm_gate",
    "muse_norm_residual", "muse_device_error", "muse_stream_copy",
    "muse_norm_backward_workspace_bytes", "muse_rms_norm_backward",
    "muse_input_scale_norm_backward", "muse_norm_residual_backward",
    "muse_output_norm_gate_backward", "muse_qk_norm_rope_backward",
    "muse_rms_norm_backward_noalloc", "muse_norm_residual_rms_norm", "muse_rms_norm_grouped",
    "muse_vision_rope", "muse_vision_rope_frequencies", "muse_rms_norm_stall_probe",
    "muse_residual_blend", "muse_residual", "muse_residual_gate_angles",
    "muse_residual_backward_workspace_bytes", "muse_residual_blend_backward", "muse_residual_backward",
    "muse_residual_blend_rms_norm",
)


class MuseError(RuntimeError):
    def __init__(self, status: int, fn: str, detail: str):
        self.status = status
        super().__init__(f"{fn} -> {_STATUS.get(status, status)}: {detail}")


_STATUS = {0: "MUSE_OK", 1: "MUSE_ERR_INVALID_ARGUMENT", 2: "MUSE_ERR_UNSUPPORTED", 3: "MUSE_ERR_CUDA"}

_lock = threading.Lock()
_lib = None


def load() -> ctypes.CDLL:
    """Load the library (raises OSError with a build hint when it is missing)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise OSError(f"{LIB_PATH} is not built; run `python -m gate_cores_b200.build` "
                          "(the CUDA library is required, there is no fallback)")
        lib = ctypes.CDLL(LIB_PATH)
        P, i64, i32, f32, c_int = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                   ctypes.c_float, ctypes.c_int)
        lib.muse_version.restype = c_int
        lib.muse_version.argtypes = []
        lib.muse_status_string.restype = ctypes.c_char_p
        lib.muse_status_string.argtypes = [c_int]
        lib.muse_last_error.restype = ctypes.c_char_p
        lib.muse_last_error.argtypes = []
        row = [P, P, c_int, i64, i64, i64, i64, P, f32, f32, P]
        lib.muse_rms_norm.argtypes = row
        lib.muse_input_scale_norm.argtypes = row
        lib.muse_rms_norm_stall_probe.argtypes = row[:-1] + [ctypes.c_uint32, i64, P]
        lib.muse_residual_blend.argtypes = [P, P, P, c_int, i64, i64, P, P]
        lib.muse_residual.argtypes = [P, P, P, c_int, i64, i64, P, f32, f32, P]
        lib.muse_residual_gate_angles.argtypes = [P, P, i64, f32, f32, P]
        lib.muse_residual_backward_workspace_bytes.argtypes = [i64, i64]
        lib.muse_residual_blend_rms_norm.argtypes = [P, P, P, P, c_int, c_int, i64, i64, P, P, f32, f32, P]
        lib.muse_residual_blend_backward.argtypes = [P, P, P, P, P, c_int, i64, i64, P, P, P, ctypes.c_size_t, P]
        lib.muse_residual_backward.argtypes = [P, P, P, P, P, c_int, i64, i64, P, f32, f32, P, P,
                                               ctypes.c_size_t, P]
        lib.muse_qk_norm_rope.argtypes = [P, P, P, P, c_int, c_int, i64, i64, P, i32, i64, P,
                                          i32, i32, i32, i64, i64, i64, i64, f32, f32, c_int,
                                          c_int, f32, P]
        lib.muse_output_norm_gate.argtypes = [P, P, P, c_int, i64, i32, i32, i32, f32, P]
        lib.muse_norm_residual.argtypes = [P, P, P, c_int, i64, i64, P, f32, P, c_int, f32, P]
        lib.muse_stream_copy.argtypes = [P, P, i64, P]
        lib.muse_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint), c_int]
        sz = ctypes.c_size_t
        lib.muse_norm_backward_workspace_bytes.argtypes = [i64, i64]
        rbwd = [P, P, P, c_int, i64, i64, i64, i64, i64, P, f32, f32, P, P, sz, P]
        lib.muse_rms_norm_backward.argtypes = rbwd
        lib.muse_input_scale_norm_backward.argtypes = rbwd
        lib.muse_norm_residual_backward.argtypes = [P, P, P, P, P, c_int, i64, i64, P, f32, P,
                                                    c_int, f32, P, P, P, sz, P]
        lib.muse_rms_norm_grouped.argtypes = [P, P, c_int, i64, i64, i64, i64, P, f32, P, i32, f32, P]
        lib.muse_norm_residual_rms_norm.argtypes = [P, P, P, P, c_int, c_int, i64, i64, P, f32, P,
                                                    c_int, f32, P, f32, f32, P]
        lib.muse_rms_norm_backward_noalloc.argtypes = [P, P, P, c_int, i64, i64, i64, i64, i64, P,
                                                       f32, f32, P, P]
        lib.muse_output_norm_gate_backward.argtypes = [P, P, P, P, P, c_int, i64, i32, i32, i32,
                                                       f32, P]
        lib.muse_qk_norm_rope_backward.argtypes = [P, P, P, P, P, P, c_int, c_int, i64, i64, P,
                                                   i32, i64, P, i32, i32, i32, i64, i64, i64, i64,
                                                   i64, i64, f32, f32, c_int, c_int, f32, P]
        lib.muse_vision_rope.argtypes = [P, P, P, P, c_int, i64, i32, i32, i32, i64, i64, i64, i64, P, P]
        lib.muse_vision_rope_frequencies.argtypes = [P, i32, i32, i32, f32, P]
        for name in EXPORTS[3:]:
            getattr(lib, name).restype = c_int
        lib.muse_norm_backward_workspace_bytes.restype = sz
        lib.muse_residual_backward_workspace_bytes.restype = sz
        _lib = lib
        return lib


def _call(name: str, *args) -> None:
    lib = load()
    st = getattr(lib, name)(*args)
    if st != MUSE_OK:
        raise MuseError(st, name, lib.muse_last_error().decode(errors="replace"))


def muse_version() -> int:
    return load().muse_version()


def muse_status_string(status: int) -> str:
    return load().muse_status_string(status).decode()


def muse_last_error() -> str:
    return load().muse_last_error().decode(errors="replace")


def muse_rms_norm(x, y, dtype, rows, hidden, x_row_stride, y_row_stride, gain, gain_offset,
                  eps, stream) -> None:
    _call("muse_rms_norm", x, y, dtype, rows, hidden, x_row_stride, y_row_stride, gain,
          gain_offset, eps, stream)


def muse_input_scale_norm(x, y, dtype, rows, hidden, x_row_stride, y_row_stride, gain,
                          gain_offset, eps, stream) -> None:
    _call("muse_input_scale_norm", x, y, dtype, rows, hidden, x_row_stride, y_row_stride, gain,
          gain_offset, eps, stream)


def muse_qk_norm_rope(q, k, q_out, k_out, dtype, layout, batch, seqlen, cu_seqlens, num_seqs,
                      total_tokens, positions, hq, hkv, head_dim, q_tok_stride, k_tok_stride,
                      q_out_tok_stride, k_out_tok_stride, eps, query_scale, use_rope,
                      upcast_rope, rope_base, stream) -> None:
    _call("muse_qk_norm_rope", q, k, q_out, k_out, dtype, layout, batch, seqlen, cu_seqlens,
          num_seqs, total_tokens, positions, hq, hkv, head_dim, q_tok_stride, k_tok_stride,
          q_out_tok_stride, k_out_tok_stride, eps, query_scale, int(use_rope), int(upcast_rope),
          rope_base, stream)


def muse_output_norm_gate(o, gate, y, dtype, tokens, heads, head_dim, norm_group, eps,
                          stream) -> None:
    _call("muse_output_norm_gate", o, gate, y, dtype, tokens, heads, head_dim, norm_group, eps,
          stream)


def muse_norm_residual(stream_in, branch, stream_out, branch_dtype, rows, hidden, gain,
                       gain_offset, theta, input_scale, norm_eps, stream) -> None:
    _call("muse_norm_residual", stream_in, branch, stream_out, branch_dtype, rows, hidden, gain,
          gain_offset, theta, int(input_scale), norm_eps, stream)


def muse_device_error(clear: bool = False) -> int:
    """Device-side error flags of the current device (bit 0: a bounded mbarrier
    wait in a row kernel timed out; bit 1: one in the Q/K kernel).  Synchronous."""
    flags = ctypes.c_uint(0)
    _call("muse_device_error", ctypes.byref(flags), int(clear))
    return flags.value


def muse_stream_copy(src, dst, nbytes, stream) -> None:
    _call("muse_stream_copy", src, dst, nbytes, stream)


def muse_norm_backward_workspace_bytes(rows, hidden) -> int:
    return load().muse_norm_backward_workspace_bytes(rows, hidden)


def muse_rms_norm_backward(x, dy, dx, dtype, rows, hidden, x_row_stride, dy_row_stride,
                           dx_row_stride, gain, gain_offset, eps, dgain, workspace,
                           workspace_bytes, stream) -> None:
    _call("muse_rms_norm_backward", x, dy, dx, dtype, rows, hidden, x_row_stride, dy_row_stride,
          dx_row_stride, gain, gain_offset, eps, dgain, workspace, workspace_bytes, stream)


def muse_input_scale_norm_backward(x, dy, dx, dtype, rows, hidden, x_row_stride, dy_row_stride,
                                   dx_row_stride, gain, gain_offset, eps, dgain, workspace,
                                   workspace_bytes, stream) -> None:
    _call("muse_input_scale_norm_backward", x, dy, dx, dtype, rows, hidden, x_row_stride,
          dy_row_stride, dx_row_stride, gain, gain_offset, eps, dgain, workspace, workspace_bytes,
          stream)


def muse_norm_residual_backward(stream_in, branch, dstream_out, dstream_in, dbranch, branch_dtype,
                                rows, hidden, gain, gain_offset, theta, input_scale, norm_eps,
                                dgain, dtheta, workspace, workspace_bytes, stream) -> None:
    _call("muse_norm_residual_backward", stream_in, branch, dstream_out, dstream_in, dbranch,
          branch_dtype, rows, hidden, gain, gain_offset, theta, int(input_scale), norm_eps, dgain,
          dtheta, workspace, workspace_bytes, stream)


def muse_output_norm_gate_backward(o, gate, dy, d_o, dgate, dtype, tokens, heads, head_dim,
                                   norm_group, eps, stream) -> None:
    _call("muse_output_norm_gate_backward", o, gate, dy, d_o, dgate, dtype, tokens, heads, head_dim,
          norm_group, eps, stream)


def muse_qk_norm_rope_backward(q, k, dq_out, dk_out, dq, dk, dtype, layout, batch, seqlen,
                               cu_seqlens, num_seqs, total_tokens, positions, hq, hkv, head_dim,
                               q_tok_stride, k_tok_stride, dq_out_tok_stride, dk_out_tok_stride,
                               dq_tok_stride, dk_tok_stride, eps, query_scale, use_rope, upcast_rope,
                               rope_base, stream) -> None:
    _call("muse_qk_norm_rope_backward", q, k, dq_out, dk_out, dq, dk, dtype, layout, batch, seqlen,
          cu_seqlens, num_seqs, total_tokens, positions, hq, hkv, head_dim, q_tok_stride,
          k_tok_stride, dq_out_tok_stride, dk_out_tok_stride, dq_tok_stride, dk_tok_stride, eps,
          query_scale, int(use_rope), int(upcast_rope), rope_base, stream)


def muse_rms_norm_backward_noalloc(x, dy, dx, dtype, rows, hidden, x_row_stride, dy_row_stride,
                                   dx_row_stride, gain, gain_offset, eps, dgain, stream) -> None:
    _call("muse_rms_norm_backward_noalloc", x, dy, dx, dtype, rows, hidden, x_row_stride,
          dy_row_stride, dx_row_stride, gain, gain_offset, eps, dgain, stream)


def muse_norm_residual_rms_norm(stream_in, branch, stream_out, y, branch_dtype, y_dtype, rows,
                                hidden, gain, gain_offset, theta, input_scale, norm_eps, next_gain,
                                next_gain_offset, next_eps, stream) -> None:
    _call("muse_norm_residual_rms_norm", stream_in, branch, stream_out, y, branch_dtype, y_dtype, rows,
          hidden, gain, gain_offset, theta, int(input_scale), norm_eps, next_gain, next_gain_offset,
          next_eps, stream)


def muse_rms_norm_grouped(x, y, dtype, rows, hidden, x_row_stride, y_row_stride, gains, gain_offset,
                          group_offsets, num_groups, eps, stream) -> None:
    _call("muse_rms_norm_grouped", x, y, dtype, rows, hidden, x_row_stride, y_row_stride, gains,
          gain_offset, group_offsets, num_groups, eps, stream)


def muse_vision_rope(q, k, q_out, k_out, dtype, tokens, hq, hk, head_dim, q_tok_stride, k_tok_stride,
                     q_out_tok_stride, k_out_tok_stride, freqs, stream) -> None:
    _call("muse_vision_rope", q, k, q_out, k_out, dtype, tokens, hq, hk, head_dim, q_tok_stride,
          k_tok_stride, q_out_tok_stride, k_out_tok_stride, freqs, stream)


def muse_rms_norm_stall_probe(x, y, dtype, rows, hidden, x_row_stride, y_row_stride, gain, gain_offset,
                              eps, spin_limit, stall_row, stream) -> None:
    _call("muse_rms_norm_stall_probe", x, y, dtype, rows, hidden, x_row_stride, y_row_stride, gain,
          gain_offset, eps, spin_limit, stall_row, stream)


def muse_residual_blend(stream_in, branch, stream_out, branch_dtype, rows, hidden, theta, stream) -> None:
    _call("muse_residual_blend", stream_in, branch, stream_out, branch_dtype, rows, hidden, theta, stream)


def muse_residual(stream_in, branch, stream_out, branch_dtype, rows, hidden, gate, temperature, eps,
                  stream) -> None:
    _call("muse_residual", stream_in, branch, stream_out, branch_dtype, rows, hidden, gate, temperature, eps,
          stream)


def muse_residual_backward_workspace_bytes(rows, hidden) -> int:
    return load().muse_residual_backward_workspace_bytes(rows, hidden)


def muse_residual_blend_backward(stream_in, branch, dstream_out, dstream_in, dbranch, branch_dtype, rows, hidden,
                                 theta, dtheta, workspace, workspace_bytes, stream) -> None:
    _call("muse_residual_blend_backward", stream_in, branch, dstream_out, dstream_in, dbranch, branch_dtype, rows,
          hidden, theta, dtheta, workspace, workspace_bytes, stream)


def muse_residual_backward(stream_in, branch, dstream_out, dstream_in, dbranch, branch_dtype, rows, hidden, gate,
                           temperature, eps, dgate, workspace, workspace_bytes, stream) -> None:
    _call("muse_residual_backward", stream_in, branch, dstream_out, dstream_in, dbranch, branch_dtype, rows, hidden,
          gate, temperature, eps, dgate, workspace, workspace_bytes, stream)


def muse_residual_blend_rms_norm(stream_in, branch, stream_out, y, branch_dtype, y_dtype, rows, hidden, theta,
                                 next_gain, next_gain_offset, next_eps, stream) -> None:
    _call("muse_residual_blend_rms_norm", stream_in, branch, stream_out, y, branch_dtype, y_dtype, rows, hidden,
          theta, next_gain, next_gain_offset, next_eps, stream)


def muse_residual_gate_angles(gate, theta, hidden, temperature, eps, stream) -> None:
    _call("muse_residual_gate_angles", gate, theta, hidden, temperature, eps, stream)


def muse_vision_rope_frequencies(out, head_dim, grid_h, grid_w, theta, stream) -> None:
    _call("muse_vision_rope_frequencies", out, head_dim, grid_h, grid_w, theta, stream)
