"""B200-native (sm_100a) fused per-token normalisation cores of the Muse Spark
Open decoder layer, behind the C ABI declared in include/muse_cores.h.

    from gate_cores_b200 import rms_norm, input_scale_norm, qk_norm_rope, \\
        output_norm_gate, norm_residual

Every call runs in libmuse_cores.so (built by ``python -m gate_cores_b200.build``);
without the library the first call raises - there is no CPU fallback.
"""
from ._lib import MuseError, load as load_library  # noqa: F401
from .cores import (  # noqa: F401
    input_scale_norm,
    norm_residual,
    output_norm_gate,
    qk_norm_rope,
    residual,
    residual_blend,
    residual_gate_angles,
    rms_norm,
    stream_copy,
)

__all__ = ["rms_norm", "input_scale_norm", "qk_norm_rope", "output_norm_gate", "norm_residual",
           "residual_blend", "residual", "residual_gate_angles", "stream_copy", "MuseError",
           "load_library"]
