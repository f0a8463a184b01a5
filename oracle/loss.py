"""The layer output loss (oracle).

Cites: AI Radio episode, "Problem Setup and Goal": T_W and T_X minimise the L2
output loss of the quantised product against W^T X, averaged over d_out and the
batch.  The extracted formula lost its norm bars and exponent; it is read as
    l = || q(T_W W)^T q(T_X X) - W^T X ||_F^2 / (d_out * d_batch).
"""
from __future__ import annotations

import numpy as np

from ._checks import require_finite
from .calibrate import nvfp4_global_scale
from .quant import transform_quantize


def output_loss(y_quant: np.ndarray, y_ref: np.ndarray) -> float:
    require_finite("output_loss", y_quant, y_ref)
    d = np.asarray(y_quant, dtype=np.float64) - np.asarray(y_ref, dtype=np.float64)
    return float(np.sum(d * d) / d.size)


def layer_loss(x_rows, w_rows, t_x, t_w, fmt: str, x_global_scale=None) -> float:
    """Loss of one quantised linear layer on activations x_rows [tokens, d_in]
    and weights w_rows [d_out, d_in], with transforms t_x, t_w [d_in/b, b, b]."""
    require_finite("layer_loss", x_rows, w_rows, t_x, t_w)
    w_global = None
    if fmt == "nvfp4":
        from .transforms import apply_block_transform
        w_global = nvfp4_global_scale(apply_block_transform(w_rows, t_w).astype(np.float32))
        if x_global_scale is None:
            x_global_scale = nvfp4_global_scale(apply_block_transform(x_rows, t_x).astype(np.float32))
    qx = transform_quantize(x_rows, t_x, fmt, x_global_scale)
    qw = transform_quantize(w_rows, t_w, fmt, w_global)
    y_q = qx["dq"] @ qw["dq"].T
    y_ref = np.asarray(x_rows, dtype=np.float64) @ np.asarray(w_rows, dtype=np.float64).T
    return output_loss(y_q, y_ref)
