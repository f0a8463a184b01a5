"""GEMM on dequantised operands (oracle).

Cites: AI Radio episode, "Conclusion" (the FP4 MatMul that gives the per-layer
speed-up) and "Problem Setup and Goal" (the product q(T_W W)^T q(T_X X)).

Storage follows the CUDA path: activations X^T as [tokens, d_in] (M x K), weights
W^T as [d_out, d_in] (N x K), output y^T as [tokens, d_out] (M x N):
    y[t, o] = alpha * sum_k a[t, k] * b[o, k]
in fp64 on the dequantised operand values.
"""
from __future__ import annotations

import numpy as np

from ._checks import require_finite


def gemm_dequantized(a_dq: np.ndarray, b_dq: np.ndarray, alpha: float = 1.0) -> np.ndarray:
    require_finite("gemm_dequantized", a_dq, b_dq, alpha)
    a = np.asarray(a_dq, dtype=np.float64)
    b = np.asarray(b_dq, dtype=np.float64)
    if a.shape[1] != b.shape[1]:
        raise ValueError("K mismatch")
    return float(alpha) * (a @ b.T)
