"""ITQ3_S-style 3-bit weight path with a 256-wide Walsh-Hadamard rotation (oracle).

Cites: ITQ3_S article, section "核心技术：FWHT预旋转与TurboQuant的完美融合":
before the 3-bit quantiser, every 256-dimensional weight vector is rotated with
the fast Walsh-Hadamard transform, which spreads outlier energy so the rotated
values are close to Gaussian; the codes are uniform; an exact inverse transform,
fused into the shared-memory load of the GPU kernel, restores the rotated
weights at inference ("zero-error round trip" of the transform itself).

Readings (the article prints no formulas):
  * A block is 256 consecutive d_in weights of one output row.
  * Rotation r = H_256 w / 16 (orthonormal; the 1/16 is exact in binary).
  * Eight uniform mid-rise levels (c - 3.5) * s, c in 0..7, s = fp16(amax|r| / 3.5),
    c = clamp(rint(r / s + 3.5), 0, 7), all in fp64; c = 0 when s = 0.  (The
    article's "三值" -- ternary -- is read as a slip for the 3-bit code.)
  * Dequantised weight w_hat = H_256 ((c - 3.5) s) / 16 (H/16 is its own inverse).
"""
from __future__ import annotations

import numpy as np

from ._checks import require_finite
from .transforms import fwht

BLOCK = 256


def rotate(w_rows: np.ndarray) -> np.ndarray:
    require_finite("rotate", w_rows)
    w = np.asarray(w_rows, dtype=np.float64)
    d_out, d_in = w.shape
    if d_in % BLOCK:
        raise ValueError("d_in must be a multiple of 256")
    return (fwht(w.reshape(d_out, d_in // BLOCK, BLOCK)) / 16.0).reshape(d_out, d_in)


def quantize(w_rows: np.ndarray):
    """(codes uint8 [d_out, d_in] in 0..7, scales fp16 [d_out, d_in/256])."""
    r = rotate(w_rows)
    d_out, d_in = r.shape
    rb = r.reshape(d_out, d_in // BLOCK, BLOCK)
    amax = np.max(np.abs(rb), axis=2)
    s16 = (amax / 3.5).astype(np.float16)
    s = s16.astype(np.float64)
    safe = np.where(s == 0, 1.0, s)
    c = np.clip(np.rint(rb / safe[..., None] + 3.5), 0, 7)
    c = np.where((s == 0)[..., None], 0, c)
    return c.astype(np.uint8).reshape(d_out, d_in), s16


def rotated_levels(codes: np.ndarray, scales16: np.ndarray) -> np.ndarray:
    """(c - 3.5) * s per element, fp64: the quantised weights in the rotated domain."""
    d_out, d_in = codes.shape
    c = codes.astype(np.float64).reshape(d_out, d_in // BLOCK, BLOCK)
    return ((c - 3.5) * scales16.astype(np.float64)[..., None]).reshape(d_out, d_in)


def dequantize(codes: np.ndarray, scales16: np.ndarray) -> np.ndarray:
    """w_hat = H_256 ((c - 3.5) s) / 16 per block, fp64 [d_out, d_in]."""
    lv = rotated_levels(codes, scales16)
    d_out, d_in = lv.shape
    return (fwht(lv.reshape(d_out, d_in // BLOCK, BLOCK)) / 16.0).reshape(d_out, d_in)


def gemv(codes: np.ndarray, scales16: np.ndarray, x_rows: np.ndarray) -> np.ndarray:
    """y[t, o] = sum_k w_hat[o, k] x[t, k], fp64; x_rows [tokens, d_in]."""
    require_finite("gemv", scales16, x_rows)
    return np.asarray(x_rows, dtype=np.float64) @ dequantize(codes, scales16).T
