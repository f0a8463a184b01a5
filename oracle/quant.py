"""Microscaled block quantisers: MXFP4, NVFP4, INT4 (oracle).

Test infrastructure: only the tests, the smoke check and the benchmark's CPU
legs use this module; the library never does.

Cites: WUSH news article, paragraph 5 (layer-wise loss measured with the MXFP4,
NVFP4 and INT4 formats) and AI Radio episode, "Conclusion" (MXFP4, INT4).  The
pages name the formats only; the rules below are the published format
definitions, written as plain quotients and evaluated in fp64.

Input to every quantiser is the transformed tensor as fp32, [rows, d_in], blocks
of ``b`` consecutive d_in elements of a row.  Each decision that turns a number
into an integer (a block scale, an element code) rounds the exact quotient once,
to nearest with ties to even:

MXFP4 (b = 32): amax = max |y|; e = floor(log2 amax) - 2, clamped to
  [-127, 127] (e = -127 when amax = 0); scale byte = e + 127 (UE8M0);
  code = E2M1_RNE_sat(y / 2^e).  (OCP MX: shared exponent = floor(log2 amax)
  minus the element format's largest exponent, 2 for E2M1.)
NVFP4 (b = 16), with the per-tensor fp32 scale s_g:
  s_b = UE4M3_RNE_sat(amax / (6 s_g));  d = s_b s_g;  code = E2M1_RNE_sat(y / d);
  codes 0 when s_b = 0.  Dequantised value = E2M1(code) * s_b * s_g.
INT4 (b = 32), symmetric: s = fp16_RNE(amax / 7); q = clamp(RNE(y / s), -7, 7);
  q = 0 when s = 0.  Dequantised q * s.

Why fp64 decides these exactly: y is fp32 (24 significant bits), s_g is fp32,
a UE4M3 value has at most 4 significant bits and an fp16 scale 11, and every
rounding boundary (E2M1 and INT4 midpoints, E4M3 and fp16 midpoints) has a short
significand.  A quotient that is not exactly on a boundary therefore lies at
least about 2^-32 relative away from it, while an fp64 quotient is within 2^-53
of the real one; an exact boundary is representable and comes out exact.  So
these fp64 expressions give the real-number result, ties included (checked
against exact rational arithmetic in the pins).

A block whose amax is 0 gets codes +0.  Otherwise the E2M1 sign bit is the sign
bit of y, also when the magnitude rounds to 0.

Each quantiser also returns, for the parity tests, the distance (in units of y)
from every element to the nearest rounding boundary of its code and from every
block's amax to the nearest boundary of its scale decision.
"""
from __future__ import annotations

import numpy as np

from ._checks import require_finite
from .formats import (E2M1_BOUNDARIES, E4M3_MIDPOINTS, INT4_MIDPOINTS, distance_to_boundary,
                      e2m1_code, e2m1_value, e4m3_code_unsigned, e4m3_value, fp16_rne_sat)

F32 = np.float32


def _blocks(y32: np.ndarray, b: int) -> np.ndarray:
    y = np.asarray(y32)
    if y.dtype != np.float32:
        raise TypeError("quantisers take the fp32 transformed tensor")
    rows, d = y.shape
    if d % b:
        raise ValueError("d_in must be a multiple of the block size")
    return y.reshape(rows, d // b, b)


def quantize_mxfp4(y32: np.ndarray) -> dict:
    require_finite("quantize_mxfp4", y32)
    yb = _blocks(y32, 32).astype(np.float64)
    amax = np.max(np.abs(yb), axis=2)
    _, p = np.frexp(amax)                       # amax = f * 2^p, f in [0.5, 1)
    e = np.clip(p - 1 - 2, -127, 127)
    e = np.where(amax == 0, -127, e)
    scale = np.ldexp(1.0, e)
    v = yb / scale[..., None]                    # exact: division by a power of 2
    codes = e2m1_code(v)
    codes = np.where((amax == 0)[..., None], 0, codes).astype(np.uint8)
    dq = e2m1_value(codes) * scale[..., None]
    elem_margin = distance_to_boundary(np.abs(v), E2M1_BOUNDARIES) * scale[..., None]
    # scale decision flips where amax crosses a power of two
    lo = np.ldexp(1.0, p - 1)
    block_margin = np.where(amax == 0, np.inf, np.minimum(amax - lo, 2 * lo - amax))
    rows = yb.shape[0]
    return dict(codes=codes.reshape(rows, -1), scale_bytes=(e + 127).astype(np.uint8),
                scale=scale, dq=dq.reshape(rows, -1),
                elem_margin=elem_margin.reshape(rows, -1), block_margin=block_margin)


def quantize_nvfp4(y32: np.ndarray, s_g) -> dict:
    require_finite("quantize_nvfp4", y32, s_g)
    yb = _blocks(y32, 16).astype(np.float64)
    s_g = np.float64(F32(s_g))                   # the per-tensor scale is an fp32 number
    amax = np.max(np.abs(yb), axis=2)
    den = 6.0 * s_g                              # exact in fp64
    t = amax / den
    sb = e4m3_code_unsigned(t)
    d = e4m3_value(sb) * s_g                     # exact: 4 x 24 significant bits
    live = (sb != 0) & (amax > 0)
    v = yb / np.where(live, d, 1.0)[..., None]
    codes = e2m1_code(v)
    codes = np.where(live[..., None], codes, 0).astype(np.uint8)
    dq = e2m1_value(codes) * d[..., None]
    elem_margin = np.where(live[..., None],
                           distance_to_boundary(np.abs(v), E2M1_BOUNDARIES) * d[..., None], np.inf)
    block_margin = distance_to_boundary(t, E4M3_MIDPOINTS) * den
    rows = yb.shape[0]
    return dict(codes=codes.reshape(rows, -1), scale_bytes=sb, scale=e4m3_value(sb),
                global_scale=F32(s_g), dq=dq.reshape(rows, -1),
                elem_margin=elem_margin.reshape(rows, -1), block_margin=block_margin)


def _fp16_midpoint_distance(v: np.ndarray) -> np.ndarray:
    """Distance from each non-negative value to the nearest fp16 rounding boundary."""
    v = np.asarray(v, dtype=np.float64)
    h = v.astype(np.float16).astype(np.float64)
    up = np.nextafter(h.astype(np.float16), np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(h.astype(np.float16), np.float16(0)).astype(np.float64)
    return np.minimum(np.abs(v - (h + up) / 2), np.abs(v - (h + dn) / 2))


def quantize_int4(y32: np.ndarray) -> dict:
    require_finite("quantize_int4", y32)
    yb = _blocks(y32, 32).astype(np.float64)
    amax = np.max(np.abs(yb), axis=2)
    pre = amax / 7.0
    s16 = fp16_rne_sat(pre)
    s = s16.astype(np.float64)
    live = s > 0
    v = yb / np.where(live, s, 1.0)[..., None]
    q = np.clip(np.rint(v), -7, 7).astype(np.int64)
    q = np.where(live[..., None], q, 0)
    dq = q * s[..., None]
    elem_margin = np.where(live[..., None],
                           distance_to_boundary(np.abs(v), INT4_MIDPOINTS) * s[..., None], np.inf)
    block_margin = _fp16_midpoint_distance(pre) * 7.0
    rows = yb.shape[0]
    return dict(codes=(q & 0xF).astype(np.uint8).reshape(rows, -1), q=q.reshape(rows, -1),
                scale_fp16=s16, scale=s, dq=dq.reshape(rows, -1),
                elem_margin=elem_margin.reshape(rows, -1), block_margin=block_margin)


def quantize(y32: np.ndarray, fmt: str, global_scale=None) -> dict:
    if fmt == "mxfp4":
        return quantize_mxfp4(y32)
    if fmt == "nvfp4":
        return quantize_nvfp4(y32, global_scale)
    if fmt == "int4":
        return quantize_int4(y32)
    raise ValueError(fmt)


BLOCK = {"mxfp4": 32, "nvfp4": 16, "int4": 32}


def transform_quantize(x_rows: np.ndarray, t: np.ndarray, fmt: str, global_scale=None) -> dict:
    """Transform every row block with t (fp64), round to fp32, then quantise.

    The fp32 rounding of the transformed value is the precision the CUDA kernel
    holds it in before its quantisation decisions.
    """
    from .transforms import apply_block_transform
    y64 = apply_block_transform(x_rows, t)
    y32 = y64.astype(np.float32)
    out = quantize(y32, fmt, global_scale)
    out["y64"] = y64
    out["y32"] = y32
    return out
