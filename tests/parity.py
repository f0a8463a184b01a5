"""Parity helpers: decode the library's byte layouts and compare against the oracle.

The decoders restate the layouts documented in include/wush.h; they are test
code, written independently of both the CUDA kernels and the oracle.
"""
from __future__ import annotations

import os

import numpy as np

from oracle import quant as Q
from oracle import transforms as T

# Element-code and scale decisions closer than this (relative to the size of the
# terms summed to form the value) to a rounding boundary may differ between the
# fp32 kernel and the fp64-then-fp32 oracle; they are counted, not compared.
BOUNDARY_TOL = 1e-6
# Transformed fp32 values: |gpu - oracle| <= Y_TOL * sum_k |T_ik x_k|.
Y_TOL = 1e-5
# At most this fraction of elements may differ from the oracle by way of a
# boundary-window exemption (mismatches excused; exact agreement inside a window
# needs no excuse and is not counted against the budget).
MAX_EXEMPT_FRACTION = 1e-4
GEMM_REL_FRO = 1e-3

# Boundary-window counts of every comparison made in this process: the session
# report in conftest prints them per test and per format (and writes them as JSON
# to $WUSH_PARITY_REPORT when that is set).
WINDOW_LOG: list = []


def unpack_nibbles(packed: np.ndarray, rows: int, d_in: int) -> np.ndarray:
    b = np.asarray(packed, dtype=np.uint8).reshape(rows, d_in // 2)
    out = np.empty((rows, d_in), np.uint8)
    out[:, 0::2] = b & 0xF
    out[:, 1::2] = b >> 4
    return out


def unswizzle_scales(buf: np.ndarray, rows: int, n_cols: int) -> np.ndarray:
    """[rows, n_cols] scale bytes from the 128x4-atom MMA scale-factor layout."""
    buf = np.asarray(buf, dtype=np.uint8)
    n_atom_cols = (n_cols + 3) // 4
    r = np.arange(rows)[:, None]
    c = np.arange(n_cols)[None, :]
    off = ((r // 128) * n_atom_cols + c // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (c % 4)
    return buf[off]


def swizzle_scales(scales: np.ndarray) -> np.ndarray:
    """Inverse of unswizzle_scales (pads rows to 128 and columns to 4 with zeros)."""
    rows, n_cols = scales.shape
    n_atom_rows, n_atom_cols = (rows + 127) // 128, (n_cols + 3) // 4
    buf = np.zeros(n_atom_rows * n_atom_cols * 512, np.uint8)
    r = np.arange(rows)[:, None]
    c = np.arange(n_cols)[None, :]
    off = ((r // 128) * n_atom_cols + c // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (c % 4)
    buf[off] = scales
    return buf


def decode_scales(buf: np.ndarray, rows: int, d_in: int, fmt: str) -> np.ndarray:
    nb = d_in // Q.BLOCK[fmt]
    if fmt == "int4":
        return np.asarray(buf, dtype=np.uint8)[: rows * nb * 2].view(np.float16).reshape(rows, nb)
    return unswizzle_scales(buf, rows, nb)


def magnitude(x_rows: np.ndarray, t: np.ndarray) -> np.ndarray:
    return T.block_magnitude(x_rows, t)


def compare_transform_quant(x_rows, t, fmt, gs, codes_gpu, scales_gpu, y_gpu=None, rows_sel=None, strict=False):
    """Compare GPU outputs for rows ``rows_sel`` (all if None) of x_rows against the oracle.

    Returns a dict of counts; raises AssertionError on any non-exempt mismatch.
    codes_gpu/scales_gpu/y_gpu are already decoded to [rows, d_in] / [rows, nb] / [rows, d_in].
    ``strict``: every code and scale must equal the oracle's (for inputs whose
    transformed values are exact in fp32 on both sides, e.g. the identity transform).
    """
    x = np.asarray(x_rows, dtype=np.float64)
    if rows_sel is not None:
        x = x[rows_sel]
        codes_gpu = codes_gpu[rows_sel]
        scales_gpu = scales_gpu[rows_sel]
        y_gpu = None if y_gpu is None else y_gpu[rows_sel]
    b = Q.BLOCK[fmt]
    ref = Q.transform_quantize(x, t, fmt, gs)
    mag = magnitude(x, t)
    rows, d_in = x.shape
    nb = d_in // b
    out = {"elements": rows * d_in}
    if y_gpu is not None:
        err = np.abs(np.asarray(y_gpu, np.float64) - ref["y64"])
        bad = err > Y_TOL * mag
        out["y_max_rel"] = float(np.max(err / np.maximum(mag, 1e-300)))
        assert not bad.any(), f"transformed values off at {np.argwhere(bad)[:5]}: max rel {out['y_max_rel']}"
    # scale decisions
    mag_b = mag.reshape(rows, nb, b)
    yb = np.abs(ref["y32"].reshape(rows, nb, b))
    amax_i = np.argmax(yb, axis=2)
    mag_amax = np.take_along_axis(mag_b, amax_i[..., None], axis=2)[..., 0]
    blk_exempt = ref["block_margin"] <= BOUNDARY_TOL * mag_amax
    if fmt == "int4":
        want_sc = ref["scale_fp16"].view(np.uint16)
        got_sc = np.asarray(scales_gpu).view(np.uint16)
    else:
        want_sc = ref["scale_bytes"]
        got_sc = np.asarray(scales_gpu, np.uint8)
    sc_bad = (want_sc != got_sc) & ~blk_exempt
    assert not sc_bad.any(), (f"{int(sc_bad.sum())} scale mismatches, first at "
                              f"{np.argwhere(sc_bad)[:5].tolist()}: want {want_sc[sc_bad][:5]}, got {got_sc[sc_bad][:5]}")
    # element codes
    el_exempt = (ref["elem_margin"] <= BOUNDARY_TOL * mag) | np.repeat(blk_exempt, b, axis=1)
    code_bad = (ref["codes"] != codes_gpu) & ~el_exempt
    assert not code_bad.any(), (f"{int(code_bad.sum())} code mismatches, first at "
                                f"{np.argwhere(code_bad)[:5].tolist()}: want {ref['codes'][code_bad][:8]}, "
                                f"got {codes_gpu[code_bad][:8]}")
    out["in_window"] = int(el_exempt.sum())
    out["exempt"] = int(((ref["codes"] != codes_gpu) & el_exempt).sum())
    out["scale_exempt"] = int(((want_sc != got_sc) & blk_exempt).sum())
    out["blocks"] = rows * nb
    out["scale_in_window"] = int(blk_exempt.sum())
    WINDOW_LOG.append(dict(out, fmt=fmt, rows=rows, d_in=d_in,
                           test=os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]))
    assert out["exempt"] <= max(MAX_EXEMPT_FRACTION * out["elements"], 1), out
    if strict:
        assert out["exempt"] == 0 and out["scale_exempt"] == 0, out
    return out
