"""Element and scale number formats (oracle).

The WUSH news article's experiments paragraph and the AI Radio episode name the
formats MXFP4, NVFP4 and INT4 but print none of their rules. The readings used
here are the published format definitions:

  * E2M1 (FP4 element of MXFP4 and NVFP4): sign bit, 2 exponent bits, 1
    mantissa bit, no inf/NaN. Magnitudes by 3-bit code 0..7:
    0, 0.5, 1, 1.5, 2, 3, 4, 6. Code = sign << 3 | magnitude code.
  * E4M3 (the "fn" variant: no inf, 0x7F/0xFF NaN), bias 7, largest finite 448,
    smallest subnormal 2^-9.  Used unsigned (UE4M3) for NVFP4 block scales.
  * E8M0 (UE8M0): a biased power of two, value 2^(byte - 127), byte 0xFF NaN.
  * fp16 for the INT4 group scale.

Rounding everywhere is round-to-nearest, ties to the even code (the code whose
mantissa LSB is 0), saturating at the largest finite magnitude ("satfinite").
"""
from __future__ import annotations

import numpy as np

# E2M1 magnitudes indexed by their 3-bit code.
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E2M1_MAX = 6.0


def _e4m3_grid() -> np.ndarray:
    """All finite non-negative E4M3 values, indexed by their 7-bit code 0..126."""
    vals = []
    for code in range(127):
        e = code >> 3
        m = code & 7
        if e == 0:
            vals.append(m * 2.0 ** -9)                 # subnormal: m/8 * 2^(1-7)
        else:
            vals.append((1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals)


E4M3_GRID = _e4m3_grid()
E4M3_MAX = 448.0


def round_to_grid(mag: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the nearest grid value to each non-negative ``mag``.

    ``grid`` is sorted ascending and indexed by code, so an even index is an even
    code. An exact midpoint goes to the even index; magnitudes above the last
    grid value saturate to it.
    """
    mag = np.asarray(mag, dtype=np.float64)
    hi = np.searchsorted(grid, mag, side="left")          # first grid value >= mag
    hi = np.clip(hi, 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    d_lo = np.abs(mag - grid[lo])
    d_hi = np.abs(grid[hi] - mag)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(mag >= grid[-1], len(grid) - 1, idx)
    return idx.astype(np.int64)


def e2m1_code(v: np.ndarray) -> np.ndarray:
    """4-bit E2M1 code of each value: RNE onto the grid, saturating at 6.

    The sign bit is the sign bit of the input, also when the magnitude rounds to
    zero (a negative value in (-0.25, 0] gives code 0x8, i.e. -0).
    """
    v = np.asarray(v, dtype=np.float64)
    mag_code = round_to_grid(np.abs(v), E2M1_GRID)
    sign = np.signbit(v).astype(np.int64)
    return (sign << 3 | mag_code).astype(np.uint8)


def e2m1_value(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code).astype(np.int64)
    mag = E2M1_GRID[code & 7]
    return np.where(code & 8, -mag, mag)


def e4m3_code_unsigned(v: np.ndarray) -> np.ndarray:
    """7-bit UE4M3 code of each non-negative value, RNE with saturation at 448."""
    v = np.asarray(v, dtype=np.float64)
    if np.any(v < 0):
        raise ValueError("UE4M3 takes non-negative values")
    return round_to_grid(v, E4M3_GRID).astype(np.uint8)


def e4m3_value(code: np.ndarray) -> np.ndarray:
    return E4M3_GRID[np.asarray(code).astype(np.int64) & 0x7F]


def e8m0_value(byte: np.ndarray) -> np.ndarray:
    return np.ldexp(1.0, np.asarray(byte).astype(np.int64) - 127)


def fp16_rne_sat(v: np.ndarray) -> np.ndarray:
    """Round fp32/fp64 values to fp16 (RNE), clamping magnitudes to 65504."""
    v = np.clip(np.asarray(v, dtype=np.float64), -65504.0, 65504.0)
    return v.astype(np.float16)


# Rounding boundaries (midpoints between adjacent representable magnitudes) that
# the parity tests use to find elements whose code depends on the last bits of
# the pre-rounding value.
E2M1_MIDPOINTS = (E2M1_GRID[:-1] + E2M1_GRID[1:]) / 2.0
# An E2M1 code also carries the sign of a value that rounds to zero magnitude, so
# zero is a decision boundary of the code as well.
E2M1_BOUNDARIES = np.concatenate([[0.0], E2M1_MIDPOINTS])
INT4_MIDPOINTS = np.arange(7) + 0.5                        # 0.5 .. 6.5
E4M3_MIDPOINTS = (E4M3_GRID[:-1] + E4M3_GRID[1:]) / 2.0


def distance_to_boundary(mag: np.ndarray, midpoints: np.ndarray) -> np.ndarray:
    """|mag - nearest midpoint| for each non-negative magnitude."""
    mag = np.asarray(mag, dtype=np.float64)
    i = np.clip(np.searchsorted(midpoints, mag), 1, len(midpoints) - 1)
    return np.minimum(np.abs(mag - midpoints[i - 1]), np.abs(mag - midpoints[i]))
