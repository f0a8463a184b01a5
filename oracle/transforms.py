"""Hadamard matrices, the fast Walsh-Hadamard transform and block transforms (oracle).

Cites:
  * WUSH news article, paragraph 2 (Hadamard as the data-agnostic baseline) and
    paragraph 3 (WUSH keeps a block-diagonal structure so blocks transform
    independently).
  * ITQ3_S article, section "核心技术：FWHT预旋转与TurboQuant的完美融合" (the
    fast Walsh-Hadamard transform on each 256-element weight vector).
"""
from __future__ import annotations

import numpy as np

from ._checks import require_finite


def sylvester_hadamard(n: int) -> np.ndarray:
    """The n x n Sylvester Hadamard matrix (entries +-1, H H^T = n I); n a power of 2.

    H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]].
    """
    if n < 1 or n & (n - 1):
        raise ValueError("n must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def normalized_hadamard(n: int) -> np.ndarray:
    """H_n / sqrt(n): symmetric and orthogonal."""
    return sylvester_hadamard(n) / np.sqrt(n)


def fwht(x: np.ndarray) -> np.ndarray:
    """Unnormalised fast Walsh-Hadamard transform along the last axis.

    log2(n) butterfly stages (a, b) -> (a + b, a - b) with stride 1, 2, 4, ...;
    the result equals sylvester_hadamard(n) @ x for each vector.
    """
    require_finite("fwht", x)
    y = np.array(x, dtype=np.float64, copy=True)
    n = y.shape[-1]
    if n & (n - 1):
        raise ValueError("length must be a power of two")
    h = 1
    while h < n:
        y = y.reshape(y.shape[:-1] + (n // (2 * h), 2, h))
        a = y[..., 0, :].copy()
        b = y[..., 1, :].copy()
        y[..., 0, :] = a + b
        y[..., 1, :] = a - b
        y = y.reshape(y.shape[:-3] + (n,))
        h *= 2
    return y


def apply_block_transform(x_rows: np.ndarray, t: np.ndarray) -> np.ndarray:
    """Apply a block-diagonal transform to every row, in fp64.

    x_rows: [rows, d_in] (a row is one token of X, or one output column of W);
    t: [d_in / b, b, b]; block j of a row, x_j = row[j*b:(j+1)*b], becomes
    y_j = t[j] @ x_j.  Returns [rows, d_in] fp64.
    """
    require_finite("apply_block_transform", x_rows, t)
    x = np.asarray(x_rows, dtype=np.float64)
    nb, b, _ = t.shape
    rows = x.shape[0]
    xb = x.reshape(rows, nb, b)
    y = np.einsum("jik,rjk->rji", np.asarray(t, dtype=np.float64), xb)
    return y.reshape(rows, nb * b)


def block_magnitude(x_rows: np.ndarray, t: np.ndarray) -> np.ndarray:
    """sum_k |t[j][i][k] * x_j[k]| for every output element (the size of the terms
    summed to form it); the parity tests measure rounding error against this."""
    require_finite("block_magnitude", x_rows, t)
    return apply_block_transform(np.abs(x_rows), np.abs(t))


def hadamard_blocks(d_in: int, b: int) -> np.ndarray:
    """Block-diagonal transform with every block H_b / sqrt(b), as [d_in/b, b, b]."""
    return np.broadcast_to(normalized_hadamard(b), (d_in // b, b, b)).copy()


def identity_blocks(d_in: int, b: int) -> np.ndarray:
    return np.broadcast_to(np.eye(b), (d_in // b, b, b)).copy()
