"""Input check for the oracle's entry points (test infrastructure).

The method is defined on real numbers: a calibration set, a weight matrix or an
activation batch holding NaN or an infinity has no block moments, no absolute
maximum and no scale exponent.  The oracle refuses such inputs instead of
returning an arbitrary answer.  (The host library rejects them as well; the
device kernels leave their codes unspecified.)
"""
from __future__ import annotations

import numpy as np


class NonFiniteInput(ValueError):
    """An input array holds NaN or an infinity."""


def require_finite(what: str, *arrays) -> None:
    for a in arrays:
        if a is None:
            continue
        v = np.asarray(a)
        if v.dtype.kind in "fc" and not np.isfinite(v).all():
            raise NonFiniteInput(f"{what}: input holds NaN or an infinity")
