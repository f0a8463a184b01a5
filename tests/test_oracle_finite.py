"""The oracle refuses NaN and infinite inputs at every public entry point.

Block moments, absolute maxima and scale exponents are undefined for them, so a
silent answer would be meaningless; each case below plants one bad value in an
otherwise valid input."""
import numpy as np
import pytest

from oracle import calibrate as C
from oracle import gemm as G
from oracle import itq3 as I
from oracle import loss as L
from oracle import quant as Q
from oracle import transforms as T
from oracle._checks import NonFiniteInput


def _planted(shape, bad, seed=3):
    a = np.random.default_rng(seed).standard_normal(shape)
    a.flat[len(a.flat) // 2] = bad
    return a


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
def test_entry_points_reject_non_finite(bad):
    x = _planted((8, 64), bad)
    ok = np.random.default_rng(4).standard_normal((8, 64))
    t = T.identity_blocks(64, 32)
    sig = np.stack([np.eye(32)] * 2)
    cases = [
        lambda: C.block_moments(x, 32),
        lambda: C.calibrate(x, ok, 32, "wush"),
        lambda: C.calibrate(ok, x, 32, "wush"),
        lambda: C.transforms_from_moments(_planted((2, 32, 32), bad), sig, "wush"),
        lambda: C.nvfp4_global_scale(x),
        lambda: C.nvfp4_dynamic_global_scale(x.astype(np.float32)),
        lambda: C.group_blocks(sig, _planted((2, 32, 32), bad), 1),
        lambda: C.shared_transforms(_planted((2, 32, 32), bad), sig, "wush", 1),
        lambda: Q.quantize_mxfp4(x.astype(np.float32)),
        lambda: Q.quantize_nvfp4(x[:, :32].astype(np.float32), 0.01),
        lambda: Q.quantize_nvfp4(ok[:, :32].astype(np.float32), bad),
        lambda: Q.quantize_int4(x.astype(np.float32)),
        lambda: Q.transform_quantize(x, t, "mxfp4"),
        lambda: Q.transform_quantize(ok, _planted(t.shape, bad), "int4"),
        lambda: T.fwht(x),
        lambda: T.apply_block_transform(x, t),
        lambda: T.block_magnitude(ok, _planted(t.shape, bad)),
        lambda: G.gemm_dequantized(x, ok),
        lambda: G.gemm_dequantized(ok, ok, bad),
        lambda: I.rotate(_planted((2, 256), bad)),
        lambda: I.quantize(_planted((2, 256), bad)),
        lambda: L.output_loss(x, ok),
        lambda: L.layer_loss(x, ok, t, t, "mxfp4"),
    ]
    for i, call in enumerate(cases):
        with pytest.raises(NonFiniteInput):
            call()
            pytest.fail(f"case {i} accepted a non-finite input")


def test_itq3_gemv_rejects_non_finite_activations():
    c, s = I.quantize(np.random.default_rng(5).standard_normal((4, 256)) * 0.02)
    I.gemv(c, s, np.ones((1, 256)))                  # finite: accepted
    with pytest.raises(NonFiniteInput):
        I.gemv(c, s, _planted((1, 256), np.nan))


def test_finite_extremes_are_accepted():
    # the largest and smallest finite magnitudes are valid inputs
    y = np.zeros((1, 32), np.float32)
    y[0, 0], y[0, 1] = np.finfo(np.float32).max, np.finfo(np.float32).tiny
    assert Q.quantize_mxfp4(y)["scale_bytes"][0, 0] == 127 + 125
