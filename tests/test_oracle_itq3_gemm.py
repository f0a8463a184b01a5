"""Pins for oracle.itq3, oracle.gemm and oracle.loss."""
import numpy as np

import synth
from oracle import gemm as G
from oracle import itq3 as I
from oracle import loss as L
from oracle import transforms as T


def _w(rows=8, d=512, seed=7):
    rng = np.random.default_rng(seed)
    w = rng.standard_t(4, size=(rows, d)) * 0.02
    return w.astype(np.float16).astype(np.float64)


def test_rotation_is_orthonormal_and_exact():
    w = _w()
    r = I.rotate(w)
    assert np.allclose(np.sum(r * r, axis=1), np.sum(w * w, axis=1), rtol=1e-13)
    # fp16 inputs: the butterflies and the /16 are exact in fp64
    assert np.array_equal(I.rotate(r), w)


def test_codes_and_error_bound():
    w = _w()
    c, s = I.quantize(w)
    assert c.min() >= 0 and c.max() <= 7
    r = I.rotate(w).reshape(8, 2, 256)
    lv = I.rotated_levels(c, s).reshape(8, 2, 256)
    sv = s.astype(np.float64)[..., None]
    assert np.all(np.abs(r - lv) <= sv / 2 * (1 + 1e-12) + np.abs(r) * 1e-3)
    # the element of largest |r| lands on an end level (c = 0 or 7)
    i = np.argmax(np.abs(r), axis=2)
    ends = np.take_along_axis(c.reshape(8, 2, 256), i[..., None], axis=2)
    assert np.all((ends == 0) | (ends == 7))


def test_zero_error_round_trip_and_idempotence():
    w = _w()
    c, s = I.quantize(w)
    w_hat = I.dequantize(c, s)
    assert np.array_equal(I.rotate(w_hat), I.rotated_levels(c, s))
    c2, s2 = I.quantize(w_hat)
    assert np.array_equal(c2, c) and np.array_equal(s2, s)


def test_fp64_to_fp16_is_single_rounding():
    # values one fp64 ulp either side of every fp16 midpoint round to the near side
    allh = np.arange(0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = (allh[1:] + allh[:-1]) / 2
    below, above = np.nextafter(mids, 0), np.nextafter(mids, 1e9)
    assert np.array_equal(below.astype(np.float16).astype(np.float64), allh[:-1])
    assert np.array_equal(above.astype(np.float16).astype(np.float64), allh[1:])


def test_gemv_brute_force():
    w = _w(rows=3, d=256)
    c, s = I.quantize(w)
    x = np.random.default_rng(8).standard_normal((2, 256))
    y = I.gemv(c, s, x)
    h = T.sylvester_hadamard(256) / 16
    for o in range(3):
        lv = (c[o].astype(np.float64) - 3.5) * float(s[o, 0])
        wh = h @ lv
        for t in range(2):
            assert np.isclose(y[t, o], sum(wh[k] * x[t, k] for k in range(256)), rtol=1e-12)


def test_gemm_brute_force():
    rng = np.random.default_rng(9)
    a, b = rng.standard_normal((3, 5)), rng.standard_normal((4, 5))
    y = G.gemm_dequantized(a, b, 0.5)
    for t in range(3):
        for o in range(4):
            assert np.isclose(y[t, o], 0.5 * sum(a[t, k] * b[o, k] for k in range(5)))


def test_output_loss_definition():
    a = np.array([[1.0, 2.0], [3.0, 4.0]])
    assert L.output_loss(a, a) == 0.0
    assert L.output_loss(a, a + np.array([[1.0, 0], [0, 3.0]])) == (1 + 9) / 4


def test_itq3_workload_shapes():
    w = synth.itq3_weights(64, 512)
    assert w.shape == (64, 512)
    c, s = I.quantize(w)
    assert c.shape == (64, 512) and s.shape == (64, 2) and s.dtype == np.float16
