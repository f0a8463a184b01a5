"""Pins for oracle.quant: brute-force scale and code search, grid membership,
idempotence, special cases and the boundary margins used by the parity tests."""
import numpy as np
import pytest

from oracle import formats as F
from oracle import quant as Q

F32 = np.float32


def _data(seed, rows=6, d=128, spread=True):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((rows, d))
    if spread:
        y *= 2.0 ** rng.integers(-20, 20, size=(rows, 1))
        y[:, 5] *= 37.0
    return y.astype(F32)


def _nearest_code_brute(v):
    """Nearest of all 16 E2M1 codes by exhaustive search, ties to the even code."""
    vals = F.e2m1_value(np.arange(16))
    out = []
    for x in np.asarray(v, dtype=np.float64).ravel():
        best = None
        for c in range(16):
            if (c >= 8) != np.signbit(x):
                continue
            d = abs(abs(x) - abs(vals[c])) if abs(x) <= 6 else abs(6 - abs(vals[c]))
            key = (d, c & 1)
            if best is None or key < best[0]:
                best = (key, c)
        out.append(best[1])
    return np.array(out).reshape(np.shape(v))


def test_mxfp4_brute_force():
    y = _data(1)
    q = Q.quantize_mxfp4(y)
    yb = y.reshape(6, 4, 32).astype(np.float64)
    for r in range(6):
        for j in range(4):
            amax = np.max(np.abs(yb[r, j]))
            e = 0
            while 2.0 ** (e + 2) > amax:        # largest e with 2^(e+2) <= amax
                e -= 1
            while 2.0 ** (e + 3) <= amax:
                e += 1
            assert q["scale_bytes"][r, j] == e + 127
            assert 4 <= amax / 2.0 ** e < 8
            want = _nearest_code_brute(yb[r, j] / 2.0 ** e)
            assert np.array_equal(q["codes"][r, 32 * j:32 * j + 32], want)


def test_mxfp4_special_blocks():
    y = np.zeros((1, 64), F32)
    y[0, 32:] = -1e-3
    y[0, 40] = 1.0
    q = Q.quantize_mxfp4(y)
    assert q["scale_bytes"][0, 0] == 0 and np.all(q["codes"][0, :32] == 0)
    assert q["scale_bytes"][0, 1] == 127 - 2          # amax 1 -> e = -2
    assert q["codes"][0, 33] == 8                      # -1e-3 / 0.25 rounds to -0


def test_nvfp4_brute_force():
    y = _data(2, d=64, spread=False) * F32(3.0)
    s_g = F32(np.max(np.abs(y)) / (6 * 448) * 0.7)      # some blocks saturate the scale
    q = Q.quantize_nvfp4(y, s_g)
    yb = y.reshape(6, 4, 16)
    grid = F.E4M3_GRID
    for r in range(6):
        for j in range(4):
            amax = F32(np.max(np.abs(yb[r, j])))
            t = F32(amax / F32(F32(6) * s_g))
            dist = np.abs(grid - np.float64(t))
            cands = np.flatnonzero(dist == dist.min())
            sb = 126 if t > 448 else min(cands, key=lambda c: (c & 1, c))
            assert q["scale_bytes"][r, j] == sb
            d = F32(F32(grid[sb]) * s_g)
            want = _nearest_code_brute((yb[r, j] * F32(F32(1) / d)).astype(F32))
            assert np.array_equal(q["codes"][r, 16 * j:16 * j + 16], want)


def test_int4_brute_force():
    y = _data(3, spread=False) * F32(40.0)
    q = Q.quantize_int4(y)
    yb = y.reshape(6, 4, 32)
    for r in range(6):
        for j in range(4):
            s = np.float16(F32(np.max(np.abs(yb[r, j]))) / F32(7))
            v = (yb[r, j] * F32(F32(1) / F32(s))).astype(F32)
            want = []
            for x in v.astype(np.float64):
                cands = np.arange(-7, 8)
                d = np.abs(cands - np.clip(x, -7.5, 7.5))
                best = cands[d == d.min()]
                want.append(best[best % 2 == 0][0] if len(best) > 1 else best[0])
            assert np.array_equal(q["q"][r, 32 * j:32 * j + 32], np.array(want))
            assert q["scale_fp16"][r, j] == s


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "int4"])
def test_idempotent_on_dequantised(fmt):
    y = _data(4, spread=(fmt != "nvfp4"))
    gs = F32(np.max(np.abs(y)) / (6 * 448)) if fmt == "nvfp4" else None
    q1 = Q.quantize(y, fmt, gs)
    dq = q1["dq"] if fmt != "nvfp4" else q1["dq"]
    q2 = Q.quantize(dq.astype(F32), fmt, gs)
    assert np.array_equal(q1["codes"], q2["codes"])


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4", "int4"])
def test_margins_are_exact_flip_distances(fmt):
    # Moving an element by less than its margin keeps its code; moving it past the
    # margin toward the boundary changes it (when the scale decision is unaffected).
    y = _data(5, rows=4, d=64, spread=False)
    gs = F32(np.max(np.abs(y)) / (6 * 448)) if fmt == "nvfp4" else None
    q = Q.quantize(y, fmt, gs)
    b = Q.BLOCK[fmt]
    rng = np.random.default_rng(6)
    checked = 0
    for _ in range(800):
        r, c = rng.integers(0, 4), rng.integers(0, 64)
        blk = c // b
        m = q["elem_margin"][r, c]
        amax = np.max(np.abs(y[r, blk * b:(blk + 1) * b]))
        # perturb a non-amax element only, never past the amax: the scale is unchanged
        if m == 0 or abs(np.float64(y[r, c])) + 2 * m >= amax:
            continue
        for sgn in (1.0, -1.0):
            y2 = y.copy()
            y2[r, c] = F32(np.float64(y[r, c]) + sgn * 0.5 * m)
            assert Q.quantize(y2, fmt, gs)["codes"][r, c] == q["codes"][r, c]
        flipped = False
        for sgn in (1.0, -1.0):
            y2 = y.copy()
            y2[r, c] = F32(np.float64(y[r, c]) + sgn * 1.5 * m)
            if abs(y2[r, c]) < np.max(np.abs(y[r, blk * b:(blk + 1) * b])):
                flipped |= Q.quantize(y2, fmt, gs)["codes"][r, c] != q["codes"][r, c]
        assert flipped
        checked += 1
    assert checked > 20


def test_block_margin_mxfp4_power_of_two():
    y = np.zeros((1, 32), F32)
    y[0, 0] = F32(1.0 + 2 ** -20)
    y[0, 1] = F32(0.3)
    q = Q.quantize_mxfp4(y)
    assert np.isclose(q["block_margin"][0, 0], 2 ** -20)
