"""Pins for oracle.quant: brute-force scale and code search, grid membership,
idempotence, special cases and the boundary margins used by the parity tests."""
from fractions import Fraction

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


def _exact_nearest(q, grid, even_key):
    """Index of the grid value nearest to the rational q >= 0 by exhaustive search;
    at an exact tie the candidate with even_key(index) == 0 wins; above the last
    value it saturates."""
    if q >= grid[-1]:
        return len(grid) - 1
    dist = [abs(q - g) for g in grid]
    best = min(dist)
    cands = [i for i, dd in enumerate(dist) if dd == best]
    return min(cands, key=lambda i: (even_key(i), i))


_E2M1_EXACT = [Fraction(v) for v in F.E2M1_GRID]
_E4M3_EXACT = [Fraction(v) for v in F.E4M3_GRID]


def _e2m1_exact(y, d):
    """E2M1 code of the exact quotient y / d (rationals): sign of y, magnitude RNE-sat."""
    q = abs(Fraction(y)) / d
    mag = _exact_nearest(q, _E2M1_EXACT, lambda i: i & 1)
    return (8 if np.signbit(y) else 0) | mag


def _nvfp4_exact(yb, s_g):
    """Scale byte and codes of one NVFP4 block in exact rational arithmetic."""
    amax = max(abs(Fraction(float(v))) for v in yb)
    sg = Fraction(float(s_g))
    sb = _exact_nearest(amax / (6 * sg), _E4M3_EXACT, lambda i: i & 1)
    if sb == 0 or amax == 0:
        return sb, [0] * len(yb)
    d = _E4M3_EXACT[sb] * sg
    return sb, [_e2m1_exact(float(v), d) for v in yb]


def _int4_exact(yb):
    """fp16 scale and codes of one INT4 block in exact rational arithmetic."""
    amax = max(abs(Fraction(float(v))) for v in yb)
    pre = amax / 7
    # nearest fp16 by search over the two fp16 neighbours of pre, ties to the even significand
    lo = np.float16(float(pre))
    cands = {float(lo), float(np.nextafter(lo, np.float16(np.inf))), float(np.nextafter(lo, np.float16(0)))}
    cands = sorted(c for c in cands if np.isfinite(c))
    dist = [abs(pre - Fraction(c)) for c in cands]
    best = min(dist)
    tied = [c for c, dd in zip(cands, dist) if dd == best]
    s = min(tied, key=lambda c: int(np.float16(c).view(np.uint16)) & 1)
    s = min(s, 65504.0)
    if s == 0:
        return np.float16(0), [0] * len(yb)
    sf = Fraction(s)
    out = []
    for v in yb:
        q = Fraction(float(v)) / sf
        k = int(np.floor(q))
        frac = q - k
        r = k + 1 if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and k % 2) else k
        out.append(max(-7, min(7, r)))
    return np.float16(s), out


def test_nvfp4_brute_force():
    y = _data(2, d=64, spread=False) * F32(3.0)
    s_g = F32(np.max(np.abs(y)) / (6 * 448) * 0.7)      # some blocks saturate the scale
    q = Q.quantize_nvfp4(y, s_g)
    yb = y.reshape(6, 4, 16)
    for r in range(6):
        for j in range(4):
            sb, want = _nvfp4_exact(yb[r, j], s_g)
            assert q["scale_bytes"][r, j] == sb
            assert np.array_equal(q["codes"][r, 16 * j:16 * j + 16], np.array(want))


def test_int4_brute_force():
    y = _data(3, spread=False) * F32(40.0)
    q = Q.quantize_int4(y)
    yb = y.reshape(6, 4, 32)
    for r in range(6):
        for j in range(4):
            s, want = _int4_exact(yb[r, j])
            assert q["scale_fp16"][r, j] == s
            assert np.array_equal(q["q"][r, 32 * j:32 * j + 32], np.array(want))


def _near_ties(grid_mid, scale, rng, n):
    """fp32 values exactly on scale * midpoint, and one fp32 ulp either side of it."""
    out = []
    for _ in range(n):
        m = float(rng.choice(grid_mid))
        v = F32(m * scale)
        out += [v, np.nextafter(v, F32(np.inf)), np.nextafter(v, F32(-np.inf))]
    return np.array(out, F32)


def test_nvfp4_codes_at_and_next_to_ties_are_the_exact_quotients():
    # Element values on, and one fp32 ulp off, every E2M1 midpoint of a block whose
    # scale is fixed by one element at 6 d: the code must be the rounding of the
    # real quotient y / d.  A reciprocal-multiply y * fl(1/d) flips some of these.
    rng = np.random.default_rng(11)
    s_g = F32(0.0123)
    flips = 0
    for sbv in (1.0, 1.125, 3.5, 13.0, 0.6875):
        d = np.float64(sbv) * np.float64(s_g)
        for trial in range(6):
            body = _near_ties(F.E2M1_MIDPOINTS, d, rng, 5)
            blk = np.concatenate([[F32(6.0 * d)], body])
            y = blk.reshape(1, 16)
            q = Q.quantize_nvfp4(y, s_g)
            sb, want = _nvfp4_exact(y[0], s_g)
            assert q["scale_bytes"][0, 0] == sb
            assert np.array_equal(q["codes"][0], np.array(want))
            rcp = F32(F32(1) / F32(F.e4m3_value(sb) * np.float64(s_g)))
            flips += int(np.sum(F.e2m1_code((y[0] * rcp).astype(F32).astype(np.float64)) != np.array(want)))
    assert flips > 0        # the cases do reach the order-of-operations difference


def test_int4_codes_at_and_next_to_ties_are_the_exact_quotients():
    rng = np.random.default_rng(12)
    flips = 0
    for s in (np.float16(0.0123), np.float16(1.0), np.float16(3.1e-3), np.float16(517.0)):
        for trial in range(6):
            body = _near_ties(F.INT4_MIDPOINTS, np.float64(s), rng, 10)
            blk = np.concatenate([[F32(7.0 * np.float64(s))], body])
            y = blk.reshape(1, 31)
            y = np.concatenate([y, np.zeros((1, 1), F32)], axis=1)
            q = Q.quantize_int4(y)
            sc, want = _int4_exact(y[0])
            assert q["scale_fp16"][0, 0] == sc
            assert np.array_equal(q["q"][0], np.array(want))
            rcp = F32(F32(1) / F32(sc))
            flips += int(np.sum(np.clip(np.rint((y[0] * rcp).astype(F32)), -7, 7) != np.array(want)))
    assert flips > 0


def test_scale_decisions_at_and_next_to_ties_are_exact():
    # Block amax on, and one fp32 ulp off, a UE4M3 midpoint (times 6 s_g) or an
    # fp16 midpoint (times 7): the scale is the rounding of the real quotient.
    s_g = F32(0.37)
    for mid in F.E4M3_MIDPOINTS[::5]:
        a = F32(mid * 6.0 * np.float64(s_g))
        for v in (a, np.nextafter(a, F32(np.inf)), np.nextafter(a, F32(0))):
            y = np.zeros((1, 16), F32)
            y[0, 3] = v
            assert Q.quantize_nvfp4(y, s_g)["scale_bytes"][0, 0] == _nvfp4_exact(y[0], s_g)[0]
    rng = np.random.default_rng(13)
    h = np.sort(rng.uniform(1e-3, 6e4, 60)).astype(np.float16)
    for hv in h:
        mid = (np.float64(hv) + np.float64(np.nextafter(hv, np.float16(np.inf)))) / 2
        a = F32(mid * 7.0)
        for v in (a, np.nextafter(a, F32(np.inf)), np.nextafter(a, F32(0))):
            y = np.zeros((1, 32), F32)
            y[0, 9] = -v
            assert Q.quantize_int4(y)["scale_fp16"][0, 0] == _int4_exact(y[0])[0]


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
