"""The kernels' exact-decision procedure, emulated in IEEE fp32 on the CPU, against
the exact rational decisions.

The transform kernels quantise each value twice, against its block's fp32 reciprocal
nudged by 1 -+ 2^-20, and settle disagreements by an exact comparison with the
boundary times the scale.  Here every fp32 operation of that procedure is emulated with
correct rounding (exact rationals, rounded once), on values at, and a few ulps either
side of, every kind of boundary, and the result must equal the rounding of the exact
quotient.  The GPU parity tests run the kernels themselves; this checks the procedure's
argument (the bracket contains the exact quotient, and the fix-up compares exactly).
"""
from fractions import Fraction

import numpy as np

from oracle import formats as F
from tests.test_oracle_quant import _E2M1_EXACT, _E4M3_EXACT, _e2m1_exact, _exact_nearest

F32 = np.float32
FIXUPS = {"scale": 0, "code": 0, "int4_scale": 0, "int4_code": 0}   # fix-up paths taken
KLO, KHI = Fraction(1) - Fraction(1, 2 ** 20), Fraction(1) + Fraction(1, 2 ** 20)


def r32(q) -> Fraction:
    """Correctly rounded fp32 (ties to even) of the rational q, as a rational."""
    q = Fraction(q)
    c = F32(float(q))                    # within an ulp or two of the answer
    cands = {c, np.nextafter(c, F32(np.inf)), np.nextafter(c, F32(-np.inf))}
    best = min(cands, key=lambda x: (abs(Fraction(float(x)) - q), int(np.array(x, F32).view(np.uint32)) & 1))
    return Fraction(float(best))


def mul(a, b):
    return r32(Fraction(a) * Fraction(b))


def rcp(a):
    return r32(1 / Fraction(a))


def ue4m3(t: Fraction) -> int:
    return _exact_nearest(t, _E4M3_EXACT, lambda i: i & 1)


def e2m1(p: Fraction) -> int:
    mag = _exact_nearest(abs(p), _E2M1_EXACT, lambda i: i & 1)
    return (8 if p < 0 else 0) | mag


def kernel_scale_byte(amax, sg) -> int:
    inv_den = rcp(mul(6, sg))
    t = mul(amax, inv_den)
    lo, hi = ue4m3(mul(t, KLO)), ue4m3(mul(t, KHI))
    if lo == hi:
        return lo
    FIXUPS["scale"] += 1
    m6 = 3 * (_E4M3_EXACT[lo] + _E4M3_EXACT[hi])
    e = Fraction(amax) - m6 * Fraction(sg)          # an FMA gives this sign exactly
    return hi if e > 0 else (lo if e < 0 else (hi if lo & 1 else lo))


def kernel_code(v, sbv, sg) -> int:
    r = rcp(mul(sbv, sg))
    a, b = e2m1(mul(v, mul(r, KLO))), e2m1(mul(v, mul(r, KHI)))
    if a == b:
        return a
    FIXUPS["code"] += 1
    lo, hi = min(a & 7, b & 7), max(a & 7, b & 7)
    m = (_E2M1_EXACT[lo] + _E2M1_EXACT[hi]) / 2
    e = abs(Fraction(v)) - m * Fraction(sbv) * Fraction(sg)
    mag = hi if e > 0 else (lo if e < 0 else (hi if lo & 1 else lo))
    return mag | (8 if Fraction(v) < 0 else 0)


def _around(x, k=2):
    x = F32(x)
    out = [x]
    up = down = x
    for _ in range(k):
        up, down = np.nextafter(up, F32(np.inf)), np.nextafter(down, F32(-np.inf))
        out += [up, down]
    return out


def test_nvfp4_scale_byte_procedure_is_exact_at_every_midpoint():
    flips = 0
    for sg in (F32(0.37), F32(1.0), F32(3.1e-4)):
        sgq = Fraction(float(sg))
        for mid in F.E4M3_MIDPOINTS:
            for a in _around(float(Fraction(mid) * 6 * sgq)):
                if not (a > 0 and np.isfinite(a)):
                    continue
                amax = Fraction(float(a))
                want = ue4m3(amax / (6 * sgq))
                assert kernel_scale_byte(amax, sgq) == want
                flips += ue4m3(mul(mul(amax, rcp(mul(6, sgq))), 1)) != want
    assert flips > 0        # the plain reciprocal product does miss some of these
    assert FIXUPS["scale"] > 0


def test_nvfp4_code_procedure_is_exact_at_every_midpoint():
    flips = 0
    for sg in (F32(0.0123), F32(1.0)):
        sgq = Fraction(float(sg))
        for sbv in (1.0, 1.125, 3.5, 13.0, 0.6875, 448.0):
            d = Fraction(sbv) * sgq
            for mid in F.E2M1_MIDPOINTS:
                for sign in (1, -1):
                    for v in _around(float(sign * Fraction(mid) * d), 3):
                        want = _e2m1_exact(float(v), d)
                        assert kernel_code(Fraction(float(v)), Fraction(sbv), sgq) == want
                        flips += e2m1(mul(Fraction(float(v)), rcp(mul(sbv, sgq)))) != want
    assert flips > 0 and FIXUPS["code"] > 0


def kernel_int4_scale(amax):
    pre = mul(amax, Fraction(float(F32(1 / 7))))
    lo = Fraction(float(np.float16(float(min(mul(pre, KLO), Fraction(65504))))))
    hi = Fraction(float(np.float16(float(min(mul(pre, KHI), Fraction(65504))))))
    if lo == hi:
        return lo
    FIXUPS["int4_scale"] += 1
    m7 = Fraction(7, 2) * (lo + hi)
    lo_even = int(np.float16(float(lo)).view(np.uint16)) & 1 == 0
    return hi if amax > m7 else (lo if amax < m7 else (lo if lo_even else hi))


def kernel_int4_code(v, s):
    r = rcp(s)
    def rne_clamped(p):
        q = round(p)                                   # Python rounds halves to even
        return max(-7, min(7, q))
    a, b = rne_clamped(mul(v, mul(r, KLO))), rne_clamped(mul(v, mul(r, KHI)))
    if a == b:
        return a
    FIXUPS["int4_code"] += 1
    lo, hi = min(a, b), max(a, b)
    p = (Fraction(lo) + Fraction(1, 2)) * s
    v = Fraction(v)
    return hi if v > p else (lo if v < p else (lo if lo % 2 == 0 else hi))


def test_int4_scale_and_code_procedures_are_exact_next_to_ties():
    rng = np.random.default_rng(21)
    hs = np.unique(np.sort(rng.uniform(1e-3, 6e4, 80)).astype(np.float16))
    for hv in hs:
        nxt = np.nextafter(hv, np.float16(np.inf))
        mid = (Fraction(float(hv)) + Fraction(float(nxt))) / 2
        for a in _around(float(7 * mid)):
            amax = Fraction(float(a))
            pre = amax / 7
            c1, c2 = Fraction(float(hv)), Fraction(float(nxt))
            want = c1 if abs(pre - c1) < abs(pre - c2) else c2 if abs(pre - c2) < abs(pre - c1) else \
                (c1 if int(hv.view(np.uint16)) & 1 == 0 else c2)
            assert kernel_int4_scale(amax) == want
    for s16 in (np.float16(0.0123), np.float16(1.0), np.float16(517.0), np.float16(6.1e-5)):
        s = Fraction(float(s16))
        for k in range(-7, 7):
            mid = (Fraction(k) + Fraction(1, 2)) * s
            for v in _around(float(mid), 3):
                q = Fraction(float(v)) / s
                want = max(-7, min(7, round(q)))
                assert kernel_int4_code(Fraction(float(v)), s) == want
    assert FIXUPS["int4_scale"] > 0 and FIXUPS["int4_code"] > 0   # the exact comparisons were reached
