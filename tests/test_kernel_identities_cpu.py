"""CPU checks of the exact-arithmetic identities the CUDA kernels rely on.

The kernels take integer decisions and build exact values with float tricks; each
trick is restated here in IEEE fp32 (numpy) and checked exhaustively or on the edges
that decide it.  These are checks of the kernels' arithmetic claims, not of the
oracle (the GPU parity tests compare the kernels with the oracle).
"""
import numpy as np

F32 = np.float32


def _bits_to_f32(u):
    return np.asarray(u, dtype=np.uint32).view(np.float32)


def test_itq3_level_decode_is_exact_for_every_code_and_fp16_scale():
    # code c in mantissa bits 20..22 of 1.0f gives f = 1 + c/8; the level (c - 3.5) s
    # is then f * (8 s) - 11.5 s, with 8 s and 11.5 s exact and one rounding, which
    # leaves it exact: (c - 3.5) s needs at most 15 significant bits
    s16 = np.arange(0x0001, 0x7C00, dtype=np.uint16).view(np.float16)      # every finite s > 0
    s = s16.astype(np.float32)
    s8, m = F32(8) * s, F32(-11.5) * s
    assert np.array_equal(s8.astype(np.float64), 8.0 * s.astype(np.float64))
    assert np.array_equal(m.astype(np.float64), -11.5 * s.astype(np.float64))
    for c in range(8):
        f = _bits_to_f32(0x3F800000 | (c << 20))
        assert float(f) == 1 + c / 8
        # fp32 FMA: exact product and sum in fp64 (24-bit operands), one rounding to fp32
        got = (np.float64(f) * s8.astype(np.float64) + m.astype(np.float64)).astype(np.float32)
        want = ((c - 3.5) * s.astype(np.float64)).astype(np.float32)
        assert np.array_equal(got, want)
        assert np.array_equal(want.astype(np.float64), (c - 3.5) * s.astype(np.float64))   # exact


def test_itq3_code_field_moves_with_a_multiply_and_a_mask():
    # the lane's 24 code bits, and garbage above them, times 2^(20 - 3i) + 2^31, masked
    # to bits 20..22, give code i; code 7 comes from a right shift by one
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 8, size=(4000, 8))
    garbage = rng.integers(0, 256, size=4000)
    bits = (codes << (3 * np.arange(8))).sum(axis=1) | (garbage << 24)
    for i in range(8):
        if i < 7:
            t = (bits.astype(np.uint64) * ((1 << (20 - 3 * i)) | 0x80000000)) & 0xFFFFFFFF
        else:
            t = bits >> 1
        assert np.array_equal((t.astype(np.int64) >> 20) & 7, codes[:, i])


def test_int4_bias_add_rounds_to_nearest_even_in_the_low_nibble():
    # v + 1.5 * 2^23 rounds to an integer (ulp 1) held in the low mantissa bits; the
    # low four bits are the two's-complement nibble of RNE(v) for |v| <= 7.5
    v = np.concatenate([np.linspace(-7.5, 7.5, 200001, dtype=np.float32),
                        np.arange(-15, 16, dtype=np.float32) / 2])          # every half-integer tie
    r = (v + F32(12582912.0)).view(np.uint32) & 15
    q = np.rint(v.astype(np.float64)).astype(np.int64)                       # numpy rint: ties to even
    assert np.array_equal(r.astype(np.int64), q & 15)


def test_bracket_factors_are_one_minus_and_plus_two_to_the_minus_twenty():
    lo, hi = F32(0.99999904632568359375), F32(1.00000095367431640625)
    assert float(lo) == 1 - 2.0 ** -20 and float(hi) == 1 + 2.0 ** -20


def test_int4_agreement_test_is_exact():
    # the two brackets' rounded values (1.5 * 2^23 + q) differ by 0 or 1; their
    # differences and squares are exact, so the sum of squares is zero exactly when
    # all agree
    base = F32(12582912.0)
    for qa in range(-7, 8):
        for d in (0, 1):
            a, b = base + F32(qa), base + F32(qa + d)
            diff = b - a
            assert float(diff) == d and float(diff * diff) == d


def _significant_bits(x):
    x = abs(float(x))
    if x == 0:
        return 0
    num, den = x.as_integer_ratio()
    while num % 2 == 0:
        num //= 2
    return num.bit_length()


def _ue4m3_values():
    vals = []
    for code in range(0x7F):                      # 0x7F is NaN
        e, m = code >> 3, code & 7
        vals.append(m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return vals


def test_nvfp4_scale_midpoints_are_exact_with_few_bits():
    # between adjacent UE4M3 codes the decision compares amax with 6 m s_g, m their
    # midpoint: 6 m = 3 (v_lo + v_hi) has at most 7 significant bits, so it is exact
    # in fp32 and one FMA gives the sign of amax - 6 m s_g exactly
    v = _ue4m3_values()
    for lo, hi in zip(v[:-1], v[1:]):
        m6 = 3.0 * (lo + hi)
        assert float(F32(m6)) == m6 and _significant_bits(m6) <= 7


def test_e2m1_midpoints_times_scales_are_exact():
    # code decision: |v| against m * s_b * s_g with m the E2M1 midpoint (at most 3
    # significant bits) and s_b a UE4M3 value (4): m * s_b is exact in fp32
    mags = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    for lo, hi in zip(mags[:-1], mags[1:]):
        m = 0.5 * (lo + hi)
        assert _significant_bits(m) <= 3
        for sb in _ue4m3_values():
            assert float(F32(m) * F32(sb)) == m * sb


def test_int4_scale_midpoints_are_exact():
    # fp16 scale decision: amax against 7 m, m the midpoint of adjacent fp16 values:
    # 3.5 (lo + hi) has at most 15 significant bits, exact in fp32
    h = np.arange(0x0000, 0x7BFF, dtype=np.uint16).view(np.float16).astype(np.float64)
    m7 = 3.5 * (h[:-1] + h[1:])
    assert np.array_equal(m7.astype(np.float32).astype(np.float64), m7)
    assert max(_significant_bits(x) for x in m7[::97]) <= 15
