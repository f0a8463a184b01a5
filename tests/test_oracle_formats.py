"""Pins for oracle.formats against library conversions and brute force."""
import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import formats as F


def _sweep_e2m1():
    mids = F.E2M1_MIDPOINTS
    pts = [F.E2M1_GRID, mids, np.nextafter(mids, 0), np.nextafter(mids, 10),
           np.linspace(0, 12, 20001), [6.0, 6.5, 1e30]]
    v = np.concatenate([np.asarray(p, dtype=np.float64) for p in pts])
    v = np.concatenate([v, -v])
    return v.astype(np.float32)


def test_e2m1_matches_ml_dtypes():
    v = _sweep_e2m1()
    ref = v.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    code = F.e2m1_code(v)
    got = F.e2m1_value(code)
    assert np.array_equal(got, ref)
    assert np.array_equal(np.signbit(got), np.signbit(ref))


def test_e2m1_tie_table():
    # midpoints resolve to the neighbour with an even code (mantissa bit 0)
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for v, want in ties.items():
        assert F.e2m1_value(F.e2m1_code(np.array([v]))) == want
        assert F.e2m1_value(F.e2m1_code(np.array([-v]))) == -want


def test_e2m1_codes_idempotent_and_signed_zero():
    codes = np.arange(16, dtype=np.uint8)
    assert np.array_equal(F.e2m1_code(F.e2m1_value(codes)), codes)
    assert F.e2m1_code(np.array([-0.1]))[0] == 8
    assert F.e2m1_code(np.array([0.1]))[0] == 0


def test_e4m3_grid_matches_library_decode():
    codes = np.arange(127, dtype=np.uint8)
    lib = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(F.E4M3_GRID, lib)
    assert F.E4M3_GRID[-1] == 448.0 and F.E4M3_GRID[1] == 2.0 ** -9


def test_e4m3_rne_matches_ml_dtypes_and_torch():
    g = F.E4M3_GRID
    mids = (g[:-1] + g[1:]) / 2
    rng = np.random.default_rng(1)
    v = np.concatenate([g, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e3),
                        rng.uniform(0, 448, 20000), 2.0 ** rng.uniform(-12, 8.8, 20000)])
    v = np.clip(v, 0, 448).astype(np.float32)
    got = F.e4m3_value(F.e4m3_code_unsigned(v))
    ref_ml = v.astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    ref_t = torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(got, ref_ml)
    assert np.array_equal(got, ref_t)


def test_e4m3_saturates():
    v = np.array([448.0, 449.0, 464.0, 500.0, 1e9], dtype=np.float32)
    assert np.all(F.e4m3_value(F.e4m3_code_unsigned(v)) == 448.0)


def test_e8m0_values():
    assert F.e8m0_value(np.array([127]))[0] == 1.0
    assert F.e8m0_value(np.array([0]))[0] == 2.0 ** -127
    assert F.e8m0_value(np.array([254]))[0] == 2.0 ** 127
    lib = np.arange(255, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    assert np.array_equal(F.e8m0_value(np.arange(255)), lib)


def test_fp16_rne_brute_force():
    allh = np.arange(0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)  # finite >= 0
    rng = np.random.default_rng(2)
    v = np.concatenate([2.0 ** rng.uniform(-26, 16, 5000), (allh[1:] + allh[:-1]) / 2])
    v = v[v <= 65504]
    got = F.fp16_rne_sat(v).astype(np.float64)
    idx = np.searchsorted(allh, v)
    lo, hi = allh[np.maximum(idx - 1, 0)], allh[np.minimum(idx, len(allh) - 1)]
    bits_hi = np.minimum(idx, len(allh) - 1)
    pick_hi = (hi - v < v - lo) | ((hi - v == v - lo) & (bits_hi % 2 == 0))
    want = np.where(v == hi, hi, np.where(pick_hi, hi, lo))
    assert np.array_equal(got, want)
    assert F.fp16_rne_sat(np.array([1e6]))[0] == np.float16(65504)


@pytest.mark.parametrize("mids", [F.E2M1_MIDPOINTS, F.INT4_MIDPOINTS])
def test_distance_to_boundary_brute(mids):
    v = np.random.default_rng(3).uniform(0, 8, 5000)
    want = np.min(np.abs(v[:, None] - mids[None, :]), axis=1)
    assert np.allclose(F.distance_to_boundary(v, mids), want, rtol=0, atol=1e-15)
