"""Pins for oracle.transforms: Hadamard closed form, FWHT vs dense product, block apply."""
import numpy as np
import pytest

from oracle import transforms as T


def _hadamard_closed_form(n):
    i = np.arange(n)
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i[:, None] & i[None, :])
    return (-1.0) ** pc


@pytest.mark.parametrize("n", [1, 2, 16, 32, 256])
def test_hadamard_orthogonality_and_closed_form(n):
    h = T.sylvester_hadamard(n)
    assert np.array_equal(h @ h.T, n * np.eye(n))
    assert np.array_equal(h, _hadamard_closed_form(n))
    hn = T.normalized_hadamard(n)
    assert np.allclose(hn @ hn, np.eye(n), atol=1e-14)


@pytest.mark.parametrize("n", [16, 32, 256])
def test_fwht_equals_dense_product_exactly_on_integers(n):
    x = np.random.default_rng(n).integers(-1000, 1000, size=(7, n)).astype(np.float64)
    assert np.array_equal(T.fwht(x), x @ T.sylvester_hadamard(n).T)


def test_fwht_twice_is_n_identity():
    x = np.random.default_rng(5).standard_normal((3, 256))
    assert np.allclose(T.fwht(T.fwht(x)), 256 * x, rtol=1e-13, atol=1e-12)


def test_block_transform_matches_loop():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((5, 96))
    t = rng.standard_normal((3, 32, 32))
    want = np.empty_like(x)
    for r in range(5):
        for j in range(3):
            want[r, 32 * j:32 * j + 32] = t[j] @ x[r, 32 * j:32 * j + 32]
    assert np.allclose(T.apply_block_transform(x, t), want, rtol=1e-14, atol=1e-14)
    mag = T.block_magnitude(x, t)
    for r in range(5):
        for j in range(3):
            xs = x[r, 32 * j:32 * j + 32]
            assert np.allclose(mag[r, 32 * j:32 * j + 32], np.abs(t[j]) @ np.abs(xs))


def test_hadamard_and_identity_blocks():
    assert np.array_equal(T.identity_blocks(64, 32)[1], np.eye(32))
    assert np.allclose(T.hadamard_blocks(64, 16)[3], T.sylvester_hadamard(16) / 4.0)
