"""Pins for the oracle's random streams and rotations (CPU only)."""

import os

import numpy as np
import pytest
from scipy import linalg, stats

from oracle import codebook, rng, rotation

MASK = (1 << 64) - 1


def _read_ints(path):
    with open(path) as f:
        return [int(x) for x in f.read().split("\n") if x and not x.startswith("#")]


def _splitmix_sequential(seed, n):
    """SplitMix64 as a plain stateful loop over Python integers."""
    state = seed & MASK
    out = []
    for _ in range(n):
        state = (state + 0x9E3779B97F4A7C15) & MASK
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
        out.append(z ^ (z >> 31))
    return out


def test_splitmix64_published_vector(golden_dir):
    vals = _read_ints(os.path.join(golden_dir, "splitmix64_vigna_seed1234567.txt"))
    seed, expected = vals[0], vals[1:]
    assert [int(v) for v in rng.splitmix64(seed, len(expected))] == expected


@pytest.mark.parametrize("seed", [0, 1, 1000, 2063, (1 << 64) - 5, 0xDEADBEEFCAFEF00D])
def test_splitmix64_vector_form_equals_stateful_loop(seed):
    assert [int(v) for v in rng.splitmix64(seed, 300)] == _splitmix_sequential(seed, 300)


def test_uniform_and_sign_streams():
    u = rng.uniforms(5, 200_000)
    assert u.min() >= 0.0 and u.max() < 1.0
    assert stats.kstest(u, "uniform").pvalue > 1e-3
    s = rng.signs(5, 200_000)
    assert set(np.unique(s)) == {-1.0, 1.0}
    # top bit of the same draws
    top = np.array([v >> 63 for v in _splitmix_sequential(5, 1000)])
    assert np.array_equal(s[:1000], np.where(top == 1, -1.0, 1.0))
    assert abs(np.mean(s)) < 4.0 / np.sqrt(len(s))


def test_gaussian_stream_is_standard_normal():
    g = rng.gaussians(123, 400_000)
    assert stats.kstest(g, "norm").pvalue > 1e-3
    assert abs(g.mean()) < 4.0 / np.sqrt(len(g))
    assert abs(g.var() - 1.0) < 4.0 * np.sqrt(2.0 / len(g))
    # odd n returns the prefix of the even stream
    assert np.array_equal(rng.gaussians(123, 7), g[:7])


@pytest.mark.parametrize("d", [2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_is_sylvester(d):
    h = rotation.hadamard(d)
    assert np.array_equal(h, linalg.hadamard(d).astype(np.float64))
    assert np.array_equal(h @ h.T, d * np.eye(d))


def _fwht_butterfly(x):
    """In-place iterative Walsh-Hadamard butterfly (natural order), unnormalised."""
    x = np.array(x, dtype=np.float64)
    d = x.shape[-1]
    h = 1
    while h < d:
        x = x.reshape(*x.shape[:-1], d // (2 * h), 2, h)
        a = x[..., 0, :].copy()
        b = x[..., 1, :].copy()
        x[..., 0, :] = a + b
        x[..., 1, :] = a - b
        x = x.reshape(*x.shape[:-3], d)
        h *= 2
    return x


@pytest.mark.parametrize("d", [64, 128, 256])
def test_wht_rotation_properties(d):
    r = rotation.wht_rotation(d, 1000)
    assert np.max(np.abs(r @ r.T - np.eye(d))) < 1e-14
    d1, d2 = rotation.wht_signs(d, 1000)
    # column 0 of H is all ones: R e0 = d^-1/2 * D2[0] * D1
    assert np.allclose(r[:, 0], d ** -0.5 * d2[0] * d1, atol=0, rtol=0)
    x = np.random.default_rng(0).standard_normal((16, d))
    y = x @ r.T
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    # a butterfly (different algorithm) gives the same rotation
    y_fast = d ** -0.5 * d1 * _fwht_butterfly(x * d2)
    assert np.max(np.abs(y - y_fast)) < 1e-12
    # determinism
    assert np.array_equal(r, rotation.wht_rotation(d, 1000))
    assert not np.array_equal(r, rotation.wht_rotation(d, 1001))


@pytest.mark.parametrize("d", [8, 64, 128, 256])
def test_haar_rotation_properties(d):
    q = rotation.haar_rotation(d, 1000)
    assert np.max(np.abs(q @ q.T - np.eye(d))) < 1e-12
    assert abs(np.linalg.det(q) - 1.0) < 1e-9
    assert np.array_equal(q, rotation.haar_rotation(d, 1000))
    assert not np.allclose(q, rotation.haar_rotation(d, 1001))
    # q is the orthogonal factor of the seeded Gaussian: q^T G is upper
    # triangular with a positive diagonal (row 0 may be negated by the det fix)
    g = rng.gaussians(1000, d * d).reshape(d, d)
    r = q.T @ g
    assert np.max(np.abs(np.tril(r, -1))) < 1e-9 * np.max(np.abs(r))
    assert np.all(np.diag(r)[1:] > 0)


def test_haar_columns_are_uniform_on_the_sphere():
    """Coordinates of Q e0 over many seeds follow the sphere marginal f (Bk = d)."""
    d = 16
    samples = np.concatenate([rotation.haar_rotation(d, s)[:, 0] for s in range(3000, 3400)])
    cdf = lambda x: 1.0 - codebook.upper_tail(x, d)
    assert stats.kstest(samples, cdf).pvalue > 1e-3
    # and the det fix does not bias the sign of Q[0, 0]
    signs = np.array([np.sign(rotation.haar_rotation(d, s)[0, 0]) for s in range(3000, 3400)])
    assert abs(signs.mean()) < 4.0 / np.sqrt(len(signs))


def test_gaussian_projection_shape_and_stream():
    s = rotation.gaussian_projection(128, 64, 2000)
    assert s.shape == (128, 64)
    assert np.array_equal(s.ravel(), rng.gaussians(2000, 128 * 64))
