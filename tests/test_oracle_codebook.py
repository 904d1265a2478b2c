"""Pins for the oracle's block-sphere density and Lloyd-Max codebook."""

import os

import numpy as np
import pytest
from scipy import integrate, special, stats

from oracle import codebook


def _read_levels(path):
    out = {}
    with open(path) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            out[int(parts[0])] = np.array([float(v) for v in parts[1:]])
    return out


@pytest.mark.parametrize("block", [3, 4, 8, 16, 32, 64])
def test_density_normalised_with_second_moment(block):
    f = lambda x: codebook.density(np.array([x]), block)[0]
    total, _ = integrate.quad(f, -1, 1, epsabs=1e-14, limit=200)
    m2, _ = integrate.quad(lambda x: x * x * f(x), -1, 1, epsabs=1e-14, limit=200)
    assert abs(total - 1.0) < 1e-10
    assert abs(m2 - 1.0 / block) < 1e-10


@pytest.mark.parametrize("block", [4, 8, 32])
def test_density_is_the_sphere_marginal(block):
    """Monte Carlo: a coordinate of a normalised Gaussian vector in R^Bk."""
    z = np.random.default_rng(11).standard_normal((100_000, block))
    u = z[:, 0] / np.linalg.norm(z, axis=1)
    assert stats.kstest(u, lambda x: 1.0 - codebook.upper_tail(x, block)).pvalue > 1e-3


def test_cdf_tail_matches_quadrature():
    for block in (4, 32):
        for x in (-0.7, -0.1, 0.0, 0.2, 0.45, 0.9):
            q, _ = integrate.quad(lambda t: codebook.density(np.array([t]), block)[0],
                                  x, 1.0, epsabs=1e-14, limit=200)
            assert abs(q - codebook.upper_tail(x, block)) < 1e-12


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("block", [4, 8, 16, 32])
def test_lloyd_max_fixed_point(bits, block):
    c, t = codebook.lloyd_max(bits, block)
    n = 1 << bits
    assert len(c) == n and len(t) == n - 1
    assert np.all(np.diff(c) > 0)
    assert np.max(np.abs(c + c[::-1])) < 1e-13           # symmetric
    assert np.max(np.abs(t - 0.5 * (c[1:] + c[:-1]))) == 0.0
    # centroid condition by quadrature (independent of the incomplete beta)
    edges = np.concatenate(([-1.0], t, [1.0]))
    f = lambda x: codebook.density(np.array([x]), block)[0]
    for i in range(n):
        m0, _ = integrate.quad(f, edges[i], edges[i + 1], epsabs=1e-15, epsrel=1e-13, limit=200)
        m1, _ = integrate.quad(lambda x: x * f(x), edges[i], edges[i + 1],
                               epsabs=1e-15, epsrel=1e-13, limit=200)
        assert abs(m1 / m0 - c[i]) < 1e-11


@pytest.mark.parametrize("block", [4, 8, 16, 32, 128])
def test_one_bit_closed_form(block):
    """b = 1: c = E|X| = Gamma(Bk/2) / (sqrt(pi) Gamma((Bk+1)/2))."""
    c, t = codebook.lloyd_max(1, block)
    expect = np.exp(special.gammaln(block / 2) - special.gammaln((block + 1) / 2)) / np.sqrt(np.pi)
    assert abs(c[1] - expect) < 1e-13 and abs(c[0] + expect) < 1e-13
    assert t[0] == 0.0
    if block == 32:
        assert round(c[1], 7) == 0.1421535


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_uniform_density_gives_uniform_quantizer(bits):
    """Bk = 3: f = 1/2 on [-1, 1], whose Lloyd-Max quantizer is uniform."""
    c, _ = codebook.lloyd_max(bits, 3)
    n = 1 << bits
    assert np.max(np.abs(c - (-1.0 + (2 * np.arange(n) + 1) / n))) < 1e-13


def test_gaussian_limit_matches_max_1960(golden_dir):
    levels = _read_levels(os.path.join(golden_dir, "max1960_gaussian_lloyd_max.txt"))
    block = 1 << 16
    for bits, table in levels.items():
        c, _ = codebook.lloyd_max(bits, block)
        pos = c[len(c) // 2:] * np.sqrt(block)
        # table printed to 4 significant digits
        assert np.all(np.abs(pos - table) <= 0.6e-3 * np.maximum(1.0, table)), (bits, pos, table)


def test_distortion_decreases_with_bits():
    d = [codebook.distortion(codebook.lloyd_max(b, 32)[0], 32) for b in (1, 2, 3, 4)]
    assert all(a > b for a, b in zip(d, d[1:]))
    # b = 1: D = E X^2 - c^2 = 1/Bk - c^2
    c1 = codebook.lloyd_max(1, 32)[0][1]
    assert abs(d[0] - (1.0 / 32 - c1 * c1)) < 1e-12


def test_fixed_point_is_a_local_minimum():
    """Moving any single centroid (boundaries re-derived) raises the distortion."""
    for bits in (2, 3):
        c, _ = codebook.lloyd_max(bits, 32)
        base = codebook.distortion(c, 32)
        for i in range(len(c)):
            for eps in (-1e-3, 1e-3):
                cc = c.copy()
                cc[i] += eps
                assert codebook.distortion(cc, 32) > base
