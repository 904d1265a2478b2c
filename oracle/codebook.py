"""Lloyd-Max scalar codebook on the density of one block-normalised rotated
coordinate.

TEST INFRASTRUCTURE (oracle).  Not imported by the product path.

The upstream guide names a Lloyd-Max codebook module and a "centroid table"
(section 1.2, section 5.2 commit 2) and, for the block layout, a per-block
norm extraction and rescale (section 5.1) with the block size decoupled from
the head dimension (section 6.1, commits 099ceab / a696962).  The density the
codebook is fitted to is not printed.  Reading taken here: after a random
rotation and division by the block norm, a block of ``Bk`` coordinates is a
uniform point on the unit sphere S^(Bk-1), so one coordinate X has density

    f(x) = (1 - x^2)^((Bk-3)/2) / B(1/2, (Bk-1)/2),   -1 <= x <= 1,

equivalently X^2 ~ Beta(1/2, (Bk-1)/2) with a symmetric sign.  The codebook
therefore depends on (bits, Bk) only.

Lloyd-Max (Lloyd 1957 / Max 1960): 2^b centroids c_0 < ... < c_{2^b-1};
boundaries are midpoints t_i = (c_{i-1} + c_i) / 2, i = 1 .. 2^b - 1; each
centroid is the conditional mean of its cell.  Started from the quantiles
F^-1((i + 1/2) / 2^b) and iterated until no centroid moves by 1e-14.  The
density is log-concave, so the fixed point is unique (Fleischer 1964) and the
start does not matter.

Cell masses come from the regularised incomplete beta function (a library
routine for the integral of f); cell first moments from the closed form
  integral x f(x) dx = -(1 - x^2)^((Bk-1)/2) / ((Bk-1) B(1/2, (Bk-1)/2)).
"""

import numpy as np
from scipy import integrate, special


def beta_param(block):
    """Second shape parameter of X^2 ~ Beta(1/2, (Bk-1)/2)."""
    return (block - 1) / 2.0


def density(x, block):
    """f(x) for one coordinate of a uniform point on S^(block-1)."""
    x = np.asarray(x, dtype=np.float64)
    a = (block - 3) / 2.0
    norm = special.beta(0.5, beta_param(block))
    inside = np.abs(x) <= 1.0
    out = np.zeros_like(x)
    out[inside] = (1.0 - x[inside] ** 2) ** a / norm
    return out


def upper_tail(x, block):
    """P(X > x), evaluated through the complementary incomplete beta."""
    x = np.asarray(x, dtype=np.float64)
    q = 0.5 * special.betaincc(0.5, beta_param(block), np.minimum(x * x, 1.0))
    return np.where(x >= 0.0, q, 1.0 - q)


def cell_mass(lo, hi, block):
    """P(lo < X <= hi)."""
    return upper_tail(lo, block) - upper_tail(hi, block)


def moment_antiderivative(x, block):
    """G(x) with G' = x f(x): -(1 - x^2)^((Bk-1)/2) / ((Bk-1) B(1/2, (Bk-1)/2))."""
    x = np.asarray(x, dtype=np.float64)
    b = beta_param(block)
    norm = special.beta(0.5, b)
    return -((1.0 - np.minimum(x * x, 1.0)) ** b) / (2.0 * b * norm)


def cell_first_moment(lo, hi, block):
    """Integral of x f(x) over (lo, hi]."""
    return moment_antiderivative(hi, block) - moment_antiderivative(lo, block)


def quantile(p, block):
    """F^-1(p) through the inverse incomplete beta."""
    p = np.asarray(p, dtype=np.float64)
    b = beta_param(block)
    upper = p >= 0.5
    tail = np.where(upper, 1.0 - p, p)          # mass beyond |x|
    y = special.betainccinv(0.5, b, 2.0 * tail)   # P(X^2 > y) = 2 * tail
    x = np.sqrt(y)
    return np.where(upper, x, -x)


def boundaries_from_centroids(c):
    """Midpoints between consecutive centroids (nearest-neighbour rule)."""
    c = np.asarray(c, dtype=np.float64)
    return 0.5 * (c[:-1] + c[1:])


def lloyd_max(bits, block, tol=1e-14, max_iter=200000):
    """Lloyd-Max centroids and boundaries (float64) for ``bits`` and ``block``.

    Returns (centroids[2^bits], boundaries[2^bits - 1]).
    """
    n = 1 << bits
    c = quantile((np.arange(n) + 0.5) / n, block)
    for _ in range(max_iter):
        t = boundaries_from_centroids(c)
        edges = np.concatenate(([-1.0], t, [1.0]))
        mass = cell_mass(edges[:-1], edges[1:], block)
        mom = cell_first_moment(edges[:-1], edges[1:], block)
        c_new = mom / mass
        moved = np.max(np.abs(c_new - c))
        c = c_new
        if moved < tol:
            break
    else:
        raise RuntimeError("Lloyd-Max did not converge")
    return c, boundaries_from_centroids(c)


def distortion(centroids, block):
    """Per-coordinate MSE E[(X - Q(X))^2] of the codebook, by quadrature."""
    c = np.asarray(centroids, dtype=np.float64)
    t = boundaries_from_centroids(c)
    edges = np.concatenate(([-1.0], t, [1.0]))
    total = 0.0
    for i in range(len(c)):
        val, _ = integrate.quad(
            lambda x, ci=c[i]: (x - ci) ** 2 * density(np.array([x]), block)[0],
            edges[i], edges[i + 1], epsabs=1e-15, epsrel=1e-12, limit=200)
        total += val
    return total


def stored_table(bits, block):
    """The codebook as stored by the packed format: the reconstruction table
    at fp16 precision -- each centroid the nearest binary16 value (ties to
    even) of the float64 fixed point, as the GPU path's fp16 centroid lookup
    table keeps it (upstream guide section 5.3, Metal backend list) -- returned
    as float32, and the float64 boundaries of the unrounded fixed point used for
    the oracle's decisions."""
    c, t = lloyd_max(bits, block)
    return c.astype(np.float16).astype(np.float32), t
