"""Seeded rotations: the Walsh-Hadamard form, the dense Haar form, and the
Gaussian projection used by QJL.

TEST INFRASTRUCTURE (oracle).  Not imported by the product path.

Upstream guide, section 4: two rotations exist side by side -- a dense QR
rotation (exact, O(d^2) per vector) and the structured ``D1 @ H @ D2``
Walsh-Hadamard form (O(d log d)).  Section 3 (Codex finding 6): the dense one
is the Q of a QR factorisation of a seeded Gaussian matrix, Haar distributed,
with ``slogdet`` used to make det = +1.

Readings taken where the pages are silent:

* H is the Sylvester Hadamard matrix in natural order,
  H[i, j] = (-1)^popcount(i & j), unnormalised (H H^T = d I); the rotation is
  R = d^-1/2 * D1 * H * D2 with D2 applied to the input first.
* D1 is the first d signs of the stream for ``seed``; D2 the next d.
* Haar: G[i, j] = gaussian draw i*d + j; G = Q R (any QR); Q <- Q diag(sign
  diag R) makes the factor unique and Haar (Mezzadri 2007); if det Q < 0,
  column 0 of Q is negated.  The rotation applied to a vector is y = Q x.
* QJL projection S (m x d): S[i, j] = gaussian draw i*d + j from the QJL seed.

This file builds H densely from its definition; it does not use a butterfly.
"""

import numpy as np

from . import rng


def hadamard(d):
    """Unnormalised Sylvester Hadamard matrix, H[i, j] = (-1)^popcount(i & j)."""
    i = np.arange(d)[:, None]
    j = np.arange(d)[None, :]
    anded = i & j
    parity = np.zeros_like(anded)
    bits = anded.copy()
    while np.any(bits):
        parity ^= bits & 1
        bits >>= 1
    return np.where(parity == 1, -1.0, 1.0)


def wht_signs(d, seed):
    """(D1, D2): the first d and the next d signs of the stream for ``seed``."""
    s = rng.signs(seed, 2 * d)
    return s[:d].copy(), s[d:].copy()


def wht_rotation(d, seed):
    """Dense matrix of R = d^-1/2 * D1 * H * D2 (float64, d x d)."""
    d1, d2 = wht_signs(d, seed)
    return (d ** -0.5) * (np.diag(d1) @ hadamard(d) @ np.diag(d2))


def haar_rotation(d, seed):
    """Haar orthogonal matrix with det = +1 from the QR of a seeded Gaussian."""
    g = rng.gaussians(seed, d * d).reshape(d, d)
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diag(r))[None, :]
    sign, _ = np.linalg.slogdet(q)
    if sign < 0:
        q[:, 0] = -q[:, 0]
    return q


def gaussian_projection(m, d, seed):
    """QJL projection S (m x d) with i.i.d. standard normal entries."""
    return rng.gaussians(seed, m * d).reshape(m, d)


def rotation(kind, d, seed):
    """Dispatch on the rotation kind name: 'wht' or 'haar'."""
    if kind == "wht":
        return wht_rotation(d, seed)
    if kind == "haar":
        return haar_rotation(d, seed)
    raise ValueError(f"unknown rotation kind {kind!r}")
