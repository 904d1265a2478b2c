"""QJL residual stage: one sign bit per Gaussian projection of the residual.

TEST INFRASTRUCTURE (oracle).  Not imported by the product path.

"Google TurboQuant deep dive", section 2.2: the residual left by the first
stage goes through a random Gaussian projection and each projected value is
reduced to its sign; the query stays in full precision, so the asymmetric
inner product absorbs the error (section 4.3).  "Plan de Integracion",
"Implementacion conceptual": one sign bit per value, bit i of byte i/8 -- the
listing there applies the sign to the raw residual, which contradicts the
projection described on the same page, so the projection reading is taken.

Readings taken where the pages are silent:

* residual r = y - x_hat in the rotated frame, x_hat built with the *stored*
  fp16 block norms and fp32 centroids;
* S is m x d with i.i.d. N(0, 1) entries from the QJL seed; z = S r;
  sign bit s_i = [z_i >= 0] (zero counts as +), stored as bit (i mod 32) of
  uint32 word i / 32;
* rho = fp16(||r||_2) is stored per row (saturating at 65504);
* estimator of <q_rot, r>:  sqrt(pi/2) / m * rho * sum_i (S q_rot)_i (2 s_i - 1),
  unbiased because E[sign(<s, r>) <s, q>] = sqrt(2/pi) <q, r> / ||r|| for a
  standard Gaussian vector s.
"""

import numpy as np

from .quant import FP16_MAX


def residual(y, x_hat_rot):
    return np.asarray(y, dtype=np.float64) - np.asarray(x_hat_rot, dtype=np.float64)


def projections(r, S):
    """z = S r for every row r."""
    return np.asarray(r, dtype=np.float64) @ np.asarray(S, dtype=np.float64).T


def sign_bits(z):
    """Boolean [n, m]: z >= 0."""
    return np.asarray(z) >= 0.0


def pack_signs(bits_bool):
    """Bool [n, m] -> uint32 [n, m/32], bit i of the row in word i/32, LSB first."""
    b = np.asarray(bits_bool, dtype=np.uint64)
    n, m = b.shape
    out = np.zeros((n, m // 32), dtype=np.uint64)
    for i in range(m):
        out[:, i // 32] |= b[:, i] << np.uint64(i % 32)
    return out.astype(np.uint32)


def unpack_signs(words, m):
    w = np.asarray(words, dtype=np.uint64)
    n = w.shape[0]
    out = np.zeros((n, m), dtype=bool)
    for i in range(m):
        out[:, i] = ((w[:, i // 32] >> np.uint64(i % 32)) & np.uint64(1)) == 1
    return out


def residual_norms(r):
    """(fp16 rho, saturated mask)."""
    rn = np.sqrt(np.sum(np.asarray(r, dtype=np.float64) ** 2, axis=1))
    return np.minimum(rn, FP16_MAX).astype(np.float16), rn > FP16_MAX


def encode(y, x_hat_rot, S):
    """Residual signs (packed) and fp16 residual norm for each row."""
    r = residual(y, x_hat_rot)
    z = projections(r, S)
    rho, sat = residual_norms(r)
    return {"r": r, "z": z, "signs": pack_signs(sign_bits(z)), "rnorm": rho,
            "saturated": sat}


def estimate(q_rot, S, signs_bool, rnorm):
    """QJL estimate of <q_rot, r_t> for each stored row t.

    q_rot: [d]; signs_bool: [n, m]; rnorm: [n] (fp16 or float).
    """
    S = np.asarray(S, dtype=np.float64)
    m = S.shape[0]
    w = S @ np.asarray(q_rot, dtype=np.float64)
    pm = np.where(np.asarray(signs_bool), 1.0, -1.0)
    rho = np.asarray(rnorm).astype(np.float64)
    return np.sqrt(np.pi / 2.0) / m * rho * (pm @ w)
