"""Pins for the oracle's inner-product search over codes (CPU only)."""

import numpy as np
import pytest

from oracle import codebook, quant, rotation, search


def test_topk_equals_brute_force_selection():
    """Against a plain Python selection, including exact ties (ties by index)."""
    rng = np.random.default_rng(1)
    s = np.round(rng.standard_normal((5, 40)), 1)     # many exact ties
    for k in (1, 3, 7, 40, 50):
        vals, idx = search.topk(s, k)
        for i in range(5):
            ref = sorted(range(40), key=lambda j: (-s[i, j], j))[:min(k, 40)]
            assert list(idx[i]) == ref
            assert np.array_equal(vals[i], s[i, ref])


def test_scores_are_original_frame_inner_products():
    """<R q, x_hat> = <q, R^T x_hat> (upstream guide, section 5.3)."""
    d, n = 64, 50
    rng = np.random.default_rng(2)
    rot = rotation.haar_rotation(d, 1000)
    c, t = codebook.stored_table(3, 32)
    x = rng.standard_normal((n, d))
    qz = quant.quantize(x, rot, c, t, 3, 32)
    q = rng.standard_normal((4, d))
    s = search.scores(q, rot, qz["codes"], qz["norms"], c, 32)
    x_orig = quant.dequantize_rotated(qz["codes"], qz["norms"], c, 32) @ rot
    assert np.allclose(s, q @ x_orig.T, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("bits", [2, 4])
def test_planted_neighbours_are_found(bits):
    """Each query is a database row plus small noise, so that row is the exact
    maximum-inner-product answer by a wide margin (<x, x> ~ d against
    |<x, x'>| ~ sqrt(d)); the search over 2- and 4-bit codes returns it first."""
    d, n, n_q = 128, 2000, 40
    rng = np.random.default_rng(3)
    x = rng.standard_normal((n, d))
    planted = rng.choice(n, n_q, replace=False)
    q = x[planted] + 0.05 * rng.standard_normal((n_q, d))
    rot = rotation.wht_rotation(d, 1000)
    c, t = codebook.stored_table(bits, 32)
    qz = quant.quantize(x, rot, c, t, bits, 32)
    _, idx = search.topk(search.scores(q, rot, qz["codes"], qz["norms"], c, 32), 1)
    assert np.array_equal(idx[:, 0], planted)
