"""Pins for the oracle's QJL estimator, logits and decode (CPU only)."""

import numpy as np
import pytest
from scipy import special

from oracle import attention, codebook, qjl, quant, rotation


def test_gaussian_sign_identity():
    """E[sign(<s, r>) <s, q>] = sqrt(2/pi) <q, r> / ||r|| for s ~ N(0, I)."""
    rng = np.random.default_rng(0)
    d = 16
    q = rng.standard_normal(d)
    r = rng.standard_normal(d)
    s = rng.standard_normal((400_000, d))
    vals = np.sign(s @ r) * (s @ q)
    expect = np.sqrt(2 / np.pi) * (q @ r) / np.linalg.norm(r)
    assert abs(vals.mean() - expect) < 4 * vals.std() / np.sqrt(len(vals))


def test_sign_packing_and_zero_is_positive():
    z = np.array([[0.0, -1.0, 2.0] + [-0.5] * 29 + [1.0] * 32])
    bits = qjl.sign_bits(z)
    w = qjl.pack_signs(bits)
    assert w.shape == (1, 2)
    assert w[0, 0] == 0b101 and w[0, 1] == 0xFFFFFFFF
    assert np.array_equal(qjl.unpack_signs(w, 64), bits)


def test_qjl_estimator_unbiased_over_64_seeds():
    """Monte Carlo over the 64 QJL seeds 2000..2063 and 1024 (q, r) pairs."""
    d, m, n_pairs = 128, 128, 1024
    rng = np.random.default_rng(42)
    q = rng.standard_normal((n_pairs, d))
    r = rng.standard_normal((n_pairs, d)) * 0.3
    truth = np.sum(q * r, axis=1)
    errs = []
    for seed in range(2000, 2064):
        S = rotation.gaussian_projection(m, d, seed)
        enc_bits = qjl.sign_bits(r @ S.T)
        rn = np.linalg.norm(r, axis=1)
        est = np.array([qjl.estimate(q[i], S, enc_bits[i:i + 1], rn[i:i + 1])[0]
                        for i in range(n_pairs)])
        errs.append(est - truth)
    errs = np.array(errs)                    # [seeds, pairs]
    mean_err = errs.mean()
    se = errs.std() / np.sqrt(errs.size)
    assert abs(mean_err) < 4 * se
    # each projected term X_i = sqrt(pi/2) ||r|| sign(<s_i, r>) <s_i, q> has
    # E X_i^2 = (pi/2) ||q||^2 ||r||^2, so Var = ((pi/2)||q||^2||r||^2 - <q,r>^2) / m
    var_exact = (np.pi / 2 * np.sum(q * q, 1) * np.sum(r * r, 1) - truth ** 2) / m
    var_ratio = errs.var(axis=0) / var_exact
    assert 0.8 < np.median(var_ratio) < 1.2


def _small_cache(bits_k, bits_v, batch=2, n_kv=2, ctx=37, d=64, seed=0):
    rng = np.random.default_rng(seed)
    rot = rotation.wht_rotation(d, 1000)
    ck, tk = codebook.stored_table(bits_k, 32)
    cv, tv = codebook.stored_table(bits_v, 32)
    k = rng.standard_normal((batch * n_kv * ctx, d)) * 2.0
    v = rng.standard_normal((batch * n_kv * ctx, d))
    qk = quant.quantize(k, rot, ck, tk, bits_k, 32)
    qv = quant.quantize(v, rot, cv, tv, bits_v, 32)
    return rot, ck, cv, qk, qv


def test_logits_equal_original_frame_dot_products():
    """<R q, x_hat_rot> == <q, R^T x_hat_rot>, with q heads grouped over kv heads."""
    batch, n_kv, n_q, ctx, d = 2, 2, 4, 37, 64
    rot, ck, _, qk, _ = _small_cache(4, 3, batch, n_kv, ctx, d)
    q = np.random.default_rng(9).standard_normal((batch, n_q, d))
    lg = attention.logits(q, rot, qk["codes"], qk["norms"], ck, 32, n_kv, ctx)
    k_orig = quant.dequantize_rotated(qk["codes"], qk["norms"], ck, 32) @ rot
    k_orig = k_orig.reshape(batch, n_kv, ctx, d)
    for b in range(batch):
        for h in range(n_q):
            assert np.allclose(lg[b, h], k_orig[b, h // 2] @ q[b, h], rtol=1e-12, atol=1e-12)


def test_decode_equals_softmax_attention_in_original_frame():
    batch, n_kv, n_q, ctx, d = 2, 2, 8, 37, 64
    rot, ck, cv, qk, qv = _small_cache(4, 3, batch, n_kv, ctx, d)
    q = np.random.default_rng(10).standard_normal((batch, n_q, d))
    out = attention.decode(q, rot, qk["codes"], qk["norms"], ck, qv["codes"], qv["norms"], cv,
                           32, n_kv, ctx)
    kk = (quant.dequantize_rotated(qk["codes"], qk["norms"], ck, 32) @ rot).reshape(batch, n_kv, ctx, d)
    vv = (quant.dequantize_rotated(qv["codes"], qv["norms"], cv, 32) @ rot).reshape(batch, n_kv, ctx, d)
    for b in range(batch):
        for h in range(n_q):
            g = h // 4
            p = special.softmax(kk[b, g] @ q[b, h] / np.sqrt(d))
            assert np.allclose(out[b, h], p @ vv[b, g], rtol=1e-11, atol=1e-12)


def test_decode_single_token_returns_dequantized_value():
    rot, ck, cv, qk, qv = _small_cache(2, 2, batch=1, n_kv=1, ctx=1, d=64)
    q = np.random.default_rng(1).standard_normal((1, 2, 64))
    out = attention.decode(q, rot, qk["codes"], qk["norms"], ck, qv["codes"], qv["norms"], cv,
                           32, 1, 1)
    v_orig = quant.dequantize_rotated(qv["codes"], qv["norms"], cv, 32) @ rot
    assert np.allclose(out[0, 0], v_orig[0], atol=1e-12)
    assert np.allclose(out[0, 1], v_orig[0], atol=1e-12)


def test_decode_equal_keys_average_values():
    d, ctx = 64, 11
    rot = rotation.wht_rotation(d, 1000)
    ck, tk = codebook.stored_table(3, 32)
    k = np.tile(np.random.default_rng(2).standard_normal((1, d)), (ctx, 1))
    v = np.random.default_rng(3).standard_normal((ctx, d))
    qk = quant.quantize(k, rot, ck, tk, 3, 32)
    qv = quant.quantize(v, rot, ck, tk, 3, 32)
    q = np.random.default_rng(4).standard_normal((1, 1, d))
    out = attention.decode(q, rot, qk["codes"], qk["norms"], ck, qv["codes"], qv["norms"], ck,
                           32, 1, ctx)
    v_orig = quant.dequantize_rotated(qv["codes"], qv["norms"], ck, 32) @ rot
    assert np.allclose(out[0, 0], v_orig.mean(axis=0), atol=1e-12)


def test_decode_error_shrinks_with_bits():
    batch, n_kv, n_q, ctx, d = 1, 2, 4, 200, 128
    rng = np.random.default_rng(6)
    k = rng.standard_normal((batch * n_kv * ctx, d))
    v = rng.standard_normal((batch * n_kv * ctx, d))
    q = rng.standard_normal((batch, n_q, d)) * 2.0
    exact = np.empty((batch, n_q, d))
    for h in range(n_q):
        g = h // 2
        kk = k.reshape(n_kv, ctx, d)[g]
        vv = v.reshape(n_kv, ctx, d)[g]
        exact[0, h] = special.softmax(kk @ q[0, h] / np.sqrt(d)) @ vv
    rot = rotation.wht_rotation(d, 1000)
    errs = []
    for bits in (2, 3, 4):
        c, t = codebook.stored_table(bits, 32)
        qk = quant.quantize(k, rot, c, t, bits, 32)
        qv = quant.quantize(v, rot, c, t, bits, 32)
        out = attention.decode(q, rot, qk["codes"], qk["norms"], c, qv["codes"], qv["norms"], c,
                               32, n_kv, ctx)
        errs.append(np.linalg.norm(out - exact) / np.linalg.norm(exact))
    assert errs[0] > errs[1] > errs[2]


def test_logits_qjl_term_removes_the_mse_bias():
    """The QJL term is an unbiased estimate of <R q, r>: averaged over the 64
    QJL seeds the corrected logits approach the exact scores, far closer than
    the MSE-only logits (one draw alone has variance (pi/2)||q||^2||r||^2/m,
    larger than the MSE-stage error, so the check is on the seed average)."""
    d, ctx, m = 128, 300, 128
    rng = np.random.default_rng(8)
    k = rng.standard_normal((ctx, d))
    q = rng.standard_normal((1, 1, d))
    rot = rotation.wht_rotation(d, 1000)
    c, t = codebook.stored_table(2, 32)
    qk = quant.quantize(k, rot, c, t, 2, 32)
    xh = quant.dequantize_rotated(qk["codes"], qk["norms"], c, 32)
    mse = attention.logits(q, rot, qk["codes"], qk["norms"], c, 32, 1, ctx)[0, 0]
    exact = k @ q[0, 0]
    full = []
    for seed in range(2000, 2064):
        S = rotation.gaussian_projection(m, d, seed)
        enc = qjl.encode(qk["y"], xh, S)
        full.append(attention.logits(q, rot, qk["codes"], qk["norms"], c, 32, 1, ctx,
                                     qjl={"S": S, "signs": qjl.unpack_signs(enc["signs"], m),
                                          "rnorm": enc["rnorm"]})[0, 0])
    avg = np.mean(full, axis=0)
    assert np.mean((avg - exact) ** 2) < 0.2 * np.mean((mse - exact) ** 2)
    # the MSE-only stage shrinks inner products; the corrected one does not
    slope_mse = np.polyfit(exact, mse, 1)[0]
    slope_full = np.polyfit(exact, avg, 1)[0]
    assert slope_mse < 0.97 and abs(slope_full - 1.0) < 0.02
