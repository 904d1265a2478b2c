"""Attention over the packed cache: raw logits and single-token decode.

TEST INFRASTRUCTURE (oracle).  Not imported by the product path.

Upstream guide, section 5.3 (pre-rotate-queries): because the rotation is
fixed and shared, <q, R^T c[idx]> = <R q, c[idx]>; the query is rotated once
instead of inverse-rotating every cached key.  "Google TurboQuant deep dive",
section 4.3: Attention(Q, K, V) = softmax(Q K^T / sqrt(d)) V with Q kept in
full precision.  Upstream guide, section 6.1: the inverse-rotation fix -- the
value sum, accumulated in the rotated frame, is rotated back with R^T.
Section 5.4: K and V may use different bit widths.

Readings taken where the pages are silent:

* layouts: cache rows are ordered [batch][kv_head][token]; queries are
  [batch][q_head][d]; q_head h reads kv_head h // (Hq / Hkv) (contiguous
  grouped-query sharing);
* one rotation R serves K and V of a layer;
* ``logits`` returns the raw score <R q, x_hat_rot> (+ the QJL term when
  present) without the 1/sqrt(d) factor; ``decode`` uses scale 1/sqrt(d)
  unless another scale is given;
* the decode output is float (fp32 in the library), in the original frame.
"""

import numpy as np

from . import qjl as qjl_mod
from .quant import dequantize_rotated


def rotate_queries(q, rot):
    """q_rot = R q for q of shape [..., d]."""
    q = np.asarray(q, dtype=np.float64)
    return q @ np.asarray(rot, dtype=np.float64).T


def _cache_view(arr, batch, n_kv_heads, ctx):
    return np.asarray(arr).reshape(batch, n_kv_heads, ctx, *np.asarray(arr).shape[1:])


def logits(q, rot, k_codes, k_norms, k_centroids, block, n_kv_heads, ctx,
           qjl=None, norm_dtype="f16"):
    """Raw scores [B, Hq, T].

    q: [B, Hq, d]; k_codes: unpacked codes [B*Hkv*T, d]; k_norms: stored
    norms [B*Hkv*T, d/block] (fp16, or fp32 with ``norm_dtype="f32"``); qjl:
    optional dict with ``S`` (m x d), ``signs`` (bool [B*Hkv*T, m]) and
    ``rnorm`` (fp16 [B*Hkv*T]).
    """
    q = np.asarray(q, dtype=np.float64)
    batch, n_q_heads, d = q.shape
    group = n_q_heads // n_kv_heads
    q_rot = rotate_queries(q, rot)
    k_hat = dequantize_rotated(k_codes, k_norms, k_centroids, block, norm_dtype)
    k_hat = k_hat.reshape(batch, n_kv_heads, ctx, d)
    out = np.empty((batch, n_q_heads, ctx), dtype=np.float64)
    for b in range(batch):
        for h in range(n_q_heads):
            g = h // group
            s = k_hat[b, g] @ q_rot[b, h]
            if qjl is not None:
                rows = slice((b * n_kv_heads + g) * ctx, (b * n_kv_heads + g + 1) * ctx)
                s = s + qjl_mod.estimate(q_rot[b, h], qjl["S"], qjl["signs"][rows],
                                         qjl["rnorm"][rows])
            out[b, h] = s
    return out


def softmax(z):
    """Max-subtracted softmax along the last axis."""
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(z - np.max(z, axis=-1, keepdims=True))
    return e / np.sum(e, axis=-1, keepdims=True)


def decode(q, rot, k_codes, k_norms, k_centroids, v_codes, v_norms, v_centroids,
           block, n_kv_heads, ctx, scale=None, qjl=None, norm_dtype="f16"):
    """Single-step decode output [B, Hq, d] in the original frame.

    p = softmax(scale * logits); o_rot = sum_t p_t * v_hat_rot[t];
    o = R^T o_rot.
    """
    q = np.asarray(q, dtype=np.float64)
    batch, n_q_heads, d = q.shape
    group = n_q_heads // n_kv_heads
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    s = logits(q, rot, k_codes, k_norms, k_centroids, block, n_kv_heads, ctx, qjl, norm_dtype)
    p = softmax(scale * s)
    v_hat = dequantize_rotated(v_codes, v_norms, v_centroids, block, norm_dtype)
    v_hat = v_hat.reshape(batch, n_kv_heads, ctx, d)
    rot = np.asarray(rot, dtype=np.float64)
    out = np.empty((batch, n_q_heads, d), dtype=np.float64)
    for b in range(batch):
        for h in range(n_q_heads):
            o_rot = p[b, h] @ v_hat[b, h // group]
            out[b, h] = rot.T @ o_rot
    return out
