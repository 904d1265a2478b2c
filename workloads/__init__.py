"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the method (no rotation, norm, codebook or
attention): only random numbers and the shapes, scales and dtypes of the
workloads.  The CUDA library and the oracle both consume what it produces;
neither is imported here.

Recipe (stand-in for the pages' wikitext-2 / NIAH / LongBench / GloVe data,
none of which is available or needed for the hot path):

* keys and values are z * s[h, c]: z ~ N(0, 1) per element; s[h, c] =
  exp(N(0, 1)) per (KV head, channel); in every head 4 channels drawn without
  replacement are multiplied by 20 (outlier channels, as seen in real K/V
  activations).  K and V draw independent scales.  Rounded to bf16 (RNE).
* queries are N(0, 1), bf16 (or fp32 for the 4096-key fp32 workload).
* every array is a pure function of its seed and shape.

Workloads (sizes as the benchmark configurations state them):

* ``keys4096``   4096 fp32 keys ~ N(0,1) (numpy PCG64 seed 0), d=128, one KV
  head, one fp32 query (seed 1); WHT rotation, 4-bit, block 32.
* ``llama8b_32k`` B=1, Hkv=8, Hq=32, T=32768, d=128, 3-bit K and V.
* ``qjl_16k``    B=16, Hkv=8, Hq=32, T=16384, d=128, 2-bit + QJL m=128.
* ``decode_128k`` B=8, Hkv=8, Hq=32, T=131072, d=128, 4-bit K, 3-bit V.
* ``prefill_1m`` 2^20 bf16 rows of one head, d in {64,128,256}, bits in
  {2,3,4}, WHT and Haar rotations.
"""

import numpy as np

SEED_K = 0
SEED_V = 1
SEED_Q = 7
SEED_ROT = 1000
SEED_QJL = 2000

WORKLOADS = {
    "keys4096": dict(batch=1, n_kv_heads=1, n_q_heads=1, ctx=4096, head_dim=128,
                     k_bits=4, v_bits=4, block=32, rot="wht", dtype="f32"),
    "llama8b_32k": dict(batch=1, n_kv_heads=8, n_q_heads=32, ctx=32768, head_dim=128,
                        k_bits=3, v_bits=3, block=32, rot="wht", dtype="bf16"),
    "qjl_16k": dict(batch=16, n_kv_heads=8, n_q_heads=32, ctx=16384, head_dim=128,
                    k_bits=2, v_bits=2, block=32, rot="wht", dtype="bf16", qjl_m=128),
    "decode_128k": dict(batch=8, n_kv_heads=8, n_q_heads=32, ctx=131072, head_dim=128,
                        k_bits=4, v_bits=3, block=32, rot="wht", dtype="bf16"),
    "prefill_1m": dict(rows=1 << 20, head_dims=(64, 128, 256), bits=(2, 3, 4),
                       block=32, rots=("wht", "haar"), dtype="bf16"),
    # the 128K decode workload on a paged cache (pages of 256 tokens, a random
    # block table), one decode step that appends its own token
    "paged_128k": dict(batch=8, n_kv_heads=8, n_q_heads=32, ctx=131072, head_dim=128,
                       k_bits=4, v_bits=3, block=32, rot="wht", dtype="bf16", page_size=256),
    # inner-product search: 2^20 database rows of one head, 64 queries, top 10
    "search_1m": dict(n_db=1 << 20, n_queries=64, k=10, head_dim=128, bits=4, block=32,
                      rot="wht", dtype="bf16"),
}


def outlier_scales(seed, n_heads, d, n_outliers=4, factor=20.0):
    """Per (head, channel) scale exp(N(0,1)); ``n_outliers`` channels per head x20."""
    rng = np.random.default_rng(seed)
    s = np.exp(rng.standard_normal((n_heads, d)))
    for h in range(n_heads):
        idx = rng.choice(d, size=n_outliers, replace=False)
        s[h, idx] *= factor
    return s


def _to_bf16_f64(x):
    """Round a float array to bf16 (RNE) and return it as float64."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.to(torch.float64).numpy()


def kv_host(batch, n_kv_heads, ctx, d, seed, dtype="bf16"):
    """Host K or V cache input [batch*n_kv_heads*ctx, d] as float64 values
    exactly representable in ``dtype`` (rows ordered [batch][head][token])."""
    scales = outlier_scales(seed + 10_000, n_kv_heads, d)
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((batch, n_kv_heads, ctx, d))
    x = z * scales[None, :, None, :]
    x = x.reshape(batch * n_kv_heads * ctx, d)
    if dtype == "bf16":
        return _to_bf16_f64(x)
    return x.astype(np.float32).astype(np.float64)


def kv_device(batch, n_kv_heads, ctx, d, seed, device="cuda"):
    """Device bf16 K or V cache input [batch*n_kv_heads*ctx, d] (torch),
    same recipe as ``kv_host`` but drawn with torch's generator on ``device``.
    Generated in head-sized pieces to bound the fp32 temporary."""
    import torch
    scales = torch.from_numpy(outlier_scales(seed + 10_000, n_kv_heads, d)).to(
        device=device, dtype=torch.float32)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    out = torch.empty((batch, n_kv_heads, ctx, d), dtype=torch.bfloat16, device=device)
    for b in range(batch):
        for h in range(n_kv_heads):
            z = torch.randn((ctx, d), generator=gen, device=device, dtype=torch.float32)
            out[b, h] = (z * scales[h][None, :]).to(torch.bfloat16)
    return out.reshape(batch * n_kv_heads * ctx, d)


def normal_rows_host(n, d, seed, dtype="f32"):
    """n x d N(0,1) rows from numpy PCG64 (``default_rng(seed)``)."""
    x = np.random.default_rng(seed).standard_normal((n, d))
    if dtype == "bf16":
        return _to_bf16_f64(x)
    return x.astype(np.float32).astype(np.float64)


def prefill_rows_host(n, d, seed):
    """n bf16 rows of one head with outlier channels (host, float64 values)."""
    return kv_host(1, 1, n, d, seed, "bf16")


def prefill_rows_device(n, d, seed, device="cuda"):
    return kv_device(1, 1, n, d, seed, device)


def queries_host(batch, n_q_heads, d, seed=SEED_Q, dtype="bf16"):
    """Queries [batch, n_q_heads, d] ~ N(0,1) as float64 values of ``dtype``."""
    x = np.random.default_rng(seed).standard_normal((batch, n_q_heads, d))
    if dtype == "bf16":
        return _to_bf16_f64(x)
    return x.astype(np.float32).astype(np.float64)


def keys4096_host():
    """The 4096-key fp32 workload: keys (seed 0) and one query (seed 1)."""
    keys = np.random.default_rng(0).standard_normal((4096, 128)).astype(np.float32)
    query = np.random.default_rng(1).standard_normal((1, 1, 128)).astype(np.float32)
    return keys.astype(np.float64), query.astype(np.float64)
