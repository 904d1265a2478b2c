"""Pins for the oracle's paged cache and decode-time append (CPU only)."""

import numpy as np

from oracle import attention, codebook, paged, quant, rotation


def _setup(batch=2, n_kv=2, n_q=4, ctx=37, d=64, page=8, seed=0):
    rng = np.random.default_rng(seed)
    rot = rotation.wht_rotation(d, 1000)
    kc, kt = codebook.stored_table(4, 32)
    vc, vt = codebook.stored_table(3, 32)
    k = rng.standard_normal((batch, n_kv, ctx, d))
    v = rng.standard_normal((batch, n_kv, ctx, d))
    q = rng.standard_normal((batch, n_q, d))
    max_pages = (ctx + page - 1) // page
    n_pages = batch * max_pages + 3
    table = rng.permutation(n_pages)[:batch * max_pages].reshape(batch, max_pages)
    return rng, rot, kc, kt, vc, vt, k, v, q, table, n_pages, max_pages


def test_scatter_gather_round_trip_and_row_map():
    """Gathering what was scattered through the table returns the flat rows,
    and every (b, hk, t) lands on a distinct physical row of its own page."""
    batch, n_kv, ctx, page = 3, 2, 29, 8
    rng = np.random.default_rng(1)
    max_pages = (ctx + page - 1) // page
    n_pages = batch * max_pages + 2
    table = rng.permutation(n_pages)[:batch * max_pages].reshape(batch, max_pages)
    flat = rng.integers(0, 1 << 30, size=(batch * n_kv * ctx, 5))
    pages = np.zeros((n_pages * n_kv * page, 5), dtype=flat.dtype)
    pages = paged.scatter(pages, flat, table, page, n_kv, batch, ctx)
    assert np.array_equal(paged.gather(pages, table, page, n_kv, batch, ctx), flat)
    seen = set()
    for b in range(batch):
        for hk in range(n_kv):
            for t in range(ctx):
                r = paged.physical_row(table, page, n_kv, b, hk, t)
                assert r // (n_kv * page) == table[b][t // page]
                seen.add(r)
    assert len(seen) == batch * n_kv * ctx


def test_append_then_decode_equals_flat_quantize_and_decode():
    """Appending the new token through the table and decoding over the pages
    gives exactly the flat computation: quantize all ctx rows (row-wise, so
    the new row's codes do not depend on the others) and decode."""
    batch, n_kv, n_q, ctx, d, page = 2, 2, 4, 37, 64, 8
    rng, rot, kc, kt, vc, vt, k, v, q, table, n_pages, _ = _setup(batch, n_kv, n_q, ctx, d, page)
    qk = quant.quantize(k.reshape(-1, d), rot, kc, kt, 4, 32)
    qv = quant.quantize(v.reshape(-1, d), rot, vc, vt, 3, 32)
    flat_out = attention.decode(q, rot, qk["codes"], qk["norms"], kc, qv["codes"], qv["norms"], vc,
                                32, n_kv, ctx)
    # pages hold the first ctx - 1 tokens; position ctx - 1 holds garbage
    rows = n_pages * n_kv * page

    def fill(qz):
        codes = rng.integers(0, 8, size=(rows, d))
        norms = rng.standard_normal((rows, d // 32)).astype(np.float16)
        keep = np.ones(batch * n_kv * ctx, dtype=bool)
        keep.reshape(batch, n_kv, ctx)[:, :, ctx - 1] = False
        old_c = paged.gather(codes, table, page, n_kv, batch, ctx)
        old_n = paged.gather(norms, table, page, n_kv, batch, ctx)
        old_c[keep] = qz["codes"][keep]
        old_n[keep] = qz["norms"][keep]
        return {"codes": paged.scatter(codes, old_c, table, page, n_kv, batch, ctx),
                "norms": paged.scatter(norms, old_n, table, page, n_kv, batch, ctx)}
    kp, vp = fill(qk), fill(qv)
    out, kp2, vp2 = paged.append_and_decode(q, rot, k[:, :, ctx - 1], v[:, :, ctx - 1], kp, vp,
                                            table, page, n_kv, ctx, kc, kt, 4, vc, vt, 3)
    assert np.array_equal(out, flat_out)
    assert np.array_equal(paged.gather(kp2["codes"], table, page, n_kv, batch, ctx), qk["codes"])
    assert np.array_equal(paged.gather(vp2["norms"], table, page, n_kv, batch, ctx), qv["norms"])
