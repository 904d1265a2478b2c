"""Paged KV cache with the new token appended during decode.

TEST INFRASTRUCTURE (oracle).  Not imported by the product path.

Upstream guide, section 5.2 (Phase 1 file table): the KV-cache manager
(``src/llama-kv-cache.cpp``) owns the compressed cache and the graph quantizes
each new token's K and V into it before attention reads it.  The pages print no
page layout; the reading taken here is the usual block-table paging:

* the cache of every kv head is cut into pages of ``page_size`` tokens; page
  storage is [n_pages][n_kv_heads][page_size][row] (a row is one token's packed
  codes, or its norms), so one physical page holds a run of tokens of one
  sequence for all its kv heads;
* ``block_table[b][j]`` is the physical page holding tokens
  [j * page_size, (j + 1) * page_size) of sequence b;
* a decode step with context length ``ctx`` (the new token included) first
  quantizes the new token's K and V rows exactly like ``quant.quantize`` and
  stores them at position ctx - 1, then attends over tokens 0 .. ctx - 1 with
  ``attention.decode``.
"""

import numpy as np

from . import attention, quant


def physical_row(block_table, page_size, n_kv_heads, b, hk, t):
    """Row index into [n_pages * n_kv_heads * page_size] page storage."""
    page = int(block_table[b][t // page_size])
    return (page * n_kv_heads + hk) * page_size + t % page_size


def gather(pages, block_table, page_size, n_kv_heads, batch, ctx):
    """Flat [batch * n_kv_heads * ctx, ...] rows ([b][hk][t] order) of the
    first ctx tokens of every sequence, read through the block table."""
    pages = np.asarray(pages)
    out = []
    for b in range(batch):
        for hk in range(n_kv_heads):
            for t in range(ctx):
                out.append(pages[physical_row(block_table, page_size, n_kv_heads, b, hk, t)])
    return np.stack(out)


def scatter(pages, rows, block_table, page_size, n_kv_heads, batch, ctx):
    """Write flat rows ([b][hk][t] order, ctx per sequence) into page storage."""
    pages = np.array(pages, copy=True)
    rows = np.asarray(rows)
    i = 0
    for b in range(batch):
        for hk in range(n_kv_heads):
            for t in range(ctx):
                pages[physical_row(block_table, page_size, n_kv_heads, b, hk, t)] = rows[i]
                i += 1
    return pages


def append_and_decode(q, rot, k_new, v_new, k_pages, v_pages, block_table, page_size,
                      n_kv_heads, ctx, kc, kt, kbits, vc, vt, vbits, block=32, scale=None):
    """One decode step on a paged cache.

    k_new, v_new: [batch, n_kv_heads, d] new rows; k_pages / v_pages: dicts
    with unpacked ``codes`` [rows, d] and ``norms`` [rows, d / block] page
    storage.  Returns (output [batch, n_q_heads, d], updated k_pages,
    updated v_pages)."""
    q = np.asarray(q, dtype=np.float64)
    batch, _, d = q.shape
    pages = {}
    for name, new, pg, c, t, bits in (("k", k_new, k_pages, kc, kt, kbits),
                                       ("v", v_new, v_pages, vc, vt, vbits)):
        rows = np.asarray(new, dtype=np.float64).reshape(batch * n_kv_heads, d)
        qz = quant.quantize(rows, rot, c, t, bits, block)
        codes = np.array(pg["codes"], copy=True)
        norms = np.array(pg["norms"], copy=True)
        for b in range(batch):
            for hk in range(n_kv_heads):
                r = physical_row(block_table, page_size, n_kv_heads, b, hk, ctx - 1)
                codes[r] = qz["codes"][b * n_kv_heads + hk]
                norms[r] = qz["norms"][b * n_kv_heads + hk]
        pages[name] = {"codes": codes, "norms": norms}
    kf = gather(pages["k"]["codes"], block_table, page_size, n_kv_heads, batch, ctx)
    kn = gather(pages["k"]["norms"], block_table, page_size, n_kv_heads, batch, ctx)
    vf = gather(pages["v"]["codes"], block_table, page_size, n_kv_heads, batch, ctx)
    vn = gather(pages["v"]["norms"], block_table, page_size, n_kv_heads, batch, ctx)
    out = attention.decode(q, rot, kf, kn, kc, vf, vn, vc, block, n_kv_heads, ctx, scale=scale)
    return out, pages["k"], pages["v"]
