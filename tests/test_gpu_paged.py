"""GPU parity of tq_decode_append_paged: one decode step over a block-table
paged cache that first quantizes the step's own K / V rows into token
ctx - 1 ("TurboQuant+ upstream guide", section 5.2: the KV-cache manager and
the graph-side quantize of each new token).

The cache of the first ctx - 1 tokens is written by tq_quantize_kv and
scattered into pages through a random block table (token ctx - 1's slots hold
garbage).  Checks: the appended rows equal the oracle's quantization of the
new rows (codes bit-exact outside the 1e-5 band, norms within one fp16 ulp);
the output equals the oracle's decode over the cache gathered back through
the table; pages no sequence owns are untouched; consecutive steps that
cross into a new page work; both rotations, every head dim, GQA groups of
4 and 8, ragged contexts."""

import numpy as np
import pytest

import workloads as W
from oracle import paged as opaged
from tests import parity as P

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tq():
    import kv_cache_vector_11_b200 as lib
    assert torch.cuda.is_available(), "GPU tests need CUDA"
    return lib


def _rows(table, page, n_kv, batch, ctx):
    return np.array([opaged.physical_row(table, page, n_kv, b, hk, t)
                     for b in range(batch) for hk in range(n_kv) for t in range(ctx)])


def _run(tq, kind, d, kb, vb, batch, n_kv, n_q, ctx0, page, steps, seed=5):
    rng = np.random.default_rng(seed)
    ctx_max = ctx0 + steps - 1
    max_pages = (ctx_max + page - 1) // page
    n_pages = batch * max_pages + 3
    table = rng.permutation(n_pages)[:batch * max_pages].reshape(batch, max_pages).astype(np.int32)
    k64 = W.kv_host(batch, n_kv, ctx_max, d, seed=seed + 1).reshape(batch, n_kv, ctx_max, d)
    v64 = W.kv_host(batch, n_kv, ctx_max, d, seed=seed + 2).reshape(batch, n_kv, ctx_max, d)
    rot = tq.Rotation(kind, d, d, W.SEED_ROT)
    kcb, vcb = tq.build_codebook(kb), tq.build_codebook(vb)
    wk, wv, nb = tq.code_words_per_row(kb, 32, d), tq.code_words_per_row(vb, 32, d), d // 32
    # pages full of garbage, then the first ctx0 - 1 tokens written through the table
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    pages = {
        "k_codes": torch.randint(-2**31, 2**31 - 1, (n_pages, n_kv, page, wk), generator=g,
                                 device="cuda", dtype=torch.int32),
        "k_norms": torch.randint(0, 2**14, (n_pages, n_kv, page, nb), generator=g, device="cuda",
                                 dtype=torch.int16),
        "v_codes": torch.randint(-2**31, 2**31 - 1, (n_pages, n_kv, page, wv), generator=g,
                                 device="cuda", dtype=torch.int32),
        "v_norms": torch.randint(0, 2**14, (n_pages, n_kv, page, nb), generator=g, device="cuda",
                                 dtype=torch.int16)}
    pre = ctx0 - 1
    if pre > 0:
        for name, x64, bits, cb in (("k", k64, kb, kcb), ("v", v64, vb, vcb)):
            xq = tq.quantize_kv(rot, bits, cb[0], cb[1],
                                torch.from_numpy(x64[:, :, :pre].reshape(-1, d)).to("cuda", torch.bfloat16))
            idx = torch.from_numpy(_rows(table, page, n_kv, batch, pre)).cuda()
            pages[name + "_codes"].view(-1, pages[name + "_codes"].shape[-1])[idx] = xq["codes"]
            pages[name + "_norms"].view(-1, nb)[idx] = xq["norms"]
    owned = set(table.ravel().tolist())
    spare = [p for p in range(n_pages) if p not in owned]
    spare_before = {k: v[spare].clone() for k, v in pages.items()}
    bt = torch.from_numpy(table).cuda()
    q64 = W.queries_host(batch, n_q, d)
    q = torch.from_numpy(q64).to("cuda", torch.bfloat16)
    rot64 = P.oracle_rotation(kind, d, W.SEED_ROT)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for step in range(steps):
        ctx = ctx0 + step
        kn = torch.from_numpy(k64[:, :, ctx - 1]).to("cuda", torch.bfloat16).contiguous()
        vn = torch.from_numpy(v64[:, :, ctx - 1]).to("cuda", torch.bfloat16).contiguous()
        out = tq.decode_append_paged(rot, kb, vb, kcb, vcb, q, kn, vn, pages, bt, n_kv, ctx, page,
                                     status=status)
        torch.cuda.synchronize()
        rows = _rows(table, page, n_kv, batch, ctx)
        kc = P.to_np_u32(pages["k_codes"].view(-1, wk))[rows]
        kno = P.to_np_f16(pages["k_norms"].view(-1, nb))[rows]
        vc = P.to_np_u32(pages["v_codes"].view(-1, wv))[rows]
        vno = P.to_np_f16(pages["v_norms"].view(-1, nb))[rows]
        last = np.arange(batch * n_kv) * ctx + ctx - 1
        new_k = k64[:, :, ctx - 1].reshape(-1, d)
        new_v = v64[:, :, ctx - 1].reshape(-1, d)
        P.compare_quantize(new_k, rot64, kb, kc[last], kno[last])
        P.compare_quantize(new_v, rot64, vb, vc[last], vno[last])
        ref = P.oracle_decode_on_cache(q64, rot64, kb, vb, kc, kno, vc, vno, n_kv, ctx)
        P.check_decode(out.cpu().numpy().astype(np.float64), ref)
    assert int(status.item()) == 0
    for k, v in pages.items():
        assert torch.equal(v[spare], spare_before[k]), k


@pytest.mark.parametrize("kind", ["wht", "haar"])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_append_paged_parity(tq, kind, d):
    _run(tq, kind, d, 4, 3, batch=2, n_kv=2, n_q=8, ctx0=1001, page=64, steps=1)


@pytest.mark.parametrize("page,ctx0,steps", [(16, 30, 4), (128, 127, 3), (256, 1, 2)])
def test_append_paged_crosses_pages(tq, page, ctx0, steps):
    # 30..33 crosses the 32-token boundary of 16-token pages; 127..129 the
    # 128 boundary; 1..2 starts from an empty cache
    _run(tq, "wht", 128, 3, 3, batch=3, n_kv=2, n_q=16, ctx0=ctx0, page=page, steps=steps)


def test_append_paged_bit_mixes_and_mha(tq):
    _run(tq, "wht", 128, 2, 4, batch=1, n_kv=4, n_q=4, ctx0=333, page=32, steps=1)
