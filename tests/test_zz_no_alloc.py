"""GPU tests of tq_decode_attention_static, the decode entry point for callers
that cannot allocate device memory while they enqueue work (its split partials
live in a fixed array inside the library instead of a caller workspace).  Kept
in its own file so that pytest collects it last.

Checks, through the C ABI:
* two calls in a row, with a call of a different, larger shape between them
  (so the shared array holds unrelated partials when the second call starts),
  each give exactly the output of the workspace-taking tq_decode_attention run
  on a NaN-filled workspace (a partial slot that the split step failed to write
  would leak NaN or stale data into the result);
* the output matches the oracle within the decode tolerance of the other tests;
* a shape whose partials do not fit the array is rejected before anything is
  launched (real, full-size device buffers, so nothing could be read out of
  bounds even if the check were missing)."""

import numpy as np
import pytest

import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _cache(tq, rot, batch, n_kv, n_q, ctx, d, kb, vb, seed):
    ck, tk = tq.build_codebook(kb)
    cv, tv = tq.build_codebook(vb)
    k64 = W.kv_host(batch, n_kv, ctx, d, seed=seed)
    v64 = W.kv_host(batch, n_kv, ctx, d, seed=seed + 1)
    q64 = W.queries_host(batch, n_q, d)
    k = torch.from_numpy(k64).to("cuda", torch.bfloat16)
    v = torch.from_numpy(v64).to("cuda", torch.bfloat16)
    q = torch.from_numpy(q64).to("cuda", torch.bfloat16)
    kq = tq.quantize_kv(rot, kb, ck, tk, k)
    vq = tq.quantize_kv(rot, vb, cv, tv, v)
    return dict(ck=ck, cv=cv, q=q, q64=q64, kq=kq, vq=vq)


def test_static_scratch_decode_matches_workspace_decode_and_oracle():
    import kv_cache_vector_11_b200 as tq
    assert torch.cuda.is_available()
    d, kb, vb = 128, 4, 3
    rot = tq.Rotation("wht", d, d, W.SEED_ROT)
    small = dict(batch=2, n_kv=4, n_q=16, ctx=5000)
    large = dict(batch=4, n_kv=8, n_q=32, ctx=3000)
    for s in (small, large):
        assert tq.decode_workspace_size(s["batch"], s["n_q"], s["n_kv"], s["ctx"], d) <= \
            tq.DECODE_STATIC_SCRATCH_BYTES
    a = _cache(tq, rot, small["batch"], small["n_kv"], small["n_q"], small["ctx"], d, kb, vb, 31)
    b = _cache(tq, rot, large["batch"], large["n_kv"], large["n_q"], large["ctx"], d, kb, vb, 33)

    def workspace_decode(c, s):
        need = tq.decode_workspace_size(s["batch"], s["n_q"], s["n_kv"], s["ctx"], d)
        ws = torch.full((max(need, 16) // 4 + 1,), float("nan"), dtype=torch.float32,
                        device="cuda")
        return tq.decode_attention(rot, kb, vb, c["ck"], c["cv"], c["q"], c["kq"]["codes"],
                                   c["kq"]["norms"], c["vq"]["codes"], c["vq"]["norms"],
                                   s["n_kv"], s["ctx"], workspace=ws.view(torch.uint8))

    def static_decode(c, s, out):
        out.fill_(float("nan"))
        tq.decode_attention_static(rot, kb, vb, c["ck"], c["cv"], c["q"], c["kq"]["codes"],
                                   c["kq"]["norms"], c["vq"]["codes"], c["vq"]["norms"],
                                   s["n_kv"], s["ctx"], out=out)
        torch.cuda.synchronize()
        return out.cpu().numpy()

    ref_a = workspace_decode(a, small).cpu().numpy()
    ref_b = workspace_decode(b, large).cpu().numpy()
    assert np.all(np.isfinite(ref_a)) and np.all(np.isfinite(ref_b))
    out_a = torch.empty(ref_a.shape, dtype=torch.float32, device="cuda")
    out_b = torch.empty(ref_b.shape, dtype=torch.float32, device="cuda")

    first = static_decode(a, small, out_a)
    assert np.array_equal(first, ref_a)
    between = static_decode(b, large, out_b)     # fills the array with other partials
    assert np.array_equal(between, ref_b)
    second = static_decode(a, small, out_a)
    assert np.array_equal(second, ref_a)

    oracle = P.oracle_decode_on_cache(
        a["q64"], P.oracle_rotation("wht", d, W.SEED_ROT), kb, vb,
        P.to_np_u32(a["kq"]["codes"]), P.to_np_f16(a["kq"]["norms"]),
        P.to_np_u32(a["vq"]["codes"]), P.to_np_f16(a["vq"]["norms"]), small["n_kv"], small["ctx"])
    P.check_decode(second.astype(np.float64), oracle)


def test_static_scratch_rejects_oversized_shapes():
    import kv_cache_vector_11_b200 as tq
    batch, n_kv, n_q, ctx, d, bits = 64, 32, 128, 512, 256, 3
    assert tq.decode_workspace_size(batch, n_q, n_kv, ctx, d) > tq.DECODE_STATIC_SCRATCH_BYTES
    rows = batch * n_kv * ctx
    words = tq.code_words_per_row(bits, 32, d)
    rot = tq.Rotation("wht", d, d, W.SEED_ROT)
    c, _ = tq.build_codebook(bits)
    kc = torch.zeros((rows, words), dtype=torch.int32, device="cuda")
    kn = torch.zeros((rows, d // 32), dtype=torch.int16, device="cuda")
    vc = torch.zeros_like(kc)
    vn = torch.zeros_like(kn)
    q = torch.zeros((batch, n_q, d), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((batch, n_q, d), dtype=torch.float32, device="cuda")
    with pytest.raises(tq.TQError) as err:
        tq.decode_attention_static(rot, bits, bits, c, c, q, kc, kn, vc, vn, n_kv, ctx, out=out)
    assert err.value.status == 2   # TQ_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert int(torch.count_nonzero(out).item()) == 0   # nothing was launched
