"""GPU parity of tq_attn_logits and tq_decode_attention against the oracle,
scored on the library's own packed cache (needs a B200)."""

import numpy as np
import pytest

import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tq():
    import kv_cache_vector_11_b200 as lib
    assert torch.cuda.is_available(), "GPU tests need CUDA"
    return lib


def _quantize(tq, rot, bits, x64, dtype="bf16"):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = torch.from_numpy(x64).to(device="cuda", dtype=tdt)
    c, t = tq.build_codebook(bits)
    return tq.quantize_kv(rot, bits, c, t, x), c


def test_keys4096_logits(tq):
    keys, query = W.keys4096_host()
    rot = tq.Rotation("wht", 128, 128, W.SEED_ROT)
    kq, c = _quantize(tq, rot, 4, keys, "f32")
    q = torch.from_numpy(query).to(device="cuda", dtype=torch.float32)
    lg = tq.attn_logits(rot, 4, c, q, kq["codes"], kq["norms"], 1, 4096)
    torch.cuda.synchronize()
    ref = P.oracle_logits_on_cache(query, P.oracle_rotation("wht", 128, W.SEED_ROT), 4,
                                   P.to_np_u32(kq["codes"]), P.to_np_f16(kq["norms"]), 1, 4096)
    P.check_logits(lg.cpu().numpy().astype(np.float64), ref, query, keys, 1, 4096)


@pytest.mark.parametrize("kind", ["wht", "haar"])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_logits_gqa_ragged(tq, kind, d):
    batch, n_kv, n_q, ctx = 2, 2, 8, 2500
    k64 = W.kv_host(batch, n_kv, ctx, d, seed=11)
    q64 = W.queries_host(batch, n_q, d)
    rot = tq.Rotation(kind, d, d, W.SEED_ROT)
    kq, c = _quantize(tq, rot, 3, k64)
    q = torch.from_numpy(q64).to(device="cuda", dtype=torch.bfloat16)
    lg = tq.attn_logits(rot, 3, c, q, kq["codes"], kq["norms"], n_kv, ctx)
    torch.cuda.synchronize()
    ref = P.oracle_logits_on_cache(q64, P.oracle_rotation(kind, d, W.SEED_ROT), 3,
                                   P.to_np_u32(kq["codes"]), P.to_np_f16(kq["norms"]), n_kv, ctx)
    P.check_logits(lg.cpu().numpy().astype(np.float64), ref, q64, k64, n_kv, ctx)


# tensor-core scores: CTA ranges that meet several (batch, kv head, group) units,
# tiny contexts (4 slabs per unit), 8 heads per kv head (two groups), Haar
@pytest.mark.parametrize("kind,d,bits,batch,n_kv,n_q,ctx", [
    ("wht", 128, 4, 4, 8, 32, 3000), ("wht", 128, 2, 3, 4, 16, 64), ("haar", 64, 3, 2, 2, 16, 520),
    ("wht", 64, 4, 1, 1, 1, 24)])
def test_logits_tensor_core_shapes(tq, kind, d, bits, batch, n_kv, n_q, ctx):
    k64 = W.kv_host(batch, n_kv, ctx, d, seed=13)
    q64 = W.queries_host(batch, n_q, d)
    rot = tq.Rotation(kind, d, d, W.SEED_ROT)
    kq, c = _quantize(tq, rot, bits, k64)
    q = torch.from_numpy(q64).to("cuda", torch.bfloat16)
    lg = tq.attn_logits(rot, bits, c, q, kq["codes"], kq["norms"], n_kv, ctx)
    torch.cuda.synchronize()
    ref = P.oracle_logits_on_cache(q64, P.oracle_rotation(kind, d, W.SEED_ROT), bits,
                                   P.to_np_u32(kq["codes"]), P.to_np_f16(kq["norms"]), n_kv, ctx)
    P.check_logits(lg.cpu().numpy().astype(np.float64), ref, q64, k64, n_kv, ctx)


def _decode_case(tq, kind, d, kbits, vbits, batch, n_kv, n_q, ctx, q_dtype="bf16", scale=0.0):
    k64 = W.kv_host(batch, n_kv, ctx, d, seed=21)
    v64 = W.kv_host(batch, n_kv, ctx, d, seed=22)
    q64 = W.queries_host(batch, n_q, d, dtype=q_dtype)
    rot = tq.Rotation(kind, d, d, W.SEED_ROT)
    kq, ck = _quantize(tq, rot, kbits, k64)
    vq, cv = _quantize(tq, rot, vbits, v64)
    tdt = torch.bfloat16 if q_dtype == "bf16" else torch.float32
    q = torch.from_numpy(q64).to(device="cuda", dtype=tdt)
    out = tq.decode_attention(rot, kbits, vbits, ck, cv, q, kq["codes"], kq["norms"],
                              vq["codes"], vq["norms"], n_kv, ctx, scale=scale)
    torch.cuda.synchronize()
    ref = P.oracle_decode_on_cache(q64, P.oracle_rotation(kind, d, W.SEED_ROT), kbits, vbits,
                                   P.to_np_u32(kq["codes"]), P.to_np_f16(kq["norms"]),
                                   P.to_np_u32(vq["codes"]), P.to_np_f16(vq["norms"]), n_kv, ctx,
                                   scale=scale if scale > 0 else None)
    return P.check_decode(out.cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("kind", ["wht", "haar"])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_decode_gqa_ragged(tq, kind, d):
    _decode_case(tq, kind, d, 4, 3, batch=2, n_kv=2, n_q=8, ctx=3001)


@pytest.mark.parametrize("kbits,vbits", [(2, 2), (3, 3), (4, 4), (2, 4), (4, 2)])
def test_decode_bit_mixes(tq, kbits, vbits):
    _decode_case(tq, "wht", 128, kbits, vbits, batch=1, n_kv=2, n_q=4, ctx=777, q_dtype="f32")


@pytest.mark.parametrize("ctx", [1, 2, 127, 128, 129, 4096])
def test_decode_context_edges(tq, ctx):
    _decode_case(tq, "wht", 128, 4, 3, batch=1, n_kv=1, n_q=4, ctx=ctx)


def test_decode_mha_and_explicit_scale(tq):
    _decode_case(tq, "wht", 64, 3, 3, batch=3, n_kv=4, n_q=4, ctx=300, scale=0.3)
