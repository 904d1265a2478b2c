"""GPU parity of the packed-cache format variants against the oracle: norm
blocks of 64 and 128 coordinates ("TurboQuant+ upstream guide", section 5.2:
block 128 reaches 5.12x), fp32 block norms (section 1.2: turbo4 at 4.25 bits
per value) and norm correction (section 11), for both rotations, bf16 and fp32
input, every head dim and bit width; then raw logits and decode attention
over such caches (CUDA-core readers), with ragged contexts and GQA."""

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


def _quantize(tq, x64, kind, d, bits, block, f32, corr, dtype="bf16"):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = torch.from_numpy(x64).to("cuda", tdt)
    rot = tq.Rotation(kind, d, d, W.SEED_ROT)
    c, t = tq.build_codebook(bits, block)
    out = tq.quantize_kv(rot, bits, c, t, x, block=block, norm_f32=f32, norm_correction=corr)
    torch.cuda.synchronize()
    return rot, c, out


def _norms_np(t, f32):
    return t.cpu().numpy() if f32 else P.to_np_f16(t)


@pytest.mark.parametrize("kind", ["wht", "haar"])
@pytest.mark.parametrize("d,block", [(64, 32), (64, 64), (128, 64), (128, 128), (256, 128),
                                     (256, 32)])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("f32,corr", [(False, False), (True, False), (False, True), (True, True)])
def test_variant_quantize_parity(tq, kind, d, block, bits, f32, corr):
    x64 = W.kv_host(1, 1, 333, d, seed=5 + d + block + bits)
    x64[17] = 0.0                                          # a zero row
    _, _, out = _quantize(tq, x64, kind, d, bits, block, f32, corr)
    P.compare_quantize(x64, P.oracle_rotation(kind, d, W.SEED_ROT), bits,
                       P.to_np_u32(out["codes"]), _norms_np(out["norms"], f32), block=block,
                       norm_dtype="f32" if f32 else "f16", norm_correction=corr)


def test_variant_quantize_fp32_input_and_many_rows(tq):
    n, d = 3 * 148 * 64 + 7, 128
    x64 = W.normal_rows_host(n, d, seed=9)
    _, _, out = _quantize(tq, x64, "wht", d, 4, 128, True, False, dtype="f32")
    stats = P.compare_quantize(x64, P.oracle_rotation("wht", d, W.SEED_ROT), 4,
                               P.to_np_u32(out["codes"]), out["norms"].cpu().numpy(), block=128,
                               norm_dtype="f32")
    assert stats["band"] < 1e-3 * stats["elements"]


@pytest.mark.parametrize("d,block,f32,kbits,vbits,ctx", [
    (128, 64, False, 4, 3, 1001), (128, 128, True, 4, 4, 777), (64, 32, True, 3, 2, 500),
    (256, 128, False, 2, 3, 300), (128, 32, True, 4, 3, 1)])
def test_variant_logits_and_decode(tq, d, block, f32, kbits, vbits, ctx):
    batch, n_kv, n_q = 2, 2, 8
    k64 = W.kv_host(batch, n_kv, ctx, d, seed=81)
    v64 = W.kv_host(batch, n_kv, ctx, d, seed=82)
    q64 = W.queries_host(batch, n_q, d)
    rot, ck, kq = _quantize(tq, k64, "wht", d, kbits, block, f32, True)
    _, cv, vq = _quantize(tq, v64, "wht", d, vbits, block, f32, False)
    q = torch.from_numpy(q64).to("cuda", torch.bfloat16)
    nd = "f32" if f32 else "f16"
    rot64 = P.oracle_rotation("wht", d, W.SEED_ROT)
    lg = tq.attn_logits(rot, kbits, ck, q, kq["codes"], kq["norms"], n_kv, ctx, block=block,
                        norm_f32=f32)
    out = tq.decode_attention(rot, kbits, vbits, ck, cv, q, kq["codes"], kq["norms"], vq["codes"],
                              vq["norms"], n_kv, ctx, block=block, norm_f32=f32)
    torch.cuda.synchronize()
    kn, vn = _norms_np(kq["norms"], f32), _norms_np(vq["norms"], f32)
    ref_lg = P.oracle_logits_on_cache(q64, rot64, kbits, P.to_np_u32(kq["codes"]), kn, n_kv, ctx,
                                      block=block, norm_dtype=nd)
    P.check_logits(lg.cpu().numpy().astype(np.float64), ref_lg, q64, k64, n_kv, ctx)
    ref = P.oracle_decode_on_cache(q64, rot64, kbits, vbits, P.to_np_u32(kq["codes"]), kn,
                                   P.to_np_u32(vq["codes"]), vn, n_kv, ctx, block=block,
                                   norm_dtype=nd)
    P.check_decode(out.cpu().numpy().astype(np.float64), ref)


def test_variant_rejections(tq):
    d = 64
    x = torch.zeros((4, d), dtype=torch.bfloat16, device="cuda")
    rot = tq.Rotation("wht", d, d, W.SEED_ROT)
    qjl = tq.Rotation("gauss", 64, d, W.SEED_QJL)
    c, t = tq.build_codebook(3, 128)
    with pytest.raises(tq.TQError) as e:        # block larger than the head
        tq.quantize_kv(rot, 3, c, t, x, block=128)
    assert e.value.status == 2
    c, t = tq.build_codebook(3, 64)
    with pytest.raises(tq.TQError) as e:        # QJL needs the default format
        tq.quantize_kv(rot, 3, c, t, x, block=64, qjl=qjl)
    assert e.value.status == 2
