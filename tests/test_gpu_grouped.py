"""GPU parity of the lane-grouped code order (TQ_FMT_GROUPED): the quantizer
writes it, the decode reads the value codes in it.

* quantize: the grouped codes and norms match the oracle (codes exact outside
  the 1e-5 boundary band) and are bit for bit the oracle's re-ordering of the
  same launch's default-order codes;
* decode: grouped value codes give the oracle's output within the decode bar
  and exactly the output of the default order on the same cache (tensor-core
  path for aligned contexts, with and without QJL keys; CUDA-core path for odd
  contexts);
* rejections: QJL signs with the flag."""

import numpy as np
import pytest

import workloads as W
from oracle import quant as oq
from oracle import rotation as orot
from tests import parity as P

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tq():
    import kv_cache_vector_11_b200 as lib
    assert torch.cuda.is_available(), "GPU tests need CUDA"
    return lib


def _regroup(codes_u32, bits, d=128):
    return oq.pack(oq.unpack(codes_u32, bits, 32, d), bits, 32, layout="grouped")


@pytest.mark.parametrize("kind", ["wht", "haar"])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_grouped_quantize_parity(tq, kind, bits):
    d = 128
    n = 3 * 148 * 128 + 77          # several tiles per CTA and a ragged last tile
    x64 = W.kv_host(1, 1, n, d, seed=300 + bits)
    x = torch.from_numpy(x64).to("cuda", torch.bfloat16)
    rot = tq.Rotation(kind, d, d, W.SEED_ROT)
    c, t = tq.build_codebook(bits)
    plain = tq.quantize_kv(rot, bits, c, t, x)
    grp = tq.quantize_kv(rot, bits, c, t, x, grouped=True)
    torch.cuda.synchronize()
    gc, gn = P.to_np_u32(grp["codes"]), P.to_np_f16(grp["norms"])
    # the same codes and norms as the default order, only moved
    assert np.array_equal(gc, _regroup(P.to_np_u32(plain["codes"]), bits))
    assert np.array_equal(gn, P.to_np_f16(plain["norms"]))
    sel = np.r_[0:600, n - 300:n]
    xr = x.float().cpu().numpy().astype(np.float64)[sel]
    P.compare_quantize(xr, P.oracle_rotation(kind, d, W.SEED_ROT), bits, gc[sel], gn[sel],
                       layout="grouped")


# aligned contexts run on the tensor cores (ragged last slab at 1000 and
# 4000), 1537 and 777 on the CUDA-core decode
@pytest.mark.parametrize("kb,vb,ctx,n_q", [
    (4, 3, 1000, 8), (4, 3, 1537, 8), (2, 2, 4096, 16), (3, 4, 4000, 8), (4, 2, 777, 4),
    (2, 3, 2048, 16)])
def test_grouped_decode_parity(tq, kb, vb, ctx, n_q):
    d, batch, n_kv = 128, 2, 2
    rot = tq.Rotation("wht", d, d, W.SEED_ROT)
    ck, tk = tq.build_codebook(kb)
    cv, tv = tq.build_codebook(vb)
    k = torch.from_numpy(W.kv_host(batch, n_kv, ctx, d, seed=11 + ctx)).to("cuda", torch.bfloat16)
    v = torch.from_numpy(W.kv_host(batch, n_kv, ctx, d, seed=12 + ctx)).to("cuda", torch.bfloat16)
    q64 = W.queries_host(batch, n_q, d)
    q = torch.from_numpy(q64).to("cuda", torch.bfloat16)
    kq = tq.quantize_kv(rot, kb, ck, tk, k.reshape(-1, d))
    vp = tq.quantize_kv(rot, vb, cv, tv, v.reshape(-1, d))
    vg = tq.quantize_kv(rot, vb, cv, tv, v.reshape(-1, d), grouped=True)
    out_p = tq.decode_attention(rot, kb, vb, ck, cv, q, kq["codes"], kq["norms"], vp["codes"],
                                vp["norms"], n_kv, ctx)
    out_g = tq.decode_attention(rot, kb, vb, ck, cv, q, kq["codes"], kq["norms"], vg["codes"],
                                vg["norms"], n_kv, ctx, v_grouped=True)
    torch.cuda.synchronize()
    og = out_g.cpu().numpy()
    if ctx % 2 == 0:
        # both run on the tensor cores with the same arithmetic (odd contexts:
        # two different CUDA-core kernels, compared with the oracle only)
        assert np.array_equal(og, out_p.cpu().numpy())
    P.check_decode(out_p.cpu().numpy().astype(np.float64),
                   P.oracle_decode_on_cache(q64, P.oracle_rotation("wht", d, W.SEED_ROT), kb, vb,
                                            P.to_np_u32(kq["codes"]), P.to_np_f16(kq["norms"]),
                                            P.to_np_u32(vp["codes"]), P.to_np_f16(vp["norms"]),
                                            n_kv, ctx))
    ref = P.oracle_decode_on_cache(q64, P.oracle_rotation("wht", d, W.SEED_ROT), kb, vb,
                                   P.to_np_u32(kq["codes"]), P.to_np_f16(kq["norms"]),
                                   P.to_np_u32(vg["codes"]), P.to_np_f16(vg["norms"]), n_kv, ctx,
                                   v_layout="grouped")
    P.check_decode(og.astype(np.float64), ref)


# 1000: tensor cores, 777: CUDA cores
@pytest.mark.parametrize("ctx", [1000, 777])
def test_grouped_values_with_qjl_keys(tq, ctx):
    d, batch, n_kv, n_q, m = 128, 2, 2, 8, 128
    rot = tq.Rotation("wht", d, d, W.SEED_ROT)
    qjl = tq.Rotation("gauss", m, d, W.SEED_QJL)
    ck, tk = tq.build_codebook(2)
    cv, tv = tq.build_codebook(3)
    k = torch.from_numpy(W.kv_host(batch, n_kv, ctx, d, seed=21)).to("cuda", torch.bfloat16)
    v = torch.from_numpy(W.kv_host(batch, n_kv, ctx, d, seed=22)).to("cuda", torch.bfloat16)
    q64 = W.queries_host(batch, n_q, d)
    q = torch.from_numpy(q64).to("cuda", torch.bfloat16)
    kq = tq.quantize_kv(rot, 2, ck, tk, k.reshape(-1, d), qjl=qjl)
    vg = tq.quantize_kv(rot, 3, cv, tv, v.reshape(-1, d), grouped=True)
    out = tq.decode_attention(rot, 2, 3, ck, cv, q, kq["codes"], kq["norms"], vg["codes"],
                              vg["norms"], n_kv, ctx, qjl=qjl, qjl_signs=kq["signs"],
                              qjl_rnorm=kq["rnorm"], v_grouped=True)
    torch.cuda.synchronize()
    S = orot.gaussian_projection(m, d, W.SEED_QJL)
    ref = P.oracle_decode_on_cache(
        q64, P.oracle_rotation("wht", d, W.SEED_ROT), 2, 3, P.to_np_u32(kq["codes"]),
        P.to_np_f16(kq["norms"]), P.to_np_u32(vg["codes"]), P.to_np_f16(vg["norms"]), n_kv, ctx,
        qjl=P.qjl_oracle_arrays(P.to_np_u32(kq["signs"]), P.to_np_f16(kq["rnorm"]), m, S),
        v_layout="grouped")
    P.check_decode(out.cpu().numpy().astype(np.float64), ref)


def test_grouped_rejects_qjl_signs(tq):
    d = 128
    rot = tq.Rotation("wht", d, d, W.SEED_ROT)
    qjl = tq.Rotation("gauss", 128, d, W.SEED_QJL)
    c, t = tq.build_codebook(2)
    x = torch.zeros((256, d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tq.TQError) as err:
        tq.quantize_kv(rot, 2, c, t, x, qjl=qjl, grouped=True)
    assert err.value.status == 2


def test_grouped_quantize_unaligned_norms_and_haar_decode(tq):
    """Norms only 4-byte aligned (the quantizer's scalar-store branch) and a
    Haar rotation through the grouped decode."""
    d, batch, n_kv, n_q, ctx, bits = 128, 1, 2, 8, 2000, 3
    rot = tq.Rotation("haar", d, d, W.SEED_ROT)
    ck, tk = tq.build_codebook(4)
    cv, tv = tq.build_codebook(bits)
    v64 = W.kv_host(batch, n_kv, ctx, d, seed=41)
    v = torch.from_numpy(v64).to("cuda", torch.bfloat16).reshape(-1, d)
    n = v.shape[0]
    words = tq.code_words_per_row(bits, 32, d)
    norms_buf = torch.zeros((n * 4 + 2,), dtype=torch.int16, device="cuda")
    out = {"codes": torch.zeros((n, words), dtype=torch.int32, device="cuda"),
           "norms": norms_buf[2:].view(n, 4)}           # 4-byte aligned, not 16
    tq.quantize_kv(rot, bits, cv, tv, v, out=out, grouped=True)
    ref = tq.quantize_kv(rot, bits, cv, tv, v, grouped=True)
    torch.cuda.synchronize()
    assert np.array_equal(P.to_np_u32(out["codes"]), P.to_np_u32(ref["codes"]))
    assert np.array_equal(P.to_np_f16(out["norms"]), P.to_np_f16(ref["norms"]))
    k64 = W.kv_host(batch, n_kv, ctx, d, seed=42)
    q64 = W.queries_host(batch, n_q, d)
    kq = tq.quantize_kv(rot, 4, ck, tk, torch.from_numpy(k64).to("cuda", torch.bfloat16).reshape(-1, d))
    q = torch.from_numpy(q64).to("cuda", torch.bfloat16)
    o = tq.decode_attention(rot, 4, bits, ck, cv, q, kq["codes"], kq["norms"], ref["codes"],
                            ref["norms"], n_kv, ctx, v_grouped=True)
    torch.cuda.synchronize()
    oracle = P.oracle_decode_on_cache(q64, P.oracle_rotation("haar", d, W.SEED_ROT), 4, bits,
                                      P.to_np_u32(kq["codes"]), P.to_np_f16(kq["norms"]),
                                      P.to_np_u32(ref["codes"]), P.to_np_f16(ref["norms"]), n_kv,
                                      ctx, v_layout="grouped")
    P.check_decode(o.cpu().numpy().astype(np.float64), oracle)
