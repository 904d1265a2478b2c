"""GPU parity at the full sizes of the workload table, in the launch
configurations the library picks for them: the Llama-3-8B-shaped 32K-context
layer (quantize K and V + decode, checked in full), the QJL 16K-context batch
of 16 (quantize with signs + logits, checked on sampled rows and kv heads) and
the 2^20-row prefill sweep (every head dim, bit width and rotation, checked on
sampled rows).  Inputs are generated on the device with the seeded recipe."""

import numpy as np
import pytest

import workloads as W
from oracle import attention as oatt
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


def _rows64(x, idx):
    return x[torch.from_numpy(idx).to(x.device)].float().cpu().numpy().astype(np.float64)


def test_llama8b_32k_layer_in_full(tq):
    cfg = W.WORKLOADS["llama8b_32k"]
    B, Hkv, Hq, T, d = cfg["batch"], cfg["n_kv_heads"], cfg["n_q_heads"], cfg["ctx"], cfg["head_dim"]
    kb, vb = cfg["k_bits"], cfg["v_bits"]
    rot = tq.Rotation("wht", d, d, W.SEED_ROT)
    ck, tk = tq.build_codebook(kb)
    cv, tv = tq.build_codebook(vb)
    k = W.kv_device(B, Hkv, T, d, seed=W.SEED_K)
    v = W.kv_device(B, Hkv, T, d, seed=W.SEED_V)
    kq = tq.quantize_kv(rot, kb, ck, tk, k)
    vq = tq.quantize_kv(rot, vb, cv, tv, v)
    q64 = W.queries_host(B, Hq, d)
    q = torch.from_numpy(q64).to("cuda", torch.bfloat16)
    out = tq.decode_attention(rot, kb, vb, ck, cv, q, kq["codes"], kq["norms"], vq["codes"],
                              vq["norms"], Hkv, T)
    torch.cuda.synchronize()
    rot64 = P.oracle_rotation("wht", d, W.SEED_ROT)
    all_rows = np.arange(B * Hkv * T)
    stats = P.compare_quantize(_rows64(k, all_rows), rot64, kb, P.to_np_u32(kq["codes"]),
                               P.to_np_f16(kq["norms"]))
    assert stats["band"] < 1e-3 * stats["elements"]
    P.compare_quantize(_rows64(v, all_rows), rot64, vb, P.to_np_u32(vq["codes"]),
                       P.to_np_f16(vq["norms"]))
    ref = P.oracle_decode_on_cache(q64, rot64, kb, vb, P.to_np_u32(kq["codes"]),
                                   P.to_np_f16(kq["norms"]), P.to_np_u32(vq["codes"]),
                                   P.to_np_f16(vq["norms"]), Hkv, T)
    P.check_decode(out.cpu().numpy().astype(np.float64), ref)


def test_qjl_16k_batch16_sampled(tq):
    cfg = W.WORKLOADS["qjl_16k"]
    B, Hkv, Hq, T, d, m = (cfg["batch"], cfg["n_kv_heads"], cfg["n_q_heads"], cfg["ctx"],
                           cfg["head_dim"], cfg["qjl_m"])
    bits = cfg["k_bits"]
    rot = tq.Rotation("wht", d, d, W.SEED_ROT)
    qjl = tq.Rotation("gauss", m, d, W.SEED_QJL)
    c, t = tq.build_codebook(bits)
    k = W.kv_device(B, Hkv, T, d, seed=W.SEED_K)
    kq = tq.quantize_kv(rot, bits, c, t, k, qjl=qjl)
    q64 = W.queries_host(B, Hq, d)
    q = torch.from_numpy(q64).to("cuda", torch.bfloat16)
    lg = tq.attn_logits(rot, bits, c, q, kq["codes"], kq["norms"], Hkv, T, qjl=qjl,
                        qjl_signs=kq["signs"], qjl_rnorm=kq["rnorm"])
    torch.cuda.synchronize()
    rot64 = P.oracle_rotation("wht", d, W.SEED_ROT)
    S = orot.gaussian_projection(m, d, W.SEED_QJL)
    idx = np.sort(np.random.default_rng(5).choice(B * Hkv * T, 8192, replace=False))
    codes = P.to_np_u32(kq["codes"])[idx]
    norms = P.to_np_f16(kq["norms"])[idx]
    x64 = _rows64(k, idx)
    P.compare_quantize(x64, rot64, bits, codes, norms)
    P.compare_qjl(x64, rot64, bits, S, codes, norms, P.to_np_u32(kq["signs"])[idx],
                  P.to_np_f16(kq["rnorm"])[idx])
    G = Hq // Hkv
    c64, _ = P.oracle_codebook(bits)
    lg = lg.cpu().numpy().astype(np.float64)
    for b, hk in [(0, 0), (9, 3), (15, 7)]:
        rows = slice((b * Hkv + hk) * T, (b * Hkv + hk + 1) * T)
        qj = P.qjl_oracle_arrays(P.to_np_u32(kq["signs"][rows]), P.to_np_f16(kq["rnorm"][rows]), m, S)
        ref = oatt.logits(q64[b:b + 1, hk * G:(hk + 1) * G], rot64,
                          oq.unpack(P.to_np_u32(kq["codes"][rows]), bits, 32, d),
                          P.to_np_f16(kq["norms"][rows]), c64, 32, 1, T, qjl=qj)
        P.check_logits(lg[b:b + 1, hk * G:(hk + 1) * G], ref, q64[b:b + 1, hk * G:(hk + 1) * G],
                       _rows64(k, np.arange((b * Hkv + hk) * T, (b * Hkv + hk + 1) * T)), 1, T)


@pytest.mark.parametrize("kind", ["wht", "haar"])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_prefill_1m_sweep_sampled(tq, kind, d):
    cfg = W.WORKLOADS["prefill_1m"]
    n = cfg["rows"]
    x = W.kv_device(1, 1, n, d, seed=W.SEED_K + d)
    rot = tq.Rotation(kind, d, d, W.SEED_ROT)
    rot64 = P.oracle_rotation(kind, d, W.SEED_ROT)
    idx = np.sort(np.concatenate([np.random.default_rng(d).choice(n, 2048, replace=False),
                                  np.arange(n - 64, n)]))
    x64 = _rows64(x, np.unique(idx))
    idx = np.unique(idx)
    for bits in cfg["bits"]:
        c, t = tq.build_codebook(bits)
        out = tq.quantize_kv(rot, bits, c, t, x)
        torch.cuda.synchronize()
        P.compare_quantize(x64, rot64, bits, P.to_np_u32(out["codes"])[idx],
                           P.to_np_f16(out["norms"])[idx])
