"""GPU parity of the warp-streamed tensor-core decode path against the oracle.

tq_decode_attention takes this path for keys without the QJL stage whenever
every (batch, kv head) section of codes and norms starts on a 16-byte
boundary (ctx * row bytes a multiple of 16 for K codes, V codes and norms:
an even context for d = 128); the other shapes run the split kernels, which
test_gpu_attention covers with odd contexts.  Cases here: every head dim and
bit mix, GQA groups of 1, 2, 4 and 8 (two head groups per kv head), ragged
last slabs, tiny contexts where there are fewer slabs than warps, warp
ranges that cross many (batch, kv head) boundaries, and the full 128K-context
decode workload checked on sampled heads."""

import numpy as np
import pytest

import workloads as W
from oracle import attention as oatt
from oracle import quant as oq
from tests import parity as P

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tq():
    import kv_cache_vector_11_b200 as lib
    assert torch.cuda.is_available(), "GPU tests need CUDA"
    return lib


def _case(tq, kind, d, kbits, vbits, batch, n_kv, n_q, ctx, q_dtype="bf16", scale=0.0, seed=41):
    k64 = W.kv_host(batch, n_kv, ctx, d, seed=seed)
    v64 = W.kv_host(batch, n_kv, ctx, d, seed=seed + 1)
    q64 = W.queries_host(batch, n_q, d, dtype=q_dtype)
    rot = tq.Rotation(kind, d, d, W.SEED_ROT)
    ck, tk = tq.build_codebook(kbits)
    cv, tv = tq.build_codebook(vbits)
    k = torch.from_numpy(k64).to("cuda", torch.bfloat16)
    v = torch.from_numpy(v64).to("cuda", torch.bfloat16)
    qt = torch.from_numpy(q64).to("cuda", torch.bfloat16 if q_dtype == "bf16" else torch.float32)
    kq = tq.quantize_kv(rot, kbits, ck, tk, k)
    vq = tq.quantize_kv(rot, vbits, cv, tv, v)
    out = tq.decode_attention(rot, kbits, vbits, ck, cv, qt, kq["codes"], kq["norms"],
                              vq["codes"], vq["norms"], n_kv, ctx, scale=scale)
    torch.cuda.synchronize()
    ref = P.oracle_decode_on_cache(q64, P.oracle_rotation(kind, d, W.SEED_ROT), kbits, vbits,
                                   P.to_np_u32(kq["codes"]), P.to_np_f16(kq["norms"]),
                                   P.to_np_u32(vq["codes"]), P.to_np_f16(vq["norms"]), n_kv, ctx,
                                   scale=scale if scale > 0 else None)
    return P.check_decode(out.cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("kind", ["wht", "haar"])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_mma_head_dims_ragged(tq, kind, d):
    _case(tq, kind, d, 4, 3, batch=2, n_kv=2, n_q=8, ctx=2002)


@pytest.mark.parametrize("kbits,vbits", [(2, 2), (3, 3), (4, 4), (2, 4), (4, 2), (3, 2)])
@pytest.mark.parametrize("d", [64, 128])
def test_mma_bit_mixes(tq, kbits, vbits, d):
    _case(tq, "wht", d, kbits, vbits, batch=1, n_kv=2, n_q=4, ctx=776, q_dtype="f32")


@pytest.mark.parametrize("n_kv,n_q", [(4, 4), (4, 8), (2, 8), (1, 8), (2, 16), (1, 6)])
def test_mma_group_sizes(tq, n_kv, n_q):
    _case(tq, "wht", 128, 4, 3, batch=2, n_kv=n_kv, n_q=n_q, ctx=1000)


@pytest.mark.parametrize("ctx", [2, 16, 18, 32, 46, 256])
def test_mma_tiny_contexts(tq, ctx):
    _case(tq, "wht", 128, 4, 3, batch=1, n_kv=1, n_q=4, ctx=ctx)


def test_mma_ranges_cross_many_groups(tq):
    # 4 * 8 groups of 250 slabs over ~2k warps: most warps span two groups
    _case(tq, "wht", 128, 4, 3, batch=4, n_kv=8, n_q=32, ctx=4000)


def test_mma_explicit_scale_sharp_softmax(tq):
    _case(tq, "haar", 128, 4, 3, batch=1, n_kv=2, n_q=8, ctx=3000, scale=0.5)


def test_decode_128k_sampled_heads(tq):
    """The 128K-context decode workload at full size (8 x 8 kv heads x 131072
    tokens, 32 query heads, 4-bit K / 3-bit V, WHT), quantized and decoded on
    the GPU in one call each, as the benchmark runs them: the K and V codes and
    norms (V also in the lane-grouped order the benchmark stores) are compared
    with the oracle on ~7000 sampled rows each, the decode over grouped V
    equals the decode over default-order V exactly, and the oracle recomputes
    three (batch, kv head) groups of four query heads from the same packed
    cache."""
    cfg = W.WORKLOADS["decode_128k"]
    batch, n_kv, n_q, ctx, d = (cfg["batch"], cfg["n_kv_heads"], cfg["n_q_heads"], cfg["ctx"],
                                cfg["head_dim"])
    kb, vb = cfg["k_bits"], cfg["v_bits"]
    rot = tq.Rotation("wht", d, d, W.SEED_ROT)
    ck, tk = tq.build_codebook(kb)
    cv, tv = tq.build_codebook(vb)
    rot64 = P.oracle_rotation("wht", d, W.SEED_ROT)
    # sampled rows of both quantize launches: random rows over the whole
    # 2 GiB input, every row of the last 128-row tile, and rows in the last
    # 1/8 of the input (byte offsets above 1.75 GiB)
    n = batch * n_kv * ctx
    idx = np.unique(np.concatenate([
        np.random.default_rng(128).choice(n, 6000, replace=False),
        np.arange(n - 128, n),
        np.random.default_rng(129).choice(np.arange(n - n // 8, n), 1000, replace=False)]))
    it = torch.from_numpy(idx).cuda()
    k = W.kv_device(batch, n_kv, ctx, d, seed=W.SEED_K).reshape(-1, d)
    kq = tq.quantize_kv(rot, kb, ck, tk, k)
    k_rows = k[it].float().cpu().numpy().astype(np.float64)
    del k
    v = W.kv_device(batch, n_kv, ctx, d, seed=W.SEED_V).reshape(-1, d)
    vq = tq.quantize_kv(rot, vb, cv, tv, v)
    # the benchmark's value cache: the same rows in the lane-grouped order
    vg = tq.quantize_kv(rot, vb, cv, tv, v, grouped=True)
    v_rows = v[it].float().cpu().numpy().astype(np.float64)
    del v
    torch.cuda.synchronize()
    P.compare_quantize(k_rows, rot64, kb, P.to_np_u32(kq["codes"][it]), P.to_np_f16(kq["norms"][it]))
    P.compare_quantize(v_rows, rot64, vb, P.to_np_u32(vq["codes"][it]), P.to_np_f16(vq["norms"][it]))
    P.compare_quantize(v_rows, rot64, vb, P.to_np_u32(vg["codes"][it]), P.to_np_f16(vg["norms"][it]),
                       layout="grouped")
    assert np.array_equal(P.to_np_u32(vg["codes"][it]),
                          oq.pack(oq.unpack(P.to_np_u32(vq["codes"][it]), vb, 32, d), vb, 32,
                                  layout="grouped"))
    q64 = W.queries_host(batch, n_q, d)
    q = torch.from_numpy(q64).to("cuda", torch.bfloat16)
    out = tq.decode_attention(rot, kb, vb, ck, cv, q, kq["codes"], kq["norms"], vq["codes"],
                              vq["norms"], n_kv, ctx)
    out_g = tq.decode_attention(rot, kb, vb, ck, cv, q, kq["codes"], kq["norms"], vg["codes"],
                                vg["norms"], n_kv, ctx, v_grouped=True)
    torch.cuda.synchronize()
    out = out.cpu().numpy().astype(np.float64)
    assert np.array_equal(out_g.cpu().numpy().astype(np.float64), out)
    c_k, _ = P.oracle_codebook(kb)
    c_v, _ = P.oracle_codebook(vb)
    G = n_q // n_kv
    for b, hk in [(0, 0), (3, 5), (7, 7)]:
        rows = slice((b * n_kv + hk) * ctx, (b * n_kv + hk + 1) * ctx)
        ki = oq.unpack(P.to_np_u32(kq["codes"][rows]), kb, 32, d)
        vi = oq.unpack(P.to_np_u32(vq["codes"][rows]), vb, 32, d)
        kn = P.to_np_f16(kq["norms"][rows])
        vn = P.to_np_f16(vq["norms"][rows])
        qs = q64[b:b + 1, hk * G:(hk + 1) * G]
        ref = oatt.decode(qs, rot64, ki, kn, c_k, vi, vn, c_v, 32, 1, ctx)
        P.check_decode(out[b:b + 1, hk * G:(hk + 1) * G], ref)
