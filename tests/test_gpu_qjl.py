"""GPU parity of the QJL stage (quantize + logits) against the oracle, and
a Monte Carlo check of unbiasedness over the 64 QJL seeds 2000..2063."""

import numpy as np
import pytest

import workloads as W
from oracle import rotation as orot
from tests import parity as P

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tq():
    import kv_cache_vector_11_b200 as lib
    assert torch.cuda.is_available(), "GPU tests need CUDA"
    return lib


def _qjl_quantize(tq, x64, kind, d, bits, m, qseed, dtype="bf16"):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = torch.from_numpy(x64).to("cuda", tdt)
    rot = tq.Rotation(kind, d, d, W.SEED_ROT)
    qjl = tq.Rotation("gauss", m, d, qseed)
    c, t = tq.build_codebook(bits)
    out = tq.quantize_kv(rot, bits, c, t, x, qjl=qjl)
    torch.cuda.synchronize()
    return rot, qjl, c, out


@pytest.mark.parametrize("kind", ["wht", "haar"])
@pytest.mark.parametrize("d,m", [(128, 128), (64, 256), (256, 64), (128, 32), (64, 128), (128, 96)])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_qjl_quantize_parity(tq, kind, d, m, bits):
    x64 = W.kv_host(1, 1, 777, d, seed=40 + d + m)
    _, _, _, out = _qjl_quantize(tq, x64, kind, d, bits, m, W.SEED_QJL)
    codes, norms = P.to_np_u32(out["codes"]), P.to_np_f16(out["norms"])
    rot64 = P.oracle_rotation(kind, d, W.SEED_ROT)
    P.compare_quantize(x64, rot64, bits, codes, norms)
    S = orot.gaussian_projection(m, d, W.SEED_QJL)
    P.compare_qjl(x64, rot64, bits, S, codes, norms, P.to_np_u32(out["signs"]),
                  P.to_np_f16(out["rnorm"]))


def test_qjl_fp32_input_and_zero_rows(tq):
    x64 = W.normal_rows_host(300, 128, seed=3)
    x64[7] = 0.0
    _, _, _, out = _qjl_quantize(tq, x64, "wht", 128, 2, 128, W.SEED_QJL, dtype="f32")
    rot64 = P.oracle_rotation("wht", 128, W.SEED_ROT)
    S = orot.gaussian_projection(128, 128, W.SEED_QJL)
    P.compare_qjl(x64, rot64, 2, S, P.to_np_u32(out["codes"]), P.to_np_f16(out["norms"]),
                  P.to_np_u32(out["signs"]), P.to_np_f16(out["rnorm"]))
    assert P.to_np_f16(out["rnorm"])[7] == 0


@pytest.mark.parametrize("d", [64, 128])
def test_qjl_bf16_zero_rows_tiny_and_flags(tq, d):
    x64 = W.kv_host(1, 1, 300, d, seed=14 + d)
    x64[0] = 0.0
    x64[129] = 0.0
    rot64 = P.oracle_rotation("wht", d, W.SEED_ROT)
    S = orot.gaussian_projection(128, d, W.SEED_QJL)
    _, _, _, out = _qjl_quantize(tq, x64, "wht", d, 3, 128, W.SEED_QJL)
    P.compare_qjl(x64, rot64, 3, S, P.to_np_u32(out["codes"]), P.to_np_f16(out["norms"]),
                  P.to_np_u32(out["signs"]), P.to_np_f16(out["rnorm"]))
    assert np.all(P.to_np_f16(out["rnorm"])[[0, 129]] == 0)
    one = x64[5:6].copy()
    _, _, _, out = _qjl_quantize(tq, one, "wht", d, 2, 128, W.SEED_QJL)
    P.compare_qjl(one, rot64, 2, S, P.to_np_u32(out["codes"]), P.to_np_f16(out["norms"]),
                  P.to_np_u32(out["signs"]), P.to_np_f16(out["rnorm"]))
    big = x64.copy()
    big[200] *= 1e5
    x = torch.from_numpy(big).to("cuda", torch.bfloat16)
    rot = tq.Rotation("wht", d, d, W.SEED_ROT)
    qjl = tq.Rotation("gauss", 128, d, W.SEED_QJL)
    c, t = tq.build_codebook(2)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.quantize_kv(rot, 2, c, t, x, qjl=qjl, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & tq.STATUS_NORM_SATURATED
    big[201, 3] = np.inf
    x = torch.from_numpy(big).to("cuda", torch.bfloat16)
    status.zero_()
    tq.quantize_kv(rot, 2, c, t, x, qjl=qjl, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & tq.STATUS_NONFINITE


# ctx = 1500: residual norms not 16-byte aligned per (batch, kv head) -> CUDA-core
# scores; the others take the tensor-core scores (ragged last slab at 1496 and 1000,
# m = 96 and 64, two groups of four heads, two heads per kv head)
@pytest.mark.parametrize("ctx,d,m,bits,n_kv,n_q", [
    (1500, 128, 128, 2, 2, 8), (1496, 128, 128, 2, 2, 8), (4096, 64, 64, 3, 1, 4),
    (2048, 128, 96, 4, 2, 4), (1000, 128, 128, 2, 3, 6)])
def test_qjl_logits_parity(tq, ctx, d, m, bits, n_kv, n_q):
    batch = 2
    k64 = W.kv_host(batch, n_kv, ctx, d, seed=51)
    q64 = W.queries_host(batch, n_q, d)
    rot, qjl, c, out = _qjl_quantize(tq, k64, "wht", d, bits, m, W.SEED_QJL)
    q = torch.from_numpy(q64).to("cuda", torch.bfloat16)
    lg = tq.attn_logits(rot, bits, c, q, out["codes"], out["norms"], n_kv, ctx, qjl=qjl,
                        qjl_signs=out["signs"], qjl_rnorm=out["rnorm"])
    torch.cuda.synchronize()
    S = orot.gaussian_projection(m, d, W.SEED_QJL)
    ref = P.oracle_logits_on_cache(
        q64, P.oracle_rotation("wht", d, W.SEED_ROT), bits, P.to_np_u32(out["codes"]),
        P.to_np_f16(out["norms"]), n_kv, ctx,
        qjl=P.qjl_oracle_arrays(P.to_np_u32(out["signs"]), P.to_np_f16(out["rnorm"]), m, S))
    P.check_logits(lg.cpu().numpy().astype(np.float64), ref, q64, k64, n_kv, ctx)


def test_qjl_monte_carlo_unbiased_on_gpu(tq):
    """Over the 64 QJL seeds, the mean error of the corrected logits against
    the exact <q, k> is within 4 standard errors of zero, while the MSE-only
    logits are biased (shrunk)."""
    n_kv, n_q, ctx, d, m = 1, 4, 256, 128, 128
    k64 = W.kv_host(1, n_kv, ctx, d, seed=61)
    q64 = W.queries_host(1, n_q, d, dtype="f32")
    exact = np.einsum("hd,td->ht", q64[0], k64)
    q = torch.from_numpy(q64).to("cuda", torch.float32)
    errs, mse_errs = [], None
    for seed in range(2000, 2064):
        rot, qjl, c, out = _qjl_quantize(tq, k64, "wht", d, 2, m, seed)
        lg = tq.attn_logits(rot, 2, c, q, out["codes"], out["norms"], n_kv, ctx, qjl=qjl,
                            qjl_signs=out["signs"], qjl_rnorm=out["rnorm"])
        errs.append(lg.cpu().numpy()[0].astype(np.float64) - exact)
        if mse_errs is None:
            mse = tq.attn_logits(rot, 2, c, q, out["codes"], out["norms"], n_kv, ctx)
            mse_errs = mse.cpu().numpy()[0].astype(np.float64) - exact
    errs = np.array(errs)                         # [seeds, heads, tokens]
    scale = np.abs(exact).mean()
    mean_err = errs.mean()
    se = errs.std() / np.sqrt(errs.size)
    assert abs(mean_err) < 4 * se, (mean_err, se)
    # per (head, token) averages over seeds shrink toward the exact scores
    avg = errs.mean(axis=0)
    assert np.mean(avg ** 2) < 0.2 * np.mean(mse_errs ** 2)
    assert scale > 0


@pytest.mark.parametrize("d,m", [(128, 128), (64, 256), (64, 128)])
def test_qjl_many_tiles_per_cta(tq, d, m):
    # several 128-row tiles per resident CTA, so the projection's TMEM
    # accumulator and its mbarrier phase are reused, plus a ragged last tile
    n = 3 * 2 * 148 * 128 + 45
    x64 = W.kv_host(1, 1, n, d, seed=90 + d)
    _, _, _, out = _qjl_quantize(tq, x64, "wht", d, 2, m, W.SEED_QJL)
    rot64 = P.oracle_rotation("wht", d, W.SEED_ROT)
    S = orot.gaussian_projection(m, d, W.SEED_QJL)
    stats = P.compare_qjl(x64, rot64, 2, S, P.to_np_u32(out["codes"]), P.to_np_f16(out["norms"]),
                          P.to_np_u32(out["signs"]), P.to_np_f16(out["rnorm"]))
    assert stats["band"] < 1e-3 * stats["signs"]


# decode over keys that carry QJL signs.  Contexts that are multiples of 8 run
# on the tensor cores (ragged last slab at 1000, 4000 and 520; m = 64, 96, 128;
# two groups of four heads per kv head at n_q = 16), the others (1537, 777, 1)
# on CUDA cores
@pytest.mark.parametrize("d,m,kbits,vbits,ctx,n_q", [
    (128, 128, 2, 2, 1000, 8), (128, 64, 2, 3, 1537, 8), (64, 128, 3, 2, 777, 8),
    (64, 64, 4, 4, 2048, 8), (128, 128, 3, 4, 1, 8), (128, 96, 3, 3, 4000, 16),
    (64, 128, 2, 4, 520, 8), (128, 32, 4, 3, 64, 4)])
def test_qjl_decode_parity(tq, d, m, kbits, vbits, ctx, n_q):
    batch, n_kv = 2, 2
    k64 = W.kv_host(batch, n_kv, ctx, d, seed=71 + ctx)
    v64 = W.kv_host(batch, n_kv, ctx, d, seed=72 + ctx)
    q64 = W.queries_host(batch, n_q, d)
    rot, qjl, ck, kq = _qjl_quantize(tq, k64, "wht", d, kbits, m, W.SEED_QJL)
    cv, tv = tq.build_codebook(vbits)
    vq = tq.quantize_kv(rot, vbits, cv, tv, torch.from_numpy(v64).to("cuda", torch.bfloat16))
    q = torch.from_numpy(q64).to("cuda", torch.bfloat16)
    out = tq.decode_attention(rot, kbits, vbits, ck, cv, q, kq["codes"], kq["norms"],
                              vq["codes"], vq["norms"], n_kv, ctx, qjl=qjl,
                              qjl_signs=kq["signs"], qjl_rnorm=kq["rnorm"])
    torch.cuda.synchronize()
    S = orot.gaussian_projection(m, d, W.SEED_QJL)
    ref = P.oracle_decode_on_cache(
        q64, P.oracle_rotation("wht", d, W.SEED_ROT), kbits, vbits, P.to_np_u32(kq["codes"]),
        P.to_np_f16(kq["norms"]), P.to_np_u32(vq["codes"]), P.to_np_f16(vq["norms"]), n_kv, ctx,
        qjl=P.qjl_oracle_arrays(P.to_np_u32(kq["signs"]), P.to_np_f16(kq["rnorm"]), m, S))
    P.check_decode(out.cpu().numpy().astype(np.float64), ref)
