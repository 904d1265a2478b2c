"""GPU parity of tq_quantize_kv against the oracle (needs a B200)."""

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


def _run(tq, x64, dtype, kind, d, bits, seed=W.SEED_ROT, status=None):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = torch.from_numpy(x64).to(device="cuda", dtype=tdt)
    rot = tq.Rotation(kind, d, d, seed)
    c, t = tq.build_codebook(bits)
    out = tq.quantize_kv(rot, bits, c, t, x, status=status)
    torch.cuda.synchronize()
    return P.to_np_u32(out["codes"]), P.to_np_f16(out["norms"])


def test_keys4096_fp32_wht_4bit(tq):
    keys, _ = W.keys4096_host()
    codes, norms = _run(tq, keys, "f32", "wht", 128, 4)
    stats = P.compare_quantize(keys, P.oracle_rotation("wht", 128, W.SEED_ROT), 4, codes, norms)
    assert stats["band"] < 0.001 * stats["elements"]


@pytest.mark.parametrize("kind", ["wht", "haar"])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_sweep_small(tq, kind, d, bits, dtype):
    n = 1537   # several warps / CTAs and a ragged tail for every lane layout
    x64 = W.kv_host(1, 1, n, d, seed=d + bits, dtype=dtype)
    codes, norms = _run(tq, x64, dtype, kind, d, bits)
    P.compare_quantize(x64, P.oracle_rotation(kind, d, W.SEED_ROT), bits, codes, norms)


def test_single_row_and_empty(tq):
    x64 = W.kv_host(1, 1, 1, 128, seed=3)
    codes, norms = _run(tq, x64, "bf16", "wht", 128, 3)
    P.compare_quantize(x64, P.oracle_rotation("wht", 128, W.SEED_ROT), 3, codes, norms)
    rot = tq.Rotation("wht", 128, 128, 1)
    c, t = tq.build_codebook(3)
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    out = tq.quantize_kv(rot, 3, c, t, x)
    assert out["codes"].shape == (0, 12)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_zero_blocks_store_middle_code(tq, bits):
    x64 = W.kv_host(1, 1, 64, 128, seed=5)
    x64[10] = 0.0
    x64[20] = 0.0
    codes, norms = _run(tq, x64, "bf16", "wht", 128, bits)
    P.compare_quantize(x64, P.oracle_rotation("wht", 128, W.SEED_ROT), bits, codes, norms)
    from oracle import quant as oq
    idx = oq.unpack(codes, bits, 32, 128)
    assert np.all(idx[10] == 1 << (bits - 1)) and np.all(norms[10] == 0)


def test_saturated_norm_and_nonfinite_flags(tq):
    x64 = W.kv_host(1, 1, 32, 128, seed=6)
    x64[3] *= 1e4           # block norms above the fp16 range
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, norms = _run(tq, x64, "f32", "wht", 128, 4, status=status)
    assert int(status.item()) & tq.STATUS_NORM_SATURATED
    assert np.all(norms[3].astype(np.float32) == 65504.0)
    P.compare_quantize(x64, P.oracle_rotation("wht", 128, W.SEED_ROT), 4, codes, norms)
    x64[7, 5] = np.nan
    status.zero_()
    _run(tq, x64, "f32", "wht", 128, 4, status=status)
    assert int(status.item()) & tq.STATUS_NONFINITE


@pytest.mark.parametrize("kind", ["haar", "wht"])
@pytest.mark.parametrize("d,bits", [(64, 3), (128, 4), (128, 2), (128, 3), (256, 3)])
def test_bf16_many_tiles_per_cta(tq, kind, d, bits):
    # enough 128-row tiles that every resident CTA loops over several of them
    # and the copy ring wraps (d = 256 Haar also streams P in 64-column chunks)
    n = 4 * 148 * 4 * 128 + 45 if d == 64 else 3 * 148 * 2 * 128 + 45
    x64 = W.kv_host(1, 1, n, d, seed=11 + d + bits, dtype="bf16")
    codes, norms = _run(tq, x64, "bf16", kind, d, bits)
    stats = P.compare_quantize(x64, P.oracle_rotation(kind, d, W.SEED_ROT), bits, codes, norms)
    assert stats["band"] < 0.001 * stats["elements"]


@pytest.mark.parametrize("kind", ["haar", "wht"])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_bf16_zero_rows_flags_and_tiny(tq, kind, d):
    x64 = W.kv_host(1, 1, 300, d, seed=12, dtype="bf16")
    x64[0] = 0.0
    x64[129] = 0.0
    codes, norms = _run(tq, x64, "bf16", kind, d, 3)
    P.compare_quantize(x64, P.oracle_rotation(kind, d, W.SEED_ROT), 3, codes, norms)
    from oracle import quant as oq
    idx = oq.unpack(codes, 3, 32, d)
    assert np.all(idx[[0, 129]] == 4) and np.all(norms[[0, 129]] == 0)
    one = x64[5:6].copy()
    codes, norms = _run(tq, one, "bf16", kind, d, 4)
    P.compare_quantize(one, P.oracle_rotation(kind, d, W.SEED_ROT), 4, codes, norms)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    big = x64.copy()
    big[200] *= 1e5
    codes, norms = _run(tq, big, "bf16", kind, d, 4, status=status)
    assert int(status.item()) == tq.STATUS_NORM_SATURATED
    big[201, 3] = np.inf
    status.zero_()
    _run(tq, big, "bf16", kind, d, 4, status=status)
    assert int(status.item()) & tq.STATUS_NONFINITE
