"""GPU test of tq_decode_attention_static, the decode entry point for callers
that cannot allocate device memory (its split partials live in a fixed array
inside the library).  Kept in its own file so that pytest collects it last.

Checks, through the C ABI: two calls in a row give the same output as the
workspace-taking tq_decode_attention, within the decode tolerance of the
other tests; a shape whose scratch would not fit is rejected before launch."""

import ctypes

import numpy as np
import pytest

import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def test_static_scratch_decode_matches_workspace_decode():
    import kv_cache_vector_11_b200 as tq
    assert torch.cuda.is_available()
    batch, n_kv, n_q, ctx, d, kb, vb = 2, 4, 16, 5000, 128, 4, 3
    assert tq.decode_workspace_size(batch, n_q, n_kv, ctx, d) <= tq.DECODE_STATIC_SCRATCH_BYTES
    rot = tq.Rotation("wht", d, d, W.SEED_ROT)
    ck, tk = tq.build_codebook(kb)
    cv, tv = tq.build_codebook(vb)
    k = torch.from_numpy(W.kv_host(batch, n_kv, ctx, d, seed=31)).to("cuda", torch.bfloat16)
    v = torch.from_numpy(W.kv_host(batch, n_kv, ctx, d, seed=32)).to("cuda", torch.bfloat16)
    q = torch.from_numpy(W.queries_host(batch, n_q, d)).to("cuda", torch.bfloat16)
    kq = tq.quantize_kv(rot, kb, ck, tk, k)
    vq = tq.quantize_kv(rot, vb, cv, tv, v)
    ref = tq.decode_attention(rot, kb, vb, ck, cv, q, kq["codes"], kq["norms"], vq["codes"],
                              vq["norms"], n_kv, ctx)
    torch.cuda.synchronize()
    ref_np = ref.cpu().numpy().astype(np.float64)
    out = torch.empty_like(ref)
    for _ in range(2):
        out.fill_(float("nan"))
        tq.decode_attention_static(rot, kb, vb, ck, cv, q, kq["codes"], kq["norms"],
                                   vq["codes"], vq["norms"], n_kv, ctx, out=out)
        torch.cuda.synchronize()
        P.check_decode(out.cpu().numpy().astype(np.float64), ref_np)


def test_static_scratch_rejects_oversized_shapes():
    import kv_cache_vector_11_b200 as tq
    batch, n_kv, n_q, ctx, d = 512, 8, 64, 1 << 20, 256
    assert tq.decode_workspace_size(batch, n_q, n_kv, ctx, d) > tq.DECODE_STATIC_SCRATCH_BYTES
    rot = tq.Rotation("wht", d, d, W.SEED_ROT)
    ck, _ = tq.build_codebook(3)
    lib = ctypes.CDLL(tq.lib_path())
    fake = 1 << 20   # never dereferenced: the size check returns before any launch
    lib.tq_decode_attention_static.restype = ctypes.c_int32
    vp = ctypes.c_void_p
    lib.tq_decode_attention_static.argtypes = [
        vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, vp, vp, vp, vp, ctypes.c_int32,
        ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
        vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp]
    st = lib.tq_decode_attention_static(rot.handle, 3, 3, 32, ck.ctypes.data, ck.ctypes.data,
                                        None, fake, 1, batch, n_q, n_kv, ctx, d, fake, fake,
                                        None, None, fake, fake, 0.0, fake, None)
    assert st == 2   # TQ_ERR_UNSUPPORTED
