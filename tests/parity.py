"""Comparison helpers for the GPU parity tests (library output vs oracle).

Bars (fixed by the method's statement of parity):
* packed codes: bit-exact, except coordinates whose normalised value lies
  within 1e-5 of a decision boundary (oracle float64 u); those are counted;
* fp16 norms: equal or one fp16 ulp apart (fp32 vs float64 norm before the
  final rounding); the one-ulp cases are counted;
* logits: |gpu - oracle| <= 1e-3 * ||q|| * ||k|| with the oracle scoring the
  library's own packed cache;
* decode outputs: relative L2 error <= 2e-3 per (batch, query head) vector,
  again on the library's packed cache.
"""

import numpy as np

from oracle import attention as oatt
from oracle import codebook as ocb
from oracle import qjl as oqjl
from oracle import quant as oq
from oracle import rotation as orot

BAND = 1e-5
LOGIT_TOL = 1e-3
DECODE_TOL = 2e-3


def to_np_u32(t):
    return t.detach().cpu().numpy().view(np.uint32)


def to_np_f16(t):
    return t.detach().cpu().numpy().view(np.float16)


def oracle_rotation(kind, d, seed):
    return orot.rotation(kind, d, seed)


def oracle_codebook(bits, block=32):
    return ocb.stored_table(bits, block)


def compare_quantize(x64, rot64, bits, gpu_codes, gpu_norms, block=32, norm_dtype="f16",
                     norm_correction=False, layout="plain"):
    """Returns a dict of counts; raises AssertionError on a violation.

    fp32 norms (``norm_dtype="f32"``) must agree to 1e-5 relative (the kernel
    rotates and sums squares in fp32 and takes approximate square roots; the
    oracle is float64 -- the same 1e-5 scale as the code band); fp16 norms to
    one fp16 ulp.  With norm correction the ulp bar
    applies to gamma / ||c[idx]|| computed on the library's own codes."""
    c32, t64 = oracle_codebook(bits, block)
    n, d = x64.shape
    ref = oq.quantize(x64, rot64, c32, t64, bits, block, norm_dtype=norm_dtype,
                      norm_correction=norm_correction)
    gi = oq.unpack(gpu_codes, bits, block, d, layout=layout)
    dist = oq.boundary_distance(ref["y"], ref["gamma"], t64, block)
    band = dist < BAND
    mism = gi != ref["codes"]
    outside = mism & ~band
    assert not outside.any(), (
        f"{int(outside.sum())} code mismatches outside the 1e-5 band; first at "
        f"{np.argwhere(outside)[:5].tolist()}")
    ref_norms = ref["norms"]
    if norm_correction:
        # codes inside the band may differ; the stored norm follows the codes
        ref_norms, _ = oq.stored_norms(ref["gamma"] / oq.reconstruction_norms(gi, c32, block),
                                       norm_dtype)
    gn = gpu_norms.astype(np.float32)
    rn = ref_norms.astype(np.float32)
    if norm_dtype == "f32":
        rel = np.abs(gn.astype(np.float64) - rn) / np.maximum(rn, 1e-30)
        rel = np.where(rn == 0, np.abs(gn), rel)
        assert np.all(rel <= 1e-5), f"fp32 norms differ by > 1e-5 at {np.argwhere(rel > 1e-5)[:5].tolist()}"
        return {"elements": int(gi.size), "band": int(band.sum()),
                "band_mismatch": int((mism & band).sum()), "norm_rel_max": float(rel.max(initial=0))}
    ulp = np.abs(gpu_norms.view(np.int16).astype(np.int32) - ref_norms.view(np.int16).astype(np.int32))
    assert np.all(ulp <= 1), f"norms differ by > 1 ulp at {np.argwhere(ulp > 1)[:5].tolist()}"
    return {"elements": int(gi.size), "band": int(band.sum()),
            "band_mismatch": int((mism & band).sum()), "norm_ulp1": int((ulp == 1).sum()),
            "max_norm_rel": float(np.max(np.abs(gn - rn) / np.maximum(rn, 1e-30)))}


def oracle_logits_on_cache(q64, rot64, bits, codes_u32, norms_f16, n_kv_heads, ctx, block=32,
                           qjl=None, norm_dtype="f16"):
    """Oracle logits scoring the library's packed cache."""
    c32, _ = oracle_codebook(bits, block)
    d = q64.shape[-1]
    idx = oq.unpack(codes_u32, bits, block, d)
    return oatt.logits(q64, rot64, idx, norms_f16, c32, block, n_kv_heads, ctx, qjl=qjl,
                       norm_dtype=norm_dtype)


def check_logits(gpu, ref, q64, k_orig64, n_kv_heads, ctx):
    """|gpu - ref| <= 1e-3 * ||q|| * ||k|| per (b, h, t)."""
    batch, n_q, _ = q64.shape
    group = n_q // n_kv_heads
    kn = np.linalg.norm(k_orig64, axis=1).reshape(batch, n_kv_heads, ctx)
    qn = np.linalg.norm(q64, axis=2)
    worst = 0.0
    for b in range(batch):
        for h in range(n_q):
            tol = LOGIT_TOL * qn[b, h] * kn[b, h // group]
            err = np.abs(gpu[b, h] - ref[b, h])
            worst = max(worst, float(np.max(err / np.maximum(tol, 1e-30))))
    assert worst <= 1.0, f"logit error reaches {worst:.3f} of the tolerance"
    return worst


def oracle_decode_on_cache(q64, rot64, kbits, vbits, kc, kn, vc, vn, n_kv_heads, ctx, block=32,
                           scale=None, qjl=None, norm_dtype="f16", v_layout="plain"):
    ck, _ = oracle_codebook(kbits, block)
    cv, _ = oracle_codebook(vbits, block)
    d = q64.shape[-1]
    ki = oq.unpack(kc, kbits, block, d)
    vi = oq.unpack(vc, vbits, block, d, layout=v_layout)
    return oatt.decode(q64, rot64, ki, kn, ck, vi, vn, cv, block, n_kv_heads, ctx, scale=scale,
                       qjl=qjl, norm_dtype=norm_dtype)


def check_decode(gpu, ref):
    num = np.linalg.norm(gpu - ref, axis=-1)
    den = np.maximum(np.linalg.norm(ref, axis=-1), 1e-30)
    rel = num / den
    worst = float(np.max(rel))
    assert worst <= DECODE_TOL, f"decode relative L2 error {worst:.3e} > {DECODE_TOL}"
    return worst


def qjl_oracle_arrays(signs_u32, rnorm_f16, m, S):
    return {"S": S, "signs": oqjl.unpack_signs(signs_u32, m), "rnorm": rnorm_f16}


def compare_qjl(x64, rot64, bits, S, gpu_codes, gpu_norms, gpu_signs, gpu_rnorm, block=32):
    """QJL stage on the library's own codes and norms: sign bits bit-exact
    except where |(S r)_i| < 1e-5 * ||S_i|| * ||r|| (counted); fp16 residual
    norms equal or one ulp apart."""
    c32, _ = oracle_codebook(bits, block)
    n, d = x64.shape
    y = oq.rotate_rows(x64, rot64)
    idx = oq.unpack(gpu_codes, bits, block, d)
    xh = oq.dequantize_rotated(idx, gpu_norms, c32, block)
    enc = oqjl.encode(y, xh, S)
    m = S.shape[0]
    gs = oqjl.unpack_signs(gpu_signs, m)
    rs = oqjl.unpack_signs(enc["signs"], m)
    band = np.abs(enc["z"]) < BAND * np.linalg.norm(S, axis=1)[None, :] * np.linalg.norm(enc["r"], axis=1)[:, None]
    mism = gs != rs
    outside = mism & ~band
    assert not outside.any(), f"{int(outside.sum())} QJL sign mismatches outside the band"
    ulp = np.abs(gpu_rnorm.view(np.int16).astype(np.int32) - enc["rnorm"].view(np.int16).astype(np.int32))
    assert np.all(ulp <= 1), "QJL residual norms differ by > 1 ulp"
    return {"signs": int(gs.size), "band": int(band.sum()), "band_mismatch": int((mism & band).sum())}
