"""CPU tests of the C-ABI library: it loads, exports every symbol tq.h
declares, its host generators match the oracle, and host-detectable errors
are rejected before any launch (no GPU needed)."""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import kv_cache_vector_11_b200 as tq
from oracle import codebook as ocb
from oracle import rotation as orot

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    declared = _declared_functions()
    assert len(declared) >= 12
    out = subprocess.run(["nm", "-D", "--defined-only", tq.lib_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(tq_[a-z0-9_]+)$", out, flags=re.M))
    missing = [n for n in declared if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(tq.lib_path())
    for n in declared:
        assert hasattr(lib, n)
    assert set(tq.exported_symbols()) <= set(declared)


def test_product_package_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "kv_cache_vector_11_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".cpp", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", text, flags=re.M), f
                assert "oracle/" not in text, f


@pytest.mark.parametrize("d", [64, 128, 256])
def test_wht_matrix_matches_oracle(d):
    for seed in (1000, 7, (1 << 64) - 1):
        lib = tq.rotation_generate("wht", d, d, seed)
        ref = orot.wht_rotation(d, seed)
        assert np.array_equal(np.sign(lib), np.sign(ref))      # every sign identical
        assert np.max(np.abs(lib - ref)) < 1e-15               # d^-1/2 to the last ulp


@pytest.mark.parametrize("d", [8, 64, 128, 256])
def test_haar_matrix_matches_oracle(d):
    lib = tq.rotation_generate("haar", d, d, 1000)
    ref = orot.haar_rotation(d, 1000)
    assert np.max(np.abs(lib - ref)) < 1e-12
    assert np.max(np.abs(lib @ lib.T - np.eye(d))) < 1e-13
    assert np.linalg.det(lib) > 0


def test_gaussian_projection_matches_oracle():
    lib = tq.rotation_generate("gauss", 128, 128, 2000)
    assert np.max(np.abs(lib - orot.gaussian_projection(128, 128, 2000))) < 1e-13
    lib2 = tq.rotation_generate("gauss", 64, 256, 2063)
    assert np.max(np.abs(lib2 - orot.gaussian_projection(64, 256, 2063))) < 1e-13


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("block", [4, 8, 16, 32, 64, 128])
def test_codebook_matches_oracle(bits, block):
    c, t = tq.build_codebook(bits, block)
    oc, ot = ocb.lloyd_max(bits, block)
    assert np.array_equal(c, oc.astype(np.float16).astype(np.float32))
    assert np.array_equal(c, ocb.stored_table(bits, block)[0])
    assert np.max(np.abs(t.astype(np.float64) - ot)) <= np.spacing(np.float32(0.5))
    assert np.all(c == -c[::-1]) and np.all(t == -t[::-1])


def test_codebook_uniform_density_closed_form():
    c, _ = tq.build_codebook(3, 3)
    assert np.allclose(c, -1 + (2 * np.arange(8) + 1) / 8, atol=1e-7, rtol=0)


def test_words_per_row_and_format_sizes():
    assert tq.code_words_per_row(4, 32, 128) == 16
    assert tq.code_words_per_row(3, 32, 128) == 12
    assert tq.code_words_per_row(2, 32, 256) == 16
    assert tq.code_words_per_row(3, 32, 100) == -1


def test_host_rejects_bad_arguments():
    with pytest.raises(tq.TQError):
        tq.rotation_generate("wht", 96, 96, 0)   # not a power of two
    with pytest.raises(tq.TQError):
        tq.build_codebook(5, 32)
    lib = ctypes.CDLL(tq.lib_path())
    assert lib.tq_build_codebook(2, 2, None, None) == 1
    lib.tq_status_string.restype = ctypes.c_char_p
    assert lib.tq_status_string(2) == b"unsupported configuration"


def test_quantize_argument_checks_happen_before_launch():
    """A WHT handle needs no device; bad sizes are rejected on the host."""
    lib = ctypes.CDLL(tq.lib_path())
    lib.tq_make_rotation.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_uint64, ctypes.POINTER(ctypes.c_void_p)]
    h = ctypes.c_void_p()
    assert lib.tq_make_rotation(0, 128, 128, 1000, ctypes.byref(h)) == 0
    c, t = tq.build_codebook(4)
    lib.tq_quantize_kv.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                   ctypes.c_int32] + [ctypes.c_void_p] * 6
    fake = 1 << 20  # never dereferenced: every call below fails its host checks
    args = lambda bits, block, d, n, x: (h, bits, block, c.ctypes.data, t.ctypes.data, None,
                                         x, 1, n, d, fake, fake, None, None, None, None)
    assert lib.tq_quantize_kv(*args(5, 32, 128, 10, fake)) == 2       # bits
    assert lib.tq_quantize_kv(*args(4, 16, 128, 10, fake)) == 2       # block
    assert lib.tq_quantize_kv(*args(4, 32, 64, 10, fake)) == 1        # size mismatch
    assert lib.tq_quantize_kv(*args(4, 32, 128, -1, fake)) == 1       # n_rows < 0
    assert lib.tq_quantize_kv(*args(4, 32, 128, 10, None)) == 1       # null x
    assert lib.tq_quantize_kv(*args(4, 32, 128, 10, fake + 4)) == 1   # misaligned
    assert lib.tq_quantize_kv(*args(4, 32, 128, 0, None)) == 0        # empty: no-op
    lib.tq_free_rotation.argtypes = [ctypes.c_void_p]
    lib.tq_free_rotation(h)


def test_decode_argument_checks_happen_before_launch():
    lib = ctypes.CDLL(tq.lib_path())
    lib.tq_make_rotation.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_uint64, ctypes.POINTER(ctypes.c_void_p)]
    h = ctypes.c_void_p()
    assert lib.tq_make_rotation(0, 128, 128, 1000, ctypes.byref(h)) == 0
    c, _ = tq.build_codebook(3)
    vp = ctypes.c_void_p
    lib.tq_decode_attention.argtypes = [vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, vp, vp,
                                        vp, vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                        ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, vp, vp,
                                        vp, vp, vp, vp, ctypes.c_float, vp, vp, ctypes.c_size_t, vp]
    fake = 1 << 20
    def call(n_q, n_kv, ctx, ws_bytes, kbits=3):
        return lib.tq_decode_attention(h, kbits, 3, 32, c.ctypes.data, c.ctypes.data, None, fake, 1,
                                       1, n_q, n_kv, ctx, 128, fake, fake, None, None, fake, fake,
                                       0.0, fake, fake, ws_bytes, None)
    assert call(6, 4, 100, 1 << 30) == 1          # n_q not a multiple of n_kv
    assert call(72, 8, 100, 1 << 30) == 2         # group of 9 > 8
    assert call(32, 8, 0, 1 << 30) == 1           # empty context
    assert call(32, 8, 100, 0) == 1               # workspace too small
    assert call(32, 8, 100, 1 << 30, kbits=1) == 2
    lib.tq_free_rotation.argtypes = [vp]
    lib.tq_free_rotation(h)


def test_format_search_and_append_checks_happen_before_launch():
    """The format variants, the search and the paged append reject bad
    arguments on the host (fake device pointers are never dereferenced)."""
    lib = ctypes.CDLL(tq.lib_path())
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    lib.tq_make_rotation.argtypes = [i32, i32, i32, ctypes.c_uint64, ctypes.POINTER(vp)]
    h = vp()
    assert lib.tq_make_rotation(0, 64, 64, 1000, ctypes.byref(h)) == 0
    c, t = tq.build_codebook(3, 64)
    fake = 1 << 20
    lib.tq_quantize_kv_ex.argtypes = [vp, i32, i32, vp, vp, vp, vp, i32, i64, i32, ctypes.c_uint32,
                                      vp, vp, vp, vp, vp, vp]
    q = lambda block, fmt, d=64: lib.tq_quantize_kv_ex(h, 3, block, c.ctypes.data, t.ctypes.data,
                                                      None, fake, 1, 10, d, fmt, fake, fake, None,
                                                      None, None, None)
    assert q(48, 0) == 2            # block not 32 / 64 / 128
    assert q(128, 0) == 2           # block larger than the head
    assert q(64, 8) == 1            # unknown format flag
    assert q(64, 4) == 2            # lane-grouped rows need head_dim 128
    assert lib.tq_quantize_kv_ex(h, 3, 64, c.ctypes.data, t.ctypes.data, None, fake, 1, 0, 64, 3,
                                 None, None, None, None, None, None) == 0   # empty: no-op
    lib.tq_search_topk.argtypes = [vp, i32, i32, vp, vp, i32, i32, i32, vp, vp, i64, i32, vp, vp,
                                   vp, ctypes.c_size_t, vp]
    lib.tq_search_workspace_size.restype = ctypes.c_size_t
    lib.tq_search_workspace_size.argtypes = [i32, i64, i32, i32]
    need = lib.tq_search_workspace_size(4, 1000, 64, 10)
    assert need >= 4 * 10 * 8             # at least k candidate keys per query
    s = lambda k, n_db, ws, block=32: lib.tq_search_topk(h, 3, block, c.ctypes.data, fake, 1, 4, 64,
                                                         fake, fake, n_db, k, fake, fake, fake, ws,
                                                         None)
    assert s(0, 1000, need) == 2          # k < 1
    assert s(257, 1000, need) == 2        # k > 256
    assert s(11, 10, need) == 2           # k > n_db
    assert s(10, 1000, 0) == 1            # workspace too small
    assert s(10, 1000, need, block=64) == 2
    lib.tq_decode_append_paged.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, vp, i32, vp, vp, i32,
                                           i32, i32, i32, i64, i32, i32, i32, vp, i32, vp, vp, vp,
                                           vp, ctypes.c_float, vp, vp, ctypes.c_size_t, vp, vp]
    c32, t32 = tq.build_codebook(3)

    def ap(page, ctx, max_pages=8, n_pages=16, ws=1 << 30):
        return lib.tq_decode_append_paged(h, 3, 3, 32, c32.ctypes.data, t32.ctypes.data,
                                          c32.ctypes.data, t32.ctypes.data, fake, 1, fake, fake, 1,
                                          1, 4, 1, ctx, 64, page, n_pages, fake, max_pages, fake,
                                          fake, fake, fake, 0.0, fake, fake, ws, None, None)
    assert ap(24, 100) == 2               # page size not a power of two
    assert ap(8, 100) == 2                # page size below 16
    assert ap(16, 200) == 1               # ctx > max_pages * page_size
    assert ap(16, 100, ws=0) == 1         # workspace too small
    lib.tq_free_rotation.argtypes = [vp]
    lib.tq_free_rotation(h)


def test_grouped_format_checks_happen_before_launch():
    """TQ_FMT_GROUPED is accepted only where a kernel writes or reads it: bf16
    rows at head_dim 128 with block 32 and no other flag in the quantizer
    (QJL signs: tests/test_gpu_grouped.py, the projection needs a device),
    value codes in the decode, never the keys of the logits (fake device
    pointers are never dereferenced)."""
    lib = ctypes.CDLL(tq.lib_path())
    vp, i32, i64, u32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32
    lib.tq_make_rotation.argtypes = [i32, i32, i32, ctypes.c_uint64, ctypes.POINTER(vp)]
    h = vp()
    assert lib.tq_make_rotation(0, 128, 128, 1000, ctypes.byref(h)) == 0
    c, t = tq.build_codebook(3)
    fake = 1 << 20
    lib.tq_quantize_kv_ex.argtypes = [vp, i32, i32, vp, vp, vp, vp, i32, i64, i32, u32,
                                      vp, vp, vp, vp, vp, vp]

    def q(fmt, dtype=1, block=32, qjl=None, n=10):
        return lib.tq_quantize_kv_ex(h, 3, block, c.ctypes.data, t.ctypes.data, qjl, fake, dtype,
                                     n, 128, fmt, fake, fake, fake, fake, None, None)
    assert q(4, dtype=0) == 2        # fp32 rows
    assert q(4 | 1) == 2             # with fp32 norms
    assert q(4 | 2) == 2             # with norm correction
    assert q(4, block=64) == 2       # block 64
    assert q(4, n=0) == 0            # empty: accepted, nothing launched
    lib.tq_attn_logits_ex.argtypes = [vp, i32, i32, vp, vp, vp, i32, i32, i32, i32, i64, i32, u32,
                                      vp, vp, vp, vp, vp, vp]
    assert lib.tq_attn_logits_ex(h, 3, 32, c.ctypes.data, None, fake, 1, 1, 4, 1, 64, 128, 4,
                                 fake, fake, None, None, fake, None) == 2   # keys are never grouped
    lib.tq_decode_attention_ex.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, i32, i32, i32, i32,
                                           i64, i32, u32, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp,
                                           vp, ctypes.c_size_t, vp]
    h64 = vp()
    assert lib.tq_make_rotation(0, 64, 64, 1000, ctypes.byref(h64)) == 0
    assert lib.tq_decode_attention_ex(h64, 3, 3, 32, c.ctypes.data, c.ctypes.data, None, fake, 1,
                                      1, 4, 1, 64, 64, 4, fake, fake, None, None, fake, fake, 0.0,
                                      fake, fake, 1 << 30, None) == 2   # head_dim 64
