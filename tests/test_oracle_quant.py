"""Pins for the oracle's quantize / pack / dequantize (CPU only)."""

import itertools
import os

import numpy as np
import pytest

from oracle import codebook, quant, rotation


def _bitstring_pack(idx_row, bits, block):
    """Pack one row through an explicit '0'/'1' string: each block's codes LSB
    first, then cut into 32-bit words read LSB first."""
    words = []
    for k in range(len(idx_row) // block):
        s = "".join(format(int(v), f"0{bits}b")[::-1] for v in idx_row[k * block:(k + 1) * block])
        for w in range(len(s) // 32):
            words.append(int(s[32 * w:32 * w + 32][::-1], 2))
    return np.array(words, dtype=np.uint64)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("block,d", [(32, 128), (32, 64), (32, 256), (8, 8), (16, 32)])
def test_pack_layout_and_round_trip(bits, block, d):
    if bits * block % 32:
        pytest.skip("block does not fill whole words")
    idx = np.random.default_rng(bits * 100 + d).integers(0, 1 << bits, size=(9, d))
    words = quant.pack(idx, bits, block)
    assert words.shape == (9, quant.words_per_row(bits, block, d))
    for r in range(9):
        assert np.array_equal(words[r].astype(np.uint64), _bitstring_pack(idx[r], bits, block))
    assert np.array_equal(quant.unpack(words, bits, block, d), idx)


def _bitstring_pack_grouped(idx_row, bits):
    """Grouped rows through an explicit '0'/'1' string: for each group of four
    coordinates g = 0..7, for each 32-value block, that block's four codes
    (LSB first); then 32-bit words read LSB first."""
    nb = len(idx_row) // 32
    s = ""
    for g in range(8):
        for b in range(nb):
            for e in range(4):
                s += format(int(idx_row[32 * b + 4 * g + e]), f"0{bits}b")[::-1]
    return np.array([int(s[32 * w:32 * w + 32][::-1], 2) for w in range(len(s) // 32)], dtype=np.uint64)


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_grouped_layout_and_round_trip(bits, d):
    idx = np.random.default_rng(bits * 7 + d).integers(0, 1 << bits, size=(7, d))
    words = quant.pack(idx, bits, 32, layout="grouped")
    assert words.shape == (7, quant.words_per_row(bits, 32, d))
    for r in range(7):
        assert np.array_equal(words[r].astype(np.uint64), _bitstring_pack_grouped(idx[r], bits))
    assert np.array_equal(quant.unpack(words, bits, 32, d, layout="grouped"), idx)
    # the same codes as the plain layout, only moved
    plain = quant.pack(idx, bits, 32)
    assert sorted(np.unpackbits(words.view(np.uint8)).tolist()) == \
        sorted(np.unpackbits(plain.view(np.uint8)).tolist())


def test_grouped_layout_hand_example():
    # d = 128, 3-bit: code 7 at block 1, coordinate 5 (group 1, position 1)
    # starts at bit 3 * (4 * (4 * 1 + 1) + 1) = 63: word 1 bit 31, word 2 bits 0-1
    idx = np.zeros((1, 128), dtype=np.int64)
    idx[0, 32 + 5] = 0b111
    w = quant.pack(idx, 3, 32, layout="grouped")
    assert w[0, 1] == 1 << 31 and w[0, 2] == 0b11 and np.count_nonzero(w) == 2
    with pytest.raises(ValueError):
        quant.pack(idx, 3, 64, layout="grouped")


def test_three_bit_codes_straddle_words():
    idx = np.zeros((1, 32), dtype=np.int64)
    idx[0, 10] = 0b111   # bits 30..32: two in word 0, one in word 1
    w = quant.pack(idx, 3, 32)
    assert w[0, 0] == (0b11 << 30) and w[0, 1] == 1 and w[0, 2] == 0


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codes_are_nearest_centroid(bits):
    c, t = codebook.lloyd_max(bits, 32)
    x = np.random.default_rng(3).standard_normal((500, 128))
    y = x @ rotation.wht_rotation(128, 1000).T
    g = quant.block_norms(y, 32)
    idx = quant.codes(y, g, t, bits, 32)
    u = (y.reshape(500, 4, 32) / g[:, :, None]).reshape(500, 128)
    nearest = np.argmin(np.abs(u[..., None] - c[None, None, :]), axis=-1)
    far = quant.boundary_distance(y, g, t, 32) > 1e-12
    assert np.array_equal(idx[far], nearest[far])


@pytest.mark.parametrize("bits,d", [(1, 4), (2, 4), (3, 4), (4, 4), (1, 8), (2, 8)])
def test_brute_force_joint_argmin(bits, d):
    """On d = Bk, the separable rule equals the joint argmin over every code
    vector of ||u - c[idx]||^2."""
    c, t = codebook.lloyd_max(bits, d)
    allcodes = np.array(list(itertools.product(range(1 << bits), repeat=d)))
    recon = c[allcodes]                                   # [K, d]
    u = np.random.default_rng(bits * 10 + d).standard_normal((40, d))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    idx = quant.codes(u, np.ones((40, 1)), t, bits, d)
    for r in range(40):
        err = np.sum((u[r][None, :] - recon) ** 2, axis=1)
        assert np.array_equal(allcodes[np.argmin(err)], idx[r])


def test_ties_go_up_and_zero_blocks():
    c, t = codebook.lloyd_max(3, 32)
    gamma = np.array([[4.0]])
    y = np.zeros((1, 32))
    y[0, :7] = t * 4.0                  # exactly on each boundary (power-of-two scale)
    idx = quant.codes(y, gamma, t, 3, 32)
    assert list(idx[0, :7]) == [1, 2, 3, 4, 5, 6, 7]
    z = quant.codes(np.zeros((2, 64)), np.zeros((2, 2)), t, 3, 32)
    assert np.all(z == 4)


def test_stored_norms_round_and_saturate():
    g = np.array([[1.0, 1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11, 70000.0]])
    s, sat = quant.stored_norms(g)
    assert s.dtype == np.float16
    assert s[0, 1] == np.float16(1.0)              # tie -> even
    assert s[0, 2] == np.float16(1.0 + 2 ** -9)    # tie -> even (upwards)
    assert s[0, 3] == np.float16(65504.0)
    assert list(sat[0]) == [False, False, False, True]


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_empirical_mse_matches_codebook_distortion(bits):
    c, t = codebook.lloyd_max(bits, 32)
    dist = codebook.distortion(c, 32)
    x = np.random.default_rng(bits).standard_normal((20_000, 32))
    u = x / np.linalg.norm(x, axis=1, keepdims=True)
    idx = quant.codes(u, np.ones((20_000, 1)), t, bits, 32)
    err = np.mean(np.sum((u - c[idx]) ** 2, axis=1)) / 32
    assert abs(err - dist) < 0.03 * dist


def test_dequantize_hand_built_blocks():
    """Two rows of two 32-blocks with norms that are not fp16 values: every
    coordinate must come back as fp16(norm of its own block) * c[code]
    (upstream guide section 5.1: the per-block norm is stored and multiplied
    back).  The fp16 values are written out by hand; the products are exact in
    float64 (11 + 24 significant bits)."""
    c32, _ = codebook.stored_table(3, 32)
    gamma = np.array([[2.0 + 1.25 * 2 ** -9, 0.75],            # -> 2 + 2^-9, 0.75
                      [1000.3, 3.0 + 2 ** -12]])                # -> 1000.5, 3.0
    gamma_f16 = [[2.001953125, 0.75], [1000.5, 3.0]]
    idx = np.zeros((2, 64), dtype=np.int64)
    idx[0, :32] = np.arange(32) % 8
    idx[0, 32:] = 7 - np.arange(32) % 8
    idx[1, :32] = (3 * np.arange(32)) % 8
    idx[1, 32:] = 5
    out = quant.dequantize_rotated(idx, gamma, c32, 32)
    for r in range(2):
        for j in range(64):
            expect = gamma_f16[r][j // 32] * float(c32[idx[r, j]])
            assert out[r, j] == expect, (r, j, out[r, j], expect)
    # fp16 norm arrays are taken as they are
    out16 = quant.dequantize_rotated(idx, np.array(gamma_f16, dtype=np.float16), c32, 32)
    assert np.array_equal(out16, out)


@pytest.mark.parametrize("bits,block,norm_dtype", [
    (2, 32, "f16"), (3, 32, "f16"), (4, 32, "f16"), (3, 64, "f16"), (4, 128, "f32"),
    (2, 128, "f16")])
def test_round_trip_distortion_equals_codebook_distortion(bits, block, norm_dtype):
    """quantize -> dequantize_rotated -> R^T on Haar-rotated N(0, 1) rows.

    Every 32-block of y = R x is Gaussian, so its direction u is uniform on the
    sphere and independent of its norm gamma; hence
    E||x - R^T x_hat||^2 / E||x||^2 = E||u - c[idx]||^2 = Bk * D_b, with D_b the
    per-coordinate distortion of the Lloyd-Max fixed point.  Storing gamma as
    fp16 (relative error <= 2^-11) and the centroids at fp16 adds at most
    ~1e-6 + 2 * 2^-11 * E||c|| * E||u - c|| relative, far inside the 3 %
    Monte Carlo band (80 000 blocks).  A dropped or misplaced norm, a wrong
    block index or a transposed rotation moves the ratio by far more."""
    n, d = 20_000, 128
    x = np.random.default_rng(77 + bits + block).standard_normal((n, d))
    rot = rotation.haar_rotation(d, 1000)
    c32, t = codebook.stored_table(bits, block)
    c64, _ = codebook.lloyd_max(bits, block)
    q = quant.quantize(x, rot, c32, t, bits, block, norm_dtype=norm_dtype)
    xr = quant.dequantize_rotated(q["codes"], q["norms"], c32, block, norm_dtype=norm_dtype) @ rot
    ratio = np.sum((x - xr) ** 2) / np.sum(x * x)
    expect = block * codebook.distortion(c64, block)
    # block 128 at d = 128: 20 000 blocks, so a wider (still 5-sigma) band
    tol = 0.03 if d // block * n >= 40_000 else 0.05
    assert abs(ratio - expect) < tol * expect, (ratio, expect)


@pytest.mark.parametrize("bits,block,norm_dtype", [
    (2, 32, "f16"), (3, 32, "f16"), (4, 64, "f16"), (3, 128, "f16"), (4, 128, "f32"),
    (2, 64, "f32")])
def test_norm_correction_restores_block_norms(bits, block, norm_dtype):
    """Norm correction (upstream guide, section 11): the stored norm is chosen
    so that the dequantized block has the norm of the rotated block itself, up
    to the storage rounding of the norm (fp16: 2^-11 relative; fp32: 2^-24).
    Codes are the same as without correction, and a block of zeros stays
    zero."""
    n, d = 500, 128
    x = np.random.default_rng(bits + block).standard_normal((n, d)) * 3.0
    x[7] = 0.0
    rot = rotation.wht_rotation(d, 1000)
    c32, t = codebook.stored_table(bits, block)
    plain = quant.quantize(x, rot, c32, t, bits, block, norm_dtype=norm_dtype)
    corr = quant.quantize(x, rot, c32, t, bits, block, norm_dtype=norm_dtype, norm_correction=True)
    assert np.array_equal(plain["codes"], corr["codes"])
    xh = quant.dequantize_rotated(corr["codes"], corr["norms"], c32, block, norm_dtype=norm_dtype)
    got = quant.block_norms(xh, block)
    want = quant.block_norms(corr["y"], block)
    rel = 2.0 ** -11 if norm_dtype == "f16" else 2.0 ** -24
    nz = want > 0
    assert np.all(np.abs(got[nz] - want[nz]) <= (rel + 1e-12) * want[nz])
    assert np.all(got[~nz] == 0.0) and np.all(nz[np.arange(n) != 7]) and not np.any(nz[7])
    # without correction the dequantized norm is shrunk: ||c[idx]|| < 1 on
    # average (E||c[idx]||^2 = 1 - Bk D_b for a Lloyd-Max codebook)
    xp = quant.dequantize_rotated(plain["codes"], plain["norms"], c32, block, norm_dtype=norm_dtype)
    shrink = np.mean(quant.block_norms(xp, block)[nz] ** 2 / want[nz] ** 2)
    c64, _ = codebook.lloyd_max(bits, block)
    assert abs(shrink - (1 - block * codebook.distortion(c64, block))) < 0.02


def test_round_trip_error_shrinks_with_bits():
    x = np.random.default_rng(5).standard_normal((400, 128))
    rot = rotation.wht_rotation(128, 1000)
    errs = []
    for bits in (2, 3, 4):
        c32, t = codebook.stored_table(bits, 32)
        q = quant.quantize(x, rot, c32, t, bits, 32)
        xr = quant.dequantize_rotated(q["codes"], q["norms"], c32, 32) @ rot
        errs.append(np.mean(np.sum((xr - x) ** 2, axis=1) / np.sum(x * x, axis=1)))
    assert errs[0] > errs[1] > errs[2]


def test_compression_ratios_printed_by_the_pages(golden_dir):
    """16 / (b + 16 / Bk): fp16 values vs b-bit codes plus one fp16 norm per block."""
    with open(os.path.join(golden_dir, "pages_compression_ratios.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    for bits, block, norm_bits, ratio, decimals in rows:
        bits, block, norm_bits, decimals = int(bits), int(block), int(norm_bits), int(decimals)
        d = 128
        row_bytes = quant.words_per_row(bits, block, d) * 4 + norm_bits // 8 * (d // block)
        assert round(2 * d / row_bytes, decimals) == float(ratio)
    # the stored norm arrays have exactly that many bytes per row
    x = np.random.default_rng(0).standard_normal((3, 128))
    c, t = codebook.stored_table(4, 128)
    q = quant.quantize(x, rotation.wht_rotation(128, 1000), c, t, 4, 128, norm_dtype="f32")
    assert q["norms"].dtype == np.float32 and q["norms"].shape == (3, 1)
    assert q["words"].shape == (3, 16)
