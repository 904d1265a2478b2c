"""Quantize / pack / dequantize for the MSE-only (PolarQuant-style) stage.

TEST INFRASTRUCTURE (oracle).  Not imported by the product path.

Upstream guide, section 5.1: the submitted variant is MSE-only PolarQuant with
block size 32: rotate, take the norm of each block, rescale, and quantize each
coordinate against the centroid table; section 5.2 commits 1-2 add the block
struct and the CPU quantize / dequantize.  Section 5.4: 2-, 3- and 4-bit
types.  The byte layout is never printed (section 5.1 only promises it), so
the layout below is this implementation's own:

* per row (one token of one KV head) and per block k of ``block`` coordinates:
  gamma_k = ||y_blk||_2 of the rotated row y = R x, stored as IEEE fp16
  (round to nearest even; values above 65504 saturate to 65504);
* codes idx_j = #{i : u_j >= t_i} with u = y_blk / gamma_k (unrounded gamma)
  and t the ascending Lloyd-Max boundaries -- a value exactly on a boundary
  takes the upper cell; if gamma_k == 0 every code of the block is 2^(b-1);
* packing: each block owns ``bits * block / 32`` consecutive uint32 words;
  code j of the block fills bits [j*b, j*b + b) of the little-endian bit
  stream formed by those words (word 0 bit 0 first), so 3-bit codes may
  straddle two words;
* dequantized value in the rotated frame: fp16(gamma_k) * c[idx_j], with c
  the fp32 centroid table.

Format variants (upstream guide, section 5.2: block 128 gives 5.12x with PPL
unchanged; section 11 names "norm correction" among the validated results;
section 1.2 quotes turbo4 at 4.25 bits per value):

* ``block`` may be 32, 64 or 128 (the codebook is fitted for that block);
* ``norm_dtype="f32"`` stores the block norm as IEEE fp32 (round to nearest)
  instead of fp16 -- with 4-bit codes and block 128 that is 4 + 32/128 = 4.25
  bits per value, the pages' turbo4 figure (reading taken here);
* ``norm_correction=True`` stores gamma_k / ||c[idx_blk]|| instead of gamma_k,
  so that the dequantized block fp(gamma') * c[idx] has the block's own norm
  up to the storage rounding (the pages name the step but print no formula;
  this is the plainest reading).  Codes are unchanged.
"""

import numpy as np

FP16_MAX = 65504.0


def rotate_rows(x, rot):
    """y = R x for every row of x (rows are vectors)."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(rot, dtype=np.float64).T


def block_norms(y, block):
    """gamma[row, k] = ||y[row, k*block:(k+1)*block]||_2 in float64."""
    n, d = y.shape
    return np.sqrt(np.sum(y.reshape(n, d // block, block) ** 2, axis=2))


def stored_norms(gamma, norm_dtype="f16"):
    """(stored norms, saturated mask).  fp16: RNE after clamping to 65504;
    fp32: RNE, nothing saturates below the fp32 range."""
    gamma = np.asarray(gamma, dtype=np.float64)
    if norm_dtype == "f32":
        return gamma.astype(np.float32), np.zeros(gamma.shape, dtype=bool)
    saturated = gamma > FP16_MAX
    return np.minimum(gamma, FP16_MAX).astype(np.float16), saturated


def reconstruction_norms(idx, centroids_f32, block):
    """||c[idx_blk]||_2 per row and block (float64 over the stored table)."""
    idx = np.asarray(idx)
    n, d = idx.shape
    c = np.asarray(centroids_f32, dtype=np.float32).astype(np.float64)
    return np.sqrt(np.sum(c[idx].reshape(n, d // block, block) ** 2, axis=2))


def codes(y, gamma, boundaries, bits, block):
    """Per-coordinate code = number of boundaries at or below u = y / gamma."""
    n, d = y.shape
    nb = d // block
    yb = y.reshape(n, nb, block)
    g = gamma.reshape(n, nb, 1)
    zero = g == 0.0
    u = yb / np.where(zero, 1.0, g)
    t = np.asarray(boundaries, dtype=np.float64)
    idx = np.sum(u[..., None] >= t[None, None, None, :], axis=-1)
    idx = np.where(zero, 1 << (bits - 1), idx)
    return idx.reshape(n, d).astype(np.int64)


def words_per_row(bits, block, d):
    return (d // block) * (bits * block // 32)


def code_bit_offsets(bits, block, d, layout="plain"):
    """Bit offset of the code of coordinate j in its row's little-endian bit
    stream.  ``plain``: block k owns bits [k*block*bits, (k+1)*block*bits) and
    code j of a block sits at j*bits inside it.  ``grouped`` (32-value blocks
    only): the row is ordered by groups of four consecutive coordinates -- the
    group g of every block (blocks 0 .. d/32 - 1), then group g + 1 -- so code
    (block b, coordinate 4g + e) sits at bits * (4 * (nb*g + b) + e), nb = d/32.
    The grouped order is this library's layout for value caches (a reading:
    the pages fix no byte layout); it keeps the four codes that one lane of
    the decode's value product reads together with those of the other blocks."""
    j = np.arange(d)
    if layout == "plain":
        return (j // block) * block * bits + (j % block) * bits
    if layout != "grouped" or block != 32:
        raise ValueError("grouped layout: 32-value blocks only")
    nb = d // 32
    b, c = j // 32, j % 32
    return bits * (4 * (nb * (c // 4) + b) + c % 4)


def pack(idx, bits, block, layout="plain"):
    """Pack codes [n, d] into uint32 words [n, (d/block) * bits*block/32]."""
    idx = np.asarray(idx, dtype=np.int64)
    n, d = idx.shape
    off = code_bit_offsets(bits, block, d, layout)
    out = np.zeros((n, d * bits // 32), dtype=np.uint64)
    for j in range(d):
        for q in range(bits):
            pos = int(off[j]) + q
            bit = (idx[:, j] >> q) & 1
            out[:, pos // 32] |= bit.astype(np.uint64) << np.uint64(pos % 32)
    return out.astype(np.uint32)


def unpack(words, bits, block, d, layout="plain"):
    """Inverse of ``pack``: uint32 words [n, W] -> codes [n, d]."""
    w = np.asarray(words, dtype=np.uint64)
    n = w.shape[0]
    off = code_bit_offsets(bits, block, d, layout)
    idx = np.zeros((n, d), dtype=np.int64)
    for j in range(d):
        for q in range(bits):
            pos = int(off[j]) + q
            bit = (w[:, pos // 32] >> np.uint64(pos % 32)) & np.uint64(1)
            idx[:, j] |= bit.astype(np.int64) << q
    return idx


def dequantize_rotated(idx, norms_f16, centroids_f32, block, norm_dtype="f16"):
    """x_hat in the rotated frame: the stored norm of the block (rounded to
    the storage type: fp16, or fp32 for ``norm_dtype="f32"``) times c[idx]."""
    idx = np.asarray(idx)
    n, d = idx.shape
    c = np.asarray(centroids_f32, dtype=np.float32).astype(np.float64)
    store = np.float32 if norm_dtype == "f32" else np.float16
    g = np.asarray(norms_f16, dtype=store).astype(np.float64)
    vals = c[idx].reshape(n, d // block, block) * g[:, :, None]
    return vals.reshape(n, d)


def quantize(x, rot, centroids_f32, boundaries, bits, block, norm_dtype="f16",
             norm_correction=False):
    """Full MSE-only quantization of the rows of x.

    Returns a dict with the rotated rows ``y``, float64 norms ``gamma``,
    ``codes`` (unpacked), ``words`` (packed uint32), stored ``norms`` (fp16,
    or fp32 for ``norm_dtype="f32"``; divided by ||c[idx_blk]|| with
    ``norm_correction``) and the ``saturated`` mask.
    """
    y = rotate_rows(x, rot)
    gamma = block_norms(y, block)
    idx = codes(y, gamma, boundaries, bits, block)
    stored = gamma
    if norm_correction:
        stored = gamma / reconstruction_norms(idx, centroids_f32, block)
    norms, sat = stored_norms(stored, norm_dtype)
    return {
        "y": y,
        "gamma": gamma,
        "codes": idx,
        "words": pack(idx, bits, block),
        "norms": norms,
        "saturated": sat,
    }


def boundary_distance(y, gamma, boundaries, block):
    """min_i |u_j - t_i| per coordinate (float64); inf where gamma == 0."""
    n, d = y.shape
    nb = d // block
    g = gamma.reshape(n, nb, 1)
    zero = g == 0.0
    u = y.reshape(n, nb, block) / np.where(zero, 1.0, g)
    t = np.asarray(boundaries, dtype=np.float64)
    dist = np.min(np.abs(u[..., None] - t[None, None, None, :]), axis=-1)
    dist = np.where(zero, np.inf, dist)
    return dist.reshape(n, d)
