"""Maximum-inner-product search over TurboQuant codes.

TEST INFRASTRUCTURE (oracle).  Not imported by the product path.

"Google TurboQuant deep dive", section 3.4: the codes also serve vector
search (recall measured against product quantization).  The pages print no
procedure; the plainest reading, and the one taken here, is the attention
score without the softmax: a database row j, quantized like a cache row, is
scored against a query q by the same pre-rotated inner product as a key

    score(q, j) = <R q, x_hat_j> = sum_k gamma_jk sum_{i in k} (R q)_i c[idx_ji]

(upstream guide, section 5.3: <q, R^T c[idx]> = <R q, c[idx]>), and the k
largest scores are returned, largest first; equal scores are ordered by
ascending row index.
"""

import numpy as np

from .quant import dequantize_rotated


def scores(q, rot, codes, norms, centroids, block, norm_dtype="f16"):
    """[n_q, n_db] float64: <R q_i, x_hat_j> for unpacked codes [n_db, d]."""
    q = np.asarray(q, dtype=np.float64)
    q_rot = q @ np.asarray(rot, dtype=np.float64).T
    x_hat = dequantize_rotated(codes, norms, centroids, block, norm_dtype)
    return q_rot @ x_hat.T


def topk(s, k):
    """(values, indices) [n_q, k]: the k largest entries of every row of s,
    largest first, ties by ascending index."""
    s = np.asarray(s, dtype=np.float64)
    n_q, n = s.shape
    k = min(k, n)
    idx = np.empty((n_q, k), dtype=np.int64)
    for i in range(n_q):
        order = np.lexsort((np.arange(n), -s[i]))   # primary: -score; then index
        idx[i] = order[:k]
    return np.take_along_axis(s, idx, axis=1), idx
