"""2:4 magnitude pruning of a 16/32-bit weight (oracle; test infrastructure).

The page "Add CUTLASS-based row-wise scaled sparse FP8 kernel" (pytorch/ao
pull request 1671) takes a weight that is already 2:4 sparse ("sparsify/
quantize method" in its list of remaining tasks) and does not say how it is
pruned.  The plainest reading, used here: in every group of four consecutive
elements along K, keep the two of largest magnitude and set the other two to
+0.0.  Magnitude compares |w|, so -0.0 counts as zero (the point of the page's
item 3).  Ties go to the lower index.

With m_j = |w_j| in a group, element j's rank is

    rank_j = #{i : m_i > m_j} + #{i < j : m_i == m_j}

and j is kept iff rank_j < 2.  Kept elements keep their exact bits.
"""

import numpy as np


def group_ranks(mag):
    """Ranks (see module docstring) of a [..., 4] magnitude array."""
    mag = np.asarray(mag)
    assert mag.shape[-1] == 4
    ranks = np.zeros(mag.shape, dtype=np.int64)
    for j in range(4):
        r = np.zeros(mag.shape[:-1], dtype=np.int64)
        for i in range(4):
            if i == j:
                continue
            r += (mag[..., i] > mag[..., j]).astype(np.int64)
            if i < j:
                r += (mag[..., i] == mag[..., j]).astype(np.int64)
        ranks[..., j] = r
    return ranks


def prune_24(w32):
    """Prune float32 values [N, K] (K % 4 == 0) to 2:4; returns float32.

    Dropped positions become +0.0; kept positions are the input values
    bit for bit (so a kept -0.0 stays -0.0).
    """
    w32 = np.asarray(w32, dtype=np.float32)
    n, k = w32.shape
    if k % 4:
        raise ValueError("K must be a multiple of 4")
    if np.isnan(w32).any():
        raise ValueError("NaN input is outside the pruner's contract")
    g = w32.reshape(n, k // 4, 4)
    keep = group_ranks(np.abs(g.astype(np.float64))) < 2
    out = np.where(keep, g, np.float32(0.0)).astype(np.float32)
    return out.reshape(n, k)
