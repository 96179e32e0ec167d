"""2:4 compression of FP8 codes (oracle; test infrastructure).

Page "Add CUTLASS-based row-wise scaled sparse FP8 kernel" (pytorch/ao pull
request 1671), item 1: a converter of FP8 data to the sparse semi-structured
format -- the kept values plus per-group index metadata; item 3: -0.0 must be
treated as zero when deciding what is kept.

Per group g of four codes c_0..c_3 along K (k = 4g .. 4g+3):

* magnitudes m_j = |decode(c_j)|, so 0x80 (-0.0) has magnitude 0;
* keep the two with rank < 2, rank as in :mod:`oracle.prune` (ties to the
  lower index); call their indices i0 < i1;
* kept values: c_{i0}, c_{i1}, the source codes unchanged;
* index nibble: i0 | (i1 << 2).  The six possible nibbles are listed in
  NIBBLES_VALID.

This is the *logical* result: values [N, K/2] and nibbles [N, K/4].  How the
library lays these out in memory is specified in :mod:`oracle.layout`.
"""

import numpy as np

from .fp8 import decode
from .prune import group_ranks

NIBBLES_VALID = tuple(sorted(i0 | (i1 << 2) for i0 in range(4)
                             for i1 in range(i0 + 1, 4)))


def compress_24(q, fmt):
    """Compress FP8 codes [N, K] (K % 4 == 0).

    Returns (vals uint8 [N, K/2], nibbles uint8 [N, K/4]).
    """
    q = np.asarray(q, dtype=np.uint8)
    n, k = q.shape
    if k % 4:
        raise ValueError("K must be a multiple of 4")
    groups = q.reshape(n, k // 4, 4)
    mag = np.abs(decode(groups, fmt))
    if np.isnan(mag).any():
        raise ValueError("NaN codes are outside the compressor's contract")
    keep = group_ranks(mag) < 2                      # exactly two per group
    idx = np.argsort(~keep, axis=-1, kind="stable")[..., :2]   # kept, ascending
    i0 = idx[..., 0]
    i1 = idx[..., 1]
    assert np.all(i0 < i1)
    v0 = np.take_along_axis(groups, i0[..., None], axis=-1)[..., 0]
    v1 = np.take_along_axis(groups, i1[..., None], axis=-1)[..., 0]
    vals = np.stack([v0, v1], axis=-1).reshape(n, k // 2).astype(np.uint8)
    nib = (i0 | (i1 << 2)).astype(np.uint8)
    return vals, nib


def decompress_24(vals, nib, k):
    """Inverse of :func:`compress_24`: codes [N, K], dropped slots 0x00."""
    vals = np.asarray(vals, dtype=np.uint8)
    nib = np.asarray(nib, dtype=np.uint8)
    n = vals.shape[0]
    if vals.shape != (n, k // 2) or nib.shape != (n, k // 4):
        raise ValueError("shape mismatch")
    bad = ~np.isin(nib, np.array(NIBBLES_VALID, dtype=np.uint8))
    if bad.any():
        raise ValueError("invalid index nibble")
    out = np.zeros((n, k // 4, 4), dtype=np.uint8)
    i0 = (nib & 3).astype(np.int64)
    i1 = ((nib >> 2) & 3).astype(np.int64)
    v = vals.reshape(n, k // 4, 2)
    np.put_along_axis(out, i0[..., None], v[..., 0:1], axis=-1)
    np.put_along_axis(out, i1[..., None], v[..., 1:2], axis=-1)
    return out.reshape(n, k)
