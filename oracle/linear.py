"""The row-wise scaled 2:4 sparse FP8 linear in fp64 (oracle; test infra).

Page "Add CUTLASS-based row-wise scaled sparse FP8 kernel" (pytorch/ao pull
request 1671), item 1: a row-wise scaled linear operator with a sparse FP8
weight and an FP8 activation:

    y[m, n] = s_a[m] * s_w[n] * sum_{g, j in {i0, i1}}
                  dec(A_q[m, 4g + j]) * dec(kept value of W row n at slot j)
              (+ bias[n])

computed here in float64 from the *logical* compressed weight (kept values
and index nibbles; see :mod:`oracle.compress`).  The dense decompressed weight
goes through one fp64 matrix product (a library primitive).  For e4m3 x e4m3
every product has at most 8 significant bits between 2^-18 and 2^17, so all
partial sums fit in 53 bits for K up to 2^14 and the sum is exact in any
order; for e5m2 operands it is exact to a few fp64 ulps.

Acceptance (the stated tolerance for the linear's output, against this fp64
value):

    |y - y_ref| <= 8e-3 * |y_ref| + 1e-3 * s_a[m] * s_w[n] * sum_k |a_q * w_q|
"""

import numpy as np

from .fp8 import decode
from .compress import decompress_24

REL_TOL = 8e-3
ABS_DOT_TOL = 1e-3


def _dense_weight(vals, nib, k, w_fmt):
    codes = decompress_24(vals, nib, k)
    w = decode(codes, w_fmt)
    # dropped slots are code 0x00 -> +0.0, which contributes nothing
    return w


def sparse_linear_ref(a_q, a_fmt, s_a, vals, nib, w_fmt, s_w, bias=None,
                      rows=None, cols=None):
    """fp64 reference output and the |a|.|w| sums used by the bound.

    a_q [M, K] uint8, s_a [M] float32, vals [N, K/2], nib [N, K/4],
    s_w [N] float32, bias [N] float (bf16 values) or None.  ``rows`` /
    ``cols`` select a subset of output rows (m) / columns (n); the result
    is then [len(rows), len(cols)].

    Returns (y_ref float64, absdot float64, scale float64) where
    scale[m, n] = s_a[m] * s_w[n].
    """
    a_q = np.asarray(a_q, dtype=np.uint8)
    m, k = a_q.shape
    vals = np.asarray(vals, dtype=np.uint8)
    nib = np.asarray(nib, dtype=np.uint8)
    s_a = np.asarray(s_a, dtype=np.float32).astype(np.float64)
    s_w = np.asarray(s_w, dtype=np.float32).astype(np.float64)
    if rows is None:
        rows = np.arange(m)
    if cols is None:
        cols = np.arange(vals.shape[0])
    rows = np.asarray(rows, dtype=np.int64)
    cols = np.asarray(cols, dtype=np.int64)
    a = decode(a_q[rows], a_fmt)                      # [r, K] float64
    w = _dense_weight(vals[cols], nib[cols], k, w_fmt)   # [c, K] float64
    if np.isnan(a).any() or np.isnan(w).any():
        raise ValueError("NaN codes are outside the linear's contract")
    acc = a @ w.T                                     # exact for e4m3 x e4m3
    absdot = np.abs(a) @ np.abs(w).T
    scale = s_a[rows][:, None] * s_w[cols][None, :]
    y = acc * scale
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[cols][None, :]
    return y, absdot, scale


def acceptance_bound(y_ref, absdot, scale):
    return REL_TOL * np.abs(y_ref) + ABS_DOT_TOL * scale * absdot


def check_linear(y_gpu, y_ref, absdot, scale):
    """Elementwise acceptance; returns (ok bool, worst ratio err/bound)."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    err = np.abs(y_gpu - y_ref)
    bound = acceptance_bound(y_ref, absdot, scale)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / np.where(bound > 0, bound, 1.0),
                         np.where(err > 0, np.inf, 0.0))
    ok = bool(np.all(err <= bound)) and bool(np.all(np.isfinite(y_gpu)))
    worst = float(ratio.max()) if ratio.size else 0.0
    return ok, worst
