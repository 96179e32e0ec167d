"""Dynamic row-wise FP8 quantisation (oracle; test infrastructure).

Page "Add CUTLASS-based row-wise scaled sparse FP8 kernel" (pytorch/ao pull
request 1671): the title and item 1 make both operands row-wise scaled; item 4
names the dynamic-activation path (``Float8DynamicActivationFloat8SemiSparse-
WeightConfig``), where the activation is quantised at run time.  The weight is
quantised with the same rule once, when it is prepared.

Per row m of a K-wide matrix x (values widened exactly to float32):

    amax[m] = max_k |x[m, k]|                        (float32, exact)
    s[m]    = max(amax[m], 1e-12f) / FP8_MAX         (one IEEE float32 division)
    q[m, k] = RNE_satfinite_fp8(x[m, k] / s[m])      (float32 division, then
                                                      one rounding to FP8)

Readings of what the page leaves open:

* the guard 1e-12 (as a float32 constant) keeps s positive and normal for an
  all-zero row, whose codes are then all zero (sign kept);
* ``x / s`` is a true division, correctly rounded to float32, and only then
  rounded to FP8 (not x / s in higher precision straight to FP8);
* saturation on overflow, for both formats.
"""

import numpy as np

from .fp8 import encode_rne_sat, fp8_max

GUARD_AMAX = np.float32(1e-12)


def quantize_rowwise(x32, fmt):
    """Quantise float32 rows to FP8 codes and per-row float32 scales.

    ``x32``: float32 array [M, K] (exact widening of a bf16/fp16/fp32 input).
    Returns (q uint8 [M, K], s float32 [M]).  K may be 0 (scales only).
    """
    x32 = np.asarray(x32, dtype=np.float32)
    if x32.ndim != 2:
        raise ValueError("x must be 2-D [rows, cols]")
    m, k = x32.shape
    if k == 0:
        amax = np.zeros((m,), dtype=np.float32)
    else:
        amax = np.max(np.abs(x32), axis=1).astype(np.float32)
    denom = np.float32(fp8_max(fmt))
    s = (np.maximum(amax, GUARD_AMAX) / denom).astype(np.float32)
    assert s.dtype == np.float32
    t = (x32 / s[:, None]).astype(np.float32)   # float32 / float32, IEEE
    q = encode_rne_sat(t, fmt)
    return q, s
