"""Tensor-wise (one global amax) FP8 quantisation (oracle; test infrastructure).

Page "[float8nocompile] Add alternate Triton kernels for FP8 conversion which
use atomic_max-based algo instead of reduction-based algo" (pytorch/ao pull
request 1455), Summary: one global amax for the whole tensor, found either by
a reduction over per-block partial maxima (deterministic, the reviewer's
point) or by every block folding its local amax into one shared scalar with
an atomic max; both strategies give the same amax, since a maximum is exact
and independent of order.  The page does not restate the conversion itself;
the reading here is the row-wise rule of the page "Add CUTLASS-based row-wise
scaled sparse FP8 kernel" (pytorch/ao pull request 1671) with the whole tensor
as the one group:

    amax = max over all elements |x|                  (float32, exact)
    s    = max(amax, 1e-12f) / FP8_MAX                (one IEEE float32 division)
    q    = RNE_satfinite_fp8(x / s)                   (float32 division, then
                                                       one rounding to FP8)

so a tensor of one row quantises exactly as the row-wise quantiser does.
"""

import numpy as np

from .fp8 import encode_rne_sat, fp8_max
from .quantize import GUARD_AMAX


def quantize_tensorwise(x32, fmt):
    """Quantise a float32 array (any shape, exact widening of a bf16/fp16/fp32
    input) with one scale.  Returns (q uint8, same shape; s float32 scalar).
    An empty array gives the guard scale."""
    x32 = np.asarray(x32, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0.0)
    s = np.float32(np.maximum(amax, GUARD_AMAX) / np.float32(fp8_max(fmt)))
    t = (x32 / s).astype(np.float32)            # float32 / float32, IEEE
    return encode_rne_sat(t, fmt), s
