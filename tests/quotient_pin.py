"""Expected FP8 codes of the quotient x/s, computed without the oracle (CPU pin).

The row-wise rule of the page "Add CUTLASS-based row-wise scaled sparse FP8
kernel" (pytorch/ao pull request 1671, title and item 1) scales each row by
s = amax / FP8_MAX and casts x / s.  The reading pinned here: the quotient is
one correctly rounded float32 division, RN32(x / s), then one saturating
round-to-nearest-even to FP8 -- not x * RN32(1 / s), which differs near FP8
midpoints.

Independence from the oracle's arithmetic:

* the quotient of two float32 numbers, evaluated in float64 and rounded once
  to float32, is the correctly rounded float32 quotient, because float64 has
  53 >= 2 * 24 + 2 significand bits (double rounding is innocuous for a
  division at that width);
* the FP8 rounding below FP8_MAX is ml_dtypes' cast; at or above FP8_MAX the
  code is the largest finite one with x's sign (saturation), taken from the
  format definitions (0x7E for e4m3, 0x7B for e5m2), not from the oracle.
"""
import ml_dtypes
import numpy as np

E4M3, E5M2 = "e4m3", "e5m2"
LIB = {E4M3: ml_dtypes.float8_e4m3fn, E5M2: ml_dtypes.float8_e5m2}
MAX_VALUE = {E4M3: 448.0, E5M2: 57344.0}
MAX_CODE = {E4M3: 0x7E, E5M2: 0x7B}


def scale(amax, fmt):
    """RN32(max(amax, 1e-12f) / FP8_MAX), through float64 (exact argument above)."""
    a = np.maximum(np.asarray(amax, np.float32), np.float32(1e-12)).astype(np.float64)
    return (a / MAX_VALUE[fmt]).astype(np.float32)


def codes(x32, s, fmt):
    """FP8 codes of RN32(x / s) with saturation; s broadcasts against x."""
    t = (np.asarray(x32, np.float32).astype(np.float64)
         / np.asarray(s, np.float32).astype(np.float64)).astype(np.float32)
    big = np.abs(t) >= np.float32(MAX_VALUE[fmt])
    c = np.where(big, np.float32(0), t).astype(LIB[fmt]).view(np.uint8)
    sat = (np.uint8(MAX_CODE[fmt]) | (np.signbit(t).astype(np.uint8) << 7)).astype(np.uint8)
    return np.where(big, sat, c)


def inexact_scale_rows(seed, fmt):
    """float32 rows (exact bf16 values) whose scales are not powers of two.

    Row amax values take all 128 bf16 significands at five binary exponents
    (640 rows).  Each row holds its amax once, N(0, amax/3) values, and values
    placed next to the FP8 midpoints of x/s (x = bf16(amax * mid / FP8_MAX)),
    where RN32(x/s) and RN32(x * RN32(1/s)) are most likely to round apart.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    sig = np.arange(128, dtype=np.uint32)
    exps = np.array([-40, -3, 0, 5, 37])
    amax_bits = (((127 + exps[:, None]) << 7) | sig[None, :]).ravel().astype(np.uint32)
    amax = (amax_bits << 16).view(np.float32)
    table = np.arange(256, dtype=np.uint8).view(LIB[fmt]).astype(np.float64)
    pos = np.unique(table[np.isfinite(table) & (table >= 0)])
    pos = pos[pos <= MAX_VALUE[fmt]]
    mids = (pos[1:] + pos[:-1]) / 2
    mids = mids[mids > pos[1]]                      # skip the subnormal corner
    k_rand, k_mid = 512, 64
    rows = []
    for a in amax:
        r = (rng.standard_normal(k_rand) * (float(a) / 3)).astype(np.float32)
        r = np.clip(r, -a, a)
        m = rng.choice(mids, k_mid) * float(a) / MAX_VALUE[fmt] * rng.choice([-1.0, 1.0], k_mid)
        row = np.concatenate([[a], r, m]).astype(np.float32)
        row = row.astype(ml_dtypes.bfloat16).astype(np.float32)
        row = np.clip(row, -a, a)
        rng.shuffle(row)
        rows.append(row)
    return np.stack(rows)
