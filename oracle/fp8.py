"""FP8 formats, written out from their bit fields (oracle; test infrastructure).

The two formats that the page "Add CUTLASS-based row-wise scaled sparse FP8
kernel" (pytorch/ao pull request 1671) instantiates its operator for are e4m3
and e5m2 (the four ``..._e4m3e4m3`` ... ``..._e5m2e5m2`` instantiations it
lists, repeated in the file table of issue 3516).  The page relies on their
public definition, the OCP 8-bit floating point specification (OFP8):

* e4m3 ("e4m3fn"): 1 sign, 4 exponent, 3 mantissa bits, bias 7.  Exponent 0
  is subnormal (m * 2^-9).  Exponent 15 with mantissa 7 is NaN; there is no
  infinity, so exponent 15 with mantissa 0..6 is normal.  Max finite 448.
* e5m2: 1 sign, 5 exponent, 2 mantissa bits, bias 15.  Exponent 0 is
  subnormal (m * 2^-16).  Exponent 31 is infinity (mantissa 0) or NaN.  Max
  finite 57344.

The encoder is round-to-nearest, ties to the code with an even mantissa LSB,
with saturation to the largest finite value ("satfinite"), and it keeps the
sign, including the sign of a value that rounds to zero.  Saturation rather
than a NaN/inf on overflow is the reading taken for the NaN outputs that the
same page reports from FP16->FP8 quantisation (its item 2, issue 1766).
"""

import math

import numpy as np

E4M3 = "e4m3"
E5M2 = "e5m2"

# exponent bits, mantissa bits, bias, and how the all-ones exponent is used.
FORMATS = {
    E4M3: {"ebits": 4, "mbits": 3, "bias": 7, "ieee_specials": False},
    E5M2: {"ebits": 5, "mbits": 2, "bias": 15, "ieee_specials": True},
}

_TABLE_CACHE = {}


def _decode_code(code, fmt):
    f = FORMATS[fmt]
    eb, mb, bias = f["ebits"], f["mbits"], f["bias"]
    sign = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> mb) & ((1 << eb) - 1)
    m = code & ((1 << mb) - 1)
    e_all_ones = (1 << eb) - 1
    if f["ieee_specials"]:
        if e == e_all_ones:
            return sign * math.inf if m == 0 else math.nan
    else:
        # e4m3fn: only S.1111.111 is NaN.
        if e == e_all_ones and m == (1 << mb) - 1:
            return math.nan
    if e == 0:
        mag = m * 2.0 ** (1 - bias - mb)
    else:
        mag = (1.0 + m / 2.0 ** mb) * 2.0 ** (e - bias)
    return math.copysign(mag, sign)


def decode_table(fmt):
    """256-entry float64 table: code -> value (NaN where the code is NaN)."""
    if fmt not in _TABLE_CACHE:
        t = np.array([_decode_code(c, fmt) for c in range(256)], dtype=np.float64)
        t.setflags(write=False)
        _TABLE_CACHE[fmt] = t
    return _TABLE_CACHE[fmt]


def decode(codes, fmt):
    """Decode an array of uint8 codes to float64."""
    return decode_table(fmt)[np.asarray(codes, dtype=np.uint8)]


def max_code(fmt):
    """Largest positive finite code (0x7E for e4m3, 0x7B for e5m2)."""
    t = decode_table(fmt)
    best = None
    for c in range(0x80):
        if np.isfinite(t[c]) and (best is None or t[c] > t[best]):
            best = c
    return best


def fp8_max(fmt):
    """Largest finite magnitude (448 for e4m3, 57344 for e5m2)."""
    return float(decode_table(fmt)[max_code(fmt)])


def encode_rne_sat(t, fmt):
    """Encode float32 values to FP8 codes: RNE, satfinite, sign kept.

    For |t| >= max finite the result is the max-finite code of t's sign.
    Otherwise the code whose value is nearest to |t|; when |t| is exactly
    halfway between two neighbouring codes, the one with an even mantissa LSB
    (code & 1 == 0) -- for non-negative codes the value grows with the code,
    so neighbours differ by one and exactly one of them is even.  NaN input is
    outside the contract and raises.
    """
    t = np.asarray(t, dtype=np.float32)
    if np.isnan(t).any():
        raise ValueError("NaN input is outside the quantiser's contract")
    table = decode_table(fmt)
    top = max_code(fmt)
    pos = table[: top + 1]                     # codes 0..top, ascending values
    assert np.all(np.diff(pos) > 0)
    a = np.abs(t.astype(np.float64))           # exact
    hi = np.searchsorted(pos, a, side="left")  # first code with value >= a
    hi_c = np.minimum(hi, top)
    lo_c = np.maximum(hi - 1, 0)
    d_hi = pos[hi_c] - a
    d_lo = a - pos[lo_c]
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((hi_c & 1) == 0))
    mag = np.where(pick_hi, hi_c, lo_c)
    mag = np.where(a >= pos[top], top, mag)    # saturate (covers +inf too)
    mag = np.where(a == pos[hi_c], hi_c, mag)  # exact hit
    sign = np.signbit(t).astype(np.int64) << 7
    return (mag.astype(np.int64) | sign).astype(np.uint8)


def bf16_bits_to_f32(bits):
    """bfloat16 bit patterns (uint16) -> float32 values (exact widening)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def f16_bits_to_f32(bits):
    """IEEE binary16 bit patterns -> float32 values (exact widening)."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float32)


def round_to_bf16(y):
    """Round float64 values to the nearest bfloat16 value, ties to even.

    Written from the bfloat16 definition (8 significand bits, the float32
    exponent range) in one rounding step, so there is no fp64->fp32->bf16
    double rounding.  Returns float64 values that are bf16-representable.
    Subnormal bf16 results use the fixed spacing 2^-133.
    """
    y = np.asarray(y, dtype=np.float64)
    out = np.empty_like(y)
    flat_in = y.reshape(-1)
    flat_out = out.reshape(-1)
    for i, v in enumerate(flat_in):
        if not math.isfinite(v) or v == 0.0:
            flat_out[i] = v
            continue
        _, e = math.frexp(abs(v))          # |v| = f * 2^e, 0.5 <= f < 1
        exp = max(e - 1, -126)             # unbiased exponent of the binade
        spacing = 2.0 ** (exp - 7)         # 8 significant bits
        q = abs(v) / spacing               # exact: power-of-two scaling
        r = round(q)                       # Python round: ties to even
        mag = r * spacing
        if mag > 3.3895313892515355e38:    # beyond max bf16 -> inf
            mag = math.inf
        flat_out[i] = math.copysign(mag, v)
    return out
