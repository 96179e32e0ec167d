"""Pins for the oracle's row-wise quantiser (CPU).

* the hand-worked row (golden file) in both formats;
* an exhaustive sweep: every finite bf16 value with |x| <= FP8_MAX, placed in
  rows whose amax is FP8_MAX, so that s == 1 exactly and each code must equal
  an independent library cast of x itself;
* the all-zero row, saturation, and the error bound of the round trip.
"""
import json
import os

import ml_dtypes
import numpy as np
import pytest

import oracle
import quotient_pin
from oracle import E4M3, E5M2

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "hand_worked_examples.json")))
LIB = {E4M3: ml_dtypes.float8_e4m3fn, E5M2: ml_dtypes.float8_e5m2}


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_hand_worked_row(fmt):
    row = GOLDEN["activation_row"]
    bits = np.array([int(b, 16) for b in row["x_bf16_bits"]], dtype=np.uint16)
    x = oracle.bf16_bits_to_f32(bits)[None, :]
    q, s = oracle.quantize_rowwise(x, fmt)
    want = [int(c, 16) for c in row[fmt]["codes"]]
    assert s[0] == np.float32(row[fmt]["scale"])
    assert list(q[0]) == want
    dec = oracle.decode(q[0], fmt)
    assert np.array_equal(dec, np.array(row[fmt]["decoded"]))
    assert np.array_equal(np.signbit(dec), np.signbit(np.array(row[fmt]["decoded"])))


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_exhaustive_bf16_unit_scale(fmt):
    mx = np.float32(oracle.fp8_max(fmt))
    v = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) <= mx)]
    width = 256
    pad = (-v.size) % (width - 1)
    v = np.concatenate([v, np.zeros(pad, dtype=np.float32)])
    body = v.reshape(-1, width - 1)
    x = np.concatenate([np.full((body.shape[0], 1), mx, dtype=np.float32), body], axis=1)
    q, s = oracle.quantize_rowwise(x, fmt)
    assert np.all(s == np.float32(1.0))
    lib = body.astype(LIB[fmt]).view(np.uint8)
    # |x| == FP8_MAX casts exactly in the library as well
    assert np.array_equal(q[:, 1:], lib)
    assert np.all(q[:, 0] == oracle.max_code(fmt))


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_zero_row_guard(fmt):
    x = np.zeros((3, 64), dtype=np.float32)
    x[1, 5] = -0.0
    x[2, :] = -0.0
    q, s = oracle.quantize_rowwise(x, fmt)
    mx = oracle.fp8_max(fmt)
    for si in s:
        assert si > 0 and np.isfinite(si)
        assert abs(float(si) * mx - 1e-12) <= 1e-12 * 2.0 ** -22   # s = 1e-12 / max
        assert si >= np.finfo(np.float32).tiny                     # normal
    assert np.all(q[0] == 0x00)
    assert q[1, 5] == 0x80 and np.all(np.delete(q[1], 5) == 0x00)
    assert np.all(q[2] == 0x80)


def test_empty_k():
    q, s = oracle.quantize_rowwise(np.zeros((4, 0), dtype=np.float32), E4M3)
    assert q.shape == (4, 0) and np.all(s == np.float32(1e-12) / np.float32(448))


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_roundtrip_error_bound(fmt):
    """|dec(q)*s - x| <= (half the FP8 spacing at x/s) * s, plus fp32 slack."""
    rng = np.random.Generator(np.random.PCG64(11))
    x = (rng.standard_t(3, size=(64, 512)) * np.exp(rng.uniform(-8, 8, (64, 1)))).astype(np.float32)
    q, s = oracle.quantize_rowwise(x, fmt)
    dec = oracle.decode(q, fmt)
    mx = oracle.fp8_max(fmt)
    assert np.all(np.abs(dec) <= mx)
    t = np.abs(x.astype(np.float64) / s[:, None].astype(np.float64))
    table = oracle.decode_table(fmt)
    pos = np.sort(table[: oracle.max_code(fmt) + 1])
    # local spacing: distance between the two codes around t
    hi = np.clip(np.searchsorted(pos, t), 1, pos.size - 1)
    spacing = pos[hi] - pos[hi - 1]
    err = np.abs(np.abs(dec) - t)
    assert np.all(err <= 0.5 * spacing * (1 + 1e-6) + 1e-6 * t)
    assert np.all(np.abs(dec).max(axis=1) >= mx * (1 - 2.0 ** -3))   # amax maps near max


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_scale_is_ieee_float32_division(fmt):
    """s equals the correctly rounded quotient amax / max (checked in fp64)."""
    rng = np.random.Generator(np.random.PCG64(5))
    x = rng.standard_normal((2000, 33)).astype(np.float32)
    _, s = oracle.quantize_rowwise(x, fmt)
    amax = np.abs(x).max(axis=1).astype(np.float64)
    exact = amax / oracle.fp8_max(fmt)            # exact enough in fp64
    lo = np.nextafter(s, np.float32(-np.inf)).astype(np.float64)
    hi = np.nextafter(s, np.float32(np.inf)).astype(np.float64)
    sd = s.astype(np.float64)
    # s is the float32 nearest to the exact quotient
    assert np.all(np.abs(sd - exact) <= np.minimum(np.abs(lo - exact), np.abs(hi - exact)))


def test_inexact_scale_hand_worked_row():
    """A row with an inexact scale where RN32(x/s) sits on an e4m3 midpoint and
    ties to the even code, while x * RN32(1/s) would round past it (golden
    file, worked by hand with integer arithmetic)."""
    row = GOLDEN["inexact_scale_row_e4m3"]
    bits = np.array([int(b, 16) for b in row["x_bf16_bits"]], dtype=np.uint16)
    x = oracle.bf16_bits_to_f32(bits)[None, :]
    q, s = oracle.quantize_rowwise(x, E4M3)
    assert s.view(np.uint32)[0] == int(row["scale_bits"], 16)
    assert s[0] == np.float32(row["scale"])
    assert [int(c) for c in q[0]] == [int(c, 16) for c in row["codes"]]
    assert np.array_equal(oracle.decode(q[0], E4M3), np.array(row["decoded"]))
    assert row["codes"] != row["codes_if_multiplied_by_reciprocal"]


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_quotient_is_one_float32_division(fmt):
    """Codes equal RN_sat(RN32(x / s)) computed without the oracle (float64
    quotient rounded once to float32, library cast) on 640 rows whose scales
    are not powers of two, with values placed beside the FP8 midpoints."""
    x = quotient_pin.inexact_scale_rows(21, fmt)
    q, s = oracle.quantize_rowwise(x, fmt)
    s_ind = quotient_pin.scale(np.abs(x).max(axis=1), fmt)
    assert np.array_equal(s.view(np.uint32), s_ind.view(np.uint32))
    assert np.array_equal(q, quotient_pin.codes(x, s_ind[:, None], fmt))
    # the rows do separate the two readings: multiplying by RN32(1/s) moves codes
    r = (np.float32(1.0) / s_ind).astype(np.float32)
    t_mul = (x * r[:, None]).astype(np.float32)
    q_mul = quotient_pin.codes(t_mul, np.float32(1.0), fmt)
    assert np.count_nonzero(q_mul != q) > 0
