"""Pins for the oracle's FP8 formats (CPU).

The decode tables and the RNE+satfinite encoder are checked against things
other than themselves: hand-worked spot values and midpoints (golden file),
and two independent library casts (ml_dtypes and torch's CPU float8 types),
which agree with the encoder wherever neither saturates.
"""
import json
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
from oracle import E4M3, E5M2

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "hand_worked_examples.json")))
LIB = {E4M3: ml_dtypes.float8_e4m3fn, E5M2: ml_dtypes.float8_e5m2}
TORCH = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


def _gold_value(v):
    if v == "nan":
        return math.nan
    if v == "inf":
        return math.inf
    if v == "-inf":
        return -math.inf
    return float(v)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_spot_values(fmt):
    t = oracle.decode_table(fmt)
    for code, v in GOLDEN["fp8_spot_values"][fmt].items():
        want = _gold_value(v)
        got = t[int(code, 16)]
        if math.isnan(want):
            assert math.isnan(got)
        else:
            assert got == want and math.copysign(1, got) == math.copysign(1, want)


def test_max_values():
    assert oracle.fp8_max(E4M3) == 448.0 and oracle.max_code(E4M3) == 0x7E
    assert oracle.fp8_max(E5M2) == 57344.0 and oracle.max_code(E5M2) == 0x7B


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_table_matches_library_decode(fmt):
    codes = np.arange(256, dtype=np.uint8)
    lib = codes.view(LIB[fmt]).astype(np.float64)
    ours = oracle.decode_table(fmt)
    assert np.array_equal(np.isnan(lib), np.isnan(ours))
    m = ~np.isnan(lib)
    assert np.array_equal(lib[m], ours[m])
    assert np.array_equal(np.signbit(lib[m]), np.signbit(ours[m]))


def _all_finite_bf16_as_f32():
    bits = np.arange(1 << 16, dtype=np.uint32) << 16
    v = bits.view(np.float32)
    return v[np.isfinite(v)]


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encode_matches_libraries_in_range(fmt):
    """Below FP8_MAX the library casts are RNE too: all must agree bitwise."""
    rng = np.random.Generator(np.random.PCG64(7))
    mx = oracle.fp8_max(fmt)
    pool = [_all_finite_bf16_as_f32(),
            (rng.standard_normal(200_000) * 30).astype(np.float32),
            (rng.standard_normal(200_000) * 1e-3).astype(np.float32),
            rng.uniform(-mx, mx, 200_000).astype(np.float32)]
    t = np.concatenate(pool)
    t = t[np.abs(t) < mx]
    ours = oracle.encode_rne_sat(t, fmt)
    lib = t.astype(LIB[fmt]).view(np.uint8)
    assert np.array_equal(ours, lib)
    tor = torch.from_numpy(t).to(TORCH[fmt]).view(torch.uint8).numpy()
    assert np.array_equal(ours, tor)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_midpoints_and_saturation(fmt):
    for v, code in GOLDEN["rne_midpoints"][fmt]:
        got = oracle.encode_rne_sat(np.array([v], dtype=np.float32), fmt)[0]
        assert got == int(code, 16), (fmt, v, hex(got), code)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_saturation_all_large(fmt):
    mx = oracle.fp8_max(fmt)
    t = np.array([mx, np.nextafter(np.float32(mx), np.float32(np.inf)), 1e20, np.inf,
                  -mx, -1e20, -np.inf], dtype=np.float32)
    top = oracle.max_code(fmt)
    got = oracle.encode_rne_sat(t, fmt)
    assert list(got) == [top, top, top, top, top | 0x80, top | 0x80, top | 0x80]


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_signed_zero(fmt):
    t = np.array([0.0, -0.0, 1e-30, -1e-30], dtype=np.float32)
    assert list(oracle.encode_rne_sat(t, fmt)) == [0x00, 0x80, 0x00, 0x80]


def test_nan_rejected():
    with pytest.raises(ValueError):
        oracle.encode_rne_sat(np.array([np.nan], dtype=np.float32), E4M3)


def test_bf16_rounding_examples():
    g = GOLDEN["dot_product_e4m3"]
    assert oracle.round_to_bf16(np.array([g["y_exact"]]))[0] == g["y_bf16"]
    # against torch's float64 -> bfloat16 cast (one rounding) on random values
    rng = np.random.Generator(np.random.PCG64(3))
    y = rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))
    ours = oracle.round_to_bf16(y)
    lib = torch.from_numpy(y).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, lib)
