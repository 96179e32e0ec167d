"""Pins for the oracle's tensor-wise quantiser (CPU).

* the hand-worked row of the golden file, laid out as a 2 x 4 tensor, in both
  formats (its amax 14 gives s = 2^-5 / 2^-12 exactly);
* every finite bf16 value with |x| <= FP8_MAX in one tensor whose amax is
  FP8_MAX: s == 1 and each code must equal an independent library cast of x;
* one global amax, not one per row: a tensor whose rows have different amax
  values quantises with the largest, and its scale is the same as that of
  the row-wise quantiser on the flattened tensor (one row);
* scaling by a power of two leaves the codes and scales the scale; the zero
  tensor takes the guard scale and keeps the signs of its zeros.
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
def test_hand_worked_tensor(fmt):
    row = GOLDEN["activation_row"]
    bits = np.array([int(b, 16) for b in row["x_bf16_bits"]], dtype=np.uint16)
    x = oracle.bf16_bits_to_f32(bits).reshape(2, 4)
    q, s = oracle.quantize_tensorwise(x, fmt)
    assert s == np.float32(row[fmt]["scale"])
    assert q.shape == (2, 4)
    assert [int(c) for c in q.ravel()] == [int(c, 16) for c in row[fmt]["codes"]]


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_exhaustive_bf16_unit_scale(fmt):
    mx = np.float32(oracle.fp8_max(fmt))
    v = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) <= mx)]
    x = np.concatenate([[mx], v]).astype(np.float32)
    q, s = oracle.quantize_tensorwise(x, fmt)
    assert s == np.float32(1.0)
    assert np.array_equal(q[1:], v.astype(LIB[fmt]).view(np.uint8))


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_one_global_amax(fmt):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((6, 40)).astype(np.float32)
    x *= np.float32(2.0) ** np.arange(6, dtype=np.float32)[:, None]   # rows of growing amax
    q, s = oracle.quantize_tensorwise(x, fmt)
    amax = np.max(np.abs(x))
    assert s == np.float32(amax / np.float32(oracle.fp8_max(fmt)))
    q_row, s_row = oracle.quantize_rowwise(x.reshape(1, -1), fmt)
    assert s_row[0] == s and np.array_equal(q_row.reshape(x.shape), q)
    # the per-row quantiser differs on every row but the largest
    q_each, s_each = oracle.quantize_rowwise(x, fmt)
    assert len(set(s_each.tolist())) == 6
    for r in range(5):
        assert not np.array_equal(q_each[r], q[r])


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_power_of_two_scaling(fmt):
    rng = np.random.default_rng(4)
    x = (rng.standard_t(3, size=(17, 33))).astype(np.float32)
    q, s = oracle.quantize_tensorwise(x, fmt)
    for e in (-20, -3, 5, 30):
        q2, s2 = oracle.quantize_tensorwise(x * np.float32(2.0 ** e), fmt)
        assert np.array_equal(q2, q) and s2 == s * np.float32(2.0 ** e)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_zero_tensor_and_empty(fmt):
    x = np.zeros((4, 8), np.float32)
    x[1, 2] = -0.0
    q, s = oracle.quantize_tensorwise(x, fmt)
    assert s == np.float32(np.float32(1e-12) / np.float32(oracle.fp8_max(fmt)))
    assert q[1, 2] == 0x80 and np.count_nonzero(q) == 1
    q0, s0 = oracle.quantize_tensorwise(np.zeros((0,), np.float32), fmt)
    assert q0.size == 0 and s0 == s


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_quotient_is_one_float32_division(fmt):
    """Each tensor of a family with inexact scales quantises to RN_sat(RN32(x / s))
    computed without the oracle (float64 quotient rounded once, library cast)."""
    rows = quotient_pin.inexact_scale_rows(22, fmt)
    moved = 0
    for x in rows[::5]:
        q, s = oracle.quantize_tensorwise(x, fmt)
        s_ind = quotient_pin.scale(np.abs(x).max(), fmt)
        assert np.float32(s).view(np.uint32) == s_ind.view(np.uint32)
        assert np.array_equal(q, quotient_pin.codes(x, s_ind, fmt))
        t_mul = (x * (np.float32(1.0) / s_ind).astype(np.float32)).astype(np.float32)
        moved += np.count_nonzero(quotient_pin.codes(t_mul, np.float32(1.0), fmt) != q)
    assert moved > 0
