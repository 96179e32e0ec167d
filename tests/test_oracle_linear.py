"""Pins for the oracle's linear (CPU).

* the hand-worked dot product (golden file): 261.25, which rounds to 262 in
  bf16;
* exact rational arithmetic (Python Fractions, operands decoded by ml_dtypes)
  on the tiny workload's shape, with explicit loops over the kept slots only;
* scale linearity, bias, and the acceptance bound's behaviour.
"""
import json
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

import oracle
from oracle import E4M3, E5M2
from semi_structured_sparse_rowwise_b200 import synthetic

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "hand_worked_examples.json")))
LIB = {E4M3: ml_dtypes.float8_e4m3fn, E5M2: ml_dtypes.float8_e5m2}


def test_hand_worked_dot_product():
    g = GOLDEN["dot_product_e4m3"]
    a = np.array([[int(c, 16) for c in g["a_codes"]]], dtype=np.uint8)
    w_dense = np.array(g["w_dense_values"])
    # the weight row's values are e4m3-representable: encode them as they are
    wq = oracle.encode_rne_sat(w_dense.astype(np.float32)[None, :], E4M3)
    vals, nib = oracle.compress_24(wq, E4M3)
    y, absdot, scale = oracle.sparse_linear_ref(
        a, E4M3, np.array([g["s_a"]], np.float32), vals, nib, E4M3,
        np.array([g["s_w"]], np.float32))
    assert y[0, 0] == g["y_exact"]
    assert y[0, 0] / scale[0, 0] == g["sum_products"]
    assert oracle.round_to_bf16(y)[0, 0] == g["y_bf16"]


def _fraction_linear(a_q, a_fmt, s_a, vals, nib, w_fmt, s_w, bias):
    a_dec = a_q.view(LIB[a_fmt])
    v_dec = vals.view(LIB[w_fmt])
    m, k = a_q.shape
    n = vals.shape[0]
    out = [[None] * n for _ in range(m)]
    for i in range(m):
        for j in range(n):
            acc = Fraction(0)
            for g in range(k // 4):
                code = int(nib[j, g])
                i0, i1 = code & 3, code >> 2
                acc += Fraction(float(a_dec[i, 4 * g + i0])) * Fraction(float(v_dec[j, 2 * g]))
                acc += Fraction(float(a_dec[i, 4 * g + i1])) * Fraction(float(v_dec[j, 2 * g + 1]))
            y = acc * Fraction(float(s_a[i])) * Fraction(float(s_w[j]))
            if bias is not None:
                y += Fraction(float(bias[j]))
            out[i][j] = (acc, y)
    return out


@pytest.mark.parametrize("fmts", [(E4M3, E4M3), (E5M2, E4M3), (E4M3, E5M2), (E5M2, E5M2)])
def test_exact_rational_tiny(fmts):
    a_fmt, w_fmt = fmts
    x_bits, w_bits, _, _ = synthetic.workload_inputs("tiny")
    b_bits = synthetic.bias(77, 64)
    x = oracle.bf16_bits_to_f32(x_bits)
    w = oracle.prune_24(oracle.bf16_bits_to_f32(w_bits))
    a_q, s_a = oracle.quantize_rowwise(x, a_fmt)
    w_q, s_w = oracle.quantize_rowwise(w, w_fmt)
    vals, nib = oracle.compress_24(w_q, w_fmt)
    bias = oracle.bf16_bits_to_f32(b_bits)
    y, absdot, scale = oracle.sparse_linear_ref(a_q, a_fmt, s_a, vals, nib, w_fmt, s_w, bias)
    exact = _fraction_linear(a_q, a_fmt, s_a, vals, nib, w_fmt, s_w, bias)
    for i in range(y.shape[0]):
        for j in range(y.shape[1]):
            acc, ye = exact[i][j]
            # the fp64 value is the exact rational up to the roundings of the
            # scale product and the bias addition (a few fp64 ulps)
            tol = (abs(acc * Fraction(float(s_a[i])) * Fraction(float(s_w[j]))) + abs(ye)) * Fraction(1, 2 ** 50)
            assert abs(Fraction(float(y[i, j])) - ye) <= tol


def test_e4m3_accumulator_exact():
    x_bits, w_bits, _, _ = synthetic.workload_inputs("tiny")
    x = oracle.bf16_bits_to_f32(x_bits)
    w = oracle.prune_24(oracle.bf16_bits_to_f32(w_bits))
    a_q, s_a = oracle.quantize_rowwise(x, E4M3)
    w_q, s_w = oracle.quantize_rowwise(w, E4M3)
    vals, nib = oracle.compress_24(w_q, E4M3)
    ones = np.ones_like(s_a)
    y, _, _ = oracle.sparse_linear_ref(a_q, E4M3, ones, vals, nib, E4M3, np.ones_like(s_w))
    exact = _fraction_linear(a_q, E4M3, ones, vals, nib, E4M3, np.ones_like(s_w), None)
    for i in range(y.shape[0]):
        for j in range(y.shape[1]):
            assert Fraction(float(y[i, j])) == exact[i][j][0]


def test_scale_linearity_and_bias():
    x_bits, w_bits, _, _ = synthetic.workload_inputs("tiny")
    x = oracle.bf16_bits_to_f32(x_bits)
    w = oracle.prune_24(oracle.bf16_bits_to_f32(w_bits))
    a_q, s_a = oracle.quantize_rowwise(x, E4M3)
    w_q, s_w = oracle.quantize_rowwise(w, E4M3)
    vals, nib = oracle.compress_24(w_q, E4M3)
    y1, _, _ = oracle.sparse_linear_ref(a_q, E4M3, s_a, vals, nib, E4M3, s_w)
    y2, _, _ = oracle.sparse_linear_ref(a_q, E4M3, s_a, vals, nib, E4M3, s_w * np.float32(2))
    assert np.array_equal(y2, 2 * y1)
    b = np.linspace(-1, 1, 64)
    y3, _, _ = oracle.sparse_linear_ref(a_q, E4M3, s_a, vals, nib, E4M3, s_w, b)
    assert np.array_equal(y3, y1 + b[None, :])
    # sampled rows/cols agree with the full result
    y4, _, _ = oracle.sparse_linear_ref(a_q, E4M3, s_a, vals, nib, E4M3, s_w,
                                        rows=[3, 0, 15], cols=[63, 1])
    assert np.array_equal(y4, y1[[3, 0, 15]][:, [63, 1]])


def test_acceptance_bound():
    x_bits, w_bits, _, _ = synthetic.workload_inputs("tiny")
    x = oracle.bf16_bits_to_f32(x_bits)
    w = oracle.prune_24(oracle.bf16_bits_to_f32(w_bits))
    a_q, s_a = oracle.quantize_rowwise(x, E4M3)
    w_q, s_w = oracle.quantize_rowwise(w, E4M3)
    vals, nib = oracle.compress_24(w_q, E4M3)
    y, absdot, scale = oracle.sparse_linear_ref(a_q, E4M3, s_a, vals, nib, E4M3, s_w)
    assert oracle.check_linear(y, y, absdot, scale)[0]
    assert oracle.check_linear(oracle.round_to_bf16(y), y, absdot, scale)[0]
    bad = y.copy()
    bad[2, 7] += 0.05 * abs(y[2, 7]) + 0.05 * scale[2, 7] * absdot[2, 7]
    assert not oracle.check_linear(bad, y, absdot, scale)[0]
    nan = y.copy()
    nan[0, 0] = np.nan
    assert not oracle.check_linear(nan, y, absdot, scale)[0]
