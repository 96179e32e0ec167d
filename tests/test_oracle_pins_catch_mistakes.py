"""The pins are sharp: plausible mistakes planted in the oracle (on the CPU,
never in the CUDA path) make at least one pin fail.

Each case swaps one oracle function for a mutated copy and checks that the
corresponding pin would reject it.
"""
import itertools
import json
import os

import ml_dtypes
import numpy as np

import oracle
import quotient_pin
from oracle import E4M3
from oracle import prune as prune_mod

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "hand_worked_examples.json")))


def _midpoint_pin(encode):
    return all(encode(np.array([v], np.float32), E4M3)[0] == int(c, 16)
               for v, c in GOLDEN["rne_midpoints"][E4M3])


def test_ties_away_from_zero_is_caught():
    def encode_ties_away(t, fmt):
        table = oracle.decode_table(fmt)
        top = oracle.max_code(fmt)
        pos = table[: top + 1]
        a = np.abs(t.astype(np.float64))
        hi = np.minimum(np.searchsorted(pos, a), top)
        lo = np.maximum(hi - 1, 0)
        mag = np.where(pos[hi] - a <= a - pos[lo], hi, lo)   # ties go up
        mag = np.where(a >= pos[top], top, mag)
        return (mag | (np.signbit(t).astype(np.int64) << 7)).astype(np.uint8)
    assert _midpoint_pin(oracle.encode_rne_sat)
    assert not _midpoint_pin(encode_ties_away)


def test_nonsaturating_cast_is_caught():
    def encode_lib(t, fmt):
        return np.asarray(t, np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert not _midpoint_pin(encode_lib)      # 1000 -> NaN instead of 448


def _brute_force_compress_pin(compress):
    codes = [0x00, 0x80, 0x01, 0x81, 0x38, 0xB8, 0x40, 0xC0]
    groups = np.array(list(itertools.product(codes, repeat=4)), dtype=np.uint8)
    vals, nib = compress(groups, E4M3)
    mags = np.abs(groups.view(ml_dtypes.float8_e4m3fn).astype(np.float64))
    for r in range(groups.shape[0]):
        order = sorted(range(4), key=lambda j: (-mags[r, j], j))
        i0, i1 = sorted(order[:2])
        if nib[r, 0] != (i0 | (i1 << 2)):
            return False
    return True


def test_tie_to_higher_index_is_caught(monkeypatch):
    assert _brute_force_compress_pin(oracle.compress_24)

    def ranks_high(mag):
        r = np.zeros(mag.shape, dtype=np.int64)
        for j in range(4):
            for i in range(4):
                if i != j:
                    r[..., j] += (mag[..., i] > mag[..., j])
                    if i > j:
                        r[..., j] += (mag[..., i] == mag[..., j])
        return r
    import oracle.compress as comp
    monkeypatch.setattr(comp, "group_ranks", ranks_high)
    assert not _brute_force_compress_pin(comp.compress_24)


def test_negative_zero_ranked_by_code_is_caught(monkeypatch):
    import oracle.compress as comp
    real_decode = comp.decode
    # a mistake: rank by the raw byte, so 0x80 (-0.0) looks large
    monkeypatch.setattr(comp, "decode", lambda codes, fmt: np.asarray(codes, np.float64))
    assert not _brute_force_compress_pin(comp.compress_24)
    monkeypatch.setattr(comp, "decode", real_decode)


def test_swapped_nibble_fields_are_caught():
    g = GOLDEN["compress_groups_e4m3"][1]
    q = np.array([[int(c, 16) for c in g["codes"]]], dtype=np.uint8)
    vals, nib = oracle.compress_24(q, E4M3)
    swapped = ((nib & 3) << 2) | (nib >> 2)
    assert nib[0, 0] == int(g["nibble"], 16)
    assert swapped[0, 0] != int(g["nibble"], 16)


def test_dropped_term_in_linear_is_caught():
    g = GOLDEN["dot_product_e4m3"]
    a = np.array([[int(c, 16) for c in g["a_codes"]]], dtype=np.uint8)
    wq = oracle.encode_rne_sat(np.array(g["w_dense_values"], np.float32)[None, :], E4M3)
    vals, nib = oracle.compress_24(wq, E4M3)
    s = np.array([g["s_a"]], np.float32)
    y, _, _ = oracle.sparse_linear_ref(a, E4M3, s, vals, nib, E4M3, s)
    assert y[0, 0] == g["y_exact"]
    # drop the second kept slot of every group
    vals_half = vals.copy()
    vals_half[:, 1::2] = 0
    y2, _, _ = oracle.sparse_linear_ref(a, E4M3, s, vals_half, nib, E4M3, s)
    assert y2[0, 0] != g["y_exact"]
    # transposed scales (s_w applied per row m) on a 2x2 case change the result
    a2 = np.vstack([a, a])
    vals2, nib2 = np.vstack([vals, vals]), np.vstack([nib, nib])
    sa2 = np.array([1.0, 2.0], np.float32)
    sw2 = np.array([1.0, 4.0], np.float32)
    y_ok, _, _ = oracle.sparse_linear_ref(a2, E4M3, sa2, vals2, nib2, E4M3, sw2)
    y_tr, _, _ = oracle.sparse_linear_ref(a2, E4M3, sw2, vals2, nib2, E4M3, sa2)
    assert not np.array_equal(y_ok, y_tr.T) or not np.array_equal(y_ok, y_tr)


def _prune_pin(prune):
    vals = [0.0, -0.0, 1.0, -1.0, 2.0, 0.5]
    groups = np.array(list(itertools.product(vals, repeat=4)), dtype=np.float32)
    out = prune(groups)
    for r in range(groups.shape[0]):
        order = sorted(range(4), key=lambda j: (-abs(float(groups[r, j])), j))
        keep = set(order[:2])
        for j in range(4):
            want = groups[r, j] if j in keep else np.float32(0.0)
            if out[r, j].view(np.uint32) != np.float32(want).view(np.uint32):
                return False
    return True


def test_prune_mistakes_are_caught(monkeypatch):
    assert _prune_pin(oracle.prune_24)
    real = prune_mod.group_ranks
    monkeypatch.setattr(prune_mod, "group_ranks", lambda m: 3 - real(m))   # keeps the smallest
    assert not _prune_pin(prune_mod.prune_24)
    monkeypatch.setattr(prune_mod, "group_ranks", real)
    # dropped entries written as -0.0 instead of +0.0
    monkeypatch.setattr(prune_mod, "prune_24", lambda w: np.where(
        real(np.abs(w.reshape(-1, 1, 4)).astype(np.float64)).reshape(w.shape) < 2, w, np.float32(-0.0)))
    assert not _prune_pin(prune_mod.prune_24)


def _global_amax_pin(quantize_tensorwise):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((6, 40)).astype(np.float32)
    x *= np.float32(2.0) ** np.arange(6, dtype=np.float32)[:, None]
    q, s = quantize_tensorwise(x, E4M3)
    return (np.size(s) == 1 and np.float32(s) == np.float32(np.max(np.abs(x)) / np.float32(448.0))
            and np.array_equal(q, oracle.quantize_rowwise(x.reshape(1, -1), E4M3)[0].reshape(x.shape)))


def test_tensorwise_mistakes_are_caught():
    def per_block_amax(x, fmt):          # each block (row) scaled by its own amax
        q, s = oracle.quantize_rowwise(np.asarray(x, np.float32), fmt)
        return q, s

    def last_block_amax(x, fmt):         # a race: the amax read before the last block folded in
        x = np.asarray(x, np.float32)
        amax = np.float32(np.max(np.abs(x[:-1])))
        s = np.float32(amax / np.float32(oracle.fp8_max(fmt)))
        return oracle.encode_rne_sat((x / s).astype(np.float32), fmt), s

    assert _global_amax_pin(oracle.quantize_tensorwise)
    assert not _global_amax_pin(per_block_amax)
    assert not _global_amax_pin(last_block_amax)


def _quotient_pins(quantize_rowwise, quantize_tensorwise):
    """The two quotient pins: the hand-worked inexact-scale row, and codes equal
    to RN_sat(RN32(x / s)) computed without the oracle on inexact-scale rows."""
    row = GOLDEN["inexact_scale_row_e4m3"]
    x = np.array(row["x_bf16_values"], np.float32)[None, :]
    q, _ = quantize_rowwise(x, E4M3)
    golden_ok = [int(c) for c in q[0]] == [int(c, 16) for c in row["codes"]]
    rows = quotient_pin.inexact_scale_rows(23, E4M3)[:128]
    q, s = quantize_rowwise(rows, E4M3)
    rowwise_ok = np.array_equal(q, quotient_pin.codes(rows, s[:, None], E4M3))
    tensor_ok = True
    for x1 in rows[::8]:
        q1, s1 = quantize_tensorwise(x1, E4M3)
        tensor_ok &= np.array_equal(q1, quotient_pin.codes(x1, s1, E4M3))
    return golden_ok, rowwise_ok, tensor_ok


def test_multiply_by_reciprocal_is_caught():
    """x * RN32(1/s) instead of the correctly rounded x / s, in either quantiser."""
    def rowwise_recip(x32, fmt):
        x32 = np.asarray(x32, np.float32)
        amax = np.max(np.abs(x32), axis=1).astype(np.float32)
        s = (np.maximum(amax, oracle.GUARD_AMAX) / np.float32(oracle.fp8_max(fmt))).astype(np.float32)
        r = (np.float32(1.0) / s).astype(np.float32)
        return oracle.encode_rne_sat((x32 * r[:, None]).astype(np.float32), fmt), s

    def tensorwise_recip(x32, fmt):
        x32 = np.asarray(x32, np.float32)
        s = np.float32(np.maximum(np.float32(np.max(np.abs(x32))), oracle.GUARD_AMAX)
                       / np.float32(oracle.fp8_max(fmt)))
        return oracle.encode_rne_sat((x32 * np.float32(np.float32(1.0) / s)).astype(np.float32), fmt), s

    assert _quotient_pins(oracle.quantize_rowwise, oracle.quantize_tensorwise) == (True, True, True)
    golden_ok, rowwise_ok, tensor_ok = _quotient_pins(rowwise_recip, tensorwise_recip)
    assert not golden_ok and not rowwise_ok and not tensor_ok


def test_quotient_rounded_straight_from_float64_is_caught():
    """x / s evaluated in float64 and rounded once to FP8 (no float32 quotient)."""
    def rowwise_f64(x32, fmt):
        x32 = np.asarray(x32, np.float32)
        amax = np.max(np.abs(x32), axis=1).astype(np.float32)
        s = (np.maximum(amax, oracle.GUARD_AMAX) / np.float32(oracle.fp8_max(fmt))).astype(np.float32)
        t = x32.astype(np.float64) / s[:, None].astype(np.float64)
        table = oracle.decode_table(fmt)
        top = oracle.max_code(fmt)
        pos = table[: top + 1]
        a = np.abs(t)
        hi = np.minimum(np.searchsorted(pos, a), top)
        lo = np.maximum(hi - 1, 0)
        d_lo, d_hi = a - pos[lo], pos[hi] - a
        mag = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, np.where(lo % 2 == 0, lo, hi)))
        mag = np.where(a >= pos[top], top, mag)
        return (mag | (np.signbit(t).astype(np.int64) << 7)).astype(np.uint8), s

    golden_ok, rowwise_ok, _ = _quotient_pins(rowwise_f64, oracle.quantize_tensorwise)
    assert not golden_ok and not rowwise_ok
