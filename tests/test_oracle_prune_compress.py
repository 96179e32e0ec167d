"""Pins for the oracle's 2:4 prune and compress (CPU).

* brute force over every 4-tuple of a 12-code set (20 736 groups), against an
  independent selection (a stable sort by decreasing magnitude, magnitudes
  decoded by ml_dtypes rather than by the oracle's table);
* the hand-worked groups (golden file);
* invariants: two kept indices per group, ascending; decompress inverts
  compress on a pruned weight; compress is idempotent; a -0.0 swapped for
  +0.0 changes nothing.
"""
import itertools
import json
import os

import ml_dtypes
import numpy as np
import pytest

import oracle
from oracle import E4M3, E5M2

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "hand_worked_examples.json")))
# zeros of both signs, the smallest subnormals, +-1, +-2 (e4m3) / +-2, +-max,
# and two neighbouring codes
CODES = {E4M3: [0x00, 0x80, 0x01, 0x81, 0x38, 0xB8, 0x40, 0xC0, 0x7E, 0xFE, 0x45, 0x44],
         E5M2: [0x00, 0x80, 0x01, 0x81, 0x3C, 0xBC, 0x40, 0xC0, 0x7B, 0xFB, 0x45, 0x44]}
LIB = {E4M3: ml_dtypes.float8_e4m3fn, E5M2: ml_dtypes.float8_e5m2}


def _select_by_sort(mags):
    order = sorted(range(4), key=lambda j: (-mags[j], j))
    return sorted(order[:2])


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_compress_brute_force(fmt):
    groups = np.array(list(itertools.product(CODES[fmt], repeat=4)), dtype=np.uint8)
    q = groups.reshape(-1, 4)           # one group per row, K = 4
    vals, nib = oracle.compress_24(q, fmt)
    lib_mag = np.abs(groups.view(LIB[fmt]).astype(np.float64))
    for r in range(groups.shape[0]):
        i0, i1 = _select_by_sort(list(lib_mag[r]))
        assert nib[r, 0] == (i0 | (i1 << 2))
        assert vals[r, 0] == groups[r, i0] and vals[r, 1] == groups[r, i1]


def test_compress_hand_worked():
    for g in GOLDEN["compress_groups_e4m3"]:
        q = np.array([[int(c, 16) for c in g["codes"]]], dtype=np.uint8)
        vals, nib = oracle.compress_24(q, E4M3)
        assert nib[0, 0] == int(g["nibble"], 16)
        assert list(vals[0]) == [int(v, 16) for v in g["vals"]]
        i0, i1 = g["kept"]
        assert int(g["nibble"], 16) == i0 | (i1 << 2)


def test_nibble_set():
    assert oracle.NIBBLES_VALID == (0x4, 0x8, 0x9, 0xC, 0xD, 0xE)


def test_prune_brute_force():
    mags = [0.0, -0.0, 1.0, -1.0, 2.0, -2.0, 0.5, 3.0e-40]
    groups = np.array(list(itertools.product(mags, repeat=4)), dtype=np.float32)
    out = oracle.prune_24(groups.reshape(-1, 4))
    for r in range(groups.shape[0]):
        keep = _select_by_sort([abs(float(v)) for v in groups[r]])
        for j in range(4):
            if j in keep:
                assert out[r, j].view(np.uint32) == groups[r, j].view(np.uint32)
            else:
                assert out[r, j].view(np.uint32) == 0


def _random_weight(seed, n, k, negzero=0.05):
    rng = np.random.Generator(np.random.PCG64(seed))
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    w[rng.random((n, k)) < negzero] = -0.0
    return w


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_pipeline_invariants(fmt):
    w = _random_weight(3, 96, 256)
    wp = oracle.prune_24(w)
    g = wp.reshape(96, 64, 4)
    assert np.all((g != 0).sum(axis=-1) <= 2)
    q, s = oracle.quantize_rowwise(wp, fmt)
    vals, nib = oracle.compress_24(q, fmt)
    assert np.all(np.isin(nib, oracle.NIBBLES_VALID))
    back = oracle.decompress_24(vals, nib, 256)
    # by value, decompress(compress(q)) == q (dropped slots of q are zeros)
    assert np.array_equal(oracle.decode(back, fmt), oracle.decode(q, fmt) * 1.0 + 0.0)
    kept_back = back.reshape(96, 64, 4)
    qq = q.reshape(96, 64, 4)
    i0 = (nib & 3).astype(np.int64)
    i1 = (nib >> 2).astype(np.int64)
    for idx in (i0, i1):   # bitwise on kept slots
        assert np.array_equal(np.take_along_axis(kept_back, idx[..., None], -1),
                              np.take_along_axis(qq, idx[..., None], -1))
    # idempotent
    v2, n2 = oracle.compress_24(back, fmt)
    assert np.array_equal(v2, vals) and np.array_equal(n2, nib)
    # -0.0 -> +0.0 swap leaves the metadata unchanged
    q_pos = np.where(q == 0x80, np.uint8(0), q)
    v3, n3 = oracle.compress_24(q_pos, fmt)
    assert np.array_equal(n3, nib)


def test_layout_unpacker_against_loop_packer():
    """Pack by explicit loops from the layout's byte formula, then unpack."""
    n, k = 130, 256
    rng = np.random.Generator(np.random.PCG64(9))
    vals = rng.integers(0, 256, (n, k // 2), dtype=np.uint8)
    nib = rng.choice(np.array(oracle.NIBBLES_VALID, dtype=np.uint8), (n, k // 4))
    npad = oracle.padded_rows(n)
    assert npad == 256
    phys = np.zeros(npad * k * 5 // 8, dtype=np.uint8)
    assert phys.size == oracle.packed_bytes(n, k)
    for row in range(npad):
        nt, r = divmod(row, 128)
        for j in range(k // 2):
            kt, jj = divmod(j, 64)          # 64 value bytes per 128-wide K step
            c, b = divmod(jj, 16)           # 16-byte chunk c, byte b
            pos = c ^ ((r >> 1) & 3)
            byte = (nt * (k // 128) + kt) * 10240 + 64 * r + 16 * pos + b
            phys[byte] = vals[row, j] if row < n else 0
        for grp in range(k // 4):
            v = nib[row, grp] if row < n else 0x4
            kt, gg = divmod(grp, 32)
            byte = (nt * (k // 128) + kt) * 10240 + 8192 + 16 * r + gg // 2
            phys[byte] |= v << (4 * (gg % 2))
    v_out, n_out = oracle.unpack_physical(phys, n, k)
    assert np.array_equal(v_out, vals) and np.array_equal(n_out, nib)
    v_all, n_all = oracle.unpack_physical(phys, n, k, include_padding=True)
    assert np.all(v_all[n:] == 0) and np.all(n_all[n:] == 0x4)
