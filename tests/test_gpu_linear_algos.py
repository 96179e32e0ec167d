"""GPU parity of every work split ("algorithm") of the sparse linear, and the
shape-keyed table and search that pick one.

Every algorithm offered for a shape -- one-CTA kernel at each tile width,
k steps per stage and whole-tile / stream-K split; CTA-pair kernel at each
tile width, k steps per stage and weight tiles per CTA -- is run on the
same quantised operands and checked against the oracle within the stated
bound |y - y_ref| <= 8e-3 |y_ref| + 1e-3 s_a s_w sum|a w|, on shapes with
ragged token tiles, ragged weight tiles and a single or odd number of k
steps.  Each algorithm is deterministic; the table makes sfp8_sparse_linear
use the chosen algorithm bit for bit, and the search returns the fastest.
"""
import numpy as np
import pytest
import torch

import semi_structured_sparse_rowwise_b200 as S
from semi_structured_sparse_rowwise_b200 import synthetic
from gpu_pipeline import (GpuLayer, RefLayer, bf16_dev, check_output, ensure_library,
                          requires_gpu)

pytestmark = [pytest.mark.gpu, requires_gpu]

# (m, k, n): decode-like, ragged one-CTA shapes, and pair-eligible shapes
# (m >= 256) with ragged token and weight tiles.
SHAPES = [(1, 128, 1), (16, 1024, 520), (40, 512, 300), (129, 640, 200), (300, 1024, 384),
          (700, 384, 390), (1024, 256, 1000)]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_library()


def _status_clean():
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == 0 and flags == 0, (st, flags)


def _operands(m, k, n, seed):
    x = synthetic.activation(seed, m, k, dist="student_t3", zero_row_frac=0.03)
    w = synthetic.weight(seed + 1, n, k, neg_zero_frac=0.02)
    b = synthetic.bias(seed + 2, n)
    gl = GpuLayer(w, "e4m3")
    aq, sa = S.sfp8_quantize_rowwise(bf16_dev(x), "e4m3")
    rl = RefLayer(w, "e4m3")
    rows, aq_r, sa_r = rl.act(x, "e4m3")
    y_ref, absdot, scale = rl.linear(aq_r, "e4m3", sa_r, b)
    return gl, aq, sa, bf16_dev(b), rows, y_ref, absdot, scale


@pytest.mark.parametrize("m,k,n", SHAPES)
def test_every_algorithm_matches_oracle(m, k, n):
    gl, aq, sa, bias, rows, y_ref, absdot, scale = _operands(m, k, n, 12000 + m + k + n)
    count = S.sfp8_sparse_linear_algo_count(m, n, k)
    assert count >= 1
    infos = [S.sfp8_sparse_linear_algo_info(m, n, k, a) for a in range(count)]
    if m >= 256:
        assert any(i["pair"] for i in infos) and any(not i["pair"] for i in infos)
    assert len({tuple(sorted(i.items())) for i in infos}) == count    # no repeats
    for a in range(count):
        y = S.sfp8_sparse_linear_algo(aq, "e4m3", sa, gl.packed, "e4m3", gl.sw, n, k, a,
                                      bias=bias)
        check_output(y, rows, np.arange(n), y_ref, absdot, scale)
        y2 = S.sfp8_sparse_linear_algo(aq, "e4m3", sa, gl.packed, "e4m3", gl.sw, n, k, a,
                                       bias=bias)
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16)), "algo %d %s" % (
            a, infos[a])
    _status_clean()


def test_algorithm_zero_is_the_builtin_rule():
    m, k, n = 40, 512, 300
    gl, aq, sa, bias, *_ = _operands(m, k, n, 12100)
    y0 = S.sfp8_sparse_linear(aq, "e4m3", sa, gl.packed, "e4m3", gl.sw, n, k, bias=bias)
    y1 = S.sfp8_sparse_linear_algo(aq, "e4m3", sa, gl.packed, "e4m3", gl.sw, n, k, 0, bias=bias)
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
    assert (S.sfp8_sparse_linear_workspace_bytes(m, n, k)
            == S.sfp8_sparse_linear_algo_workspace_bytes(m, n, k, 0))
    _status_clean()


@pytest.mark.parametrize("m,k,n", [(40, 512, 300), (700, 384, 390)])
def test_table_and_search(m, k, n):
    gl, aq, sa, bias, rows, y_ref, absdot, scale = _operands(m, k, n, 12200 + m)
    count = S.sfp8_sparse_linear_algo_count(m, n, k)
    best, times = S.sfp8_sparse_linear_search(aq, "e4m3", sa, gl.packed, "e4m3", gl.sw, n, k,
                                              bias=bias, reps=3)
    assert 0 <= best < count and len(times) == count
    assert all(t > 0 for t in times) and times[best] == min(times)
    try:
        # a non-default algorithm through the table: the plain entry point,
        # its workspace query and the one-call forward follow it
        pick = count - 1
        S.sfp8_sparse_linear_set_algo(m, n, k, pick)
        assert S.sfp8_sparse_linear_get_algo(m, n, k) == pick
        assert (S.sfp8_sparse_linear_workspace_bytes(m, n, k)
                == S.sfp8_sparse_linear_algo_workspace_bytes(m, n, k, pick))
        y_tab = S.sfp8_sparse_linear(aq, "e4m3", sa, gl.packed, "e4m3", gl.sw, n, k, bias=bias)
        y_alg = S.sfp8_sparse_linear_algo(aq, "e4m3", sa, gl.packed, "e4m3", gl.sw, n, k, pick,
                                          bias=bias)
        assert torch.equal(y_tab.view(torch.int16), y_alg.view(torch.int16))
        check_output(y_tab, rows, np.arange(n), y_ref, absdot, scale)
        # another shape is not affected
        assert S.sfp8_sparse_linear_get_algo(m + 1, n, k) == 0
    finally:
        S.sfp8_sparse_linear_set_algo(m, n, k, 0)
    assert S.sfp8_sparse_linear_get_algo(m, n, k) == 0
    with pytest.raises(S.Sfp8Error):
        S.sfp8_sparse_linear_set_algo(m, n, k, count)
    _status_clean()


def test_layer_autotune_decode_shape():
    """The layer's autotune on the decode gate/up shape (m=16, k=4096,
    n=14336): it stores the fastest algorithm in the table and the forward
    still matches the oracle on sampled columns."""
    x, w, _, _ = synthetic.workload_inputs("decode_gate_up_8b", 2)
    m, k = x.shape
    n = w.shape[0]
    layer = S.SparseFp8Linear(bf16_dev(w))
    xd = bf16_dev(x)
    try:
        best, times = layer.autotune(xd, reps=3)
        assert S.sfp8_sparse_linear_get_algo(m, n, k) == best
        y = layer(xd)
        cols = np.arange(0, n, 37)
        rl = RefLayer(w, "e4m3", cols)
        rows, aq_r, sa_r = rl.act(x, "e4m3")
        y_ref, absdot, scale = rl.linear(aq_r, "e4m3", sa_r)
        check_output(y, rows, cols, y_ref, absdot, scale)
    finally:
        S.sfp8_sparse_linear_set_algo(m, n, k, 0)
    _status_clean()


def test_table_change_resizes_other_layers_workspace():
    """After one layer's algorithm choice lands in the table, another layer of
    the same shape (whose workspace was cached under the old choice) still
    runs: its workspace follows the table."""
    m, k, n = 16, 8192, 256
    w = synthetic.weight(12300, n, k)
    a = S.SparseFp8Linear(bf16_dev(w))
    b = S.SparseFp8Linear(bf16_dev(w))
    x = bf16_dev(synthetic.activation(12301, m, k))
    y0 = b(x).clone()                                   # caches b's workspace
    count = S.sfp8_sparse_linear_algo_count(m, n, k)
    # the algorithm with the largest workspace
    pick = max(range(count), key=lambda i: S.sfp8_sparse_linear_algo_workspace_bytes(m, n, k, i))
    try:
        S.sfp8_sparse_linear_set_algo(m, n, k, pick)
        y1 = b(x)
        y2 = a(x)
        torch.cuda.synchronize()
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
        rl = RefLayer(w, "e4m3")
        rows, aq_r, sa_r = rl.act(synthetic.activation(12301, m, k), "e4m3")
        y_ref, absdot, scale = rl.linear(aq_r, "e4m3", sa_r)
        check_output(y1, rows, np.arange(n), y_ref, absdot, scale)
        check_output(y0, rows, np.arange(n), y_ref, absdot, scale)
    finally:
        S.sfp8_sparse_linear_set_algo(m, n, k, 0)
    _status_clean()
