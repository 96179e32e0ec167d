"""GPU parity of the sparse FP8 linear against the oracle.

Bit-exact for every integer/code stage (pruned weight, codes, scales, kept
values, index nibbles); the output within the stated bound
|y - y_ref| <= 8e-3 |y_ref| + 1e-3 s_a s_w sum|a w|.  Small shapes are checked
in full; the full-size workloads on sampled rows and columns, plus properties
of the whole output.
"""
import numpy as np
import pytest
import torch

import oracle
import semi_structured_sparse_rowwise_b200 as S
from semi_structured_sparse_rowwise_b200 import synthetic
from gpu_pipeline import (GpuLayer, RefLayer, bf16_dev, check_activation, check_output,
                          check_weight_prep, ensure_library, requires_gpu, sample_indices)

pytestmark = [pytest.mark.gpu, requires_gpu]

PAIRS = [("e4m3", "e4m3"), ("e4m3", "e5m2"), ("e5m2", "e4m3"), ("e5m2", "e5m2")]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_library()


def _status_clean():
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == 0 and flags == 0, (st, flags)


def run_full(x_bits, w_bits, a_fmt, w_fmt, bias_bits=None):
    gl = GpuLayer(w_bits, w_fmt)
    aq, sa, y = gl.forward(x_bits, a_fmt, bias_bits)
    rl = RefLayer(w_bits, w_fmt)
    rows, aq_r, sa_r = rl.act(x_bits, a_fmt)
    check_weight_prep(gl, rl, np.arange(w_bits.shape[0]))
    check_activation(aq, sa, rows, aq_r, sa_r)
    y_ref, absdot, scale = rl.linear(aq_r, a_fmt, sa_r, bias_bits)
    worst = check_output(y, rows, np.arange(w_bits.shape[0]), y_ref, absdot, scale)
    _status_clean()
    return gl, y, worst


def test_tiny_workload():
    x, w, b, _ = synthetic.workload_inputs("tiny")
    run_full(x, w, "e4m3", "e4m3", b)


SHAPES = [(40, 512, 300), (200, 256, 520), (1, 128, 1), (17, 384, 129), (1024, 256, 4096),
          (300, 1024, 384), (64, 128, 128), (256, 2048, 256), (129, 640, 200)]


@pytest.mark.parametrize("m,k,n", SHAPES)
@pytest.mark.parametrize("pair", PAIRS)
def test_ragged_multi_tile(m, k, n, pair):
    a_fmt, w_fmt = pair
    seed = 7000 + m * 7 + k * 3 + n
    x = synthetic.activation(seed, m, k, dist="student_t3", zero_row_frac=0.05)
    w = synthetic.weight(seed + 1, n, k, neg_zero_frac=0.02)
    b = synthetic.bias(seed + 2, n) if (m + n) % 2 else None
    run_full(x, w, a_fmt, w_fmt, b)


# Shapes for the CTA-pair kernel (512 tokens and more): an odd count of
# 128-row weight tiles (the second CTA of the last pair has no rows), ragged
# token tiles, a single k step, and token counts that choose different tile
# widths (192, 224).  The last four have enough tiles for two weight tiles
# per CTA (512-row pair tiles), with a last group of 1, 2 or 4 valid tiles.
PAIR_SHAPES = [(512, 128, 100), (700, 384, 390), (1000, 256, 1000), (2049, 128, 260),
               (600, 640, 129), (4000, 256, 2700), (4000, 256, 2600), (2049, 384, 5000),
               (5000, 128, 1700)]


@pytest.mark.parametrize("m,k,n", PAIR_SHAPES)
@pytest.mark.parametrize("pair", PAIRS)
def test_pair_kernel_shapes(m, k, n, pair):
    a_fmt, w_fmt = pair
    seed = 9100 + m * 5 + k * 3 + n
    x = synthetic.activation(seed, m, k, dist="student_t3", zero_row_frac=0.03)
    w = synthetic.weight(seed + 1, n, k, neg_zero_frac=0.02)
    b = synthetic.bias(seed + 2, n) if (m + n) % 2 else None
    run_full(x, w, a_fmt, w_fmt, b)


def test_pair_kernel_deterministic():
    m, k, n = 1000, 512, 700
    x = synthetic.activation(31, m, k)
    w = synthetic.weight(32, n, k)
    gl = GpuLayer(w, "e4m3")
    aq, sa = S.sfp8_quantize_rowwise(bf16_dev(x), "e4m3")
    assert S.sfp8_sparse_linear_workspace_bytes(m, n, k) == 0
    y1 = S.sfp8_sparse_linear(aq, "e4m3", sa, gl.packed, "e4m3", gl.sw, n, k)
    y2 = S.sfp8_sparse_linear(aq, "e4m3", sa, gl.packed, "e4m3", gl.sw, n, k)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    _status_clean()


def test_deterministic_and_counters_reset():
    m, k, n = 40, 8192, 700            # split-K tiles (few tiles, 64 k steps each)
    x = synthetic.activation(1, m, k)
    w = synthetic.weight(2, n, k)
    gl = GpuLayer(w, "e4m3")
    xd = bf16_dev(x)
    aq, sa = S.sfp8_quantize_rowwise(xd, "e4m3")
    ws = S.new_workspace(m, n, k, xd.device)
    y1 = S.sfp8_sparse_linear(aq, "e4m3", sa, gl.packed, "e4m3", gl.sw, n, k, workspace=ws)
    y2 = S.sfp8_sparse_linear(aq, "e4m3", sa, gl.packed, "e4m3", gl.sw, n, k, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    nbytes = S.sfp8_sparse_linear_workspace_bytes(m, n, k)
    tiles = ((n + 127) // 128) * 1
    assert nbytes >= tiles * 16           # this shape is split across CTAs
    counters = ws[nbytes - tiles * 16: nbytes].view(torch.int32)
    assert int(counters.abs().sum()) == 0
    _status_clean()


def test_workspace_too_small():
    m, k, n = 16, 8192, 256
    assert S.sfp8_sparse_linear_workspace_bytes(m, n, k) > 16     # split-K shape
    gl = GpuLayer(synthetic.weight(3, n, k), "e4m3")
    aq, sa = S.sfp8_quantize_rowwise(bf16_dev(synthetic.activation(4, m, k)), "e4m3")
    small = torch.zeros((16,), dtype=torch.uint8, device="cuda")
    with pytest.raises(S.Sfp8Error) as e:
        S.sfp8_sparse_linear(aq, "e4m3", sa, gl.packed, "e4m3", gl.sw, n, k, workspace=small)
    assert e.value.status == 6


def run_sampled(name, shape_index, pairs=None, n_rows=48, n_cols=384, prep_cache=None):
    x, w, b, _ = synthetic.workload_inputs(name, shape_index)
    m, k = x.shape
    n = w.shape[0]
    rows = sample_indices(m, n_rows, 11 + shape_index, must=(0, m - 1))
    cols = sample_indices(n, n_cols, 13 + shape_index, must=(0, 127, 128, n - 1))
    pairs = pairs or synthetic.WORKLOADS[name]["dtypes"]
    worst = 0.0
    for a_fmt, w_fmt in pairs:
        key = (name, shape_index, w_fmt)
        if prep_cache is not None and key in prep_cache:
            gl, rl = prep_cache[key]
        else:
            gl = GpuLayer(w, w_fmt)
            rl = RefLayer(w, w_fmt, cols)
            check_weight_prep(gl, rl, cols)
            if prep_cache is not None:
                prep_cache[key] = (gl, rl)
        aq, sa, y = gl.forward(x, a_fmt, b)
        r, aq_r, sa_r = rl.act(x, a_fmt, rows)
        check_activation(aq, sa, r, aq_r, sa_r)
        y_ref, absdot, scale = rl.linear(aq_r, a_fmt, sa_r, b)
        worst = max(worst, check_output(y, rows, cols, y_ref, absdot, scale))
        assert bool(torch.isfinite(y.float()).all())
        _status_clean()
    return worst


@pytest.mark.parametrize("shape_index", [0, 1, 2])
def test_decode_workload(shape_index):
    run_sampled("decode_gate_up_8b", shape_index, n_rows=16, n_cols=1024)


@pytest.mark.parametrize("shape_index", [0, 1, 2, 3])
def test_prefill_workload(shape_index):
    run_sampled("prefill_8b", shape_index)


_SWEEP_CACHE = {}


@pytest.mark.parametrize("shape_index", [0, 1, 2, 3, 4])
def test_dtype_sweep_workload(shape_index):
    run_sampled("dtype_sweep_8b_up", shape_index, prep_cache=_SWEEP_CACHE)


def test_stress_workload():
    name = "stress_70b_mlp"
    x, w, b, _ = synthetic.workload_inputs(name, 0)
    m, k = x.shape
    n = w.shape[0]
    gl = GpuLayer(w, "e4m3")
    aq, sa, y = gl.forward(x, "e4m3", b)
    # all-zero activation rows give exactly zero outputs (no bias here)
    x32_rowmax = np.abs(x.view(np.int16).astype(np.int32) & 0x7FFF).max(axis=1)
    zero_rows = np.nonzero(x32_rowmax == 0)[0]
    assert zero_rows.size > 0
    zr = torch.from_numpy(zero_rows).cuda()
    assert bool((y.index_select(0, zr).float() == 0).all())
    rows = sample_indices(m, 40, 21, must=(0, m - 1, int(zero_rows[0])))
    cols = sample_indices(n, 256, 23, must=(0, n - 1))
    rl = RefLayer(w, "e4m3", cols)
    check_weight_prep(gl, rl, cols)
    r, aq_r, sa_r = rl.act(x, "e4m3", rows)
    check_activation(aq, sa, r, aq_r, sa_r)
    y_ref, absdot, scale = rl.linear(aq_r, "e4m3", sa_r, b)
    check_output(y, rows, cols, y_ref, absdot, scale)
    _status_clean()
