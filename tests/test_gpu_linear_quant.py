"""GPU parity of sfp8_sparse_linear_quant: quantise + sparse linear in one call.

a_q and s_a must equal the oracle's bit for bit, y must equal the two
separate calls (sfp8_quantize_rowwise + sfp8_sparse_linear) bit for bit and
lie within the stated bound of the oracle, for every activation dtype and
for the one-CTA and CTA-pair GEMMs.
"""
import numpy as np
import pytest
import torch

import semi_structured_sparse_rowwise_b200 as S
from semi_structured_sparse_rowwise_b200 import synthetic
from gpu_pipeline import (GpuLayer, RefLayer, bf16_dev, check_activation, check_output,
                          check_weight_prep, ensure_library, requires_gpu, sample_indices)

pytestmark = [pytest.mark.gpu, requires_gpu]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_library()


def _status_clean():
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == 0 and flags == 0, (st, flags)


def _two_calls(gl, x, a_fmt, bias):
    aq, sa = S.sfp8_quantize_rowwise(x, a_fmt)
    y = S.sfp8_sparse_linear(aq, a_fmt, sa, gl.packed, gl.w_fmt, gl.sw, gl.n, gl.k, bias=bias)
    return y, aq, sa


def _check(m, k, n, a_fmt, w_fmt, with_bias, seed, x_dtype=torch.bfloat16, ld_extra=0,
           n_cols=None):
    x_bits = synthetic.activation(seed, m, k + ld_extra, dist="student_t3", zero_row_frac=0.1)
    w_bits = synthetic.weight(seed + 1, n, k, neg_zero_frac=0.02)
    b_bits = synthetic.bias(seed + 2, n) if with_bias else None
    gl = GpuLayer(w_bits, w_fmt)
    x = bf16_dev(x_bits).to(x_dtype)[:, :k]          # row stride k + ld_extra
    bias = bf16_dev(b_bits) if b_bits is not None else None
    ws = S.new_quant_workspace(m, n, k, x.device)
    y, aq, sa = S.sfp8_sparse_linear_quant(x, a_fmt, gl.packed, w_fmt, gl.sw, n, k,
                                           bias=bias, workspace=ws)
    y2, aq2, sa2 = _two_calls(gl, x, a_fmt, bias)
    torch.cuda.synchronize()
    assert torch.equal(aq, aq2) and torch.equal(sa.view(torch.int32), sa2.view(torch.int32))
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16)), "one-call y != two calls"
    # the oracle on the activation as the device holds it (bf16-exact values)
    xr_bits = (x.float().cpu().numpy().view(np.uint32) >> 16).astype(np.uint16)
    cols = np.arange(n) if n_cols is None else sample_indices(n, n_cols, seed, must=(0, n - 1))
    rl = RefLayer(w_bits, w_fmt, cols)
    check_weight_prep(gl, rl, cols)
    rows, aq_r, sa_r = rl.act(xr_bits, a_fmt)
    check_activation(aq, sa, rows, aq_r, sa_r)
    y_ref, absdot, scale = rl.linear(aq_r, a_fmt, sa_r, b_bits)
    check_output(y, rows, cols, y_ref, absdot, scale)
    _status_clean()
    return gl, x, bias, ws, y


# (m, k, n): decode sizes (one token tile, the activation resident in shared
# memory), strided and ragged.
FUSED_SHAPES = [(1, 128, 64), (4, 256, 300), (16, 4096, 1000), (16, 6144, 384),
                (17, 2048, 700), (32, 3072, 520), (3, 512, 129)]


@pytest.mark.parametrize("m,k,n", FUSED_SHAPES)
@pytest.mark.parametrize("a_fmt,w_fmt", [("e4m3", "e4m3"), ("e5m2", "e4m3"), ("e4m3", "e5m2")])
def test_one_call_matches_two_calls_and_oracle(m, k, n, a_fmt, w_fmt):
    _check(m, k, n, a_fmt, w_fmt, with_bias=(m + n) % 2 == 1, seed=3300 + m * 11 + k + n)


def test_one_call_strided_activation():
    _check(16, 1024, 640, "e4m3", "e4m3", with_bias=True, seed=3401, ld_extra=64)


def test_one_call_decode_workload_repeated():
    """The decode workload, sampled columns, five calls in a row on one
    workspace: identical outputs every time."""
    m, k, n = 16, 4096, 14336
    gl, x, bias, ws, y = _check(m, k, n, "e4m3", "e4m3", with_bias=False, seed=3501,
                                n_cols=512)
    for _ in range(5):
        y_again, _, _ = S.sfp8_sparse_linear_quant(x, "e4m3", gl.packed, "e4m3", gl.sw, n, k,
                                                   bias=bias, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(y_again.view(torch.int16), y.view(torch.int16))
    _status_clean()


@pytest.mark.parametrize("m,k,n,x_dtype", [(16, 1024, 300, torch.float32),
                                           (16, 1024, 300, torch.float16),
                                           (64, 512, 260, torch.bfloat16),
                                           (600, 256, 390, torch.bfloat16)])
def test_other_inputs(m, k, n, x_dtype):
    """Other activation dtypes, more than one token tile, the CTA-pair GEMM."""
    _check(m, k, n, "e4m3", "e4m3", with_bias=True, seed=3600 + m + k, x_dtype=x_dtype)


def test_zero_outputs_still_quantises():
    x = bf16_dev(synthetic.activation(3700, 8, 256))
    gl = GpuLayer(synthetic.weight(3701, 128, 256), "e4m3")
    aq = torch.empty((8, 256), dtype=torch.uint8, device="cuda")
    sa = torch.empty((8,), dtype=torch.float32, device="cuda")
    ws = S.new_quant_workspace(8, 128, 256, x.device)
    y, aq, sa = S.sfp8_sparse_linear_quant(x, "e4m3", gl.packed, "e4m3", gl.sw, 0, 256,
                                           workspace=ws, a_q=aq, s_a=sa)
    aq2, sa2 = S.sfp8_quantize_rowwise(x, "e4m3")
    torch.cuda.synchronize()
    assert y.shape == (8, 0)
    assert torch.equal(aq, aq2) and torch.equal(sa.view(torch.int32), sa2.view(torch.int32))
