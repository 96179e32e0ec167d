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


@pytest.mark.parametrize("m", [3, 16])
@pytest.mark.parametrize("pinned", [True, False])
def test_host_path_matches_device_path(pinned, m):
    """sfp8_sparse_linear_quant_host (copy in, quantise, linear, copy out in
    one call) gives the device path's bits, from page-locked or pageable host
    buffers, on repeated calls; m=3 goes through the tile-high staging of the
    codes."""
    k, n = 1024, 700
    x = synthetic.activation(8100, m, k, dist="student_t3")
    w = synthetic.weight(8101, n, k)
    b = synthetic.bias(8102, n)
    layer = S.SparseFp8Linear(bf16_dev(w), bias=bf16_dev(b).float())
    x_host = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
    y_host = torch.empty((m, n), dtype=torch.bfloat16)
    if pinned:
        x_host, y_host = x_host.pin_memory(), y_host.pin_memory()
    y_dev = layer(x_host.cuda())
    for _ in range(3):
        y_host.fill_(float("nan"))
        layer.forward_host(x_host, y_host)
        torch.cuda.synchronize()
        assert torch.equal(y_host.view(torch.int16), y_dev.cpu().view(torch.int16))
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == 0 and flags == 0


def test_host_pipeline_eager_and_captured():
    """HostPipeline: copies in, forward and copies out on three streams with
    rotating buffers; each batch's y_host equals the device path's bits, both
    for eager submits and for a captured graph replayed twice."""
    m, k, n = 16, 512, 300
    w = synthetic.weight(8200, n, k)
    layer = S.SparseFp8Linear(bf16_dev(w))
    xs = [synthetic.activation(8201 + i, m, k, dist="student_t3") for i in range(5)]
    x_hosts = [torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
               .pin_memory() for x in xs]
    refs = [layer(xh.cuda()).cpu() for xh in x_hosts]
    y_hosts = [torch.empty((m, n), dtype=torch.bfloat16).pin_memory() for _ in xs]
    pipe = S.HostPipeline(layer, m, depth=3)
    for xh, yh in zip(x_hosts, y_hosts):
        pipe.submit(xh, yh)
    pipe.synchronize()
    for yh, ref in zip(y_hosts, refs):
        assert torch.equal(yh.view(torch.int16), ref.view(torch.int16))
    pipe2 = S.HostPipeline(layer, m, depth=2)
    g = pipe2.capture(x_hosts, y_hosts)
    for _ in range(2):
        for yh in y_hosts:
            yh.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for yh, ref in zip(y_hosts, refs):
            assert torch.equal(yh.view(torch.int16), ref.view(torch.int16))
    del g
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == 0 and flags == 0
