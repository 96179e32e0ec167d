"""GPU parity of the fused one-call forward (sfp8_sparse_linear_quant_fused).

In the fused form every CTA of the decode GEMM quantises the activation's
(at most 16) rows itself and writes the codes into its shared-memory tile.
Its results must equal, bit for bit, the chained form (row-wise quantiser,
then the GEMM) and the two separate calls (sfp8_quantize_rowwise +
sfp8_sparse_linear): a_q, s_a and y.  With bf16 activations a_q and s_a are
also compared with the oracle bit for bit and y against the oracle's bound.

The shapes cover each way the kernel spreads rows over its 256 quantiser
threads (1, 2, 3-4, 5-8 and 9-16 rows: 256 down to 16 threads per row, the
wider ones reducing across warps), 1, 2 and 4 k steps per pipeline stage,
the largest resident activation (k = 6144), grids smaller and larger than
the number of k steps (the codes are written to global memory split by k
step over the CTAs), strided activations, every input dtype and both code
formats, and a stream-K work split taken from the shape-keyed table.
"""
import numpy as np
import pytest
import torch

import semi_structured_sparse_rowwise_b200 as S
from semi_structured_sparse_rowwise_b200 import synthetic
from gpu_pipeline import (GpuLayer, RefLayer, bf16_dev, check_activation, check_output,
                          ensure_library, requires_gpu, sample_indices)

pytestmark = [pytest.mark.gpu, requires_gpu]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_library()


def _status_clean():
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == 0 and flags == 0, (st, flags)


def _same(a, b):
    if a.dtype == torch.bfloat16:
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    if a.dtype == torch.float32:
        return torch.equal(a.view(torch.int32), b.view(torch.int32))
    return torch.equal(a, b)


def _run(m, k, n, a_fmt, w_fmt, with_bias, seed, x_dtype=torch.bfloat16, ld_extra=0,
         n_cols=None, dist="student_t3", x_bits=None):
    if x_bits is None:
        x_bits = synthetic.activation(seed, m, k + ld_extra, dist=dist, zero_row_frac=0.1)
    w_bits = synthetic.weight(seed + 1, n, k, neg_zero_frac=0.02)
    b_bits = synthetic.bias(seed + 2, n) if with_bias else None
    gl = GpuLayer(w_bits, w_fmt)
    x = bf16_dev(x_bits).to(x_dtype)[:, :k]
    bias = bf16_dev(b_bits) if b_bits is not None else None
    assert S.sfp8_sparse_linear_quant_fusable(m, n, k)
    ws = S.new_quant_workspace(m, n, k, x.device)
    # stale codes and NaN outputs: everything must be written by the call
    aq = torch.full((m, k), 0x55, dtype=torch.uint8, device="cuda")
    sa = torch.full((m,), float("nan"), dtype=torch.float32, device="cuda")
    out = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
    y, aq, sa = S.sfp8_sparse_linear_quant_fused(x, a_fmt, gl.packed, w_fmt, gl.sw, n, k,
                                                 bias=bias, workspace=ws, a_q=aq, s_a=sa,
                                                 out=out)
    yc, aqc, sac = S.sfp8_sparse_linear_quant_chained(x, a_fmt, gl.packed, w_fmt, gl.sw, n, k,
                                                      bias=bias, workspace=ws)
    ya, aqa, saa = S.sfp8_sparse_linear_quant(x, a_fmt, gl.packed, w_fmt, gl.sw, n, k,
                                              bias=bias, workspace=ws)
    aq2, sa2 = S.sfp8_quantize_rowwise(x, a_fmt)
    y2 = S.sfp8_sparse_linear(aq2, a_fmt, sa2, gl.packed, w_fmt, gl.sw, n, k, bias=bias)
    torch.cuda.synchronize()
    for name, a, b in (("a_q", aq, aq2), ("s_a", sa, sa2), ("y", y, y2),
                       ("chained a_q", aqc, aq2), ("chained s_a", sac, sa2), ("chained y", yc, y2),
                       ("default y", ya, y2), ("default a_q", aqa, aq2)):
        assert _same(a, b), "fused and separate calls differ in " + name
    if x_dtype == torch.bfloat16:
        xr_bits = (x.float().cpu().numpy().view(np.uint32) >> 16).astype(np.uint16)
        cols = np.arange(n) if n_cols is None else sample_indices(n, n_cols, seed,
                                                                  must=(0, n - 1))
        rl = RefLayer(w_bits, w_fmt, cols)
        rows, aq_r, sa_r = rl.act(xr_bits, a_fmt)
        check_activation(aq, sa, rows, aq_r, sa_r)
        y_ref, absdot, scale = rl.linear(aq_r, a_fmt, sa_r, b_bits)
        check_output(y, rows, cols, y_ref, absdot, scale)
    _status_clean()
    return gl, x, bias, ws, y


# (m, k, n): every rows-per-thread-group case, KS 4 / 2 / 1 (k steps 32, 6, 3),
# k = 128 (fewer 16-code chunks than threads per row), the largest resident
# activation (16 x 6144 = 96 KB), n ragged, grids of 1 to 112 CTAs.
SHAPES = [(1, 4096, 1000), (2, 768, 300), (3, 384, 129), (4, 128, 64), (5, 4096, 260),
          (8, 6144, 520), (9, 2048, 700), (15, 768, 1024), (16, 4096, 1000),
          (16, 6144, 384), (16, 128, 200), (1, 256, 64), (16, 4096, 64)]


@pytest.mark.parametrize("m,k,n", SHAPES)
@pytest.mark.parametrize("a_fmt,w_fmt", [("e4m3", "e4m3"), ("e5m2", "e5m2")])
def test_fused_equals_chained_and_oracle(m, k, n, a_fmt, w_fmt):
    _run(m, k, n, a_fmt, w_fmt, with_bias=(m + n) % 2 == 0, seed=5100 + 7 * m + k + n)


@pytest.mark.parametrize("x_dtype", [torch.float16, torch.float32])
@pytest.mark.parametrize("m", [3, 16])
def test_fused_other_input_dtypes(x_dtype, m):
    _run(m, 1024, 300, "e4m3", "e4m3", with_bias=True, seed=5200 + m, x_dtype=x_dtype)


@pytest.mark.parametrize("m", [1, 7, 16])
def test_fused_strided_activation(m):
    _run(m, 2048, 640, "e5m2", "e4m3", with_bias=False, seed=5300 + m, ld_extra=64)


def test_fused_special_rows():
    """Rows of zeros, tiny (bf16 subnormal) and huge values, one nonzero per
    row, and FP8 midpoints of x / s: codes and scales identical to the
    separate quantiser's."""
    m, k, n = 6, 512, 256
    rng = np.random.Generator(np.random.PCG64(5401))
    x = np.zeros((m, k), np.float32)
    x[1] = rng.standard_normal(k) * 1e-39                      # bf16 subnormals
    x[2] = rng.standard_normal(k) * 1e30
    x[3, 17] = -3.0                                            # one nonzero
    x[4] = rng.standard_normal(k)
    x[4, ::7] = 0.0
    table = np.array([0.5, 1.5, 2.5, 3.25, 6.5, 13.0, 26.0, 52.0, 104.0, 208.0, 416.0])
    x[5] = rng.choice(table, k) * rng.choice([-1.0, 1.0], k)
    x[5, 0] = 448.0
    bits = synthetic.f32_to_bf16_bits(x.astype(np.float32))
    _run(m, k, n, "e4m3", "e4m3", with_bias=True, seed=5400, x_bits=bits)


def test_fused_decode_workload_repeated():
    """The decode workload (16 x 4096 -> 14336, sampled columns), then five
    more calls on the same buffers: identical every time."""
    m, k, n = 16, 4096, 14336
    gl, x, bias, ws, y = _run(m, k, n, "e4m3", "e4m3", with_bias=False, seed=5501,
                              n_cols=512, dist="normal")
    for _ in range(5):
        y_again, _, _ = S.sfp8_sparse_linear_quant_fused(x, "e4m3", gl.packed, "e4m3", gl.sw,
                                                         n, k, bias=bias, workspace=ws)
        torch.cuda.synchronize()
        assert _same(y_again, y)
    _status_clean()


def test_fused_with_stream_k_table_entry():
    """A stream-K split (partial sums through the workspace) set in the
    shape-keyed table: the fused form follows it and still equals the
    chained form bit for bit."""
    m, k, n = 16, 2048, 512
    pick = None
    for algo in range(1, S.sfp8_sparse_linear_algo_count(m, n, k)):
        info = S.sfp8_sparse_linear_algo_info(m, n, k, algo)
        if not info["whole_tiles"] and not info["pair"] and info["bn"] == 16:
            pick = algo
            break
    assert pick is not None
    S.sfp8_sparse_linear_set_algo(m, n, k, pick)
    try:
        _run(m, k, n, "e4m3", "e4m3", with_bias=True, seed=5601)
    finally:
        S.sfp8_sparse_linear_set_algo(m, n, k, 0)


def test_fused_form_rejects_other_shapes():
    """More than 16 tokens (or an activation too large to stay resident): no
    fused form; the default entry point falls back to the chain."""
    for m, k, n in ((17, 1024, 256), (16, 8192, 256), (64, 512, 256)):
        assert not S.sfp8_sparse_linear_quant_fusable(m, n, k)
        x = bf16_dev(synthetic.activation(5700 + m, m, k))
        gl = GpuLayer(synthetic.weight(5701, n, k), "e4m3")
        ws = S.new_quant_workspace(m, n, k, x.device)
        with pytest.raises(S.Sfp8Error) as e:
            S.sfp8_sparse_linear_quant_fused(x, "e4m3", gl.packed, "e4m3", gl.sw, n, k,
                                             workspace=ws)
        assert e.value.status == 2      # SFP8_ERR_UNSUPPORTED_SHAPE
    _status_clean()
