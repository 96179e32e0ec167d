"""Shared plumbing of the GPU parity tests: run the layer's steps through the
C-ABI (via the binding) and through the oracle on the same seeded inputs.

The oracle side may work on a subset of rows: quantisation, pruning and
compression are row-independent, and a sampled output needs only its own
activation row and weight row.
"""
import numpy as np
import pytest
import torch

import oracle
import semi_structured_sparse_rowwise_b200 as S
from semi_structured_sparse_rowwise_b200 import build

requires_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def ensure_library():
    build.build()
    S.load_library()


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_bits_of(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f32_to_bits16(v32):
    """float32 values that are bf16-representable -> bf16 bit patterns."""
    return (np.ascontiguousarray(v32, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


class GpuLayer:
    """Weight preparation and forward through the library, keeping every
    intermediate for comparison."""

    def __init__(self, w_bits, w_fmt):
        self.n, self.k = w_bits.shape
        self.w_fmt = w_fmt
        self.w = bf16_dev(w_bits)
        self.wp = S.sfp8_prune_24(self.w)
        self.wq, self.sw = S.sfp8_quantize_rowwise(self.wp, w_fmt)
        self.packed = S.sfp8_compress_24(self.wq, w_fmt)

    def forward(self, x_bits, a_fmt, bias_bits=None):
        x = bf16_dev(x_bits)
        aq, sa = S.sfp8_quantize_rowwise(x, a_fmt)
        bias = bf16_dev(bias_bits) if bias_bits is not None else None
        y = S.sfp8_sparse_linear(aq, a_fmt, sa, self.packed, self.w_fmt, self.sw,
                                 self.n, self.k, bias=bias)
        return aq, sa, y


class RefLayer:
    """The oracle on a subset of weight rows `cols` (output columns)."""

    def __init__(self, w_bits, w_fmt, cols=None):
        self.cols = np.arange(w_bits.shape[0]) if cols is None else np.asarray(cols)
        self.w_fmt = w_fmt
        w32 = oracle.bf16_bits_to_f32(w_bits[self.cols])
        self.wp = oracle.prune_24(w32)
        self.wq, self.sw = oracle.quantize_rowwise(self.wp, w_fmt)
        self.vals, self.nib = oracle.compress_24(self.wq, w_fmt)

    def act(self, x_bits, a_fmt, rows=None):
        rows = np.arange(x_bits.shape[0]) if rows is None else np.asarray(rows)
        aq, sa = oracle.quantize_rowwise(oracle.bf16_bits_to_f32(x_bits[rows]), a_fmt)
        return rows, aq, sa

    def linear(self, aq, a_fmt, sa, bias_bits=None):
        b = None
        if bias_bits is not None:
            b = oracle.bf16_bits_to_f32(bias_bits[self.cols]).astype(np.float64)
        return oracle.sparse_linear_ref(aq, a_fmt, sa, self.vals, self.nib, self.w_fmt,
                                        self.sw, b)


def sample_indices(total, count, seed, must=()):
    rng = np.random.Generator(np.random.PCG64(seed))
    pick = set(int(i) for i in rng.choice(total, size=min(total, count), replace=False))
    for i in must:
        if 0 <= i < total:
            pick.add(int(i))
    return np.array(sorted(pick), dtype=np.int64)


def check_weight_prep(gl, rl, cols):
    """Bit-exact: pruned weight, W_q, s_w, kept values and index nibbles."""
    cols_t = torch.from_numpy(cols).cuda()
    wp = bf16_bits_of(gl.wp.index_select(0, cols_t))
    assert np.array_equal(wp, f32_to_bits16(rl.wp)), "pruned weight differs"
    wq = gl.wq.index_select(0, cols_t).cpu().numpy()
    assert np.array_equal(wq, rl.wq), "quantised weight codes differ"
    sw = gl.sw.index_select(0, cols_t).cpu().numpy()
    assert np.array_equal(sw.view(np.uint32), rl.sw.view(np.uint32)), "weight scales differ"
    vals, nib = oracle.unpack_physical(gl.packed.cpu().numpy(), gl.n, gl.k,
                                       include_padding=True)
    assert np.array_equal(vals[cols], rl.vals), "kept values differ"
    assert np.array_equal(nib[cols], rl.nib), "index nibbles differ"
    npad = vals.shape[0]
    if npad > gl.n:
        assert np.all(vals[gl.n:] == 0) and np.all(nib[gl.n:] == 0x4), "padding rows"


def check_activation(aq_gpu, sa_gpu, rows, aq_ref, sa_ref):
    rows_t = torch.from_numpy(rows).cuda()
    aq = aq_gpu.index_select(0, rows_t).cpu().numpy()
    sa = sa_gpu.index_select(0, rows_t).cpu().numpy()
    assert np.array_equal(sa.view(np.uint32), sa_ref.view(np.uint32)), "activation scales differ"
    assert np.array_equal(aq, aq_ref), "activation codes differ"


def check_output(y_gpu, rows, cols, y_ref, absdot, scale):
    y = y_gpu.index_select(0, torch.from_numpy(rows).cuda()).index_select(
        1, torch.from_numpy(cols).cuda()).float().cpu().numpy().astype(np.float64)
    ok, worst = oracle.check_linear(y, y_ref, absdot, scale)
    assert ok, "linear output outside the tolerance (worst err/bound %.3g)" % worst
    return worst
