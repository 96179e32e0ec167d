"""The sparse linear entry point that allocates nothing.

sfp8_sparse_linear_noalloc serves callers that may not allocate device
memory when they call the layer -- a pre-built CUDA graph being replayed, an
allocator that forbids cudaMalloc after start-up, or a host that hands over
only inputs and outputs.  It keeps its split-K scratch (partial sums and
per-tile counters) in a buffer built into the library instead of a
caller-provided workspace.

The shapes below are chosen so that the built-in work split divides the k
range of each weight tile over several CTAs (a workspace of more than zero
bytes), so the calls really go through the built-in buffer.  Each shape is
called twice, with a call of another split shape in between that leaves its
own partial sums and counters behind; every result is checked against the
oracle's output bound and bit for bit against the workspace entry point.

This file is named so that pytest collects it last; it also passes alone.
"""
import numpy as np
import pytest
import torch

import oracle
import semi_structured_sparse_rowwise_b200 as S
from semi_structured_sparse_rowwise_b200 import synthetic
from gpu_pipeline import (GpuLayer, RefLayer, bf16_dev, check_activation, ensure_library,
                          requires_gpu)

pytestmark = [pytest.mark.gpu, requires_gpu]

LIMIT = 8 << 20            # SFP8_NOALLOC_SCRATCH_BYTES


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_library()


class Case:
    """One problem: GPU weight and activation, the oracle's output and bound."""

    def __init__(self, m, k, n, a_fmt, w_fmt, with_bias, seed):
        x = synthetic.activation(seed, m, k, dist="student_t3")
        w = synthetic.weight(seed + 1, n, k)
        b = synthetic.bias(seed + 2, n) if with_bias else None
        self.m, self.k, self.n, self.a_fmt, self.w_fmt = m, k, n, a_fmt, w_fmt
        self.gl = GpuLayer(w, w_fmt)
        self.aq, self.sa = S.sfp8_quantize_rowwise(bf16_dev(x), a_fmt)
        self.bias = bf16_dev(b) if b is not None else None
        rl = RefLayer(w, w_fmt)
        rows, aq_r, sa_r = rl.act(x, a_fmt)
        check_activation(self.aq, self.sa, rows, aq_r, sa_r)
        self.y_ref, self.absdot, self.scale = rl.linear(aq_r, a_fmt, sa_r, b)

    def workspace_bytes(self):
        return S.sfp8_sparse_linear_workspace_bytes(self.m, self.n, self.k)

    def with_workspace(self):
        return S.sfp8_sparse_linear(self.aq, self.a_fmt, self.sa, self.gl.packed, self.w_fmt,
                                    self.gl.sw, self.n, self.k, bias=self.bias)

    def noalloc(self):
        out = torch.full((self.m, self.n), float("nan"), dtype=torch.bfloat16, device="cuda")
        return S.sfp8_sparse_linear_noalloc(self.aq, self.a_fmt, self.sa, self.gl.packed,
                                            self.w_fmt, self.gl.sw, self.n, self.k,
                                            bias=self.bias, out=out)

    def check(self, y):
        torch.cuda.synchronize()
        got = y.float().cpu().numpy().astype(np.float64)
        ok, worst = oracle.check_linear(got, self.y_ref, self.absdot, self.scale)
        assert ok, "output outside the oracle's bound (worst err/bound %.3g)" % worst


@pytest.fixture(scope="module")
def other_split():
    """A problem with another split (grid, token tile, tile count), called
    between the repeated calls so that the buffer holds its leftovers."""
    return Case(17, 8192, 4096, "e4m3", "e4m3", False, 950)


@pytest.mark.parametrize("m,k,n,a_fmt,w_fmt,with_bias", [
    (16, 8192, 256, "e4m3", "e4m3", False),     # stream-K, 32 CTAs, 0.5 MB of scratch
    (1, 8192, 1024, "e5m2", "e4m3", True),      # stream-K, 128 CTAs, 2.1 MB
    (3, 16384, 384, "e4m3", "e5m2", True),      # stream-K, 96 CTAs, 1.6 MB
    (24, 8192, 640, "e5m2", "e5m2", False),     # stream-K on 32-token tiles, 2.6 MB
    (32, 4096, 256, "e4m3", "e4m3", True),      # whole tiles: no scratch at all
])
def test_noalloc_matches_oracle_and_workspace_entry_point(m, k, n, a_fmt, w_fmt, with_bias,
                                                          other_split):
    c = Case(m, k, n, a_fmt, w_fmt, with_bias, 500 + m + n)
    nbytes = c.workspace_bytes()
    assert nbytes <= LIMIT
    if (m, k, n) != (32, 4096, 256):
        assert nbytes > 0, "this shape was chosen to use the built-in scratch"
    y_ws = c.with_workspace()
    c.check(y_ws)
    other_ref = other_split.with_workspace()
    for call in range(2):
        y = c.noalloc()
        c.check(y)
        # same kernel and work split, partial sums added in the same order
        assert torch.equal(y.view(torch.int16), y_ws.view(torch.int16)), "call %d" % call
        y_other = other_split.noalloc()
        assert torch.equal(y_other.view(torch.int16), other_ref.view(torch.int16))
    other_split.check(y_other)
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == 0 and flags == 0


def test_noalloc_follows_a_stream_k_table_entry(other_split):
    """A stream-K work split stored in the shape-keyed table is used by the
    no-allocation entry point as well (its scratch fits the buffer)."""
    m, k, n = 32, 4096, 512
    c = Case(m, k, n, "e4m3", "e4m3", True, 880)
    pick = None
    for algo in range(1, S.sfp8_sparse_linear_algo_count(m, n, k)):
        info = S.sfp8_sparse_linear_algo_info(m, n, k, algo)
        ws = S.sfp8_sparse_linear_algo_workspace_bytes(m, n, k, algo)
        if not info["whole_tiles"] and 0 < ws <= LIMIT:
            pick = algo
            break
    assert pick is not None
    y_algo = S.sfp8_sparse_linear_algo(c.aq, "e4m3", c.sa, c.gl.packed, "e4m3", c.gl.sw, n, k,
                                       pick, bias=c.bias)
    c.check(y_algo)
    S.sfp8_sparse_linear_set_algo(m, n, k, pick)
    try:
        for _ in range(2):
            y = c.noalloc()
            c.check(y)
            assert torch.equal(y.view(torch.int16), y_algo.view(torch.int16))
            other_split.noalloc()
    finally:
        S.sfp8_sparse_linear_set_algo(m, n, k, 0)
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == 0 and flags == 0


def test_noalloc_rejects_problems_beyond_its_buffer():
    # 8 weight tiles: too few for the SMs even at 16 tokens per tile, and 64
    # k steps per tile, so the k range is split over 148 CTAs of 128 tokens:
    # 19.4 MB of partial sums
    m, k, n = 128, 8192, 1024
    assert S.sfp8_sparse_linear_workspace_bytes(m, n, k) > LIMIT
    aq = torch.zeros((m, k), dtype=torch.uint8, device="cuda")
    sa = torch.ones((m,), dtype=torch.float32, device="cuda")
    packed = torch.zeros((S.sfp8_compressed_bytes(n, k),), dtype=torch.uint8, device="cuda")
    sw = torch.ones((n,), dtype=torch.float32, device="cuda")
    with pytest.raises(S.Sfp8Error) as e:
        S.sfp8_sparse_linear_noalloc(aq, "e4m3", sa, packed, "e4m3", sw, n, k)
    assert e.value.status == 6      # SFP8_ERR_WORKSPACE
