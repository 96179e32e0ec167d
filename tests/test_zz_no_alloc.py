"""The sparse linear entry point that allocates nothing.

sfp8_sparse_linear_noalloc serves callers that may not allocate device
memory when they call the layer -- a pre-built CUDA graph being replayed, an
allocator that forbids cudaMalloc after start-up, or a host that hands over
only inputs and outputs.  It keeps its split-K scratch in a buffer built into
the library instead of a caller-provided workspace.  This test calls it
through the C ABI twice in a row (so the second call sees the buffer as the
first left it) and checks each result against the workspace entry point's
output on the same inputs, with the tolerance the other output tests use.

This file is named so that pytest collects it last; it also passes alone.
"""
import numpy as np
import pytest
import torch

import oracle
import semi_structured_sparse_rowwise_b200 as S
from semi_structured_sparse_rowwise_b200 import synthetic
from gpu_pipeline import GpuLayer, RefLayer, bf16_dev, ensure_library, requires_gpu

pytestmark = [pytest.mark.gpu, requires_gpu]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_library()


@pytest.mark.parametrize("m,k,n,a_fmt,w_fmt,with_bias", [
    (16, 1024, 1000, "e4m3", "e4m3", False),
    (5, 512, 300, "e5m2", "e4m3", True),
    (32, 256, 4096, "e4m3", "e5m2", True),
])
def test_noalloc_matches_workspace_entry_point(m, k, n, a_fmt, w_fmt, with_bias):
    limit = 8 << 20
    assert S.sfp8_sparse_linear_workspace_bytes(m, n, k) <= limit
    x = synthetic.activation(500 + m, m, k, dist="student_t3")
    w = synthetic.weight(600 + n, n, k)
    b = synthetic.bias(700 + n, n) if with_bias else None
    gl = GpuLayer(w, w_fmt)
    aq, sa = S.sfp8_quantize_rowwise(bf16_dev(x), a_fmt)
    bias = bf16_dev(b) if b is not None else None
    y_ws = S.sfp8_sparse_linear(aq, a_fmt, sa, gl.packed, w_fmt, gl.sw, n, k, bias=bias)
    # the acceptance bound's terms, from the oracle on the same inputs
    rl = RefLayer(w, w_fmt)
    _, aq_r, sa_r = rl.act(x, a_fmt)
    _, absdot, scale = rl.linear(aq_r, a_fmt, sa_r, b)
    ref = y_ws.float().cpu().numpy().astype(np.float64)
    for _ in range(2):
        out = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
        y_na = S.sfp8_sparse_linear_noalloc(aq, a_fmt, sa, gl.packed, w_fmt, gl.sw,
                                            n, k, bias=bias, out=out)
        torch.cuda.synchronize()
        got = y_na.float().cpu().numpy().astype(np.float64)
        ok, worst = oracle.check_linear(got, ref, absdot, scale)
        assert ok, "no-alloc output differs from the workspace entry point (%.3g)" % worst
        # same kernel and work split: the bits agree as well
        assert torch.equal(y_na.view(torch.int16), y_ws.view(torch.int16))
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == 0 and flags == 0


def test_noalloc_rejects_problems_beyond_its_buffer():
    # 8 weight tiles: too few for the SMs even at 16 tokens per tile, and 64
    # k steps per tile, so the k range is split over 148 CTAs of 128 tokens:
    # 19.4 MB of partial sums
    m, k, n = 128, 8192, 1024
    assert S.sfp8_sparse_linear_workspace_bytes(m, n, k) > 8 << 20
    aq = torch.zeros((m, k), dtype=torch.uint8, device="cuda")
    sa = torch.ones((m,), dtype=torch.float32, device="cuda")
    packed = torch.zeros((S.sfp8_compressed_bytes(n, k),), dtype=torch.uint8, device="cuda")
    sw = torch.ones((n,), dtype=torch.float32, device="cuda")
    with pytest.raises(S.Sfp8Error) as e:
        S.sfp8_sparse_linear_noalloc(aq, "e4m3", sa, packed, "e4m3", sw, n, k)
    assert e.value.status == 6      # SFP8_ERR_WORKSPACE
