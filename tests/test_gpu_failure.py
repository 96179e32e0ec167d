"""Failure paths on the GPU, without a fault or a hang.

* A bounded wait that runs out: the library's self-test waits, with the same
  bounded wait as every pipeline, on a barrier that nothing completes.  The
  status word must report SFP8_DEVICE_TIMEOUT, and the context must stay
  usable: a sparse linear run afterwards still matches the oracle.
* A device-side check: decompressing a packed weight whose index nibble was
  corrupted (i0 >= i1) must set SFP8_DEVICE_CHECK_FAIL; the result is
  written without any out-of-range access and the next call runs clean.
"""
import numpy as np
import pytest
import torch

import semi_structured_sparse_rowwise_b200 as S
from semi_structured_sparse_rowwise_b200 import synthetic
from gpu_pipeline import GpuLayer, RefLayer, check_output, ensure_library, requires_gpu

pytestmark = [pytest.mark.gpu, requires_gpu]

ERR_TIMEOUT, ERR_DEVICE_CHECK = 8, 9


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_library()


def test_bounded_wait_reports_timeout_and_context_survives():
    assert S.sfp8_read_device_status(clear=True) == (0, 0)
    S.sfp8_selftest_timeout()
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == ERR_TIMEOUT and flags == 0x1, (st, flags)
    assert S.sfp8_read_device_status(clear=True) == (0, 0)       # cleared
    # the context still computes correctly
    m, k, n = 16, 256, 300
    x = synthetic.activation(81, m, k)
    w = synthetic.weight(82, n, k)
    gl = GpuLayer(w, "e4m3")
    aq, sa, y = gl.forward(x, "e4m3")
    rl = RefLayer(w, "e4m3")
    rows, aq_r, sa_r = rl.act(x, "e4m3")
    y_ref, absdot, scale = rl.linear(aq_r, "e4m3", sa_r)
    check_output(y, rows, np.arange(n), y_ref, absdot, scale)
    assert S.sfp8_read_device_status(clear=True) == (0, 0)


def test_corrupted_index_nibble_sets_check_flag():
    n, k = 200, 256
    gl = GpuLayer(synthetic.weight(83, n, k), "e4m3")
    packed = gl.packed.clone()
    # tile (0, 0), weight row 5: metadata bytes at 8192 + 16 * 5; a zero nibble
    # means i0 = i1 = 0, which the layout never holds
    off = 8192 + 16 * 5
    packed[off] = 0x40                    # group 0 nibble 0x0, group 1 valid
    out = S.sfp8_decompress_24(packed, n, k)
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == ERR_DEVICE_CHECK and flags == 0x2, (st, flags)
    # the untouched weight decompresses clean
    ref = S.sfp8_decompress_24(gl.packed, n, k)
    assert S.sfp8_read_device_status(clear=True) == (0, 0)
    assert torch.equal(out[:5], ref[:5]) and torch.equal(out[6:], ref[6:])
