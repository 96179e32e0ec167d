"""GPU parity of the 2:4 prune and the 2:4 compressor (bit-exact)."""
import itertools

import numpy as np
import pytest
import torch

import oracle
import semi_structured_sparse_rowwise_b200 as S
from semi_structured_sparse_rowwise_b200 import synthetic
from gpu_pipeline import (GpuLayer, RefLayer, check_weight_prep, ensure_library, requires_gpu,
                          sample_indices)

pytestmark = [pytest.mark.gpu, requires_gpu]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_library()


def _device_status_clean():
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == 0 and flags == 0, (st, flags)


def test_prune_ties_and_signed_zeros():
    vals = [0.0, -0.0, 1.0, -1.0, 2.0, 0.5, 3.0e-40, -2.0]
    groups = np.array(list(itertools.product(vals, repeat=4)), dtype=np.float32)
    w32 = groups.reshape(-1, 16)              # 4 groups per row, cols = 16
    for dtype in (torch.bfloat16, torch.float16, torch.float32):
        wd = torch.from_numpy(w32).to(dtype).cuda()
        ref_in = wd.float().cpu().numpy()
        out = S.sfp8_prune_24(wd)
        ref = oracle.prune_24(ref_in)
        got = out.float().cpu().numpy()
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), dtype


@pytest.mark.parametrize("n,k", [(64, 128), (200, 256), (1, 128), (129, 1024), (300, 4096)])
@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_weight_prep_parity(n, k, fmt):
    w_bits = synthetic.weight(31 + n + k, n, k, std=0.02, neg_zero_frac=0.05)
    gl = GpuLayer(w_bits, fmt)
    rl = RefLayer(w_bits, fmt)
    check_weight_prep(gl, rl, np.arange(n))
    _device_status_clean()


def test_compress_brute_force_groups():
    codes = [0x00, 0x80, 0x01, 0x81, 0x38, 0xB8, 0x40, 0xC0, 0x7E, 0xFE, 0x45, 0x44]
    groups = np.array(list(itertools.product(codes, repeat=4)), dtype=np.uint8)   # 20736 x 4
    q = groups.reshape(-1, 128)                                                   # 648 rows
    n, k = q.shape
    packed = S.sfp8_compress_24(torch.from_numpy(q).cuda(), "e4m3")
    vals, nib = oracle.unpack_physical(packed.cpu().numpy(), n, k)
    vr, nr = oracle.compress_24(q, "e4m3")
    assert np.array_equal(vals, vr) and np.array_equal(nib, nr)
    back = S.sfp8_decompress_24(packed, n, k).cpu().numpy()
    assert np.array_equal(back, oracle.decompress_24(vr, nr, k))
    _device_status_clean()


def test_compress_idempotent_on_gpu():
    w_bits = synthetic.weight(5, 256, 512, neg_zero_frac=0.05)
    gl = GpuLayer(w_bits, "e4m3")
    back = S.sfp8_decompress_24(gl.packed, 256, 512)
    p2 = S.sfp8_compress_24(back, "e4m3")
    assert torch.equal(p2, gl.packed)


def test_stress_weight_sampled():
    n, k = 28672, 8192
    w_bits = synthetic.weight(1004 * 100 + 2, n, k, std=0.01)
    gl = GpuLayer(w_bits, "e4m3")
    cols = sample_indices(n, 96, 17, must=(0, 127, 128, n - 1))
    rl = RefLayer(w_bits, "e4m3", cols)
    check_weight_prep(gl, rl, cols)
