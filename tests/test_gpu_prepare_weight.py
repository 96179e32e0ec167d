"""GPU parity of the one-pass weight preparation (prune 2:4 -> row-wise FP8
quantisation -> compression): bit-exact against the oracle's three steps."""
import itertools

import numpy as np
import pytest
import torch

import oracle
import semi_structured_sparse_rowwise_b200 as S
from semi_structured_sparse_rowwise_b200 import synthetic
from gpu_pipeline import GpuLayer, bf16_dev, ensure_library, requires_gpu, sample_indices

pytestmark = [pytest.mark.gpu, requires_gpu]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_library()


def _device_status_clean():
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == 0 and flags == 0, (st, flags)


def _check_against_oracle(packed, sw, w32, fmt, rows=None, n_total=None):
    """packed/s_w from the GPU vs the oracle's prune -> quantise -> compress of
    the float32 rows w32 (all rows, or the sampled `rows` of an n_total-row
    weight)."""
    n, k = (w32.shape[0], w32.shape[1]) if rows is None else (n_total, w32.shape[1])
    rows = np.arange(n) if rows is None else rows
    wq, sw_ref = oracle.quantize_rowwise(oracle.prune_24(w32), fmt)
    vals_ref, nib_ref = oracle.compress_24(wq, fmt)
    got_sw = sw.cpu().numpy()[rows]
    assert np.array_equal(got_sw.view(np.uint32), sw_ref.view(np.uint32)), "weight scales differ"
    vals, nib = oracle.unpack_physical(packed.cpu().numpy(), n, k, include_padding=True)
    assert np.array_equal(vals[rows], vals_ref), "kept values differ"
    assert np.array_equal(nib[rows], nib_ref), "index nibbles differ"
    if vals.shape[0] > n:
        assert np.all(vals[n:] == 0) and np.all(nib[n:] == 0x4), "padding rows"


@pytest.mark.parametrize("n,k", [(64, 128), (200, 256), (1, 128), (129, 1024), (300, 4096),
                                 (130, 14336)])
@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_prepare_parity_bf16(n, k, fmt):
    w_bits = synthetic.weight(77 + n + k, n, k, std=0.02, neg_zero_frac=0.05)
    packed, sw = S.sfp8_prepare_weight_24(bf16_dev(w_bits), fmt)
    _check_against_oracle(packed, sw, oracle.bf16_bits_to_f32(w_bits), fmt)
    _device_status_clean()


@pytest.mark.parametrize("dtype", [torch.float16, torch.float32])
@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_prepare_parity_wide_inputs(dtype, fmt):
    n, k = 257, 512
    rng = np.random.Generator(np.random.PCG64(4242))
    w = (rng.standard_normal((n, k), dtype=np.float32) * np.float32(0.05))
    w[rng.random((n, k)) < 0.05] = -0.0
    wd = torch.from_numpy(w).to(dtype).cuda()
    packed, sw = S.sfp8_prepare_weight_24(wd, fmt)
    _check_against_oracle(packed, sw, wd.float().cpu().numpy(), fmt)
    _device_status_clean()


def test_prepare_strided_rows():
    n, k, ld = 150, 384, 512
    w_bits = synthetic.weight(91, n, ld, std=0.02)
    full = bf16_dev(w_bits)
    packed, sw = S.sfp8_prepare_weight_24(full[:, :k], "e4m3")
    _check_against_oracle(packed, sw, oracle.bf16_bits_to_f32(w_bits[:, :k]), "e4m3")


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_prepare_kept_values_that_quantise_to_zero(fmt, dtype):
    """Groups whose kept values round to a zero code (the row amax is 1, the
    values far below the smallest FP8 step) next to exact and signed zeros:
    the compressor's second selection on the codes decides those groups."""
    tiny = 1e-6 if fmt == "e4m3" else 1e-10
    vals = [0.0, -0.0, tiny, -tiny, 3 * tiny, 0.25, -0.5]
    groups = np.array(list(itertools.product(vals, repeat=4)), dtype=np.float32)   # 2401
    per_row = 31
    rows = -(-groups.shape[0] // per_row)
    pad = rows * per_row - groups.shape[0]
    groups = np.concatenate([groups, np.zeros((pad, 4), np.float32)])
    w = np.zeros((rows, 128), np.float32)
    w[:, 0] = 1.0                                        # amax 1 in every row
    w[:, 4:] = groups.reshape(rows, per_row * 4)
    wd = torch.from_numpy(w).to(dtype).cuda()
    packed, sw = S.sfp8_prepare_weight_24(wd, fmt)
    _check_against_oracle(packed, sw, wd.float().cpu().numpy(), fmt)
    _device_status_clean()


def test_prepare_equals_three_calls_llama_up():
    """At the 8B up projection's size the one-pass result is byte-identical to
    prune -> quantise -> compress through the library, and rows sampled from it
    match the oracle."""
    n, k = 14336, 4096
    w_bits = synthetic.weight(1001 * 100 + 1, n, k, std=0.02)
    gl = GpuLayer(w_bits, "e4m3")
    packed, sw = S.sfp8_prepare_weight_24(gl.w, "e4m3")
    assert torch.equal(packed, gl.packed)
    assert torch.equal(sw.view(torch.int32), gl.sw.view(torch.int32))
    rows = sample_indices(n, 64, 23, must=(0, 127, 128, n - 1))
    wq, sw_ref = oracle.quantize_rowwise(oracle.prune_24(oracle.bf16_bits_to_f32(w_bits[rows])),
                                         "e4m3")
    vals_ref, nib_ref = oracle.compress_24(wq, "e4m3")
    vals, nib = oracle.unpack_physical(packed.cpu().numpy(), n, k)
    assert np.array_equal(vals[rows], vals_ref) and np.array_equal(nib[rows], nib_ref)
    assert np.array_equal(sw.cpu().numpy()[rows].view(np.uint32), sw_ref.view(np.uint32))
    _device_status_clean()


def test_prepare_stress_70b_weight_sampled():
    n, k = 28672, 8192
    w_bits = synthetic.weight(1004 * 100 + 2, n, k, std=0.01)
    packed, sw = S.sfp8_prepare_weight_24(bf16_dev(w_bits), "e4m3")
    rows = sample_indices(n, 48, 29, must=(0, 127, 128, n - 1))
    wq, sw_ref = oracle.quantize_rowwise(oracle.prune_24(oracle.bf16_bits_to_f32(w_bits[rows])),
                                         "e4m3")
    vals_ref, nib_ref = oracle.compress_24(wq, "e4m3")
    vals, nib = oracle.unpack_physical(packed.cpu().numpy(), n, k)
    assert np.array_equal(vals[rows], vals_ref) and np.array_equal(nib[rows], nib_ref)
    assert np.array_equal(sw.cpu().numpy()[rows].view(np.uint32), sw_ref.view(np.uint32))
    _device_status_clean()
