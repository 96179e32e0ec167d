"""GPU parity of the tensor-wise quantiser (one global amax): codes and the
scale bit-exact against the oracle, in both amax modes (per-block partials
reduced, and one word folded with atomic max), for every input dtype and
both FP8 formats.

Sizes: empty, a few elements (all in the scalar tail), one tile, the pages'
65500-element case (a ragged tail), sizes that span many tiles and CTAs with
a ragged tail, and the pages' largest case (2.68e8 elements, bf16 and fp32)
checked on sampled elements: a sub-tensor that holds the global-maximum
element has the whole tensor's scale, so the oracle quantises that
sub-tensor to give the expected codes of the sampled elements.
"""
import numpy as np
import pytest
import torch

import oracle
import semi_structured_sparse_rowwise_b200 as S
from semi_structured_sparse_rowwise_b200 import synthetic
from gpu_pipeline import ensure_library, requires_gpu

pytestmark = [pytest.mark.gpu, requires_gpu]

TORCH = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_library()


def _input(numel, dtype, seed, dist="student_t3"):
    """Seeded values (Student-t by default: heavy tails stress the amax),
    widened exactly to float32 on the CPU from the device tensor."""
    rng = synthetic.rng_for(seed)
    if dist == "student_t3":
        x = rng.standard_t(3, size=numel).astype(np.float32)
    else:
        x = rng.standard_normal(numel, dtype=np.float32)
    xd = torch.from_numpy(x).to(TORCH[dtype]).cuda()
    return xd


def _check(xd, fmt, mode, q, s):
    x32 = xd.float().cpu().numpy()
    q_ref, s_ref = oracle.quantize_tensorwise(x32, fmt)
    assert np.float32(s.item()).view(np.uint32) == np.float32(s_ref).view(np.uint32)
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("mode", ["reduce", "atomic"])
@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("dtype", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("numel", [1, 7, 16, 4096, 65500, (1 << 20) + 3, 5_000_011])
def test_parity(numel, dtype, fmt, mode):
    xd = _input(numel, dtype, seed=3000 + numel % 997)
    q, s = S.sfp8_quantize_tensorwise(xd, fmt, mode)
    _check(xd, fmt, mode, q, s)
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == 0 and flags == 0


@pytest.mark.parametrize("mode", ["reduce", "atomic"])
def test_empty_tensor_gives_guard_scale(mode):
    xd = torch.empty((0,), dtype=torch.bfloat16, device="cuda")
    q, s = S.sfp8_quantize_tensorwise(xd, "e4m3", mode)
    _, s_ref = oracle.quantize_tensorwise(np.zeros((0,), np.float32), "e4m3")
    assert q.numel() == 0
    assert np.float32(s.item()).view(np.uint32) == np.float32(s_ref).view(np.uint32)


@pytest.mark.parametrize("mode", ["reduce", "atomic"])
def test_zero_tensor_keeps_signed_zeros(mode):
    x = np.zeros(4096 + 5, np.float32)
    x[1::2] = -0.0
    xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
    q, s = S.sfp8_quantize_tensorwise(xd, "e4m3", mode)
    _check(xd, "e4m3", mode, q, s)


@pytest.mark.parametrize("mode", ["reduce", "atomic"])
def test_consecutive_calls_share_workspace(mode):
    """The grid barrier and the atomic word are reset by each call: a
    smaller-amax tensor after a larger one gets its own scale, several times
    over, on one workspace."""
    ws = S.new_tensorwise_workspace(mode, torch.device("cuda"))
    for i, scale in enumerate([100.0, 0.01, 7.0, 1e-3]):
        xd = _input(3_000_017 - 1000 * i, "bf16", seed=4000 + i) * scale
        q, s = S.sfp8_quantize_tensorwise(xd, "e5m2" if i % 2 else "e4m3", mode, workspace=ws)
        _check(xd, "e5m2" if i % 2 else "e4m3", mode, q, s)
    if mode == "atomic":
        assert S.sfp8_quantize_tensorwise_workspace_bytes("atomic") == 64
    words = ws[:16].view(torch.int32).cpu().numpy()
    assert words[0] == 0 and words[2] == 0          # arrival count, atomic word: zero


def test_modes_agree_bitwise():
    xd = _input(10_000_019, "f32", seed=4100, dist="normal")
    q1, s1 = S.sfp8_quantize_tensorwise(xd, "e4m3", "reduce")
    q2, s2 = S.sfp8_quantize_tensorwise(xd, "e4m3", "atomic")
    assert torch.equal(q1, q2) and torch.equal(s1.view(torch.int32), s2.view(torch.int32))


def test_amax_element_anywhere():
    """The global maximum placed in the first element, the last vector and
    the scalar tail in turn: every CTA's partial reaches the scale."""
    n = 2_000_003
    base = _input(n, "f32", seed=4200, dist="normal")
    for pos in (0, n // 2 + 1, n - 9, n - 1):
        xd = base.clone()
        xd[pos] = -1000.0
        q, s = S.sfp8_quantize_tensorwise(xd, "e4m3", "atomic")
        _check(xd, "e4m3", "atomic", q, s)
        q2, s2 = S.sfp8_quantize_tensorwise(xd, "e4m3", "reduce")
        assert torch.equal(q, q2) and torch.equal(s.view(torch.int32), s2.view(torch.int32))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_full_size_sampled(dtype):
    """2^28 elements (the pages' largest conversion case), both modes: the
    scale exactly, the codes of 2^20 sampled elements and the tail exactly."""
    numel = 1 << 28
    g = torch.Generator(device="cuda").manual_seed(4300)
    xd = torch.randn(numel, generator=g, device="cuda", dtype=torch.float32).to(TORCH[dtype])
    x32 = xd.float().cpu().numpy()
    imax = int(np.argmax(np.abs(x32)))
    rng = synthetic.rng_for(4301)
    idx = np.unique(np.concatenate([rng.integers(0, numel, size=1 << 20),
                                    np.arange(numel - 64, numel)]))
    sub = np.concatenate([x32[imax:imax + 1], x32[idx]])
    q_sub, s_ref = oracle.quantize_tensorwise(sub, "e4m3")
    for mode in ("reduce", "atomic"):
        q, s = S.sfp8_quantize_tensorwise(xd, "e4m3", mode)
        assert np.float32(s.item()).view(np.uint32) == np.float32(s_ref).view(np.uint32)
        qi = q[torch.from_numpy(idx).cuda()].cpu().numpy()
        assert np.array_equal(qi, q_sub[1:])
        del q
    st, flags = S.sfp8_read_device_status(clear=True)
    assert st == 0 and flags == 0
