"""GPU parity of the row-wise quantiser (bit-exact codes and scales)."""
import numpy as np
import pytest
import torch

import oracle
import semi_structured_sparse_rowwise_b200 as S
from semi_structured_sparse_rowwise_b200 import synthetic
from gpu_pipeline import bf16_dev, ensure_library, requires_gpu, sample_indices

pytestmark = [pytest.mark.gpu, requires_gpu]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_library()


def _to_dev(x32, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x32))
    return t.to(dtype).cuda()


def _ref_from_dev(xd):
    """Exact float32 widening of the device tensor's values, on the CPU."""
    return xd.float().cpu().numpy()


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_exhaustive_bf16_sweep(fmt):
    mx = np.float32(oracle.fp8_max(fmt))
    v = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) <= mx)]
    width = 256
    v = np.concatenate([v, np.zeros((-v.size) % (width - 1), np.float32)])
    body = v.reshape(-1, width - 1)
    x = np.concatenate([np.full((body.shape[0], 1), mx, np.float32), body], axis=1)
    xd = _to_dev(x, torch.bfloat16)
    q, s = S.sfp8_quantize_rowwise(xd, fmt)
    q_ref, s_ref = oracle.quantize_rowwise(x, fmt)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("fmt,amax", [("e4m3", 300.0), ("e5m2", 39936.0)])
def test_exhaustive_bf16_sweep_scaled(fmt, amax):
    """Every finite bf16 value up to amax in rows whose amax is not FP8_MAX times
    a power of two, so s = amax / FP8_MAX is inexact and the quotients land all
    over the FP8 grid (midpoints included)."""
    mx = np.float32(amax)
    v = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) <= mx)]
    width = 256
    v = np.concatenate([v, np.zeros((-v.size) % (width - 1), np.float32)])
    body = v.reshape(-1, width - 1)
    x = np.concatenate([np.full((body.shape[0], 1), mx, np.float32), body], axis=1)
    xd = _to_dev(x, torch.bfloat16)
    q, s = S.sfp8_quantize_rowwise(xd, fmt)
    q_ref, s_ref = oracle.quantize_rowwise(x, fmt)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_exhaustive_bf16_many_row_scales(fmt):
    """Every finite bf16 value up to the row amax, for row amax values with
    each of the 128 bf16 significands and exponents from 2^-60 to 2^60: the
    quotients x / s fall on, next to and between FP8 rounding midpoints for
    scales of every significand."""
    rng = np.random.default_rng(7 if fmt == "e4m3" else 8)
    sig = (np.arange(128, dtype=np.uint32) | 0x3F80).astype(np.uint32)          # [1, 2)
    amax_bits = list(sig)
    for e in range(-60, 61, 3):
        amax_bits += list(((127 + e) << 7) | rng.integers(0, 128, size=2, dtype=np.uint32))
    amaxes = (np.array(amax_bits, dtype=np.uint32) << 16).view(np.float32)
    v_all = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32)
    v_all = v_all[np.isfinite(v_all)]
    width = 256
    blocks = []
    for a in amaxes:
        v = v_all[np.abs(v_all) <= a]
        v = np.concatenate([v, np.zeros((-v.size) % (width - 1), np.float32)])
        body = v.reshape(-1, width - 1)
        blocks.append(np.concatenate([np.full((body.shape[0], 1), a, np.float32), body], axis=1))
    x = np.concatenate(blocks)
    q, s = S.sfp8_quantize_rowwise(_to_dev(x, torch.bfloat16), fmt)
    q_ref, s_ref = oracle.quantize_rowwise(x, fmt)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)


def _near_midpoint_rows(fmt, seed, n_rows):
    """fp32 rows whose quotients x / s fall within a few units in the last
    place of FP8 rounding midpoints (and on both sides of them)."""
    rng = np.random.default_rng(seed)
    table = oracle.decode_table(fmt)
    pos = np.unique(table[np.isfinite(table) & (table >= 0)])
    mids = (pos[:-1] + pos[1:]) / 2.0
    fmax = np.float32(oracle.fp8_max(fmt))
    rows = []
    for _ in range(n_rows):
        amax = np.float32(rng.uniform(0.5, 3.0) * 2.0 ** int(rng.integers(-20, 20)))
        s = np.float32(amax / fmax)
        base = (mids * np.float64(s)).astype(np.float32)
        cands = [base]
        up, dn = base.copy(), base.copy()
        for _ in range(5):
            up = np.nextafter(up, np.float32(np.inf))
            dn = np.nextafter(dn, np.float32(0.0))
            cands += [up.copy(), dn.copy()]
        v = np.concatenate(cands)
        v = v[np.abs(v) <= amax]
        rows.append(np.concatenate([[amax], v, -v]).astype(np.float32))
    width = (max(r.size for r in rows) + 15) // 16 * 16
    x = np.zeros((len(rows), width), np.float32)
    for i, r in enumerate(rows):
        x[i, :r.size] = r
    return x


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_near_midpoint_quotients(fmt):
    """The quantiser's division-free quotient must be exact next to every FP8
    rounding midpoint: codes equal the oracle's (IEEE fp32 division, then one
    rounding) bit for bit."""
    x = _near_midpoint_rows(fmt, 77 if fmt == "e4m3" else 78, 48)
    q, s = S.sfp8_quantize_rowwise(_to_dev(x, torch.float32), fmt)
    q_ref, s_ref = oracle.quantize_rowwise(x, fmt)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    # the rows do exercise the near-midpoint case: quotients that a 1-ulp
    # error would round differently
    quo = x / s_ref[:, None]
    up = oracle.encode_rne_sat(np.nextafter(quo, np.float32(np.inf)), fmt)
    dn = oracle.encode_rne_sat(np.nextafter(quo, np.float32(-np.inf)), fmt)
    assert int((up != dn).sum()) > 1000


CASES = [
    # rows, cols, torch dtype, distribution
    (16, 128, torch.bfloat16, "normal"),
    (1, 4096, torch.bfloat16, "normal"),
    (4, 4096, torch.bfloat16, "normal"),
    (16, 4096, torch.bfloat16, "normal"),
    (37, 208, torch.bfloat16, "student_t3"),
    (5, 16, torch.bfloat16, "normal"),
    (1000, 4096, torch.bfloat16, "student_t3"),
    (7, 16384, torch.bfloat16, "normal"),
    (3, 65536, torch.bfloat16, "student_t3"),
    (64, 4096, torch.float16, "normal"),
    (33, 1024, torch.float32, "student_t3"),
    (9, 16384, torch.float32, "normal"),
    (3, 32768, torch.float32, "normal"),
]


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("rows,cols,dtype,dist", CASES)
def test_quantize_parity(rows, cols, dtype, dist, fmt):
    bits = synthetic.activation(4242 + rows + cols, rows, cols, dist=dist, zero_row_frac=0.1)
    x32 = oracle.bf16_bits_to_f32(bits) * np.float32(3.0)
    xd = _to_dev(x32, dtype)
    xr = _ref_from_dev(xd)
    q, s = S.sfp8_quantize_rowwise(xd, fmt)
    q_ref, s_ref = oracle.quantize_rowwise(xr, fmt)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_strided_input(fmt):
    bits = synthetic.activation(99, 24, 512, dist="student_t3")
    wide = bf16_dev(bits)
    xd = wide[:, 128:384]                  # ld = 512, cols = 256
    q, s = S.sfp8_quantize_rowwise(xd, fmt)
    q_ref, s_ref = oracle.quantize_rowwise(oracle.bf16_bits_to_f32(bits)[:, 128:384], fmt)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
@pytest.mark.parametrize("rows,cols,ld,dtype", [(300, 256, 512, torch.bfloat16),
                                                (257, 16, 16, torch.bfloat16),
                                                (600, 4096, 4096, torch.float32),
                                                (1000, 8192, 8192, torch.bfloat16),
                                                (700, 6144, 6144, torch.bfloat16)])
def test_streaming_quantiser_shapes(rows, cols, ld, dtype, fmt):
    """Row counts that use the streaming quantiser (one CTA per SM, ring of row
    buffers): strided rows, 32-byte rows, 16 KB rows, ring sizes of 24 and 16
    slots, rows not a multiple of the grid."""
    bits = synthetic.activation(5150 + rows + cols, rows, ld, dist="student_t3", zero_row_frac=0.05)
    x32 = oracle.bf16_bits_to_f32(bits)
    wide = _to_dev(x32, dtype)
    xd = wide[:, :cols]
    xr = _ref_from_dev(xd)
    q, s = S.sfp8_quantize_rowwise(xd, fmt)
    q_ref, s_ref = oracle.quantize_rowwise(xr, fmt)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_zero_and_negative_zero_rows():
    x = np.zeros((4, 64), np.float32)
    x[1, :] = -0.0
    x[2, 7] = -0.0
    x[3, 9] = 1e-30
    for fmt in ("e4m3", "e5m2"):
        q, s = S.sfp8_quantize_rowwise(_to_dev(x, torch.float32), fmt)
        q_ref, s_ref = oracle.quantize_rowwise(x, fmt)
        assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
        assert np.array_equal(q.cpu().numpy(), q_ref)


def test_empty_cols_and_rows():
    xd = torch.empty((5, 0), dtype=torch.bfloat16, device="cuda")
    q, s = S.sfp8_quantize_rowwise(xd, "e4m3")
    _, s_ref = oracle.quantize_rowwise(np.zeros((5, 0), np.float32), "e4m3")
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    q, s = S.sfp8_quantize_rowwise(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"))
    assert q.shape == (0, 64) and s.shape == (0,)


@pytest.mark.parametrize("shape,dtype", [((65536, 4096), torch.bfloat16),
                                         ((16384, 16384), torch.bfloat16),
                                         ((65536, 4096), torch.float32)])
def test_standalone_2p28_sampled(shape, dtype):
    rows, cols = shape
    g = torch.Generator(device="cpu").manual_seed(1004)
    # the full tensor is generated on the CPU with numpy, like every input
    bits = synthetic.activation(1004 * 100 + rows % 97, rows, cols, dist="normal")
    xd = bf16_dev(bits).to(dtype)
    q, s = S.sfp8_quantize_rowwise(xd, "e4m3")
    sel = sample_indices(rows, 96, 5, must=(0, rows - 1))
    q_ref, s_ref = oracle.quantize_rowwise(oracle.bf16_bits_to_f32(bits[sel]), "e4m3")
    st = torch.from_numpy(sel).cuda()
    assert np.array_equal(s.index_select(0, st).cpu().numpy().view(np.uint32),
                          s_ref.view(np.uint32))
    assert np.array_equal(q.index_select(0, st).cpu().numpy(), q_ref)
    # every row: max |code| is reached (the amax element maps to +-FP8_MAX)
    mags = (q & 0x7F).max(dim=1).values
    assert bool((mags == 0x7E).all())
