"""The C-ABI library builds, loads and exports every symbol that
include/sfp8.h declares; host-side validation answers without a GPU.

None of these tests launches a kernel.
"""
import ctypes
import os
import re

import pytest

import oracle
from semi_structured_sparse_rowwise_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sfp8.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sfp8_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("sfp8_quantize_rowwise", "sfp8_compress_24", "sfp8_sparse_linear"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert names, "no declarations parsed"
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(binding.SIGNATURES), (set(names) ^ set(binding.SIGNATURES))


def test_layout_constants_match(lib):
    assert lib.sfp8_layout_version() == 3 == oracle.layout.LAYOUT_VERSION
    for n in (0, 1, 127, 128, 129, 14336, 28672):
        assert lib.sfp8_padded_rows(n) == oracle.padded_rows(n)
        for k in (128, 4096, 14336):
            assert lib.sfp8_compressed_bytes(n, k) == oracle.packed_bytes(n, k)
            npad = oracle.padded_rows(n)
            assert lib.sfp8_compressed_values_bytes(n, k) == npad * k // 2
            assert lib.sfp8_compressed_meta_bytes(n, k) == npad * k // 8
            assert (lib.sfp8_compressed_values_bytes(n, k) + lib.sfp8_compressed_meta_bytes(n, k)
                    == lib.sfp8_compressed_bytes(n, k))


def test_status_strings(lib):
    for code in range(10):
        s = lib.sfp8_status_string(code)
        assert s and s != b"unknown status"
    assert lib.sfp8_status_string(99) == b"unknown status"


FAKE = ctypes.c_void_p(0x10000)        # never dereferenced: rejected before use
FAKE_ODD = ctypes.c_void_p(0x10001)


def test_quantize_validation_without_gpu(lib):
    q = lib.sfp8_quantize_rowwise
    assert q(FAKE, 9, 4, 16, 16, FAKE, 3, FAKE, None) == 4       # bad input dtype
    assert q(FAKE, 0, 4, 16, 16, FAKE, 0, FAKE, None) == 4       # bf16 output
    assert q(FAKE, 0, -1, 16, 16, FAKE, 3, FAKE, None) == 1      # negative rows
    assert q(FAKE, 0, 4, 16, 8, FAKE, 3, FAKE, None) == 1        # ld < cols
    assert q(FAKE, 0, 4, 24, 24, FAKE, 3, FAKE, None) == 2       # cols % 16
    assert q(FAKE, 0, 0, 16, 16, FAKE, 3, FAKE, None) == 0       # empty: no-op
    assert q(None, 0, 4, 16, 16, FAKE, 3, FAKE, None) == 1       # null x
    assert q(FAKE_ODD, 0, 4, 16, 16, FAKE, 3, FAKE, None) == 3   # misaligned x
    assert q(FAKE, 0, 4, 16, 20, FAKE, 3, FAKE, None) == 3       # ld*2 % 16


def test_quantize_tensorwise_validation_without_gpu(lib):
    q = lib.sfp8_quantize_tensorwise
    ws = 1 << 20
    assert q(FAKE, 9, 64, FAKE, 3, FAKE, 0, FAKE, ws, None) == 4       # bad input dtype
    assert q(FAKE, 0, 64, FAKE, 2, FAKE, 0, FAKE, ws, None) == 4       # f32 output
    assert q(FAKE, 0, 64, FAKE, 3, FAKE, 2, FAKE, ws, None) == 1       # unknown mode
    assert q(FAKE, 0, -1, FAKE, 3, FAKE, 0, FAKE, ws, None) == 1       # negative numel
    assert q(None, 0, 64, FAKE, 3, FAKE, 0, FAKE, ws, None) == 1       # null x
    assert q(FAKE, 0, 64, FAKE, 3, None, 0, FAKE, ws, None) == 1       # null scale
    assert q(FAKE, 0, 64, FAKE, 3, FAKE, 1, None, ws, None) == 1       # null workspace
    assert q(FAKE_ODD, 0, 64, FAKE, 3, FAKE, 0, FAKE, ws, None) == 3   # misaligned x
    assert q(FAKE, 0, 64, FAKE_ODD, 3, FAKE, 0, FAKE, ws, None) == 3   # misaligned q
    assert q(FAKE, 0, 1 << 41, FAKE, 3, FAKE, 0, FAKE, ws, None) == 2  # too large
    assert lib.sfp8_quantize_tensorwise_workspace_bytes(7) == 0


def test_host_path_validation_without_gpu(lib):
    f = lib.sfp8_sparse_linear_quant_host
    # an fp8 activation input is rejected before any device is touched
    assert f(FAKE, FAKE, 3, 3, FAKE, FAKE, 16, FAKE, 3, FAKE, 64, 128, None, FAKE, FAKE,
             FAKE, 0, None) == 4

def test_prune_compress_validation_without_gpu(lib):
    assert lib.sfp8_prune_24(FAKE, 3, 4, 16, 16, FAKE, None) == 4
    assert lib.sfp8_prune_24(FAKE, 0, 4, 20, 20, FAKE, None) == 2
    assert lib.sfp8_prune_24(FAKE, 0, 4, 16, 32, FAKE, None) == 1   # in place needs ld == cols
    assert lib.sfp8_compress_24(FAKE, 0, 4, 128, FAKE, None) == 4
    assert lib.sfp8_compress_24(FAKE, 3, 4, 192, FAKE, None) == 2
    assert lib.sfp8_compress_24(FAKE, 3, 4, 0, FAKE, None) == 2
    assert lib.sfp8_compress_24(FAKE, 3, 0, 128, FAKE, None) == 0
    assert lib.sfp8_compress_24(FAKE_ODD, 3, 4, 128, FAKE, None) == 3
    assert lib.sfp8_compress_24(FAKE, 3, 4, 128, FAKE_ODD, None) == 3
    assert lib.sfp8_decompress_24(FAKE, 4, 100, FAKE, None) == 2


def test_prepare_weight_validation_without_gpu(lib):
    f = lib.sfp8_prepare_weight_24
    assert f(FAKE, 0, 4, 128, 128, 0, FAKE, FAKE, None) == 4        # codes must be FP8
    assert f(FAKE, 3, 4, 128, 128, 3, FAKE, FAKE, None) == 4        # input must be wide
    assert f(FAKE, 0, 4, 192, 192, 3, FAKE, FAKE, None) == 2        # k % 128
    assert f(FAKE, 0, 4, 0, 0, 3, FAKE, FAKE, None) == 2
    assert f(FAKE, 0, 4, 128, 64, 3, FAKE, FAKE, None) == 1         # ld < k
    assert f(FAKE, 0, 0, 128, 128, 3, FAKE, FAKE, None) == 0        # nothing to do
    assert f(FAKE, 0, 4, 128, 128, 3, FAKE, None, None) == 1        # no scales
    assert f(FAKE_ODD, 0, 4, 128, 128, 3, FAKE, FAKE, None) == 3
    assert f(FAKE, 0, 4, 128, 132, 3, FAKE, FAKE, None) == 3        # row stride 264 bytes
    assert f(FAKE, 0, 4, 128, 128, 3, FAKE_ODD, FAKE, None) == 3


def test_linear_validation_without_gpu(lib):
    f = lib.sfp8_sparse_linear
    args = [FAKE, 3, FAKE, 16, FAKE, 3, FAKE, 64, 128, None, FAKE, FAKE, 1 << 20, None]

    def call(**kw):
        a = list(args)
        names = ["a_q", "a_dt", "s_a", "m", "packed", "w_dt", "s_w", "n", "k", "bias",
                 "y", "ws", "wsb", "stream"]
        for key, v in kw.items():
            a[names.index(key)] = v
        return f(*a)
    assert call(a_dt=0) == 4
    assert call(w_dt=2) == 4
    assert call(k=0) == 2
    assert call(k=192) == 2
    assert call(m=-1) == 1
    assert call(m=0) == 0
    assert call(n=0) == 0
    assert call(a_q=None) == 1
    assert call(y=None) == 1
    assert call(a_q=FAKE_ODD) == 3
    assert call(bias=FAKE_ODD) == 3
    assert call(s_w=ctypes.c_void_p(0x10002)) == 3
    assert call(packed=FAKE_ODD) == 3
    na = lib.sfp8_sparse_linear_noalloc
    assert na(FAKE, 0, FAKE, 16, FAKE, 3, FAKE, 64, 128, None, FAKE, None) == 4
    assert na(FAKE, 3, FAKE, 16, FAKE, 3, FAKE, 64, 0, None, FAKE, None) == 2
    assert na(FAKE, 3, FAKE, 0, FAKE, 3, FAKE, 64, 128, None, FAKE, None) == 0
    qargs = [FAKE, 0, 128, 3, FAKE, FAKE, 16, FAKE, 3, FAKE, 64, 128, None, FAKE, FAKE,
             1 << 20, None]
    for entry in ("sfp8_sparse_linear_quant", "sfp8_sparse_linear_quant_fused",
                  "sfp8_sparse_linear_quant_chained"):
        fq = getattr(lib, entry)

        def qcall(**kw):
            a = list(qargs)
            names = ["x", "x_dt", "ld_x", "a_dt", "a_q", "s_a", "m", "packed", "w_dt", "s_w",
                     "n", "k", "bias", "y", "ws", "wsb", "stream"]
            for key, v in kw.items():
                a[names.index(key)] = v
            return fq(*a)
        assert qcall(x_dt=3) == 4          # x must be bf16 / f16 / f32
        assert qcall(ld_x=64) == 1         # ld_x < k
        assert qcall(a_dt=0) == 4          # a_q must be FP8
        assert qcall(k=192, ld_x=192) == 2
        assert qcall(m=0) == 0
    # host-only query: invalid sizes (and no device here) answer 0
    assert lib.sfp8_sparse_linear_quant_fusable(16, 14336, 100) == 0
    assert lib.sfp8_sparse_linear_quant_fusable(0, 14336, 4096) == 0


@pytest.mark.parametrize("entry", ["sfp8_sparse_linear", "sfp8_sparse_linear_noalloc",
                                   "sfp8_sparse_linear_algo"])
def test_linear_wrappers_reject_bad_arguments_without_gpu(lib, entry):
    """The binding's sparse linear wrappers check a_q's width, the bias and the
    output tensor before any call reaches the library (CPU tensors; nothing
    launches)."""
    import torch
    from semi_structured_sparse_rowwise_b200 import binding as B
    m, n, k = 4, 64, 256
    a_q = torch.zeros((m, k), dtype=torch.uint8)
    s = torch.ones((max(m, n),), dtype=torch.float32)
    packed = torch.zeros((16,), dtype=torch.uint8)
    extra = (0,) if entry == "sfp8_sparse_linear_algo" else ()
    f = getattr(B, entry)

    def call(a=a_q, bias=None, out=None):
        return f(a, "e4m3", s[:m], packed, "e4m3", s[:n], n, k, *extra, bias=bias, out=out)

    with pytest.raises(ValueError, match="columns"):
        call(a=torch.zeros((m, k - 128), dtype=torch.uint8))          # fewer than k columns
    with pytest.raises(ValueError, match="uint8"):
        call(a=torch.zeros((m, 2 * k), dtype=torch.uint8)[:, :k])     # not contiguous
    with pytest.raises(ValueError, match="bias"):
        call(bias=torch.zeros((n,), dtype=torch.float32))            # fp32 bias
    with pytest.raises(ValueError, match="bias"):
        call(bias=torch.zeros((n - 1,), dtype=torch.bfloat16))       # short bias
    with pytest.raises(ValueError, match="out"):
        call(out=torch.zeros((m, n), dtype=torch.float32))           # fp32 out
    with pytest.raises(ValueError, match="out"):
        call(out=torch.zeros((m, n + 1), dtype=torch.bfloat16))      # wrong shape
    with pytest.raises(ValueError, match="out"):
        call(out=torch.zeros((n, m), dtype=torch.bfloat16).t())      # not contiguous
    with pytest.raises(ValueError, match="CUDA"):
        call()                                                       # well-formed, on the CPU


@pytest.mark.parametrize("entry", ["sfp8_sparse_linear_quant", "sfp8_sparse_linear_quant_fused",
                                   "sfp8_sparse_linear_quant_chained"])
def test_quant_wrappers_reject_bad_outputs_without_gpu(lib, entry):
    """The one-call forward's wrappers check x, the bias and every output
    tensor they are given (y, a_q, s_a) before any call reaches the library
    (CPU tensors; nothing launches)."""
    import torch
    from semi_structured_sparse_rowwise_b200 import binding as B
    m, n, k = 4, 64, 256
    x = torch.zeros((m, k), dtype=torch.bfloat16)
    s_w = torch.ones((n,), dtype=torch.float32)
    packed = torch.zeros((16,), dtype=torch.uint8)
    f = getattr(B, entry)

    def call(x=x, **kw):
        return f(x, "e4m3", packed, "e4m3", s_w, n, k, **kw)

    with pytest.raises(ValueError, match="columns"):
        call(x=torch.zeros((m, k - 128), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="dtype"):
        call(x=torch.zeros((m, k), dtype=torch.int16))
    with pytest.raises(ValueError, match="bias"):
        call(bias=torch.zeros((n,), dtype=torch.float32))
    with pytest.raises(ValueError, match="out"):
        call(out=torch.zeros((m, n + 1), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="a_q"):
        call(a_q=torch.zeros((m, k - 1), dtype=torch.uint8))
    with pytest.raises(ValueError, match="a_q"):
        call(a_q=torch.zeros((m, 2 * k), dtype=torch.uint8)[:, :k])
    with pytest.raises(ValueError, match="s_a"):
        call(s_a=torch.zeros((m,), dtype=torch.float64))
    with pytest.raises(ValueError, match="CUDA"):
        call()                                                       # well-formed, on the CPU


def test_host_wrapper_rejects_bad_buffers_without_gpu(lib):
    """sfp8_sparse_linear_quant_host's wrapper checks the shapes, dtypes and
    layout of its host and staging buffers before any call reaches the
    library (CPU tensors; nothing launches)."""
    import torch
    from semi_structured_sparse_rowwise_b200 import binding as B
    m, n, k = 4, 64, 256
    bf = torch.bfloat16

    def call(x_host=None, x_dev=None, y_dev=None, y_host=None):
        return B.sfp8_sparse_linear_quant_host(
            torch.zeros((m, k), dtype=bf) if x_host is None else x_host, "e4m3",
            torch.zeros((16,), dtype=torch.uint8), "e4m3", torch.ones((n,)), n, k,
            torch.zeros((m, k), dtype=bf) if x_dev is None else x_dev,
            torch.zeros((m, k), dtype=torch.uint8), torch.ones((m,)),
            torch.zeros((m, n), dtype=bf) if y_dev is None else y_dev,
            torch.zeros((m, n), dtype=bf) if y_host is None else y_host,
            torch.zeros((16,), dtype=torch.uint8))

    with pytest.raises(ValueError, match="shapes"):
        call(y_dev=torch.zeros((m, n + 1), dtype=bf))
    with pytest.raises(ValueError, match="shapes"):
        call(y_dev=torch.zeros((m, n), dtype=torch.float32))
    with pytest.raises(ValueError, match="contiguous"):
        call(y_dev=torch.zeros((n, m), dtype=bf).t())
    with pytest.raises(ValueError, match="shapes"):
        call(y_host=torch.zeros((m, n - 1), dtype=bf))
    with pytest.raises(ValueError, match="dtype"):
        call(x_host=torch.zeros((m, k), dtype=torch.float16))
    with pytest.raises(ValueError, match="CUDA"):
        call()                                                       # well-formed, on the CPU


def test_workspace_size_is_counted_in_bytes():
    """A caller's workspace of any dtype is passed as its size in bytes; a
    non-contiguous or CPU workspace is refused before any call."""
    import torch
    from semi_structured_sparse_rowwise_b200 import binding as B
    with pytest.raises(ValueError, match="workspace"):
        B._ws_bytes(torch.zeros((64,), dtype=torch.uint8), "cpu")
    if torch.cuda.is_available():
        w = torch.zeros((16,), dtype=torch.float32, device="cuda")
        assert B._ws_bytes(w, w.device) == 64
        with pytest.raises(ValueError, match="workspace"):
            B._ws_bytes(torch.zeros((8, 8), device="cuda").t(), w.device)


@pytest.mark.parametrize("entry", ["sfp8_sparse_linear_quant", "sfp8_sparse_linear_quant_fused",
                                   "sfp8_sparse_linear_quant_chained"])
def test_quant_entry_points_refuse_outputs_overlapping_x(lib, entry):
    """x is read while a_q, s_a and y are written: an output sharing bytes
    with x's span (rows 0..m-1 at stride ld_x) is refused with
    SFP8_ERR_INVALID_ARG before any device is touched; disjoint buffers pass
    on to the device checks (no device here: SFP8_ERR_CUDA or _ARCH)."""
    f = getattr(lib, entry)
    X = 0x100000
    m, k, n = 16, 256, 64

    def call(a_q, s_a, y, ld=k):
        return f(ctypes.c_void_p(X), 0, ld, 3, ctypes.c_void_p(a_q), ctypes.c_void_p(s_a), m,
                 ctypes.c_void_p(0x900000), 3, ctypes.c_void_p(0xA00000), n, k, None,
                 ctypes.c_void_p(y), ctypes.c_void_p(0xB00000), 1 << 20, None)
    x_end = X + m * k * 2
    assert call(0x200000, 0x300000, 0x400000) in (5, 7)              # disjoint
    assert call(X + 256, 0x300000, 0x400000) == 1                    # a_q inside x
    assert call(0x200000, x_end - 4, 0x400000) == 1                  # s_a's first bytes in x
    assert call(0x200000, x_end, 0x400000) in (5, 7)                 # s_a right after x
    assert call(0x200000, 0x300000, X - m * n * 2 + 2) == 1          # y's last bytes in x
    assert call(0x200000, 0x300000, X - m * n * 2) in (5, 7)         # y right before x
    # x with row stride 512: its span ends with row 15's 256 values (X + 15872)
    assert call(X + 14 * 1024 + 512, 0x300000, 0x400000, ld=512) == 1   # inside the span
    assert call(X + 15 * 1024 + 512, 0x300000, 0x400000, ld=512) in (5, 7)   # right after it
