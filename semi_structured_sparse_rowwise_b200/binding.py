"""Thin Python binding of libsfp8.so (ctypes).

Argument marshalling only: tensors are passed as raw device pointers with
their sizes, on torch's current CUDA stream.  Every step of the layer runs in
the library's CUDA kernels; there is no fallback of any kind.  If the library
is missing or fails to load, every call raises.

The functions carry the C names (``sfp8_quantize_rowwise`` and so on) and
allocate their outputs with torch when none are given.
"""

import ctypes
import os

import torch

from . import build as _build

OK = 0
STATUS_NAMES = {
    0: "SFP8_OK", 1: "SFP8_ERR_INVALID_ARG", 2: "SFP8_ERR_UNSUPPORTED_SHAPE",
    3: "SFP8_ERR_MISALIGNED", 4: "SFP8_ERR_UNSUPPORTED_DTYPE", 5: "SFP8_ERR_ARCH",
    6: "SFP8_ERR_WORKSPACE", 7: "SFP8_ERR_CUDA", 8: "SFP8_ERR_TIMEOUT",
    9: "SFP8_ERR_DEVICE_CHECK",
}
DTYPE = {"bf16": 0, "f16": 1, "f32": 2, "e4m3": 3, "e5m2": 4}
TORCH_WIDE = {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32"}
AMAX_MODE = {"reduce": 0, "atomic": 1}
DEVICE_TIMEOUT = 0x1
DEVICE_CHECK_FAIL = 0x2

# Every symbol declared in include/sfp8.h, with its C signature.
_c_void_p, _i64, _sz, _i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
SIGNATURES = {
    "sfp8_quantize_rowwise": (_i32, [_c_void_p, _i32, _i64, _i64, _i64, _c_void_p, _i32,
                                     _c_void_p, _c_void_p]),
    "sfp8_quantize_tensorwise_workspace_bytes": (_sz, [_i32]),
    "sfp8_quantize_tensorwise": (_i32, [_c_void_p, _i32, _i64, _c_void_p, _i32, _c_void_p, _i32,
                                        _c_void_p, _sz, _c_void_p]),
    "sfp8_prune_24": (_i32, [_c_void_p, _i32, _i64, _i64, _i64, _c_void_p, _c_void_p]),
    "sfp8_padded_rows": (_i64, [_i64]),
    "sfp8_compressed_bytes": (_sz, [_i64, _i64]),
    "sfp8_compressed_values_bytes": (_sz, [_i64, _i64]),
    "sfp8_compressed_meta_bytes": (_sz, [_i64, _i64]),
    "sfp8_compress_24": (_i32, [_c_void_p, _i32, _i64, _i64, _c_void_p, _c_void_p]),
    "sfp8_decompress_24": (_i32, [_c_void_p, _i64, _i64, _c_void_p, _c_void_p]),
    "sfp8_prepare_weight_24": (_i32, [_c_void_p, _i32, _i64, _i64, _i64, _i32, _c_void_p,
                                      _c_void_p, _c_void_p]),
    "sfp8_sparse_linear_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "sfp8_workspace_clear": (_i32, [_c_void_p, _sz, _c_void_p]),
    "sfp8_sparse_linear": (_i32, [_c_void_p, _i32, _c_void_p, _i64, _c_void_p, _i32,
                                  _c_void_p, _i64, _i64, _c_void_p, _c_void_p, _c_void_p, _sz,
                                  _c_void_p]),
    "sfp8_sparse_linear_noalloc": (_i32, [_c_void_p, _i32, _c_void_p, _i64, _c_void_p,
                                          _i32, _c_void_p, _i64, _i64, _c_void_p,
                                          _c_void_p, _c_void_p]),
    "sfp8_sparse_linear_algo_count": (_i32, [_i64, _i64, _i64]),
    "sfp8_sparse_linear_algo_info": (_i32, [_i64, _i64, _i64, _i32,
                                            ctypes.POINTER(ctypes.c_int32)]),
    "sfp8_sparse_linear_algo_workspace_bytes": (_sz, [_i64, _i64, _i64, _i32]),
    "sfp8_sparse_linear_plan_count": (_i32, [_i64, _i64, _i64, _i32]),
    "sfp8_sparse_linear_plan_info": (_i32, [_i64, _i64, _i64, _i32, _i32,
                                            ctypes.POINTER(ctypes.c_int64)]),
    "sfp8_sparse_linear_search_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "sfp8_sparse_linear_algo": (_i32, [_c_void_p, _i32, _c_void_p, _i64, _c_void_p, _i32,
                                       _c_void_p, _i64, _i64, _c_void_p, _c_void_p, _i32,
                                       _c_void_p, _sz, _c_void_p]),
    "sfp8_sparse_linear_search": (_i32, [_c_void_p, _i32, _c_void_p, _i64, _c_void_p, _i32,
                                         _c_void_p, _i64, _i64, _c_void_p, _c_void_p,
                                         _c_void_p, _sz, _c_void_p, _sz, _i32,
                                         ctypes.POINTER(ctypes.c_int32),
                                         ctypes.POINTER(ctypes.c_float), _i32, _c_void_p]),
    "sfp8_sparse_linear_set_algo": (_i32, [_i64, _i64, _i64, _i32]),
    "sfp8_sparse_linear_get_algo": (_i32, [_i64, _i64, _i64]),
    "sfp8_sparse_linear_quant_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "sfp8_sparse_linear_quant": (_i32, [_c_void_p, _i32, _i64, _i32, _c_void_p, _c_void_p,
                                        _i64, _c_void_p, _i32, _c_void_p, _i64, _i64,
                                        _c_void_p, _c_void_p, _c_void_p, _sz, _c_void_p]),
    "sfp8_sparse_linear_quant_fused": (_i32, [_c_void_p, _i32, _i64, _i32, _c_void_p,
                                              _c_void_p, _i64, _c_void_p, _i32, _c_void_p,
                                              _i64, _i64, _c_void_p, _c_void_p, _c_void_p,
                                              _sz, _c_void_p]),
    "sfp8_sparse_linear_quant_chained": (_i32, [_c_void_p, _i32, _i64, _i32, _c_void_p,
                                                _c_void_p, _i64, _c_void_p, _i32, _c_void_p,
                                                _i64, _i64, _c_void_p, _c_void_p, _c_void_p,
                                                _sz, _c_void_p]),
    "sfp8_sparse_linear_quant_fusable": (_i32, [_i64, _i64, _i64]),
    "sfp8_selftest_timeout": (_i32, [_c_void_p]),
    "sfp8_sparse_linear_quant_host": (_i32, [_c_void_p, _c_void_p, _i32, _i32, _c_void_p,
                                             _c_void_p, _i64, _c_void_p, _i32, _c_void_p, _i64,
                                             _i64, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                             _sz, _c_void_p]),
    "sfp8_read_device_status": (_i32, [ctypes.POINTER(ctypes.c_uint32), _i32]),
    "sfp8_last_device_status": (_i32, []),
    "sfp8_status_string": (ctypes.c_char_p, [_i32]),
    "sfp8_layout_version": (_i32, []),
}

_LIB = None


class Sfp8Error(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (what, STATUS_NAMES.get(status, "?"), status))


def library_path():
    return _build.LIB_PATH


def load_library():
    """Loads libsfp8.so from the package directory (raises if absent)."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise ImportError(
                "libsfp8.so is not built (%s); run "
                "`python -m semi_structured_sparse_rowwise_b200.build`" % path)
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def _check(status, what):
    if status != OK:
        raise Sfp8Error(status, what)


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _fp8_name(d):
    if d not in ("e4m3", "e5m2"):
        raise ValueError("fp8 dtype must be 'e4m3' or 'e5m2'")
    return d


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors")


def _ws_bytes(ws, device):
    """Size in bytes of a caller's workspace (any dtype), which must be a
    contiguous CUDA tensor on `device`."""
    if not ws.is_cuda or ws.device != torch.device(device) or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor on %s" % (device,))
    return ws.numel() * ws.element_size()


def sfp8_quantize_rowwise(x, q_dtype="e4m3", q=None, scales=None):
    """x [rows, cols] bf16/f16/f32 (unit column stride) -> (q uint8, scales f32)."""
    lib = load_library()
    _require_cuda(x)
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    rows, cols = x.shape
    xd = TORCH_WIDE.get(x.dtype)
    if xd is None:
        raise ValueError("x dtype must be bfloat16, float16 or float32")
    if q is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((rows,), dtype=torch.float32, device=x.device)
    ld = x.stride(0) if rows > 1 else cols
    with torch.cuda.device(x.device):
        st = lib.sfp8_quantize_rowwise(_ptr(x), DTYPE[xd], rows, cols, ld, _ptr(q),
                                       DTYPE[_fp8_name(q_dtype)], _ptr(scales), _stream(x.device))
    _check(st, "sfp8_quantize_rowwise")
    return q, scales


def sfp8_quantize_tensorwise_workspace_bytes(mode="reduce", device=None):
    lib = load_library()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        return int(lib.sfp8_quantize_tensorwise_workspace_bytes(AMAX_MODE[mode]))


def new_tensorwise_workspace(mode, device):
    """A zeroed workspace for sfp8_quantize_tensorwise on `device`."""
    nbytes = sfp8_quantize_tensorwise_workspace_bytes(mode, device)
    return torch.zeros((max(nbytes, 16),), dtype=torch.uint8, device=device)


def sfp8_quantize_tensorwise(x, q_dtype="e4m3", mode="reduce", q=None, scale=None,
                             workspace=None):
    """x (any shape, contiguous) bf16/f16/f32 -> (q uint8 of x's shape, scale f32 [1]):
    one scale for the whole tensor, the global amax found by `mode`
    ('reduce': per-block partials, 'atomic': one word with atomic max)."""
    lib = load_library()
    _require_cuda(x)
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    xd = TORCH_WIDE.get(x.dtype)
    if xd is None:
        raise ValueError("x dtype must be bfloat16, float16 or float32")
    if mode not in AMAX_MODE:
        raise ValueError("mode must be 'reduce' or 'atomic'")
    if q is None:
        q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scale is None:
        scale = torch.empty((1,), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = new_tensorwise_workspace(mode, x.device)
    with torch.cuda.device(x.device):
        st = lib.sfp8_quantize_tensorwise(_ptr(x), DTYPE[xd], x.numel(), _ptr(q),
                                          DTYPE[_fp8_name(q_dtype)], _ptr(scale),
                                          AMAX_MODE[mode], _ptr(workspace),
                                          _ws_bytes(workspace, x.device),
                                          _stream(x.device))
    _check(st, "sfp8_quantize_tensorwise")
    return q, scale


def sfp8_prune_24(w, out=None):
    """2:4 magnitude prune along rows; w [rows, cols] bf16/f16/f32."""
    lib = load_library()
    _require_cuda(w)
    if w.dim() != 2 or w.stride(1) != 1:
        raise ValueError("w must be 2-D with unit column stride")
    wd = TORCH_WIDE.get(w.dtype)
    if wd is None:
        raise ValueError("w dtype must be bfloat16, float16 or float32")
    rows, cols = w.shape
    if out is None:
        out = torch.empty((rows, cols), dtype=w.dtype, device=w.device)
    ld = w.stride(0) if rows > 1 else cols
    with torch.cuda.device(w.device):
        st = lib.sfp8_prune_24(_ptr(w), DTYPE[wd], rows, cols, ld, _ptr(out), _stream(w.device))
    _check(st, "sfp8_prune_24")
    return out


def sfp8_padded_rows(n):
    return int(load_library().sfp8_padded_rows(n))


def sfp8_compressed_bytes(n, k):
    return int(load_library().sfp8_compressed_bytes(n, k))


def sfp8_compress_24(w_q, w_dtype="e4m3", packed=None):
    """w_q [n, k] uint8 FP8 codes -> packed compressed weight (layout v3)."""
    lib = load_library()
    _require_cuda(w_q)
    if w_q.dim() != 2 or not w_q.is_contiguous() or w_q.dtype != torch.uint8:
        raise ValueError("w_q must be a contiguous 2-D uint8 tensor")
    n, k = w_q.shape
    if packed is None:
        packed = torch.empty((lib.sfp8_compressed_bytes(n, k),), dtype=torch.uint8,
                             device=w_q.device)
    with torch.cuda.device(w_q.device):
        st = lib.sfp8_compress_24(_ptr(w_q), DTYPE[_fp8_name(w_dtype)], n, k, _ptr(packed),
                                  _stream(w_q.device))
    _check(st, "sfp8_compress_24")
    return packed


def sfp8_prepare_weight_24(w, q_dtype="e4m3", packed=None, scales=None):
    """w [n, k] bf16/f16/f32 (unit column stride) -> (packed, s_w): prune 2:4,
    quantise row-wise and compress in one pass (the same bytes as
    sfp8_prune_24 -> sfp8_quantize_rowwise -> sfp8_compress_24)."""
    lib = load_library()
    _require_cuda(w)
    if w.dim() != 2 or w.stride(1) != 1:
        raise ValueError("w must be 2-D with unit column stride")
    wd = TORCH_WIDE.get(w.dtype)
    if wd is None:
        raise ValueError("w dtype must be bfloat16, float16 or float32")
    n, k = w.shape
    if packed is None:
        packed = torch.empty((lib.sfp8_compressed_bytes(n, k),), dtype=torch.uint8,
                             device=w.device)
    if scales is None:
        scales = torch.empty((n,), dtype=torch.float32, device=w.device)
    ld = w.stride(0) if n > 1 else k
    with torch.cuda.device(w.device):
        st = lib.sfp8_prepare_weight_24(_ptr(w), DTYPE[wd], n, k, ld, DTYPE[_fp8_name(q_dtype)],
                                        _ptr(packed), _ptr(scales), _stream(w.device))
    _check(st, "sfp8_prepare_weight_24")
    return packed, scales


def sfp8_decompress_24(packed, n, k, out=None):
    lib = load_library()
    _require_cuda(packed)
    if out is None:
        out = torch.empty((n, k), dtype=torch.uint8, device=packed.device)
    with torch.cuda.device(packed.device):
        st = lib.sfp8_decompress_24(_ptr(packed), n, k, _ptr(out), _stream(packed.device))
    _check(st, "sfp8_decompress_24")
    return out


def sfp8_sparse_linear_workspace_bytes(m, n, k, device=None):
    lib = load_library()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        return int(lib.sfp8_sparse_linear_workspace_bytes(m, n, k))


def new_workspace(m, n, k, device):
    """A zeroed workspace for sfp8_sparse_linear(m, n, k) on `device`."""
    nbytes = sfp8_sparse_linear_workspace_bytes(m, n, k, device)
    return torch.zeros((max(nbytes, 16),), dtype=torch.uint8, device=device)


def sfp8_workspace_clear(workspace):
    lib = load_library()
    with torch.cuda.device(workspace.device):
        st = lib.sfp8_workspace_clear(_ptr(workspace), _ws_bytes(workspace, workspace.device),
                                      _stream(workspace.device))
    _check(st, "sfp8_workspace_clear")


def _linear_args(a_q, n, k, bias, out):
    """Shape, dtype and layout checks shared by the sparse linear wrappers,
    made before anything reaches the library; returns m."""
    if a_q.dim() != 2 or not a_q.is_contiguous() or a_q.dtype != torch.uint8:
        raise ValueError("a_q must be a contiguous 2-D uint8 tensor")
    m = a_q.shape[0]
    if a_q.shape[1] != k:
        raise ValueError("a_q has %d columns, expected k=%d" % (a_q.shape[1], k))
    if bias is not None and (bias.dtype != torch.bfloat16 or bias.dim() != 1
                             or bias.shape[0] != n or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous bfloat16 vector of n=%d elements" % n)
    if out is not None and (out.dtype != torch.bfloat16 or tuple(out.shape) != (m, n)
                            or not out.is_contiguous() or out.device != a_q.device):
        raise ValueError("out must be a contiguous (m, n) = (%d, %d) bfloat16 tensor on "
                         "a_q's device" % (m, n))
    return m


def sfp8_sparse_linear(a_q, a_dtype, s_a, packed, w_dtype, s_w, n, k, bias=None,
                       out=None, workspace=None):
    """y [m, n] bf16 = (s_a s_w^T) * (A_q . W_q^T) + bias."""
    lib = load_library()
    m = _linear_args(a_q, n, k, bias, out)
    _require_cuda(a_q, s_a, packed, s_w, bias)
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=a_q.device)
    if workspace is None:
        workspace = new_workspace(m, n, k, a_q.device)
    with torch.cuda.device(a_q.device):
        st = lib.sfp8_sparse_linear(_ptr(a_q), DTYPE[_fp8_name(a_dtype)], _ptr(s_a), m,
                                    _ptr(packed), DTYPE[_fp8_name(w_dtype)],
                                    _ptr(s_w), n, k, _ptr(bias), _ptr(out), _ptr(workspace),
                                    _ws_bytes(workspace, a_q.device), _stream(a_q.device))
    _check(st, "sfp8_sparse_linear")
    return out


def sfp8_sparse_linear_noalloc(a_q, a_dtype, s_a, packed, w_dtype, s_w, n, k,
                               bias=None, out=None):
    """sfp8_sparse_linear without a workspace, for callers that cannot
    allocate device memory at call time (see include/sfp8.h): the library's
    built-in scratch buffer is used instead.  `out` must be given by such a
    caller; only when it is None does this wrapper allocate it with torch."""
    lib = load_library()
    m = _linear_args(a_q, n, k, bias, out)
    _require_cuda(a_q, s_a, packed, s_w, bias)
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=a_q.device)
    with torch.cuda.device(a_q.device):
        st = lib.sfp8_sparse_linear_noalloc(_ptr(a_q), DTYPE[_fp8_name(a_dtype)], _ptr(s_a), m,
                                            _ptr(packed), DTYPE[_fp8_name(w_dtype)],
                                            _ptr(s_w), n, k, _ptr(bias), _ptr(out),
                                            _stream(a_q.device))
    _check(st, "sfp8_sparse_linear_noalloc")
    return out


ALGO_FIELDS = ("pair", "bn", "ks", "wt", "whole_tiles", "ra", "stages", "grid")


def _dev_ctx(device):
    return torch.cuda.device(device if device is not None else torch.cuda.current_device())


def sfp8_sparse_linear_algo_count(m, n, k, device=None):
    with _dev_ctx(device):
        return int(load_library().sfp8_sparse_linear_algo_count(m, n, k))


def sfp8_sparse_linear_algo_info(m, n, k, algo, device=None):
    """dict of the algorithm's work split (keys ALGO_FIELDS)."""
    info = (ctypes.c_int32 * 8)()
    with _dev_ctx(device):
        st = load_library().sfp8_sparse_linear_algo_info(m, n, k, algo, info)
    _check(st, "sfp8_sparse_linear_algo_info")
    return dict(zip(ALGO_FIELDS, [int(v) for v in info]))


PLAN_FIELDS = ("pair", "bn", "ks", "wt", "whole_tiles", "ra", "stages", "grid", "producers",
               "smem_bytes", "workspace_bytes", "m_tiles")


def sfp8_sparse_linear_plan(m, n, k, num_sms, algo=0):
    """Host-only: the plan of an algorithm for a device of num_sms SMs (dict
    of PLAN_FIELDS), no device involved."""
    info = (ctypes.c_int64 * len(PLAN_FIELDS))()
    st = load_library().sfp8_sparse_linear_plan_info(m, n, k, num_sms, algo, info)
    _check(st, "sfp8_sparse_linear_plan_info")
    return dict(zip(PLAN_FIELDS, [int(v) for v in info]))


def sfp8_sparse_linear_plan_count(m, n, k, num_sms):
    return int(load_library().sfp8_sparse_linear_plan_count(m, n, k, num_sms))


def sfp8_sparse_linear_algo_workspace_bytes(m, n, k, algo, device=None):
    with _dev_ctx(device):
        return int(load_library().sfp8_sparse_linear_algo_workspace_bytes(m, n, k, algo))


def sfp8_sparse_linear_search_workspace_bytes(m, n, k, device=None):
    with _dev_ctx(device):
        return int(load_library().sfp8_sparse_linear_search_workspace_bytes(m, n, k))


def sfp8_sparse_linear_algo(a_q, a_dtype, s_a, packed, w_dtype, s_w, n, k, algo, bias=None,
                            out=None, workspace=None):
    """sfp8_sparse_linear with an explicit work split (algorithm index)."""
    lib = load_library()
    m = _linear_args(a_q, n, k, bias, out)
    _require_cuda(a_q, s_a, packed, s_w, bias)
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=a_q.device)
    if workspace is None:
        nbytes = sfp8_sparse_linear_algo_workspace_bytes(m, n, k, algo, a_q.device)
        workspace = torch.zeros((max(nbytes, 16),), dtype=torch.uint8, device=a_q.device)
    with torch.cuda.device(a_q.device):
        st = lib.sfp8_sparse_linear_algo(_ptr(a_q), DTYPE[_fp8_name(a_dtype)], _ptr(s_a), m,
                                         _ptr(packed), DTYPE[_fp8_name(w_dtype)], _ptr(s_w), n,
                                         k, _ptr(bias), _ptr(out), algo, _ptr(workspace),
                                         _ws_bytes(workspace, a_q.device), _stream(a_q.device))
    _check(st, "sfp8_sparse_linear_algo")
    return out


def sfp8_sparse_linear_search(a_q, a_dtype, s_a, packed, w_dtype, s_w, n, k, bias=None,
                              reps=10, flush=None, out=None):
    """Times every work split of the shape (see include/sfp8.h); returns
    (best algorithm, [median microseconds per algorithm])."""
    lib = load_library()
    m = _linear_args(a_q, n, k, bias, out)
    _require_cuda(a_q, s_a, packed, s_w, bias, flush)
    dev = a_q.device
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
    count = sfp8_sparse_linear_algo_count(m, n, k, dev)
    nbytes = sfp8_sparse_linear_search_workspace_bytes(m, n, k, dev)
    ws = torch.zeros((max(nbytes, 16),), dtype=torch.uint8, device=dev)
    best = ctypes.c_int32(-1)
    times = (ctypes.c_float * max(count, 1))()
    with torch.cuda.device(dev):
        st = lib.sfp8_sparse_linear_search(_ptr(a_q), DTYPE[_fp8_name(a_dtype)], _ptr(s_a), m,
                                           _ptr(packed), DTYPE[_fp8_name(w_dtype)], _ptr(s_w),
                                           n, k, _ptr(bias), _ptr(out), _ptr(ws), ws.numel(),
                                           _ptr(flush),
                                           0 if flush is None else _ws_bytes(flush, dev),
                                           reps, ctypes.byref(best), times, count, _stream(dev))
    _check(st, "sfp8_sparse_linear_search")
    return int(best.value), [float(t) for t in times[:count]]


# Bumped by every change of the shape-keyed algorithm table made through this
# binding: workspaces cached for a shape are re-sized when it moves.
_ALGO_EPOCH = [0]


def algo_epoch():
    return _ALGO_EPOCH[0]


def sfp8_sparse_linear_set_algo(m, n, k, algo, device=None):
    with _dev_ctx(device):
        st = load_library().sfp8_sparse_linear_set_algo(m, n, k, algo)
    _check(st, "sfp8_sparse_linear_set_algo")
    _ALGO_EPOCH[0] += 1


def sfp8_sparse_linear_get_algo(m, n, k, device=None):
    with _dev_ctx(device):
        return int(load_library().sfp8_sparse_linear_get_algo(m, n, k))


def sfp8_sparse_linear_quant_workspace_bytes(m, n, k, device=None):
    lib = load_library()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        return int(lib.sfp8_sparse_linear_quant_workspace_bytes(m, n, k))


def new_quant_workspace(m, n, k, device):
    """A zeroed workspace for sfp8_sparse_linear_quant(m, n, k) on `device`."""
    nbytes = sfp8_sparse_linear_quant_workspace_bytes(m, n, k, device)
    return torch.zeros((max(nbytes, 16),), dtype=torch.uint8, device=device)


def sfp8_sparse_linear_quant(x, a_dtype, packed, w_dtype, s_w, n, k, bias=None, out=None,
                             workspace=None, a_q=None, s_a=None):
    """Quantise x [m, k] (bf16/f16/f32, unit column stride) row-wise and apply
    the sparse linear, one library call: returns (y [m, n] bf16,
    a_q [m, k] uint8, s_a [m] f32), by the chained form (quantiser, then
    the GEMM as its programmatic dependent)."""
    return _quant_linear("sfp8_sparse_linear_quant", x, a_dtype, packed, w_dtype, s_w, n, k,
                         bias, out, workspace, a_q, s_a)


def sfp8_sparse_linear_quant_fused(x, a_dtype, packed, w_dtype, s_w, n, k, bias=None, out=None,
                                   workspace=None, a_q=None, s_a=None):
    """sfp8_sparse_linear_quant in its fused form: one kernel in which every
    CTA quantises the (at most 16) rows itself.  Raises Sfp8Error
    (SFP8_ERR_UNSUPPORTED_SHAPE) where the form does not apply."""
    return _quant_linear("sfp8_sparse_linear_quant_fused", x, a_dtype, packed, w_dtype, s_w, n,
                         k, bias, out, workspace, a_q, s_a)


def sfp8_sparse_linear_quant_chained(x, a_dtype, packed, w_dtype, s_w, n, k, bias=None,
                                     out=None, workspace=None, a_q=None, s_a=None):
    """sfp8_sparse_linear_quant in its chained form: the row-wise quantiser,
    then the GEMM as its programmatic dependent."""
    return _quant_linear("sfp8_sparse_linear_quant_chained", x, a_dtype, packed, w_dtype, s_w,
                         n, k, bias, out, workspace, a_q, s_a)


def sfp8_sparse_linear_quant_fusable(m, n, k, device=None):
    """Whether sfp8_sparse_linear_quant_fused accepts (m, n, k) on `device`
    (host-only query)."""
    lib = load_library()
    with _dev_ctx(device):
        return bool(lib.sfp8_sparse_linear_quant_fusable(m, n, k))


def _quant_linear(name, x, a_dtype, packed, w_dtype, s_w, n, k, bias, out, workspace, a_q, s_a):
    lib = load_library()
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    m = x.shape[0]
    if x.shape[1] != k:
        raise ValueError("x has %d columns, expected k=%d" % (x.shape[1], k))
    xd = TORCH_WIDE.get(x.dtype)
    if xd is None:
        raise ValueError("x dtype must be bfloat16, float16 or float32")
    if bias is not None and bias.dtype != torch.bfloat16:
        raise ValueError("bias must be bfloat16")
    dev = x.device
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
    if a_q is None:
        a_q = torch.empty((m, k), dtype=torch.uint8, device=dev)
    if s_a is None:
        s_a = torch.empty((m,), dtype=torch.float32, device=dev)
    for t, shape, dtype, what in ((out, (m, n), torch.bfloat16, "out"),
                                  (a_q, (m, k), torch.uint8, "a_q"),
                                  (s_a, (m,), torch.float32, "s_a")):
        if (tuple(t.shape) != shape or t.dtype != dtype or not t.is_contiguous()
                or t.device != dev):
            raise ValueError("%s must be a contiguous %s tensor of shape %s on %s"
                             % (what, dtype, shape, dev))
    _require_cuda(x, packed, s_w, bias)
    if workspace is None:
        workspace = new_quant_workspace(m, n, k, dev)
    ld = x.stride(0) if m > 1 else k
    with torch.cuda.device(dev):
        st = getattr(lib, name)(_ptr(x), DTYPE[xd], ld, DTYPE[_fp8_name(a_dtype)], _ptr(a_q),
                                _ptr(s_a), m, _ptr(packed), DTYPE[_fp8_name(w_dtype)],
                                _ptr(s_w), n, k, _ptr(bias), _ptr(out), _ptr(workspace),
                                _ws_bytes(workspace, dev), _stream(dev))
    _check(st, name)
    return out, a_q, s_a


def sfp8_selftest_timeout(device=None):
    """Runs the library's failure-path self-test on `device` (a bounded wait
    that runs out, about a second); read the status word afterwards."""
    lib = load_library()
    with _dev_ctx(device):
        dev = torch.cuda.current_device()
        st = lib.sfp8_selftest_timeout(_stream(dev))
    _check(st, "sfp8_selftest_timeout")


def sfp8_sparse_linear_quant_host(x_host, a_dtype, packed, w_dtype, s_w, n, k, x_dev, a_q, s_a,
                                  y_dev, y_host, workspace, bias=None):
    """Host x [m, k] -> host y [m, n] in one library call: copy in, quantise,
    sparse linear, copy out, all on the current stream (page-locked host
    tensors keep it asynchronous).  Every buffer is given by the caller."""
    lib = load_library()
    if x_host.is_cuda or y_host.is_cuda:
        raise ValueError("x_host and y_host must be host tensors")
    if not (x_host.is_contiguous() and y_host.is_contiguous() and x_dev.is_contiguous()
            and y_dev.is_contiguous()):
        raise ValueError("x_host, x_dev, y_dev and y_host must be contiguous")
    m = x_host.shape[0]
    if (x_host.shape != (m, k) or x_dev.shape != (m, k) or y_host.shape != (m, n)
            or y_dev.shape != (m, n) or y_dev.dtype != torch.bfloat16):
        raise ValueError("shapes: x_host/x_dev [m, k], y_host/y_dev [m, n] (y bfloat16)")
    xd = TORCH_WIDE.get(x_host.dtype)
    if xd is None or x_dev.dtype != x_host.dtype or y_host.dtype != torch.bfloat16:
        raise ValueError("x dtype bfloat16/float16/float32 (same on host and device), y bfloat16")
    _require_cuda(x_dev, a_q, s_a, packed, s_w, bias, y_dev, workspace)
    dev = x_dev.device
    with torch.cuda.device(dev):
        st = lib.sfp8_sparse_linear_quant_host(
            _ptr(x_host), _ptr(x_dev), DTYPE[xd], DTYPE[_fp8_name(a_dtype)], _ptr(a_q), _ptr(s_a),
            m, _ptr(packed), DTYPE[_fp8_name(w_dtype)], _ptr(s_w), n, k, _ptr(bias), _ptr(y_dev),
            _ptr(y_host), _ptr(workspace), _ws_bytes(workspace, dev), _stream(dev))
    _check(st, "sfp8_sparse_linear_quant_host")
    return y_host


def sfp8_read_device_status(clear=True):
    """(status, flags) of the current device's status word; synchronises."""
    lib = load_library()
    flags = ctypes.c_uint32(0)
    st = lib.sfp8_read_device_status(ctypes.byref(flags), 1 if clear else 0)
    return st, flags.value


def sfp8_last_device_status():
    """Status of the current device's status word (not cleared); synchronises."""
    return int(load_library().sfp8_last_device_status())


def sfp8_compressed_values_bytes(n, k):
    return int(load_library().sfp8_compressed_values_bytes(n, k))


def sfp8_compressed_meta_bytes(n, k):
    return int(load_library().sfp8_compressed_meta_bytes(n, k))


def sfp8_status_string(status):
    return load_library().sfp8_status_string(status).decode()


def sfp8_layout_version():
    return int(load_library().sfp8_layout_version())
