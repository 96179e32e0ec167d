"""The layer a user calls: a prepared 2:4 sparse FP8 weight and its forward.

Weight preparation (once, as the page "Add CUTLASS-based row-wise scaled
sparse FP8 kernel", pytorch/ao pull request 1671, does at ``quantize_()`` time,
its items 1, 3 and 4): 2:4 magnitude prune -> row-wise FP8 quantisation ->
2:4 compression.  Forward (per call): dynamic row-wise FP8 quantisation of the
activation -> sparse FP8 GEMM with the scale/bias epilogue.  Every step is a
kernel of libsfp8.so; torch only provides memory and streams.
"""

import torch

from . import binding as B


class SparseFp8Linear:
    """y = (s_a s_w^T) * (A_q W_q^T) + bias with a 2:4 compressed FP8 weight."""

    def __init__(self, weight, bias=None, w_dtype="e4m3", a_dtype="e4m3", prune=True):
        if weight.dim() != 2:
            raise ValueError("weight must be [out_features, in_features]")
        self.n, self.k = weight.shape
        self.w_dtype = w_dtype
        self.a_dtype = a_dtype
        self.device = weight.device
        if prune:
            # prune, quantise and compress in one pass over the weight
            self.packed, self.s_w = B.sfp8_prepare_weight_24(weight.contiguous(), w_dtype)
        else:
            w_q, self.s_w = B.sfp8_quantize_rowwise(weight.contiguous(), w_dtype)
            self.packed = B.sfp8_compress_24(w_q, w_dtype)
        self.bias = None if bias is None else bias.to(torch.bfloat16).contiguous()
        self._ws = {}

    @classmethod
    def from_compressed(cls, packed, s_w, n, k, bias=None, w_dtype="e4m3", a_dtype="e4m3"):
        """A layer over an already compressed weight (packed, s_w)."""
        self = cls.__new__(cls)
        self.n, self.k = n, k
        self.w_dtype, self.a_dtype = w_dtype, a_dtype
        self.device = packed.device
        self.packed, self.s_w = packed, s_w
        self.bias = None if bias is None else bias.to(torch.bfloat16).contiguous()
        self._ws = {}
        return self

    def workspace(self, m):
        """The layer's zeroed workspace for m tokens (kept between calls; each
        call leaves its split-K counters at zero)."""
        ws = self._ws.get(m)
        if ws is None:
            ws = B.new_quant_workspace(m, self.n, self.k, self.device)
            self._ws[m] = ws
        return ws

    def autotune(self, x, reps=10, flush_bytes=256 << 20):
        """Times every work split of the GEMM for x's token count on this
        layer's weight (sfp8_sparse_linear_search; a flush_bytes write before
        each timed launch evicts the operands from L2) and stores the fastest
        in the library's shape-keyed table, which every later forward with
        that token count -- of any layer of the same shape on this device --
        uses.  Returns (best algorithm, median microseconds per algorithm)."""
        m = x.shape[0]
        a_q, s_a = B.sfp8_quantize_rowwise(x, self.a_dtype)
        flush = None
        if flush_bytes:
            flush = torch.empty((flush_bytes,), dtype=torch.uint8, device=self.device)
        best, times = B.sfp8_sparse_linear_search(a_q, self.a_dtype, s_a, self.packed,
                                                  self.w_dtype, self.s_w, self.n, self.k,
                                                  bias=self.bias, reps=reps, flush=flush)
        B.sfp8_sparse_linear_set_algo(m, self.n, self.k, best, self.device)
        self._ws.pop(m, None)       # the workspace size follows the algorithm
        return best, times

    def forward(self, x, out=None):
        """x [m, k] bf16/f16/f32 on the layer's device -> y [m, n] bf16.

        One library call (sfp8_sparse_linear_quant): the quantiser, then the
        GEMM as its programmatic dependent."""
        y, _, _ = B.sfp8_sparse_linear_quant(x, self.a_dtype, self.packed, self.w_dtype,
                                             self.s_w, self.n, self.k, bias=self.bias, out=out,
                                             workspace=self.workspace(x.shape[0]))
        return y

    __call__ = forward

    def forward_host(self, x_host, y_host, x_dev=None, y_dev=None):
        """Host-buffer forward: x_host (pinned) -> device -> layer -> y_host."""
        if x_dev is None:
            x_dev = torch.empty(x_host.shape, dtype=x_host.dtype, device=self.device)
        x_dev.copy_(x_host, non_blocking=True)
        y = self.forward(x_dev, out=y_dev)
        y_host.copy_(y, non_blocking=True)
        return y_host
