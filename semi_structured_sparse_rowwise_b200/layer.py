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
        self._act = {}
        self._host = {}

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
        self._act = {}
        self._host = {}
        return self

    def workspace(self, m):
        """The layer's zeroed workspace for m tokens (kept between calls; each
        call leaves its split-K counters at zero).  Re-sized after any change
        of the library's algorithm table (which may pick a split that needs a
        larger one)."""
        epoch = B.algo_epoch()
        hit = self._ws.get(m)
        if hit is None or hit[0] != epoch:
            # a fresh zeroed buffer: another split keeps its counters elsewhere
            ws = B.new_quant_workspace(m, self.n, self.k, self.device)
            self._ws[m] = (epoch, ws)
            return ws
        return hit[1]

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
        return best, times

    def forward(self, x, out=None):
        """x [m, k] bf16/f16/f32 on the layer's device -> y [m, n] bf16.

        One library call (sfp8_sparse_linear_quant): the quantiser, then the
        GEMM as its programmatic dependent.  The quantised activation, its
        scales and the workspace are kept per token count, so one forward of
        a layer per token count may be in flight at a time (calls on one
        stream are ordered)."""
        m = x.shape[0]
        a_q, s_a = self._act_buffers(m)
        y, _, _ = B.sfp8_sparse_linear_quant(x, self.a_dtype, self.packed, self.w_dtype,
                                             self.s_w, self.n, self.k, bias=self.bias, out=out,
                                             workspace=self.workspace(m), a_q=a_q, s_a=s_a)
        return y

    __call__ = forward

    def _act_buffers(self, m):
        """The quantised activation [m, k] and its scales [m] (kept per m)."""
        b = self._act.get(m)
        if b is None:
            b = (torch.empty((m, self.k), dtype=torch.uint8, device=self.device),
                 torch.empty((m,), dtype=torch.float32, device=self.device))
            self._act[m] = b
        return b

    def _host_buffers(self, m, x_dtype):
        """Device buffers of the host path for m tokens (kept): staging x, the
        quantised activation and its scales, staging y."""
        key = (m, x_dtype)
        b = self._host.get(key)
        if b is None:
            a_q, s_a = self._act_buffers(m)
            b = (torch.empty((m, self.k), dtype=x_dtype, device=self.device), a_q, s_a,
                 torch.empty((m, self.n), dtype=torch.bfloat16, device=self.device))
            self._host[key] = b
        return b

    def forward_host(self, x_host, y_host, x_dev=None, y_dev=None):
        """Host-buffer forward: x_host [m, k] (page-locked for an asynchronous
        copy) -> device -> quantise -> sparse linear -> y_host [m, n] bf16, in
        one library call (sfp8_sparse_linear_quant_host) on the current
        stream.  x_dev / y_dev override the layer's staging buffers."""
        m = x_host.shape[0]
        xs, a_q, s_a, ys = self._host_buffers(m, x_host.dtype)
        return B.sfp8_sparse_linear_quant_host(
            x_host, self.a_dtype, self.packed, self.w_dtype, self.s_w, self.n, self.k,
            xs if x_dev is None else x_dev, a_q, s_a, ys if y_dev is None else y_dev, y_host,
            self.workspace(m), bias=self.bias)


class HostPipeline:
    """Streams host batches of m tokens through a layer, with the host <->
    device copies of one batch overlapping the compute of its neighbours.

    Copies in run on one CUDA stream, the forward (quantise + sparse linear,
    one library call) on a second, copies out on a third; `depth` sets of
    device buffers rotate, and CUDA events order each batch's three steps and
    the reuse of a set.  With page-locked host buffers every step is
    asynchronous, so a sequence of submits can also be captured in a CUDA
    graph (`capture`) and replayed with no per-batch host work."""

    def __init__(self, layer, m, x_dtype=torch.bfloat16, depth=3):
        dev = layer.device
        self.layer, self.m = layer, m
        self.streams = [torch.cuda.Stream(dev) for _ in range(3)]
        ws = B.new_quant_workspace(m, layer.n, layer.k, dev)
        self._ws_epoch = B.algo_epoch()
        self.slots = []
        for _ in range(depth):
            self.slots.append(dict(
                x=torch.empty((m, layer.k), dtype=x_dtype, device=dev),
                y=torch.empty((m, layer.n), dtype=torch.bfloat16, device=dev),
                a_q=torch.empty((m, layer.k), dtype=torch.uint8, device=dev),
                s_a=torch.empty((m,), dtype=torch.float32, device=dev), ws=ws))
        self._reset()

    def _reset(self):
        for sl in self.slots:
            sl.update(used=False, x_in=torch.cuda.Event(), y_done=torch.cuda.Event(),
                      y_out=torch.cuda.Event())
        self.i = 0

    def submit(self, x_host, y_host, layer=None):
        """Enqueue one batch: x_host [m, k] -> y_host [m, n] bf16, through
        `layer` (default: the pipeline's; any layer of the same shape, e.g.
        the next layer of a model).  Returns the event that completes once
        y_host holds the result."""
        s_in, s_comp, s_out = self.streams
        sl = self.slots[self.i % len(self.slots)]
        self.i += 1
        L = self.layer if layer is None else layer
        if (L.n, L.k) != (self.layer.n, self.layer.k):
            raise ValueError("layer shape differs from the pipeline's")
        if self._ws_epoch != B.algo_epoch():
            # the algorithm table changed: the forward may need a larger workspace
            self.synchronize()
            ws = B.new_quant_workspace(self.m, L.n, L.k, L.device)
            for s_ in self.slots:
                s_["ws"] = ws
            self._ws_epoch = B.algo_epoch()
        # the set is free once its previous forward has read x and its
        # previous copy out has read y
        if sl["used"]:
            s_in.wait_event(sl["y_done"])
        with torch.cuda.stream(s_in):
            sl["x"].copy_(x_host, non_blocking=True)
        sl["x_in"].record(s_in)
        s_comp.wait_event(sl["x_in"])
        if sl["used"]:
            s_comp.wait_event(sl["y_out"])
        sl["used"] = True
        with torch.cuda.stream(s_comp):
            B.sfp8_sparse_linear_quant(sl["x"], L.a_dtype, L.packed, L.w_dtype, L.s_w, L.n, L.k,
                                       bias=L.bias, out=sl["y"], workspace=sl["ws"],
                                       a_q=sl["a_q"], s_a=sl["s_a"])
        sl["y_done"].record(s_comp)
        s_out.wait_event(sl["y_done"])
        with torch.cuda.stream(s_out):
            y_host.copy_(sl["y"], non_blocking=True)
        sl["y_out"].record(s_out)
        return sl["y_out"]

    def capture(self, x_hosts, y_hosts, layers=None):
        """A CUDA graph of one submit per (x_host, y_host) pair (page-locked
        host tensors); replay it with .replay().  The pipeline's buffers
        belong to the graph afterwards: use another pipeline for eager
        submits."""
        self.synchronize()
        self._reset()
        origin = torch.cuda.Stream(self.layer.device)
        origin.wait_stream(torch.cuda.current_stream(self.layer.device))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=origin):
            for s in self.streams:
                s.wait_stream(origin)
            for j, (xh, yh) in enumerate(zip(x_hosts, y_hosts)):
                self.submit(xh, yh, None if layers is None else layers[j % len(layers)])
            for s in self.streams:
                origin.wait_stream(s)
        torch.cuda.current_stream(self.layer.device).wait_stream(origin)
        return g

    def synchronize(self):
        for s in self.streams:
            s.synchronize()
