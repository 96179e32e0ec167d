#!/usr/bin/env python
"""Benchmark of the row-wise scaled 2:4 sparse FP8 linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--m 16] [--impl ours|reference]

Headline workload: the Llama-3.1-8B MLP gate/up projection at decode
(K=4096, N=14336, M in {1, 4, 16}; the headline line uses M=16), synthetic
seeded inputs (A ~ N(0,1) bf16, W ~ N(0, 0.02) bf16, magnitude-pruned 2:4,
both quantised row-wise to e4m3, no bias).  The line's `per_workload`
carries the compute-bound half of the metric from the same run: the four
Llama-3.1-8B prefill linears at M=8192 (QKV, O, up, down; A with 1 % outlier
channels), each in dense-equivalent TFLOP/s against 4 x the measured bf16
peak, burst and sustained, then the dtype sweep (K=4096, N=14336, M in
{1, 16, 128, 1024, 8192} x the four e4m3/e5m2 operand pairs) and the
Llama-3-70B-shaped stress GEMM (16384 x 8192 x 28672).

A step is one forward of the layer: dynamic row-wise FP8 quantisation of the
activation followed by the sparse FP8 GEMM with its scale epilogue (one
library call, two kernels).  The weight is prepared once before timing
(prune -> quantise -> compress), as the layer does at load time; those
kernels, and the one-pass preparation that the layer uses
(sfp8_prepare_weight_24), are timed separately under "offline".  The
metric's unit for the memory-bound decode shape is GB/s of compressed weight
bytes (kept values + metadata) per step.

Timing: W eager warm-up steps, then exactly K steps captured in one CUDA
graph; each replay of it is timed between CUDA events on the launching
stream, with a barrier and a device synchronise on both sides, and the
reported time is the median over enough replays to fill about a quarter of
a second (so the clock sampler sees the load), the max over ranks for each.
The K steps rotate over copies of the compressed weight that together exceed
the 126 MB L2 (8 x 36.7 MB at decode), so no step finds its weight in L2.
`e2e` is the same metric through the C-ABI host-buffer call
(sfp8_sparse_linear_quant_host: copy in from page-locked host memory,
quantise, linear, copy out).  Under torchrun every rank runs an independent
replica (weak scaling, no data-path collective).

`--impl reference` times the CPU oracle (test infrastructure) on a bounded
sample of the same workload instead.
"""

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "2:4 FP8 rowwise sparse linear TFLOP/s & GB/s, % roofline, M=1..8192"
WORKLOAD = "decode_gate_up_8b"
M_TO_SHAPE = {1: 0, 4: 1, 16: 2}
K_DIM, N_DIM = 4096, 14336
WEIGHT_COPIES = 8
E2E_CHUNK = 100          # steps per captured graph of the end-to-end leg
L2_NOTE = "rotating 8 copies of the compressed weight (8 x 36.7 MB > 126 MB L2)"

# ncu DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one
# sparse-GEMM launch, per (workload, M or shape), from the captures summarised
# under profiles/; valid only while the kernel sources hash to `sha1`.
KERNEL_SOURCES = ("device_common.cuh", "sparse_linear.cuh", "sparse_linear_pair.cuh")
NCU_TRAFFIC = {
    ("decode_gate_up_8b", 16): {"sha1": "646f387d0fb7837fc6ee6a17a12c47e357d03fb0", "bytes_per_launch": 36897024},
    ("prefill_8b", 0): {"sha1": "646f387d0fb7837fc6ee6a17a12c47e357d03fb0", "bytes_per_launch": 108502528},
    ("prefill_8b", 1): {"sha1": "646f387d0fb7837fc6ee6a17a12c47e357d03fb0", "bytes_per_launch": 70763008},
    ("prefill_8b", 2): {"sha1": "646f387d0fb7837fc6ee6a17a12c47e357d03fb0", "bytes_per_launch": 265653760},
    ("prefill_8b", 3): {"sha1": "646f387d0fb7837fc6ee6a17a12c47e357d03fb0", "bytes_per_launch": 313768192},
}


def compressed_weight_bytes(n, k):
    npad = ((n + 127) // 128) * 128
    return npad * k // 2 + npad * k // 8


def gemm_algorithmic_bytes(m, n, k):
    """HBM bytes one GEMM launch must move: compressed weight + metadata,
    weight scales, activation codes and scales, bf16 output."""
    return compressed_weight_bytes(n, k) + 4 * n + m * k + 4 * m + 2 * m * n



def kernel_source_sha1():
    h = hashlib.sha1()
    for name in KERNEL_SOURCES:
        p = os.path.join(ROOT, "semi_structured_sparse_rowwise_b200", "csrc", name)
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


# Secondary roofline denominators: the datasheet figures (HBM3e 8 TB/s; FP8
# with 2:4 sparsity 9 PFLOP/s dense-equivalent, at boost clock).
DATASHEET_HBM_GBS = 8000.0
DATASHEET_SPARSE_FP8_TFLOPS = 9000.0


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured hbm_gbs (MEASURED_PEAKS.json)"
    except Exception:
        return 6650.0, "fallback 6.65 TB/s"


def measured_tensor_peak(sustained=False):
    """Dense-equivalent 2:4 sparse FP8 peak: the measured bf16 peak x 2
    (FP8 vs bf16) x 2 (2:4 sparsity), the nominal B200 ratios; the burst
    figure by default, the power-capped sustained one for long runs."""
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return 4.0 * float(d[key]), "4 x measured %s (MEASURED_PEAKS.json)" % key
    except Exception:
        return 4.0 * (1400.0 if sustained else 1590.0), "4 x fallback %s" % (
            "1.4 PFLOP/s sustained" if sustained else "1.59 PFLOP/s")


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while running."""

    def __init__(self, device_index, period_s=0.002):
        self.idx = device_index
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._paused = threading.Event()
        self._thr = None
        self.ok = False

    def pause(self):
        """Stop sampling (host-only work in between: its idle clocks would
        dilute the record)."""
        self._paused.set()

    def resume(self):
        self._paused.clear()

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
            return self
        self._thr = threading.Thread(target=self._run, daemon=True)
        self._thr.start()
        return self

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
        names = {
            0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown",
            0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown",
        }
        for bit, name in names.items():
            if r & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            if not self._paused.is_set():
                try:
                    self._sample()
                except Exception:
                    pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._thr.join()
            try:
                self._sample()
            except Exception:
                pass
        return False

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup(backend):
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return rank, local, world


def dist_max(value, world, device=None):
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------- CPU oracle

_ORACLE_INPUTS = {}


def oracle_step_rate(m, seconds=10.0, n_sample=512):
    """Oracle throughput on a bounded sample of the decode step: quantise the
    activation (all m rows) and compute n_sample output columns, repeated for
    about `seconds`.  Returns (GB/s of compressed weight bytes, cores, note)."""
    import numpy as np
    import oracle
    from semi_structured_sparse_rowwise_b200 import synthetic
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = 1
    key = (m, n_sample)
    if key not in _ORACLE_INPUTS:
        x_bits, w_bits, _, _ = synthetic.workload_inputs(WORKLOAD, M_TO_SHAPE[m])
        cols = np.arange(n_sample)
        w32 = oracle.bf16_bits_to_f32(w_bits[cols])
        wq, sw = oracle.quantize_rowwise(oracle.prune_24(w32), "e4m3")
        vals, nib = oracle.compress_24(wq, "e4m3")
        _ORACLE_INPUTS[key] = (oracle.bf16_bits_to_f32(x_bits), vals, nib, sw)
    x32, vals, nib, sw = _ORACLE_INPUTS[key]
    reps = 0
    t0 = time.perf_counter()
    while True:
        aq, sa = oracle.quantize_rowwise(x32, "e4m3")
        oracle.sparse_linear_ref(aq, "e4m3", sa, vals, nib, "e4m3", sw)
        reps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    # one sample covers n_sample of the N output columns: scale the work
    frac = n_sample / N_DIM
    step_time = dt / reps / frac
    rate = compressed_weight_bytes(N_DIM, K_DIM) / step_time / 1e9
    try:
        affinity = len(os.sched_getaffinity(0))
    except Exception:
        affinity = None
    note = ("oracle (numpy fp64) quantise of the %dx%d activation + linear for %d of %d "
            "output columns, %d repetitions in %.1f s, scaled to the full N; %d BLAS threads, "
            "os.cpu_count() %s, affinity %s"
            % (m, K_DIM, n_sample, N_DIM, reps, dt, cores, os.cpu_count(), affinity))
    return rate, cores, note, step_time


def oracle_prefill_rate(x_bits, w_bits, seconds=3.0, rows=64, n_sample=1024):
    """Oracle throughput on a bounded sample of one prefill step: quantise
    `rows` activation rows and compute `n_sample` output columns, repeated for
    about `seconds`, then extrapolated linearly in M and N to the full shape.
    Returns (dense-equivalent TFLOP/s, cores, note)."""
    import numpy as np
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = 1
    m, k = x_bits.shape
    n = w_bits.shape[0]
    w32 = oracle.bf16_bits_to_f32(w_bits[:n_sample])
    wq, sw = oracle.quantize_rowwise(oracle.prune_24(w32), "e4m3")
    vals, nib = oracle.compress_24(wq, "e4m3")
    x32 = oracle.bf16_bits_to_f32(x_bits[:rows])
    reps = 0
    t0 = time.perf_counter()
    while True:
        aq, sa = oracle.quantize_rowwise(x32, "e4m3")
        oracle.sparse_linear_ref(aq, "e4m3", sa, vals, nib, "e4m3", sw)
        reps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    step_time = dt / reps * (m / rows) * (n / n_sample)
    rate = 2.0 * m * n * k / step_time / 1e12
    note = ("extrapolated: oracle (numpy fp64) quantise of %d of %d activation rows + linear "
            "for %d of %d output columns, %d repetitions in %.1f s, scaled linearly to the "
            "full M and N; %d BLAS threads, os.cpu_count() %s"
            % (rows, m, n_sample, n, reps, dt, cores, os.cpu_count()))
    return rate, cores, note


def oracle_offline_time(w_bits, seconds=2.0, n_sample=256):
    """Oracle time of the offline weight preparation on a bounded sample:
    prune (bf16), row-wise quantise and compress n_sample weight rows,
    repeated for about `seconds`, scaled to all rows.  Returns (seconds for
    the whole weight, cores, note)."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = 1
    n, k = w_bits.shape
    rows = min(n_sample, n)
    w32 = oracle.bf16_bits_to_f32(w_bits[:rows])
    reps = 0
    t0 = time.perf_counter()
    while True:
        wq, sw = oracle.quantize_rowwise(oracle.prune_24(w32), "e4m3")
        oracle.compress_24(wq, "e4m3")
        reps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    t_full = dt / reps * (n / rows)
    note = ("extrapolated: oracle prune + row-wise quantise + compress of %d of %d weight rows "
            "(k = %d), %d repetitions in %.1f s, scaled linearly to all rows; %d BLAS threads"
            % (rows, n, k, reps, dt, cores))
    return t_full, cores, note


def run_reference(args):
    rank, local, world = dist_setup("gloo")
    if rank != 0:
        return 0
    m = args.m
    # each step: a bounded sample of the workload (the oracle is slow); the
    # whole run stays around a minute whatever K and W are
    per_step_s = min(1.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_step_rate(m, seconds=per_step_s)
    rates, step_times = [], []
    note = ""
    cores = 1
    for _ in range(args.steps):
        r, cores, note, st = oracle_step_rate(m, seconds=per_step_s)
        rates.append(r)
        step_times.append(st)
    value = statistics.mean(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.mean(step_times) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "m": m, "k": K_DIM, "n": N_DIM, "a_dtype": "e4m3",
                   "w_dtype": "e4m3", "bias": False},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": note},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU path

def run_ours(args):
    import numpy as np
    import torch
    rank, local, world = dist_setup("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import semi_structured_sparse_rowwise_b200 as S
    from semi_structured_sparse_rowwise_b200 import synthetic

    S.load_library()
    prefill = args.workload == "prefill_8b"
    if prefill:
        x_bits, w_bits, _, seeds = synthetic.workload_inputs("prefill_8b", args.shape)
        m = x_bits.shape[0]
    else:
        m = args.m
        x_bits, w_bits, _, seeds = synthetic.workload_inputs(WORKLOAD, M_TO_SHAPE[m])
    n, k = w_bits.shape
    stream = torch.cuda.current_stream(dev)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
            torch.bfloat16).to(dev)

    w_dev = bf16(w_bits)
    x_dev = bf16(x_bits)

    # ---- offline weight preparation (timed separately)
    def prep():
        wp = S.sfp8_prune_24(w_dev)
        wq, sw = S.sfp8_quantize_rowwise(wp, "e4m3")
        packed = S.sfp8_compress_24(wq, "e4m3")
        return wp, wq, sw, packed

    wp, wq, sw, packed = prep()
    torch.cuda.synchronize(dev)
    off = {}
    packed1, sw1 = S.sfp8_prepare_weight_24(w_dev, "e4m3")
    for name, fn in (("prune_24", lambda: S.sfp8_prune_24(w_dev, out=wp)),
                     ("quantize_weight", lambda: S.sfp8_quantize_rowwise(wp, "e4m3", q=wq, scales=sw)),
                     ("compress_24", lambda: S.sfp8_compress_24(wq, "e4m3", packed=packed)),
                     ("prepare_weight_24", lambda: S.sfp8_prepare_weight_24(
                         w_dev, "e4m3", packed=packed1, scales=sw1))):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 10
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        e1.synchronize()
        off[name] = e0.elapsed_time(e1) / reps
    wbytes_bf16 = n * k * 2
    off_gbs = {
        "prune_24": {"ms": off["prune_24"], "GB/s": 2 * wbytes_bf16 / off["prune_24"] / 1e6},
        "quantize_weight": {"ms": off["quantize_weight"],
                            "GB/s": (wbytes_bf16 + n * k + 4 * n) / off["quantize_weight"] / 1e6},
        "compress_24": {"ms": off["compress_24"],
                        "GB/s": (n * k + compressed_weight_bytes(n, k)) / off["compress_24"] / 1e6},
        "prepare_weight_24": {"ms": off["prepare_weight_24"],
                              "GB/s": (wbytes_bf16 + compressed_weight_bytes(n, k) + 4 * n)
                              / off["prepare_weight_24"] / 1e6},
    }
    del packed1, sw1, wp, wq, w_dev

    # ---- the step's buffers
    n_copies = WEIGHT_COPIES if not prefill else max(
        2, -(-150 * 2 ** 20 // (packed.numel() + m * k + 2 * m * n)))
    copies = [(packed.clone(), sw.clone()) for _ in range(n_copies)]
    del packed
    aq = torch.empty((m, k), dtype=torch.uint8, device=dev)
    sa = torch.empty((m,), dtype=torch.float32, device=dev)
    ys = [torch.empty((m, n), dtype=torch.bfloat16, device=dev)
          for _ in range(WEIGHT_COPIES if not prefill else 2)]
    ws = S.new_workspace(m, n, k, dev)
    ws_q = S.new_quant_workspace(m, n, k, dev)

    def quantize():
        S.sfp8_quantize_rowwise(x_dev, "e4m3", q=aq, scales=sa)

    def gemm(j):
        pk, s = copies[j % len(copies)]
        S.sfp8_sparse_linear(aq, "e4m3", sa, pk, "e4m3", s, n, k, out=ys[j % len(ys)],
                             workspace=ws)

    def step(j):
        # one forward of the layer: one library call (quantiser + GEMM kernels)
        pk, s = copies[j % len(copies)]
        S.sfp8_sparse_linear_quant(x_dev, "e4m3", pk, "e4m3", s, n, k, out=ys[j % len(ys)],
                                   workspace=ws_q, a_q=aq, s_a=sa)

    for j in range(args.warmup):
        step(j)
    torch.cuda.synchronize(dev)

    def capture(fn, count, streams=()):
        """One CUDA graph of `count` calls of fn(j); `streams` join the capture
        (fork from and join back to its origin stream)."""
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for x in streams:
                    x.wait_stream(s)
                for j in range(count):
                    fn(j)
                for x in streams:
                    s.wait_stream(x)
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize(dev)
        return g

    def timed_once(g):
        """One replay of the K-step graph between CUDA events on the launching
        stream, with a barrier and a device synchronise on both sides; the max
        over ranks."""
        barrier(world)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        e1.synchronize()
        torch.cuda.synchronize(dev)
        barrier(world)
        return dist_max(e0.elapsed_time(e1), world, dev)

    def timed(g):
        """Median over R timed replays (each exactly K steps): R gives about
        `--timed-seconds` of timed work, at least 30 replays, so that the clock
        sampler sees the load and one short replay does not decide the
        number.  Returns (ms per replay, R)."""
        g.replay()                       # untimed: graph upload
        torch.cuda.synchronize(dev)
        first = timed_once(g)
        replays = args.replays or int(min(2000, max(30, args.timed_seconds * 1e3 / max(first, 1e-3))))
        return statistics.median([timed_once(g) for _ in range(replays)]), replays

    steps = args.steps
    g_step = capture(step, steps)
    with ClockSampler(local) as clk:
        ms, replays = timed(g_step)
    clocks = clk.summary()
    wbytes = compressed_weight_bytes(n, k)
    flops = 2.0 * m * n * k
    if prefill:
        value = world * flops * steps / (ms * 1e-3) / 1e12
    else:
        value = world * wbytes * steps / (ms * 1e-3) / 1e9

    # ---- the dominant kernel alone (sparse GEMM), same rotation
    quantize()
    ksteps = max(steps, args.kernel_steps)
    g_gemm = capture(gemm, ksteps)
    ms_gemm, _ = timed(g_gemm)
    gemm_us = ms_gemm * 1e3 / ksteps
    g_q = capture(lambda j: quantize(), ksteps)
    ms_q, _ = timed(g_q)
    peak, peak_kind = measured_peaks()
    # the dominant kernel of the step: the GEMM
    kernel_us = gemm_us
    alg = gemm_algorithmic_bytes(m, n, k)
    achieved = alg / (kernel_us * 1e-6) / 1e9
    if prefill:
        peak, peak_kind = measured_tensor_peak()
        achieved = flops / (gemm_us * 1e-6) / 1e12
    traffic = None
    rec = NCU_TRAFFIC.get((args.workload, args.shape if prefill else m))
    if rec is not None and rec["sha1"] == kernel_source_sha1():
        traffic = rec["bytes_per_launch"]

    # ---- the fused form of the step (one kernel in which every CTA quantises
    # the rows itself), timed beside the chained form that the step uses
    fused = None
    if not prefill and S.sfp8_sparse_linear_quant_fusable(m, n, k, dev):
        def step_fused(j):
            pk, s_ = copies[j % len(copies)]
            S.sfp8_sparse_linear_quant_fused(x_dev, "e4m3", pk, "e4m3", s_, n, k,
                                             out=ys[j % len(ys)], workspace=ws_q, a_q=aq, s_a=sa)
        for j in range(args.warmup):
            step_fused(j)
        g_f = capture(step_fused, ksteps)
        ms_f, _ = timed(g_f)
        del g_f
        g_c = capture(step, ksteps)
        ms_c, _ = timed(g_c)
        del g_c
        fused = {"call": "sfp8_sparse_linear_quant_fused", "step_us": ms_f * 1e3 / ksteps,
                 "chained_step_us": ms_c * 1e3 / ksteps,
                 "timing": "median of replays of one CUDA graph of %d steps each, same weight "
                           "rotation" % ksteps}

    # ---- end to end through the C-ABI host-buffer call
    # (sfp8_sparse_linear_quant_host: copy the activation in from page-locked
    # host memory, quantise, sparse linear, copy the result out, all in one
    # library call on one stream).  Steps go round-robin to three streams,
    # each with its own device staging buffers and host output, so one step's
    # copies overlap the others' kernels; the K steps are captured in one
    # CUDA graph (forked to the three streams and joined back) and replayed.
    x_host = torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).view(
        torch.bfloat16).pin_memory()
    e2e_streams = [torch.cuda.Stream(dev) for _ in range(3)]
    sets = [{"x_dev": torch.empty((m, k), dtype=torch.bfloat16, device=dev),
             "a_q": torch.empty((m, k), dtype=torch.uint8, device=dev),
             "s_a": torch.empty((m,), dtype=torch.float32, device=dev),
             "y_dev": torch.empty((m, n), dtype=torch.bfloat16, device=dev),
             "y_host": torch.empty((m, n), dtype=torch.bfloat16).pin_memory(),
             "ws": S.new_quant_workspace(m, n, k, dev)} for _ in e2e_streams]

    def host_step(j):
        sl = sets[j % len(sets)]
        pk, s_ = copies[j % len(copies)]
        with torch.cuda.stream(e2e_streams[j % len(e2e_streams)]):
            S.sfp8_sparse_linear_quant_host(x_host, "e4m3", pk, "e4m3", s_, n, k, sl["x_dev"],
                                            sl["a_q"], sl["s_a"], sl["y_dev"], sl["y_host"],
                                            sl["ws"])

    for s_ in e2e_streams:
        s_.wait_stream(torch.cuda.current_stream(dev))
    for j in range(args.warmup):
        host_step(j)
    torch.cuda.synchronize(dev)
    g_e2e = capture(host_step, steps, e2e_streams)
    ms_e2e, replays_e2e = timed(g_e2e)
    e2e_value = (world * flops * steps / (ms_e2e * 1e-3) / 1e12 if prefill
                 else world * wbytes * steps / (ms_e2e * 1e-3) / 1e9)
    e2e = {"value": e2e_value, "unit": "TFLOP/s" if prefill else "GB/s",
           "h2d_bytes_per_step": m * k * 2, "d2h_bytes_per_step": m * n * 2,
           "ms_per_step": ms_e2e / steps, "replays": replays_e2e,
           "path": "sfp8_sparse_linear_quant_host (C-ABI: copy in from page-locked host "
                   "memory, quantise, sparse linear, copy out), steps round-robin on three "
                   "streams with their own staging buffers, %d rotating weight copies, CUDA "
                   "graph of %d steps, median of %d replays" % (len(copies), steps, replays_e2e)}
    del g_e2e

    # the layer's own host pipeline (copies on separate streams), for context
    e2e_pipe = None
    if not args.no_pipeline:
        layers = [S.SparseFp8Linear.from_compressed(pk, s_, n, k) for pk, s_ in copies]
        y_host = torch.empty((m, n), dtype=torch.bfloat16).pin_memory()
        pipe = S.HostPipeline(layers[0], m, depth=3)
        g_pipe = pipe.capture([x_host] * steps, [y_host] * steps, layers)
        ms_pipe, replays_pipe = timed(g_pipe)
        e2e_pipe = {"value": (flops * steps / (ms_pipe * 1e-3) / 1e12 if prefill
                              else wbytes * steps / (ms_pipe * 1e-3) / 1e9) * world,
                    "unit": "TFLOP/s" if prefill else "GB/s", "ms_per_step": ms_pipe / steps,
                    "path": "HostPipeline (copy in, SparseFp8Linear forward, copy out on three "
                            "streams), CUDA graph of %d steps, median of %d replays"
                            % (steps, replays_pipe)}
        del g_pipe, pipe, layers

    # ---- the other decode batch sizes (context lines, same method)
    per_m = {}
    if args.all_m and world == 1 and not prefill:
        for m2 in (1, 4, 16):
            if m2 == m:
                continue
            x2 = bf16(synthetic.workload_inputs(WORKLOAD, M_TO_SHAPE[m2])[0])
            aq2 = torch.empty((m2, k), dtype=torch.uint8, device=dev)
            sa2 = torch.empty((m2,), dtype=torch.float32, device=dev)
            y2 = torch.empty((m2, n), dtype=torch.bfloat16, device=dev)
            ws2 = S.new_quant_workspace(m2, n, k, dev)

            def step2(j, x2=x2, aq2=aq2, sa2=sa2, y2=y2, ws2=ws2, m2=m2):
                # the same step as the headline: one library call
                pk, s = copies[j % WEIGHT_COPIES]
                S.sfp8_sparse_linear_quant(x2, "e4m3", pk, "e4m3", s, n, k, out=y2,
                                           workspace=ws2, a_q=aq2, s_a=sa2)
            for j in range(args.warmup):
                step2(j)
            g2 = capture(step2, steps)
            ms2, _ = timed(g2)
            per_m[str(m2)] = {"value": wbytes * steps / (ms2 * 1e-3) / 1e9, "unit": "GB/s",
                              "ms_per_step": ms2 / steps}
            del g2

    # ---- the prefill linears (M=8192): the compute-bound half of the metric
    per_workload = {}
    if not prefill and world == 1 and not args.no_prefill:
        del g_step, g_gemm, g_q
        g_step = g_gemm = g_q = None
        per_workload["prefill_8b"] = [
            prefill_case(args, S, synthetic, dev, bf16, capture, timed, i, steps)
            for i in range(4)]
        if not args.no_sweep:
            # the other two measured configurations: the dtype sweep (every M and
            # operand pair) and the 70B-shaped stress GEMM
            for wl in ("dtype_sweep_8b_up", "stress_70b_mlp"):
                table, clocks_wl = matrix_cases(args, wl, S, synthetic, dev, bf16)
                per_workload[wl] = {"table": table, "clocks": clocks_wl,
                                    "timing": "one CUDA graph of the case's steps, "
                                              "replayed once after an untimed replay"}
                torch.cuda.empty_cache()

    unit = "TFLOP/s" if prefill else "GB/s"
    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": ms / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": args.workload, "m": m, "k": k, "n": n, "a_dtype": "e4m3",
                   "w_dtype": "e4m3", "bias": False,
                   "l2": L2_NOTE if not prefill else
                   "rotating %d weight copies; every step's weight is evicted from L2 by the "
                   "others (%d x %.1f MB + activations and outputs > 126 MB)"
                   % (len(copies), len(copies), wbytes / 1e6),
                   "step": "sfp8_sparse_linear_quant (quantiser + GEMM kernels)",
                   "timing": "median of %d replays of one CUDA graph of the K steps, each "
                             "replay between CUDA events with a barrier and a device "
                             "synchronise on both sides" % replays,
                   "weight_bytes_per_step": wbytes, "seeds": seeds,
                   "parallelism": "replica" if world > 1 else "single"},
        "roofline": {"bound": "tensor" if prefill else "hbm", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s" if prefill else "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_datasheet": (DATASHEET_SPARSE_FP8_TFLOPS if prefill
                                        else DATASHEET_HBM_GBS),
                     "frac_datasheet": achieved / (DATASHEET_SPARSE_FP8_TFLOPS if prefill
                                                   else DATASHEET_HBM_GBS),
                     "kernel": ("sparse_linear_pair_kernel" if m >= 512 else
                                "sparse_linear_kernel"),
                     "algorithmic_bytes_per_launch": alg,
                     "algorithmic_flop_per_launch": flops, "us_per_launch": kernel_us,
                     "launches_timed": "median of replays of one CUDA graph of %d back-to-back "
                                       "launches of this kernel alone (same weight rotation)"
                                       % ksteps,
                     "peak_source": peak_kind},
        "quantize_us_per_launch": ms_q * 1e3 / ksteps,
        "fused_step": fused,
        "e2e": e2e,
        "gpu_launches": 2 * steps,
        "clocks": clocks,
        "offline": off_gbs,
    }
    if e2e_pipe is not None:
        line["e2e_pipelined"] = e2e_pipe
    if per_m:
        line["per_m"] = per_m
    if per_workload:
        line["per_workload"] = per_workload
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if prefill:
            rate, cores, note = oracle_prefill_rate(x_bits, w_bits, seconds=args.cpu_seconds)
            line["cpu_baseline"] = {"value": rate, "unit": "TFLOP/s", "cores": cores,
                                    "kind": "oracle", "sample": note}
        else:
            rate, cores, note, _ = oracle_step_rate(m, seconds=args.cpu_seconds)
            line["cpu_baseline"] = {"value": rate, "unit": "GB/s", "cores": cores,
                                    "kind": "oracle", "sample": note}
            # the offline weight preparation, beside the GPU's "prepare_weight_24"
            # (the same algorithmic bytes: bf16 weight in, packed weight and scales out)
            t_prep, cores, note = oracle_offline_time(w_bits, seconds=2.0)
            line["offline_cpu_baseline"] = {
                "value": (n * k * 2 + compressed_weight_bytes(n, k) + 4 * n) / t_prep / 1e9,
                "unit": "GB/s", "ms": t_prep * 1e3, "cores": cores, "kind": "oracle",
                "sample": note}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g_step, g_gemm, g_q
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


PREFILL_NAMES = ("qkv", "o", "up", "down")


def prefill_case(args, S, synthetic, dev, bf16, capture, timed, shape_index, steps):
    """One prefill linear (M=8192) on one GPU: the one-call forward (quantiser
    + GEMM) and the GEMM alone, each a CUDA graph of `steps` launches rotating
    weight copies beyond L2, timed like the headline; dense-equivalent TFLOP/s
    against 4 x the measured bf16 peak (burst and sustained), the clocks seen,
    ncu traffic when a capture of the current kernels exists, and the oracle
    on a bounded sample, extrapolated."""
    import torch
    x_bits, w_bits, _, seeds = synthetic.workload_inputs("prefill_8b", shape_index)
    m, k = x_bits.shape
    n = w_bits.shape[0]
    w_dev = bf16(w_bits)
    x_dev = bf16(x_bits)
    packed, sw = S.sfp8_prepare_weight_24(w_dev, "e4m3")
    del w_dev
    n_copies = max(2, -(-150 * 2 ** 20 // (packed.numel() + 2 * m * n)))
    copies = [(packed.clone(), sw.clone()) for _ in range(n_copies)]
    del packed
    aq = torch.empty((m, k), dtype=torch.uint8, device=dev)
    sa = torch.empty((m,), dtype=torch.float32, device=dev)
    ys = [torch.empty((m, n), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    ws = S.new_workspace(m, n, k, dev)
    ws_q = S.new_quant_workspace(m, n, k, dev)

    def step(j):
        pk, s_ = copies[j % len(copies)]
        S.sfp8_sparse_linear_quant(x_dev, "e4m3", pk, "e4m3", s_, n, k, out=ys[j % 2],
                                   workspace=ws_q, a_q=aq, s_a=sa)

    def gemm(j):
        pk, s_ = copies[j % len(copies)]
        S.sfp8_sparse_linear(aq, "e4m3", sa, pk, "e4m3", s_, n, k, out=ys[j % 2],
                             workspace=ws)

    for j in range(args.warmup):
        step(j)
    torch.cuda.synchronize(dev)
    g_gemm = capture(gemm, steps)
    # Burst: the regime of the burst peak it is compared with (a best-of-N
    # GEMM loop): after a short idle, the best of a few replays of the graph.
    g_gemm.replay()
    torch.cuda.synchronize(dev)
    time.sleep(0.2)
    with ClockSampler(dev.index) as clk_burst:
        burst = []
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g_gemm.replay()
            e1.record()
            e1.synchronize()
            burst.append(e0.elapsed_time(e1))
    ms_burst = min(burst)
    # Sustained: the median of replays for about --timed-seconds, long enough for
    # the power cap to settle the clock, compared with the sustained peak.
    with ClockSampler(dev.index) as clk:
        g = capture(step, steps)
        ms_step, replays = timed(g)
        del g
        ms_gemm, _ = timed(g_gemm)
    del g_gemm
    flops = 2.0 * m * n * k
    gemm_us = ms_gemm * 1e3 / steps
    burst_us = ms_burst * 1e3 / steps
    step_us = ms_step * 1e3 / steps
    tf = flops / (gemm_us * 1e-6) / 1e12
    tf_burst = flops / (burst_us * 1e-6) / 1e12
    peak, peak_kind = measured_tensor_peak()
    peak_sus, peak_sus_kind = measured_tensor_peak(sustained=True)
    traffic = None
    rec = NCU_TRAFFIC.get(("prefill_8b", shape_index))
    if rec is not None and rec["sha1"] == kernel_source_sha1():
        traffic = rec["bytes_per_launch"]
    out = {"shape": PREFILL_NAMES[shape_index], "m": m, "k": k, "n": n, "seeds": seeds,
           "steps": steps, "replays": replays, "weight_copies": len(copies),
           "gemm_us": gemm_us, "step_us": step_us, "TFLOP/s": tf,
           "step_TFLOP/s": flops / (step_us * 1e-6) / 1e12,
           "gemm_us_burst": burst_us, "TFLOP/s_burst": tf_burst,
           "roofline": {"bound": "tensor", "achieved": tf_burst, "peak": peak,
                        "frac": tf_burst / peak, "peak_source": peak_kind,
                        "timing": "frac: best of 5 replays after a 0.2 s idle (burst) against "
                                  "the burst peak; frac_sustained: median over about %.2f s of "
                                  "replays against the sustained peak" % args.timed_seconds,
                        "achieved_sustained": tf, "peak_sustained": peak_sus,
                        "frac_sustained": tf / peak_sus, "unit": "TFLOP/s",
                        "peak_datasheet": DATASHEET_SPARSE_FP8_TFLOPS,
                        "frac_datasheet": tf_burst / DATASHEET_SPARSE_FP8_TFLOPS,
                        "traffic": traffic, "kernel": "sparse_linear_pair_kernel",
                        "algorithmic_flop_per_launch": flops},
           "clocks": clk.summary(), "clocks_burst": clk_burst.summary()}
    del copies, aq, sa, ys, ws, ws_q, x_dev
    torch.cuda.empty_cache()
    if not args.no_cpu_baseline:
        rate, cores, note = oracle_prefill_rate(x_bits, w_bits, seconds=args.cpu_seconds_prefill)
        out["cpu_baseline"] = {"value": rate, "unit": "TFLOP/s", "cores": cores,
                               "kind": "oracle", "sample": note}
    return out


# ----------------------------------------------------------------- tensor-wise quantiser

# The conversion sizes of the page "[float8nocompile] Add alternate Triton
# kernels for FP8 conversion ..." (pytorch/ao pull request 1455), its tables.
TENSORWISE_SIZES = (65500, 1 << 20, 1 << 24, 1 << 28)


def run_tensorwise(args):
    """Times sfp8_quantize_tensorwise (both amax modes, bf16 and fp32 input,
    e4m3 output) on the pages' conversion sizes.  Each timed call follows a
    256 MB write that evicts the input from L2; CUDA events bracket the call
    alone, and the median over the repetitions is reported (`us`); `us_warm`
    is the mean of back-to-back calls without the flush."""
    import torch
    rank, local, world = dist_setup("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import semi_structured_sparse_rowwise_b200 as S
    S.load_library()
    peak, peak_kind = measured_peaks()
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev)
    g = torch.Generator(device=dev).manual_seed(1004)
    reps = max(args.steps, 5)
    table = []
    dtypes = {"f32": torch.float32, "bf16": torch.bfloat16}
    sizes = [int(v) for v in args.tw_numel.split(",")] if args.tw_numel else TENSORWISE_SIZES
    with ClockSampler(local) as clk:
        for dtype in [dtypes[d] for d in args.tw_dtype.split(",")]:
            for numel in sizes:
                x = torch.randn(numel, generator=g, device=dev, dtype=torch.float32).to(dtype)
                q = torch.empty((numel,), dtype=torch.uint8, device=dev)
                sc = torch.empty((1,), dtype=torch.float32, device=dev)
                for mode in ("reduce", "atomic"):
                    ws = S.new_tensorwise_workspace(mode, dev)
                    for _ in range(args.warmup):
                        S.sfp8_quantize_tensorwise(x, "e4m3", mode, q=q, scale=sc, workspace=ws)
                    ev = [(torch.cuda.Event(enable_timing=True),
                           torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
                    torch.cuda.synchronize(dev)
                    for e0, e1 in ev:
                        flush.fill_(1)
                        e0.record()
                        S.sfp8_quantize_tensorwise(x, "e4m3", mode, q=q, scale=sc, workspace=ws)
                        e1.record()
                    torch.cuda.synchronize(dev)
                    times = sorted(e0.elapsed_time(e1) * 1e3 for e0, e1 in ev)
                    us = times[len(times) // 2]
                    # warm: back-to-back calls, no flush (the input stays in
                    # L2 when it fits), the mean over the repetitions
                    w0, w1 = (torch.cuda.Event(enable_timing=True),
                              torch.cuda.Event(enable_timing=True))
                    w0.record()
                    for _ in range(reps):
                        S.sfp8_quantize_tensorwise(x, "e4m3", mode, q=q, scale=sc, workspace=ws)
                    w1.record()
                    w1.synchronize()
                    us_warm = w0.elapsed_time(w1) * 1e3 / reps
                    alg = numel * (x.element_size() + 1) + 4
                    table.append({"numel": numel, "dtype": str(dtype).replace("torch.", ""),
                                  "mode": mode, "us": us, "GB/s": alg / (us * 1e-6) / 1e9,
                                  "frac": alg / (us * 1e-6) / 1e9 / peak, "us_warm": us_warm})
                del x, q
    st, flags = S.sfp8_read_device_status(clear=True)
    if st != 0:
        raise RuntimeError("device status %d flags %#x" % (st, flags))
    big = [r for r in table if r["numel"] == max(sizes)]
    best = max(big, key=lambda r: r["GB/s"])
    line = {
        "metric": "tensor-wise FP8 quantise GB/s (one global amax)", "value": best["GB/s"],
        "unit": "GB/s", "n_gpus": world, "steps": reps, "warmup": args.warmup,
        "higher_is_better": True, "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": "quantize_tensorwise", "sizes": list(sizes),
                   "l2": "256 MB write before every timed call", "seed": 1004},
        "roofline": {"bound": "hbm", "achieved": best["GB/s"], "peak": peak, "unit": "GB/s",
                     "frac": best["GB/s"] / peak, "traffic": None,
                     "kernel": "quantize_tensorwise_kernel",
                     "algorithmic_bytes": "numel * (input bytes + 1) + 4 (one read, one write)",
                     "peak_source": peak_kind},
        "table": table, "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- dtype sweep and stress

def matrix_cases(args, workload, S, synthetic, dev, bf16, cases=None):
    """Times the one-call forward (quantiser + GEMM) and the GEMM alone for
    every case of the dtype-sweep workload (M in {1, 16, 128, 1024, 8192} x
    the four e4m3/e5m2 operand pairs, K=4096, N=14336, Student-t activations,
    bf16 bias) or for the 70B stress shape (M=16384, K=8192, N=28672, 2 %
    zero rows).  Each case's steps are one CUDA graph rotating enough
    compressed-weight copies to exceed L2, replayed once after an untimed
    replay.  Memory-bound cases (M <= 128) are reported in GB/s of compressed
    weight against the copy peak, the others in dense-equivalent TFLOP/s
    against 4 x the bf16 peak (burst and sustained).  Returns (table, clocks)."""
    import torch
    hbm_peak, hbm_kind = measured_peaks()
    fl_peak, fl_kind = measured_tensor_peak()
    fl_sus, fl_sus_kind = measured_tensor_peak(sustained=True)
    if cases is None:
        if workload == "stress_70b_mlp":
            cases = [(0, "e4m3", "e4m3")]
        else:
            cases = [(i, a, w) for i in range(5) for a in ("e4m3", "e5m2")
                     for w in ("e4m3", "e5m2")]
    table = []
    w_cache = {}
    inputs = {}
    oracle_step_s = {}
    with ClockSampler(dev.index) as clk:
        for shape_index, a_fmt, w_fmt in cases:
            if shape_index not in inputs:
                # the same seeded inputs serve every operand pair of a shape
                inputs.clear()
                inputs[shape_index] = synthetic.workload_inputs(workload, shape_index)
                if not args.no_cpu_baseline:
                    # the oracle on a bounded sample of this shape (host only)
                    clk.pause()
                    xb, wb = inputs[shape_index][0], inputs[shape_index][1]
                    rows = min(64, xb.shape[0])
                    rate, cores, note = oracle_prefill_rate(
                        xb, wb, seconds=args.cpu_seconds_matrix, rows=rows, n_sample=512)
                    m_, k_ = xb.shape
                    oracle_step_s[shape_index] = (
                        2.0 * m_ * wb.shape[0] * k_ / (rate * 1e12), cores,
                        note if rows < m_ else note.replace("extrapolated", "sampled in N"))
                    clk.resume()
            x_bits, w_bits, b_bits, seeds = inputs[shape_index]
            m, k = x_bits.shape
            n = w_bits.shape[0]
            key = (w_fmt, n, k)
            if key not in w_cache:
                w_cache.clear()
                w_dev = bf16(w_bits)
                packed, sw = S.sfp8_prepare_weight_24(w_dev, w_fmt)
                del w_dev
                n_copies = max(2, -(-200 * 2 ** 20 // packed.numel()))
                w_cache[key] = [(packed.clone(), sw.clone()) for _ in range(n_copies)]
            copies = w_cache[key]
            x = bf16(x_bits)
            bias = bf16(b_bits) if b_bits is not None else None
            ys = [torch.empty((m, n), dtype=torch.bfloat16, device=dev) for _ in range(2)]
            aq = torch.empty((m, k), dtype=torch.uint8, device=dev)
            sa = torch.empty((m,), dtype=torch.float32, device=dev)
            ws = S.new_quant_workspace(m, n, k, dev)
            steps = max(3, min(args.steps, int(4e5 / max(1.0, 2.0 * m * n * k / 1e9))))

            def step(j):
                pk, s_ = copies[j % len(copies)]
                S.sfp8_sparse_linear_quant(x, a_fmt, pk, w_fmt, s_, n, k, bias=bias,
                                           out=ys[j % 2], workspace=ws, a_q=aq, s_a=sa)

            def gemm(j):
                pk, s_ = copies[j % len(copies)]
                S.sfp8_sparse_linear(aq, a_fmt, sa, pk, w_fmt, s_, n, k, bias=bias,
                                     out=ys[j % 2], workspace=ws)

            res = {}
            for name, fn in (("step", step), ("gemm", gemm)):
                for j in range(3):
                    fn(j)
                torch.cuda.synchronize(dev)
                g = torch.cuda.CUDAGraph()
                st = torch.cuda.Stream(dev)
                st.wait_stream(torch.cuda.current_stream(dev))
                with torch.cuda.stream(st):
                    with torch.cuda.graph(g, stream=st):
                        for j in range(steps):
                            fn(j)
                torch.cuda.current_stream(dev).wait_stream(st)
                g.replay()
                torch.cuda.synchronize(dev)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                g.replay()
                e1.record()
                e1.synchronize()
                res[name] = e0.elapsed_time(e1) * 1e3 / steps
                del g
            wbytes = compressed_weight_bytes(n, k)
            flops = 2.0 * m * n * k
            row = {"m": m, "k": k, "n": n, "a": a_fmt, "w": w_fmt, "bias": bias is not None,
                   "step_us": res["step"], "gemm_us": res["gemm"], "steps": steps}
            cpu = oracle_step_s.get(shape_index)
            if m <= 128:
                gbs = gemm_algorithmic_bytes(m, n, k) / (res["gemm"] * 1e-6) / 1e9
                row.update({"bound": "hbm", "GB/s": gbs, "frac": gbs / hbm_peak,
                            "frac_datasheet": gbs / DATASHEET_HBM_GBS,
                            "step_GB/s_weight": wbytes / (res["step"] * 1e-6) / 1e9})
                if cpu is not None:
                    row["cpu_baseline"] = {"value": wbytes / cpu[0] / 1e9,
                                           "unit": "GB/s of compressed weight per step",
                                           "cores": cpu[1], "kind": "oracle", "sample": cpu[2]}
            else:
                tf = flops / (res["gemm"] * 1e-6) / 1e12
                row.update({"bound": "tensor", "TFLOP/s": tf, "frac": tf / fl_peak,
                            "frac_sustained": tf / fl_sus,
                            "frac_datasheet": tf / DATASHEET_SPARSE_FP8_TFLOPS,
                            "step_TFLOP/s": flops / (res["step"] * 1e-6) / 1e12})
                if cpu is not None:
                    row["cpu_baseline"] = {"value": flops / cpu[0] / 1e12, "unit": "TFLOP/s",
                                           "cores": cpu[1], "kind": "oracle", "sample": cpu[2]}
            table.append(row)
            del x, ys, aq, sa, ws
    return table, clk.summary()


def run_matrix(args):
    """The dtype-sweep or stress workload as its own JSON line (matrix_cases)."""
    import numpy as np
    import torch
    rank, local, world = dist_setup("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import semi_structured_sparse_rowwise_b200 as S
    from semi_structured_sparse_rowwise_b200 import synthetic
    S.load_library()
    hbm_peak, hbm_kind = measured_peaks()
    fl_peak, fl_kind = measured_tensor_peak()
    fl_sus, fl_sus_kind = measured_tensor_peak(sustained=True)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
            torch.bfloat16).to(dev)

    table, clocks = matrix_cases(args, args.workload, S, synthetic, dev, bf16)
    st_, flags = S.sfp8_read_device_status(clear=True)
    if st_ != 0:
        raise RuntimeError("device status %d flags %#x" % (st_, flags))
    big = max(table, key=lambda r: r["m"])
    line = {
        "metric": METRIC, "value": big.get("TFLOP/s", big.get("GB/s")),
        "unit": "TFLOP/s" if big["bound"] == "tensor" else "GB/s", "n_gpus": world,
        "higher_is_better": True, "dtype": "fp8", "data": "synthetic",
        "config": {"workload": args.workload, "l2": "rotating >= 200 MB of compressed weight"},
        "peaks": {"hbm": [hbm_peak, hbm_kind], "tensor": [fl_peak, fl_kind],
                  "tensor_sustained": [fl_sus, fl_sus_kind],
                  "hbm_datasheet": DATASHEET_HBM_GBS,
                  "sparse_fp8_datasheet": DATASHEET_SPARSE_FP8_TFLOPS},
        "table": table, "clocks": clocks,
    }
    if "cpu_baseline" in big:
        line["cpu_baseline"] = big["cpu_baseline"]
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--m", type=int, default=16, choices=[1, 4, 16])
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=[WORKLOAD, "prefill_8b", "quantize_tensorwise", "dtype_sweep_8b_up",
                             "stress_70b_mlp"],
                    help="decode gate/up (default, GB/s), the prefill linears (TFLOP/s), the "
                    "standalone tensor-wise quantiser on the pages' conversion sizes, the "
                    "dtype sweep (M x four FP8 operand pairs) or the 70B stress shape")
    ap.add_argument("--shape", type=int, default=2, choices=[0, 1, 2, 3],
                    help="prefill_8b shape: 0 QKV, 1 O, 2 up (default), 3 down")
    ap.add_argument("--tw-numel", default="",
                    help="quantize_tensorwise: comma-separated element counts (default: the "
                    "pages' 65500, 2^20, 2^24, 2^28)")
    ap.add_argument("--tw-dtype", default="f32,bf16",
                    help="quantize_tensorwise: input dtypes, comma-separated (f32, bf16)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--all-m", action="store_true", help="also time M=1 and M=4")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--cpu-seconds-matrix", type=float, default=1.0,
                    help="seconds of oracle work per shape of the sweep and stress tables")
    ap.add_argument("--cpu-seconds-prefill", type=float, default=3.0,
                    help="oracle seconds per prefill shape in the default run")
    ap.add_argument("--replays", type=int, default=0,
                    help="timed replays of each K-step graph (0: about --timed-seconds)")
    ap.add_argument("--timed-seconds", type=float, default=0.25)
    ap.add_argument("--kernel-steps", type=int, default=100,
                    help="launches per graph when timing the dominant kernel alone for the "
                    "roofline (at least --steps)")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the four M=8192 prefill shapes of the default run")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the dtype sweep and the stress shape of the default run")
    ap.add_argument("--no-pipeline", action="store_true",
                    help="skip the layer's HostPipeline end-to-end leg")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "quantize_tensorwise":
        return run_tensorwise(args)
    if args.workload in ("dtype_sweep_8b_up", "stress_70b_mlp"):
        return run_matrix(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
