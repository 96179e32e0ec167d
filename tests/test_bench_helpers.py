"""The bench's arithmetic, on the CPU: the algorithmic bytes behind the
roofline's numerator agree with the oracle's packed-layout size and with the
decode figures stated for the workload (36 700 160 B of compressed weight,
37 281 856 B per GEMM launch at M=16, K=4096, N=14336), and the argument
parser accepts every workload mode."""
import os
import subprocess
import sys

import pytest

import bench
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("n,k", [(1, 128), (64, 128), (129, 384), (14336, 4096), (4096, 14336),
                                 (28672, 8192)])
def test_compressed_bytes_match_the_layout(n, k):
    assert bench.compressed_weight_bytes(n, k) == oracle.packed_bytes(n, k)


def test_decode_algorithmic_bytes():
    assert bench.compressed_weight_bytes(14336, 4096) == 36700160
    assert bench.gemm_algorithmic_bytes(16, 14336, 4096) == 37281856
    # weight + s_w + A_q + s_a + y
    assert bench.gemm_algorithmic_bytes(1, 14336, 4096) == (
        36700160 + 4 * 14336 + 4096 + 4 + 2 * 14336)


def test_parser_accepts_every_mode():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--help"],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    for mode in ("decode_gate_up_8b", "prefill_8b", "quantize_tensorwise", "dtype_sweep_8b_up",
                 "stress_70b_mlp"):
        assert mode in r.stdout


class _FakeNvml:
    """Stands in for pynvml: a clock the test sets and a power-cap reason."""
    NVML_CLOCK_SM = 0

    def __init__(self):
        self.mhz = 1965

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByIndex(self, i):
        return i

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        return self.mhz

    def nvmlDeviceGetCurrentClocksThrottleReasons(self, h):
        return 0x4          # sw_power_cap


def test_clock_sampler_pause_keeps_host_only_time_out(monkeypatch):
    """Samples taken while paused (host-only work, idle GPU clocks) must not
    enter the record; the throttle reasons are named."""
    import time
    fake = _FakeNvml()
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    with bench.ClockSampler(0, period_s=0.001) as clk:
        time.sleep(0.05)
        clk.pause()
        n_before = len(clk.samples)
        fake.mhz = 345                      # what an idle GPU would report
        time.sleep(0.05)
        n_paused = len(clk.samples)
        fake.mhz = 1965
        clk.resume()
        time.sleep(0.05)
    s = clk.summary()
    assert n_before > 0
    assert n_paused <= n_before + 1          # at most one sample already in flight
    assert 345 not in clk.samples[n_before + 1:]
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == len(clk.samples)


def test_oracle_sample_extrapolates_linearly():
    """The oracle baseline on a bounded sample: a positive dense-equivalent
    rate, labelled as extrapolated from the rows and columns it timed."""
    from semi_structured_sparse_rowwise_b200 import synthetic
    x = synthetic.activation(11, 8, 256)
    w = synthetic.weight(12, 96, 256)
    rate, cores, note = bench.oracle_prefill_rate(x, w, seconds=0.05, rows=4, n_sample=32)
    assert rate > 0 and cores >= 1
    assert note.startswith("extrapolated") and "4 of 8 activation rows" in note
    assert "32 of 96 output columns" in note


def test_oracle_offline_sample_scales_to_all_rows():
    """The offline oracle baseline (prune + quantise + compress) on a sample
    of rows: a positive time for the whole weight, labelled as extrapolated."""
    from semi_structured_sparse_rowwise_b200 import synthetic
    w = synthetic.weight(13, 64, 256)
    t, cores, note = bench.oracle_offline_time(w, seconds=0.05, n_sample=16)
    assert t > 0 and cores >= 1
    assert note.startswith("extrapolated") and "16 of 64 weight rows" in note
