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
