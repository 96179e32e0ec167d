"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws random numbers and stores them as bfloat16 bit
patterns; it holds none of the layer's arithmetic (no quantisation, pruning,
compression or matrix product).  Both the CUDA path and the CPU oracle take
their inputs from here.

Shapes follow the Llama-3.1-8B / Llama-3-70B linear layers that the
``generate.py --sparsity semi -q float8dq`` run on the page "Add CUTLASS-based
row-wise scaled sparse FP8 kernel" (pytorch/ao pull request 1671, item 5)
exercises.  No model weights are used: values are drawn from the stated
distributions with ``numpy.random.Generator(PCG64(seed))``.
"""

import numpy as np

E4M3 = "e4m3"
E5M2 = "e5m2"


def rng_for(seed):
    return np.random.Generator(np.random.PCG64(seed))


def f32_to_bf16_bits(x):
    """float32 -> bfloat16 bit patterns, round to nearest even (finite x)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return r


def activation(seed, m, k, dist="normal", outlier_channel_frac=0.0,
               outlier_scale=50.0, zero_row_frac=0.0):
    """Activation [m, k] as bf16 bits.

    dist: "normal" (N(0,1)) or "student_t3" (Student-t, nu = 3).
    outlier_channel_frac: fraction of the k channels (seeded pick) scaled by
    ``outlier_scale``.  zero_row_frac: fraction of rows (seeded pick) set to
    all zero.
    """
    rng = rng_for(seed)
    if dist == "normal":
        x = rng.standard_normal((m, k), dtype=np.float32)
    elif dist == "student_t3":
        x = rng.standard_t(3, size=(m, k)).astype(np.float32)
    else:
        raise ValueError(dist)
    if outlier_channel_frac > 0 and k > 0:
        n_out = max(1, int(round(outlier_channel_frac * k)))
        ch = rng.choice(k, size=n_out, replace=False)
        x[:, ch] *= np.float32(outlier_scale)
    if zero_row_frac > 0 and m > 0:
        n_zero = max(1, int(round(zero_row_frac * m)))
        rows = rng.choice(m, size=n_zero, replace=False)
        x[rows, :] = 0.0
    return f32_to_bf16_bits(x)


def weight(seed, n, k, std=0.02, neg_zero_frac=0.0):
    """Dense (unpruned) weight [n, k] as bf16 bits, N(0, std^2).

    neg_zero_frac: fraction of entries (Bernoulli mask) forced to -0.0.
    """
    rng = rng_for(seed)
    w = rng.standard_normal((n, k), dtype=np.float32) * np.float32(std)
    bits = f32_to_bf16_bits(w)
    if neg_zero_frac > 0:
        mask = rng.random((n, k), dtype=np.float32) < np.float32(neg_zero_frac)
        bits[mask] = np.uint16(0x8000)
    return bits


def bias(seed, n, std=0.1):
    rng = rng_for(seed)
    return f32_to_bf16_bits(rng.standard_normal((n,), dtype=np.float32) * np.float32(std))


# Workloads.  Seeds are 1000 + workload index (+ a sub-index where a workload
# has several shapes), written into every result line.
WORKLOADS = {
    "tiny": {
        "index": 0, "shapes": [(16, 128, 64)],
        "a": {"dist": "normal"}, "w": {"std": 0.02, "neg_zero_frac": 0.05},
        "dtypes": [(E4M3, E4M3)], "bias": False,
    },
    "decode_gate_up_8b": {
        "index": 1, "shapes": [(1, 4096, 14336), (4, 4096, 14336), (16, 4096, 14336)],
        "a": {"dist": "normal"}, "w": {"std": 0.02},
        "dtypes": [(E4M3, E4M3)], "bias": False,
    },
    "prefill_8b": {
        "index": 2,
        "shapes": [(8192, 4096, 6144), (8192, 4096, 4096), (8192, 4096, 14336),
                   (8192, 14336, 4096)],
        "a": {"dist": "normal", "outlier_channel_frac": 0.01, "outlier_scale": 50.0},
        "w": {"std": 0.02},
        "dtypes": [(E4M3, E4M3)], "bias": False,
    },
    "dtype_sweep_8b_up": {
        "index": 3,
        "shapes": [(1, 4096, 14336), (16, 4096, 14336), (128, 4096, 14336),
                   (1024, 4096, 14336), (8192, 4096, 14336)],
        "a": {"dist": "student_t3"}, "w": {"std": 0.02},
        "dtypes": [(E4M3, E4M3), (E4M3, E5M2), (E5M2, E4M3), (E5M2, E5M2)],
        "bias": True,
    },
    "stress_70b_mlp": {
        "index": 4, "shapes": [(16384, 8192, 28672)],
        "a": {"dist": "normal", "zero_row_frac": 0.02}, "w": {"std": 0.01},
        "dtypes": [(E4M3, E4M3)], "bias": False,
    },
}


def workload_inputs(name, shape_index=0, m=None, k=None, n=None):
    """(x_bits [m,k], w_bits [n,k], bias_bits [n] or None, seeds dict).

    ``m``/``k``/``n`` override the workload's shape (same distributions),
    which the tests use to run a workload's recipe at a size the oracle
    finishes quickly.
    """
    wl = WORKLOADS[name]
    m0, k0, n0 = wl["shapes"][shape_index]
    m = m0 if m is None else m
    k = k0 if k is None else k
    n = n0 if n is None else n
    base = 1000 + wl["index"]
    seed_a = base * 100 + 10 * shape_index + 1
    seed_w = base * 100 + 10 * shape_index + 2
    seed_b = base * 100 + 10 * shape_index + 3
    x = activation(seed_a, m, k, **wl["a"])
    w = weight(seed_w, n, k, **wl["w"])
    b = bias(seed_b, n) if wl["bias"] else None
    return x, w, b, {"a": seed_a, "w": seed_w, "bias": seed_b if wl["bias"] else None}
