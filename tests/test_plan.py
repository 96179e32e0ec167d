"""The GEMM's work-split planning, on the CPU (host-only queries, no device).

Pins the built-in rule (algorithm 0) on the workloads' shapes for a 148-SM
B200 -- the choices the search on the GPU found fastest -- and checks
invariants of every algorithm offered for a sweep of shapes: shared memory
within the per-CTA limit, producers no more than ring stages, the resident
activation only for one token tile of at most 32, CTA-pair tiles in steps of
32 up to 224, k steps per stage dividing k, a workspace exactly for the
stream-K splits, no repeated algorithm.
"""
import itertools

import pytest

from semi_structured_sparse_rowwise_b200 import binding as B, build

SMS = 148
SMEM_LIMIT = 232448          # 227 KB of dynamic shared memory per CTA


@pytest.fixture(scope="module", autouse=True)
def lib():
    build.build()
    return B.load_library()


# (m, n, k) -> the built-in choice
RULE = [
    ((16, 14336, 4096), dict(pair=0, bn=16, ks=4, whole_tiles=1, ra=1, grid=112)),   # decode
    ((1, 14336, 4096), dict(pair=0, bn=16, ks=4, whole_tiles=1, ra=1, grid=112)),
    ((32, 14336, 4096), dict(pair=0, bn=32, ks=4, whole_tiles=1, grid=112)),
    ((128, 14336, 4096), dict(pair=1, bn=128, ks=2, wt=1, grid=112)),                # sweep
    ((192, 14336, 4096), dict(pair=1, bn=192, ks=2, wt=1)),
    ((100, 14336, 4096), dict(pair=1, bn=128, ks=2, wt=1)),
    ((64, 14336, 4096), dict(pair=1, bn=64, ks=2, wt=1)),
    ((96, 14336, 4096), dict(pair=1, bn=96, ks=2, wt=1)),
    ((32, 14336, 4096), dict(pair=0, bn=32)),
    ((16, 4096, 4096), dict(pair=0, bn=16, whole_tiles=1, grid=32)),              # short k
    ((128, 4096, 4096), dict(pair=0, bn=32, ks=4, whole_tiles=1, grid=128)),
    ((128, 4096, 14336), dict(pair=0, bn=32, ks=4, whole_tiles=1, grid=128)),
    ((16, 4096, 14336), dict(pair=0, bn=16, ks=4, whole_tiles=0, grid=148)),        # stream-K
    ((256, 14336, 4096), dict(pair=1, bn=128, ks=2, wt=2)),
    ((384, 14336, 4096), dict(pair=1, bn=192, ks=2, wt=2)),
    ((8192, 14336, 4096), dict(pair=1, bn=224, ks=2, wt=1, grid=148)),             # prefill up
    ((8192, 6144, 4096), dict(pair=1, bn=224, ks=2, wt=1)),                        # QKV
    ((8192, 4096, 14336), dict(pair=1, bn=224, ks=2, wt=2)),                       # down
    ((16384, 28672, 8192), dict(pair=1, bn=224, ks=2, wt=2)),                      # 70B stress
]


@pytest.mark.parametrize("shape,want", RULE)
def test_builtin_rule(shape, want):
    got = B.sfp8_sparse_linear_plan(*shape, SMS, 0)
    for key, val in want.items():
        assert got[key] == val, (shape, key, got)


SWEEP = list(itertools.product((1, 5, 16, 17, 32, 40, 64, 100, 128, 200, 256, 300, 384, 511,
                                512, 700, 1024, 8192),
                               (1, 64, 300, 1000, 4096, 14336),
                               (128, 384, 4096, 14336)))


@pytest.mark.parametrize("m,n,k", SWEEP[::7])
def test_every_algorithm_is_a_valid_plan(m, n, k):
    count = B.sfp8_sparse_linear_plan_count(m, n, k, SMS)
    assert 1 <= count <= 96
    seen = set()
    k_steps = k // 128
    for a in range(count):
        p = B.sfp8_sparse_linear_plan(m, n, k, SMS, a)
        key = (p["pair"], p["bn"], p["ks"], p["wt"], p["whole_tiles"])
        assert key not in seen
        seen.add(key)
        assert 0 < p["smem_bytes"] <= SMEM_LIMIT
        assert 1 <= p["stages"] <= 16 and 1 <= p["producers"] <= min(4, p["stages"])
        assert k_steps % p["ks"] == 0
        assert p["m_tiles"] == -(-m // p["bn"])
        assert 1 <= p["grid"] <= SMS
        if p["pair"]:
            assert p["bn"] % 32 == 0 and 32 <= p["bn"] <= 224 and p["wt"] in (1, 2)
            assert p["ks"] in (1, 2) and p["workspace_bytes"] == 0 and p["grid"] % 2 == 0
        else:
            assert p["bn"] in (16, 32, 64, 128) and p["wt"] == 1
            assert p["ks"] in (1, 2, 4) and (p["ks"] < 4 or p["bn"] <= 32)
            if p["ra"]:
                assert p["m_tiles"] == 1 and p["bn"] <= 32 and p["bn"] * k <= 96 * 1024
            assert (p["workspace_bytes"] > 0) == (p["whole_tiles"] == 0)


def test_deterministic_and_invalid_shapes():
    a = [B.sfp8_sparse_linear_plan(300, 1000, 4096, SMS, i)
         for i in range(B.sfp8_sparse_linear_plan_count(300, 1000, 4096, SMS))]
    b = [B.sfp8_sparse_linear_plan(300, 1000, 4096, SMS, i)
         for i in range(B.sfp8_sparse_linear_plan_count(300, 1000, 4096, SMS))]
    assert a == b
    assert B.sfp8_sparse_linear_plan_count(16, 64, 100, SMS) == 0      # k % 128
    assert B.sfp8_sparse_linear_plan_count(0, 64, 128, SMS) == 0
    assert B.sfp8_sparse_linear_plan_count(16, 64, 128, 1) == 0
    with pytest.raises(B.Sfp8Error):
        B.sfp8_sparse_linear_plan(16, 64, 128, SMS, 999)
