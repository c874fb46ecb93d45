"""The benchmark's accounting (CPU): the algorithmic work per step behind
the roofline, the launch count it claims, and the MaxVio it reports, on the
figures the workload definitions fix."""
import types

import pytest
import torch

import bench


def test_algorithmic_work_of_the_million_token_step():
    # N = 2^20, d = 2560, E = 384, K = 6: 2 N d E FLOP = 2.062 TFLOP; bytes
    # 2Nd (x) + 8NE (Z written and read) + 16NK (ids, gates, perm, inv) + 4N
    # (alpha) + 2Ed (W) = 8.70 GB
    flops, bytes_ = bench.algorithmic_work(1 << 20, 2560, 384, 6)
    assert flops == 2.0 * (1 << 20) * 2560 * 384
    assert round(flops / 1e12, 3) == 2.062
    assert round(bytes_ / 1e9, 2) == 8.70
    n = 1 << 20
    assert bytes_ == 2 * n * 2560 + 8 * n * 384 + 16 * n * 6 + 4 * n + 2 * 384 * 2560


def test_gemm_bytes():
    assert bench.gemm_bytes(4, 64, 16) == 2 * 4 * 64 + 4 * 4 * 16 + 2 * 16 * 64


@pytest.mark.parametrize("N,K,want", [
    (1 << 20, 6, 2 + 6 + 3),      # bracketed EQB chain, tiled permutation
    (16384, 6, 2 + 3 + 3),        # the sample is the column
    (256, 6, 2 + 3 + 1),          # one-block permutation (N K <= 4096)
])
def test_launches_per_step(N, K, want):
    assert bench.launches_per_step(N, 384, K) == want


def test_maxvio_of_loads():
    wl = types.SimpleNamespace(N=4, K=2, E=4)          # mean load N K / E = 2
    assert bench.maxvio(torch.tensor([2, 2, 2, 2], dtype=torch.int32), wl) == 0.0
    # the collapsed toy router of section 7.2: two experts take every slot
    assert bench.maxvio(torch.tensor([4, 0, 0, 4], dtype=torch.int32), wl) == 1.0
