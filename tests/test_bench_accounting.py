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
    (1 << 20, 6, 2 + 4 + 3),      # bracketed EQB chain, tiled permutation
    (16384, 6, 2 + 2 + 3),        # the sample is the column
    (256, 6, 2 + 2 + 1),          # one-block permutation (N K <= 4096)
])
def test_launches_per_step(N, K, want):
    assert bench.launches_per_step(N, 384, K) == want


def test_maxvio_of_loads():
    wl = types.SimpleNamespace(N=4, K=2, E=4)          # mean load N K / E = 2
    assert bench.maxvio(torch.tensor([2, 2, 2, 2], dtype=torch.int32), wl) == 0.0
    # the collapsed toy router of section 7.2: two experts take every slot
    assert bench.maxvio(torch.tensor([4, 0, 0, 4], dtype=torch.int32), wl) == 1.0


def test_algorithmic_work_of_the_collapsed_loop():
    # ten routings + updates over one GEMM's Z: x and the Z write once, then
    # per update Z read once, ids/gates/perm/inv and alpha
    N, d, E, K = 16384, 2560, 384, 6
    flops, bytes_ = bench.algorithmic_work(N, d, E, K, updates=10)
    assert flops == 2.0 * N * d * E
    assert bytes_ == 2 * N * d + 4 * N * E + 2 * E * d + 10 * (4 * N * E + 16 * N * K + 4 * N)
    # one update is the step's own accounting
    assert bench.algorithmic_work(N, d, E, K, updates=1) == bench.algorithmic_work(N, d, E, K)


def test_launches_of_the_collapsed_loop():
    # forward 2, permutation 3, update 2 (the sample is the column), then nine
    # times re-route 1 + update 2 + permutation 3
    assert bench.launches_per_step(16384, 384, 6, updates=10) == 2 + 2 + 3 + 9 * 6


@pytest.mark.parametrize("timed_s,reasons,kind", [
    (0.046, ["sw_power_cap"], "burst"),        # short region: the burst figure
    (1.0, [], "burst"),                        # long, but never capped
    (1.0, ["sw_power_cap"], "sustained"),      # long and capped
])
def test_bf16_peak_follows_the_run(timed_s, reasons, kind):
    peaks = {"bf16_tflops": 1622.9, "bf16_tflops_sustained": 1354.4}
    peak, got = bench.choose_bf16_peak(peaks, {"reasons": reasons}, timed_s)
    assert got == kind
    assert peak == (1622.9 if kind == "burst" else 1354.4)
