"""GPU router logits against the oracle's fp64 sums: |dZ| <= 1e-3 max(1, |Z|),
plus closed-form special cases that must be exact.  Batches of up to 1024
tokens take the clustered split-d kernel (its tile changes at 16, 32, 512
tokens and with d a multiple of 128 or not); larger ones the tcgen05 pair
GEMM."""
import numpy as np
import pytest
import torch

from expert_load_balancing_b200 import binding as B
from expert_load_balancing_b200 import workloads

from gpu_helpers import assert_logits_close, check_status, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(kolibri_lib):
    return kolibri_lib


def _run(x, w):
    z = B.kolibri_router_logits(x.cuda(), w.cuda())
    return host(z)


@pytest.mark.parametrize("N,d,E", [(1, 2560, 384), (127, 2560, 384), (128, 2560, 384),
                                   (300, 2560, 384), (1000, 2048, 128), (2049, 256, 512),
                                   (77, 64, 16), (640, 640, 272), (130, 1024, 48)])
def test_logits_random(oracle_mod, N, d, E):
    wl = workloads.Workload("t", N, d, E, 4, offsets="collapsed8" if E >= 16 else "none")
    x = workloads.make_x(wl)
    w = workloads.make_w(wl)
    z = _run(x, w)
    zr = oracle_mod.router_logits(workloads.bf16_bits(x), workloads.bf16_bits(w))
    err = assert_logits_close(z, zr)
    assert err < 1e-4, err     # fp32 accumulation of exact bf16 products
    check_status()


@pytest.mark.parametrize("N", [1, 15, 16, 17, 32, 33, 64, 65, 511, 512, 513, 1024, 1025])
@pytest.mark.parametrize("d,E", [(2560, 384), (320, 400), (1024, 48)])
def test_logits_small_batches(oracle_mod, N, d, E):
    wl = workloads.Workload("t", N, d, E, 4, offsets="collapsed8")
    x = workloads.make_x(wl)
    w = workloads.make_w(wl)
    z = _run(x, w)
    zr = oracle_mod.router_logits(workloads.bf16_bits(x), workloads.bf16_bits(w))
    err = assert_logits_close(z, zr)
    assert err < 1e-4, err
    # the split sums are added in a fixed order: a second call repeats every bit
    np.testing.assert_array_equal(_run(x, w), z)
    check_status()


def test_logits_small_constant_rows_exact():
    d, E = 2560, 384
    for N in (3, 40, 300):
        x = torch.full((N, d), 0.5, dtype=torch.bfloat16)
        w = ((torch.arange(E, dtype=torch.float32) % 7 + 1) / 16).repeat(d, 1).T.contiguous()
        z = _run(x, w.to(torch.bfloat16))
        expect = np.float32(d * 0.5) * ((np.arange(E) % 7 + 1) / 16).astype(np.float32)
        np.testing.assert_array_equal(z, np.tile(expect, (N, 1)))


def test_logits_one_hot_exact(oracle_mod):
    d, E = 256, 384
    w = (torch.randn(E, d, generator=torch.Generator().manual_seed(3))).to(torch.bfloat16)
    x = torch.zeros(d, d, dtype=torch.bfloat16)
    x[torch.arange(d), torch.arange(d)] = 1.0
    z = _run(x, w)
    np.testing.assert_array_equal(z, w.float().numpy().T)


def test_logits_constant_rows_exact():
    d, E = 2560, 384
    x = torch.full((200, d), 0.5, dtype=torch.bfloat16)
    w = ((torch.arange(E, dtype=torch.float32) % 7 + 1) / 16).repeat(d, 1).T.contiguous()
    z = _run(x, w.to(torch.bfloat16))
    expect = np.float32(d * 0.5) * ((np.arange(E) % 7 + 1) / 16).astype(np.float32)
    np.testing.assert_array_equal(z, np.tile(expect, (200, 1)))


def test_logits_many_tiles_persistent(oracle_mod):
    # more tiles than SMs: every CTA loops; checked on a sample of rows
    N, d, E = 148 * 128 * 2 + 77, 512, 384
    wl = workloads.Workload("t", N, d, E, 6)
    x = workloads.make_x(wl)
    w = workloads.make_w(wl)
    z = _run(x, w)
    rows = np.random.default_rng(0).choice(N, size=700, replace=False)
    rows = np.concatenate([rows, [0, N - 1, N - 77, 128 * 148 - 1, 128 * 148]])
    zr = oracle_mod.router_logits(workloads.bf16_bits(x[rows]), workloads.bf16_bits(w))
    assert_logits_close(z[rows], zr)
    check_status()


def test_logits_into_strided_buffer_rejected():
    x = torch.zeros(10, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(16, 64, dtype=torch.bfloat16, device="cuda")
    z = torch.empty(10, 32, dtype=torch.float32, device="cuda")[:, :16]
    with pytest.raises(ValueError):
        B.kolibri_router_logits(x, w, z)
