"""kolibri_router_forward_eqb: logits, routing and the EQB update from the
tokens, with the bracketed full pass inside the GEMM epilogue for large N.

Every output must equal, bit for bit, kolibri_router_forward followed by
kolibri_eqb_update with the alpha it returned, and the quantiles and the new
bias must equal the oracle's exact order statistics on the GPU's own logits
("Kolibri Pre-Training from Scratch" 7.1 update rule, 7.3 exactness)."""
import numpy as np
import pytest
import torch

from expert_load_balancing_b200 import binding as B
from expert_load_balancing_b200 import workloads

from gpu_helpers import assert_bit_equal, check_status, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(kolibri_lib):
    return kolibri_lib


def _separate(x, w, beta, K):
    b = beta.clone()
    z, ids, gates, alpha = B.kolibri_router_forward(x, w, b, K)
    _, q = B.kolibri_eqb_update(z, alpha, b, K)
    return z, ids, gates, alpha, q, b


def _fused(x, w, beta, K):
    b = beta.clone()
    z, ids, gates, alpha, q = B.kolibri_router_forward_eqb(x, w, b, K)
    return z, ids, gates, alpha, q, b


def _check(oracle_mod, x, w, beta, K, steps=1):
    x, w = x.cuda(), w.cuda()
    b_sep, b_fus = beta.cuda(), beta.cuda()
    N, E = x.shape[0], w.shape[0]
    m = (N * K) // E
    for step in range(steps):
        sep = _separate(x, w, b_sep, K)
        fus = _fused(x, w, b_fus, K)
        torch.cuda.synchronize()
        check_status()
        for g, s_, name in zip(fus, sep, ("z", "ids", "gates", "alpha", "quantiles", "beta")):
            assert_bit_equal(host(g), host(s_), f"step {step}: {name}")
        z, alpha = host(fus[0]), host(fus[3])
        v_o = oracle_mod.column_quantiles(z, alpha, m)
        assert_bit_equal(host(fus[4]), v_o, f"step {step}: quantiles vs oracle")
        assert_bit_equal(host(fus[5]), oracle_mod.eqb_bias(v_o), f"step {step}: beta vs oracle")
        b_sep, b_fus = sep[5], fus[5]


CASES = [
    # N, d, E, K, logit offsets, beta
    (70001, 512, 384, 6, "zipf1.1", "normal0.1"),    # bracket pass in the epilogue
    (40000, 256, 128, 8, "none", "normal0.1"),       # Origin-like: groups of 8 columns
    (16384, 512, 384, 6, "zipf1.1", "normal0.1"),    # the sample is the whole column
    (16385, 256, 384, 6, "collapsed8", "zeros"),     # smallest N with brackets
    (30000, 256, 400, 6, "none", "normal0.1"),       # E past the fused kernel
]


@pytest.mark.parametrize("N,d,E,K,offsets,beta", CASES)
def test_forward_eqb_matches_separate_and_oracle(oracle_mod, N, d, E, K, offsets, beta):
    wl = workloads.Workload("t", N, d, E, K, offsets=offsets, beta=beta)
    _check(oracle_mod, workloads.make_x(wl), workloads.make_w(wl), workloads.make_beta(wl), K)


def test_forward_eqb_three_steps_collapsed(oracle_mod):
    # a collapsed router re-balanced step after step: beta moves a lot, the
    # brackets come from each step's own sample
    wl = workloads.Workload("t", 50000, 256, 384, 6, offsets="collapsed8", beta="zeros")
    _check(oracle_mod, workloads.make_x(wl), workloads.make_w(wl), workloads.make_beta(wl), 6,
           steps=3)


def test_forward_eqb_ties_and_overflow_rows(oracle_mod):
    # a third of the tokens are zero (every score ties at 0: those rows
    # overflow the epilogue's candidate buffer and the row kernel finishes
    # both their routing and their part of the bracket pass); half the
    # router rows are equal, so many keys tie inside the brackets
    N, d, E, K = 30000, 256, 384, 6
    g = torch.Generator().manual_seed(5)
    x = torch.randn(N, d, generator=g).to(torch.bfloat16)
    x[::3] = 0
    w = torch.randn(1, d, generator=g).repeat(E, 1)
    w[E // 2:] = torch.randn(E - E // 2, d, generator=g)
    w = (w / 16).to(torch.bfloat16)
    beta = torch.zeros(E)
    beta[::7] = 0.125
    _check(oracle_mod, x, w, beta, K)
