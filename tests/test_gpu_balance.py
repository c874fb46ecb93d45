"""The balancing pieces beside the routing path, on the GPU against the oracle:
EQB with bf16 keys ("Kolibri Pre-Training from Scratch" 7.3), Load-Error
Injection and its chain rule (section 8), the intervention rate (section 9).
All bit-exact (the rate's integer overlap count exactly, the rate itself to
the last bits of a double)."""
import numpy as np
import pytest
import torch

from expert_load_balancing_b200 import binding as B
from expert_load_balancing_b200 import distributed as D
from expert_load_balancing_b200 import workloads

from gpu_helpers import assert_bit_equal, check_status, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(kolibri_lib):
    return kolibri_lib


def _column_data(N, E, seed, ties=False):
    rng = np.random.default_rng(seed)
    z = (rng.standard_normal((N, E)) * 2).astype(np.float32)
    if ties:
        z[:, ::3] = np.round(z[:, ::3] * 2) / 2          # many equal values per column
        z[::5] = 0.0
    a = (rng.standard_normal(N) * 0.5).astype(np.float32)
    return z, a


@pytest.mark.parametrize("N,E,K", [(1, 16, 2), (1000, 16, 2), (4099, 128, 8), (70001, 384, 6),
                                   (3000, 400, 6), (777, 512, 16)])
@pytest.mark.parametrize("with_alpha", [True, False])
def test_eqb_bf16_matches_oracle(oracle_mod, N, E, K, with_alpha):
    z, a = _column_data(N, E, N + E)
    alpha = a if with_alpha else None
    beta = dev(np.zeros(E, np.float32))
    _, q = B.kolibri_eqb_update_bf16(dev(z), None if alpha is None else dev(alpha), beta, K)
    torch.cuda.synchronize()
    check_status()
    m = (N * K) // E
    if alpha is None:   # as kolibri_eqb_update: alpha from the bias (zeros here)
        _, _, alpha = oracle_mod.select(z, np.zeros(E, np.float32), K)
    v_o = oracle_mod.column_quantiles_bf16(z, alpha, m)
    assert_bit_equal(host(q), v_o, "quantiles")
    assert_bit_equal(host(beta), oracle_mod.eqb_bias(v_o), "beta")


def test_eqb_bf16_ties_and_rounding_identity(oracle_mod):
    N, E, K = 20000, 384, 6
    z, a = _column_data(N, E, 7, ties=True)
    zt, at = dev(z), dev(a)
    b16 = dev(np.zeros(E, np.float32))
    _, q16 = B.kolibri_eqb_update_bf16(zt, at, b16, K)
    b32 = dev(np.zeros(E, np.float32))
    _, q32 = B.kolibri_eqb_update(zt, at, b32, K)
    torch.cuda.synchronize()
    m = (N * K) // E
    assert_bit_equal(host(q16), oracle_mod.column_quantiles_bf16(z, a, m), "quantiles")
    # rounding is monotone: the bf16 quantile is the rounding of the fp32 one
    r = host(q32.to(torch.bfloat16).to(torch.float32))
    assert_bit_equal(host(q16), r, "bf16(fp32 quantile)")


def test_eqb_bf16_pieces_equal_one_call(oracle_mod):
    # the multi-rank sequence on a single rank (no all-reduce) is the one-call update
    N, E, K = 5000, 384, 6
    z, a = _column_data(N, E, 11)
    zt, at = dev(z), dev(a)
    b1 = dev(np.zeros(E, np.float32))
    _, q1 = B.kolibri_eqb_update_bf16(zt, at, b1, K)
    b2 = dev(np.zeros(E, np.float32))
    _, q2 = D.eqb_update_bf16_distributed(zt, at, b2, K, N)
    torch.cuda.synchronize()
    assert_bit_equal(host(q2), host(q1), "quantiles")
    assert_bit_equal(host(b2), host(b1), "beta")


@pytest.mark.parametrize("N,E,K,ties", [(1, 16, 2, False), (5000, 384, 6, False), (20000, 384, 6, True),
                                        (4099, 128, 8, True), (777, 400, 6, False)])
def test_eqb_fp32_key_passes_equal_one_call(oracle_mod, N, E, K, ties):
    # the four fp32-key passes of the split form, on one rank (no all-reduce),
    # give kolibri_eqb_update's exact quantile and bias bit for bit
    z, a = _column_data(N, E, N + 3 * E, ties=ties)
    zt, at = dev(z), dev(a)
    b1 = dev(np.zeros(E, np.float32))
    _, q1 = B.kolibri_eqb_update(zt, at, b1, K)
    b2 = dev(np.zeros(E, np.float32))
    _, q2 = D.eqb_update_distributed(zt, at, b2, K, N)
    torch.cuda.synchronize()
    check_status()
    assert_bit_equal(host(q2), host(q1), "quantiles")
    assert_bit_equal(host(b2), host(b1), "beta")
    assert_bit_equal(host(q2), oracle_mod.column_quantiles(z, a, (N * K) // E), "oracle")


def test_lei_pages_example(oracle_mod):
    # section 8: loads (4, 4, 0, 0), K = 2, four tokens
    counts = dev(np.array([4, 4, 0, 0], np.int32))
    g = dev(np.zeros((4, 4), np.float32))
    B.kolibri_lei_inject(counts, g, 2)
    torch.cuda.synchronize()
    assert_bit_equal(host(g), oracle_mod.lei_inject(np.array([4, 4, 0, 0]), np.zeros((4, 4)), 2), "g")
    assert abs(float(host(g)[0, 0]) - 1e-5 * 0.7616) < 1e-9


@pytest.mark.parametrize("N,E,K,lam,tau", [(1000, 384, 6, 1e-5, 1.0), (4099, 128, 8, 1e-3, 0.25),
                                           (300, 16, 2, 1e-5, 1.0), (64, 384, 6, 1.0, 1e-4)])
def test_lei_matches_oracle(oracle_mod, N, E, K, lam, tau):
    rng = np.random.default_rng(N)
    counts = rng.multinomial(N * K, rng.dirichlet(np.full(E, 0.5))).astype(np.int32)
    g0 = rng.standard_normal((N, E)).astype(np.float32) * np.float32(1e-4)
    g = dev(g0)
    B.kolibri_lei_inject(dev(counts), g, K, lam, tau)
    torch.cuda.synchronize()
    check_status()
    assert_bit_equal(host(g), oracle_mod.lei_inject(counts, g0, K, lam, tau), "g")


def test_lei_balanced_is_identity_but_signed_zero(oracle_mod):
    N, E, K = 100, 16, 4
    counts = np.full(E, N * K // E, np.int32)
    g0 = np.random.default_rng(0).standard_normal((N, E)).astype(np.float32)
    g0[0, 0] = -0.0
    g = dev(g0)
    B.kolibri_lei_inject(dev(counts), g, K)
    torch.cuda.synchronize()
    assert_bit_equal(host(g), oracle_mod.lei_inject(counts, g0, K), "g")


def test_score_grad_to_logits_matches_oracle(oracle_mod):
    rng = np.random.default_rng(3)
    z = np.concatenate([rng.standard_normal(50000).astype(np.float32) * 8,
                        np.array([2.0, 0.0, -0.0, 700.0, 701.0, -700.0, -701.0, 1e4, -1e4, 40.0],
                                 np.float32)])
    gs = rng.standard_normal(z.shape[0]).astype(np.float32)
    gz = B.kolibri_score_grad_to_logits(dev(z), dev(gs))
    torch.cuda.synchronize()
    assert_bit_equal(host(gz), oracle_mod.score_grad_to_logits(z, gs), "gz")
    # views one element in: not 16-byte aligned, so the one-element-per-thread form runs
    gz1 = B.kolibri_score_grad_to_logits(dev(z)[1:], dev(gs)[1:])
    torch.cuda.synchronize()
    assert_bit_equal(host(gz1), oracle_mod.score_grad_to_logits(z[1:], gs[1:]), "gz misaligned")
    one = B.kolibri_score_grad_to_logits(dev(np.array([2.0], np.float32)), dev(np.array([1.0], np.float32)))
    assert abs(float(host(one)[0]) - 0.105) < 5e-4                    # section 8


def test_intervention_rate_ties_large(oracle_mod):
    # from 4096 rows the overlap runs eight lanes per row; rows with heavy
    # ties are finished by the whole warp in the same kernel
    N, E, K = 6000, 256, 4
    z = workloads.random_logits(N, E, seed=41)
    z[::3] = workloads.tied_logits(N, E, seed=42)[::3]
    ids_routed, _, _ = oracle_mod.select(z, workloads.random_logits(1, E, seed=43)[0], K)
    ids_unb, _, _ = oracle_mod.select(z, None, K)
    rate, ovl = B.kolibri_intervention_rate(dev(z), dev(ids_routed))
    torch.cuda.synchronize()
    check_status()
    assert int(host(ovl)[0]) == oracle_mod.intervention_overlap(ids_routed, ids_unb)


@pytest.mark.parametrize("N,E,K", [(1, 4, 2), (5000, 384, 6), (4099, 128, 8), (777, 400, 6)])
def test_intervention_rate_matches_oracle(oracle_mod, N, E, K):
    wl = workloads.Workload("t", N, 64, E, K, beta="normal0.1")
    z = workloads.random_logits(N, E, seed=N + E)
    beta = workloads.make_beta(wl).numpy() * np.float32(5.0)
    ids_routed, _, _ = oracle_mod.select(z, beta, K)
    ids_unb, _, _ = oracle_mod.select(z, None, K)
    rate, ovl = B.kolibri_intervention_rate(dev(z), dev(ids_routed))
    torch.cuda.synchronize()
    check_status()
    n_ovl = oracle_mod.intervention_overlap(ids_routed, ids_unb)
    assert int(host(ovl)[0]) == n_ovl                       # the exact quantity, bit for bit
    # the rate is that count in one division; the oracle's mean of N terms
    # carries up to N roundings of its running sum
    assert float(host(rate)[0]) == 1.0 - n_ovl / (N * K)
    want = oracle_mod.intervention_rate(ids_routed, ids_unb)
    assert abs(float(host(rate)[0]) - want) <= N * 2.0 ** -52


def test_intervention_rate_pages_toy(oracle_mod):
    # section 9: the toy trace re-routed after one EQB step: every token keeps
    # one of its own top-2, rate 0.5 (= 1 - K/E for E = 4, K = 2)
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "toy_router_e4k2.json")))
    z = np.array(g["logits_Z"], np.float32)
    beta = np.array(g["beta_centred"], np.float32)
    assert g["intervention_rate_after"] == 0.5
    ids_routed, _, _ = oracle_mod.select(z, beta, 2)
    rate, ovl = B.kolibri_intervention_rate(dev(z), dev(ids_routed))
    torch.cuda.synchronize()
    ids_unb, _, _ = oracle_mod.select(z, None, 2)
    assert int(host(ovl)[0]) == oracle_mod.intervention_overlap(ids_routed, ids_unb) == 4
    assert float(host(rate)[0]) == 0.5
