"""GPU parity of selection, permutation and the EQB update, fed the same fp32
logits as the oracle: ids, gates, token biases, counts, offsets,
permutation, quantiles and biases must be bit-exact."""
import json
import os

import numpy as np
import pytest
import torch

from expert_load_balancing_b200 import binding as B
from expert_load_balancing_b200 import workloads

from gpu_helpers import (assert_bit_equal, check_status, dev, gpu_eqb, gpu_permute, gpu_select,
                         host)

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module", autouse=True)
def _lib(kolibri_lib):
    return kolibri_lib


def _select_case(oracle_mod, z, beta, K):
    ids, gates, alpha = gpu_select(z, beta, K)
    ids_o, gates_o, alpha_o = oracle_mod.select(z, beta, K)
    assert_bit_equal(ids, ids_o, "ids")
    assert_bit_equal(gates, gates_o, "gates")
    assert_bit_equal(alpha, alpha_o, "alpha")
    return ids_o, alpha_o


def _permute_case(oracle_mod, ids, E):
    c, o, p, i = gpu_permute(ids, E)
    c_o, o_o, p_o, i_o = oracle_mod.permute(ids, E)
    assert_bit_equal(c, c_o, "counts")
    assert_bit_equal(o, o_o, "offsets")
    assert_bit_equal(p, p_o, "perm")
    assert_bit_equal(i, i_o, "inv")


def _eqb_case(oracle_mod, z, alpha, beta_in, K):
    N, E = z.shape
    m = oracle_mod.eqb_target_rank(N, K, E)
    a_ref = alpha if alpha is not None else oracle_mod.select(z, beta_in, K)[2]
    v_o = oracle_mod.column_quantiles(z, a_ref, m)
    b_o = oracle_mod.eqb_bias(v_o)
    b, v = gpu_eqb(z, alpha, beta_in, K)
    assert_bit_equal(v, v_o, "quantiles")
    assert_bit_equal(b, b_o, "beta")
    return b


# ------------------------------------------------------------- toy example

def test_toy_trace_on_gpu(oracle_mod):
    toy = json.load(open(os.path.join(GOLDEN, "toy_router_e4k2.json")))
    z = np.array(toy["logits_Z"], np.float32)
    ids, gates, alpha = gpu_select(z, np.zeros(4, np.float32), 2)
    np.testing.assert_array_equal(alpha, np.array(toy["alpha"], np.float32))
    assert [sorted(r) for r in ids.tolist()] == toy["top2_sets_beta0"]
    counts, _, _, _ = gpu_permute(ids, 4)
    assert counts.tolist() == toy["loads_beta0"]
    beta, v = gpu_eqb(z, alpha, np.zeros(4, np.float32), 2)
    np.testing.assert_array_equal(-v, np.array(toy["beta_before_centring"], np.float32))
    np.testing.assert_array_equal(beta, np.array(toy["beta_centred"], np.float32))
    ids2, gates2, _ = gpu_select(z, beta, 2)
    assert ids2.tolist() == [[0, 3], [1, 2], [1, 2], [0, 3]]
    counts2, _, _, _ = gpu_permute(ids2, 4)
    assert counts2.tolist() == toy["loads_after"]
    assert round(float(gates2[0, 0]), 3) == 0.881 and round(float(gates2[0, 1]), 3) == 0.269
    # alpha computed inside the update from beta_in gives the same result
    beta_b, _ = gpu_eqb(z, None, np.zeros(4, np.float32), 2)
    np.testing.assert_array_equal(beta_b, beta)
    check_status()


# ------------------------------------------------ selection, bit-exact

@pytest.mark.parametrize("N,E,K", [(1, 384, 6), (7, 384, 6), (1000, 384, 6), (2049, 128, 8),
                                   (333, 512, 16), (64, 16, 15), (100, 4, 1), (513, 388, 6),
                                   (300, 132, 2)])
def test_select_random(oracle_mod, N, E, K):
    z = workloads.random_logits(N, E, seed=N + E + K)
    beta = workloads.random_logits(1, E, seed=7)[0] * np.float32(0.3)
    _select_case(oracle_mod, z, beta, K)
    _select_case(oracle_mod, z, None, K)
    check_status()


@pytest.mark.parametrize("E,K", [(384, 6), (128, 8), (8, 3)])
def test_select_ties(oracle_mod, E, K):
    z = workloads.tied_logits(700, E, seed=3)
    beta = workloads.tied_logits(1, E, seed=4)[0] * np.float32(0.5)
    _select_case(oracle_mod, z, beta, K)
    _select_case(oracle_mod, z, None, K)
    # all-equal rows: ids 0..K-1
    ids, _, alpha = gpu_select(np.zeros((5, E), np.float32), None, K)
    assert (ids == np.arange(K)).all() and (alpha == 0).all()
    check_status()


def test_select_extreme_values(oracle_mod):
    E, K = 384, 6
    z = workloads.random_logits(256, E, seed=11) * np.float32(60.0)
    z[0, :] = np.float32(-800.0)
    z[1, :10] = np.float32(900.0)
    z[2, :] = np.float32(1e-40)           # subnormal logits
    z[3, ::2] = np.float32(-0.0)
    _select_case(oracle_mod, z, None, K)
    _select_case(oracle_mod, z, workloads.random_logits(1, E, 5)[0], K)


@pytest.mark.parametrize("N,E,K", [(16384, 384, 6), (16411, 128, 8), (16400, 256, 1),
                                   (16390, 512, 16), (20001, 384, 15), (16384, 128, 7)])
def test_select_large_batch(oracle_mod, N, E, K):
    # From 16384 rows the selection runs eight lanes per row (E in 128, 256,
    # 384, 512); rows with heavy ties (more than 32 scores at or above its
    # threshold) are left to the row kernel through a NaN alpha.  Mixed in:
    # tied rows, all-equal rows, signed zeros, large and subnormal logits.
    z = workloads.random_logits(N, E, seed=N + E + K) * np.float32(4.0)
    t = workloads.tied_logits(N, E, seed=K)
    z[::97] = t[::97]
    z[5::211] = np.float32(0.0)
    z[7::389, ::3] = np.float32(-0.0)
    z[11::401, :10] = np.float32(900.0)
    z[13::409] = np.float32(1e-40)
    z[17::419] = np.float32(-800.0)
    beta = workloads.random_logits(1, E, seed=8)[0] * np.float32(0.3)
    _select_case(oracle_mod, z, beta, K)
    _select_case(oracle_mod, z, None, K)
    check_status()


def test_gates_unchanged_by_bias():
    z = workloads.random_logits(500, 384, seed=21)
    i1, g1, _ = gpu_select(z, workloads.random_logits(1, 384, 22)[0], 6)
    i2, g2, _ = gpu_select(z, workloads.random_logits(1, 384, 23)[0] * 3, 6)
    shared = 0
    for t in range(500):
        m = dict(zip(i1[t].tolist(), g1[t].tolist()))
        for e, g in zip(i2[t].tolist(), g2[t].tolist()):
            if e in m:
                assert m[e] == g
                shared += 1
    assert shared > 0
    assert all(len(set(r)) == 6 for r in i1.tolist())


# ------------------------------------------------ permutation, bit-exact

@pytest.mark.parametrize("N,E,K", [(1, 384, 6), (256, 384, 6), (683, 384, 6), (5000, 384, 6),
                                   (40000, 128, 8), (12345, 16, 3),
                                   # one block up to N*K = 4096: its edges
                                   (512, 512, 8), (4096, 16, 1), (1, 512, 16), (13, 48, 5),
                                   (4097, 16, 1),
                                   # tiled path at each width of the expert-id grouping
                                   # (E itself marks an empty slot: 8 bits up to E = 252,
                                   # 9 bits up to 511, 10 bits at 512)
                                   (9001, 252, 3), (7000, 256, 4), (3000, 512, 8)])
def test_permute(oracle_mod, N, E, K):
    rng = np.random.default_rng(N)
    ids = np.stack([rng.choice(E, size=K, replace=False) for _ in range(N)]).astype(np.int32)
    _permute_case(oracle_mod, ids, E)
    check_status()


def test_permute_skewed(oracle_mod):
    # every token on the same few experts; empty experts in between
    N, E, K = 30000, 384, 6
    ids = np.tile(np.array([5, 17, 0, 383, 200, 6], np.int32), (N, 1))
    _permute_case(oracle_mod, ids, E)


def test_permute_skewed_one_block(oracle_mod):
    # a decode batch on the same experts: one expert's run spans every warp's segment
    N, E, K = 600, 384, 6
    ids = np.tile(np.array([5, 17, 0, 383, 200, 6], np.int32), (N, 1))
    ids[::7, 2] = 1
    _permute_case(oracle_mod, ids, E)
    check_status()


def test_permute_bad_id_sets_device_status():
    ids = np.zeros((100, 2), np.int32)
    ids[:, 1] = 1
    ids[37, 1] = 999          # out of range: skipped by the kernel, flagged
    gpu_permute(ids, 16)
    assert B.kolibri_device_status() == B.KOLIBRI_ERR_DEVICE
    assert B.kolibri_device_status() == B.KOLIBRI_OK   # cleared by the read
    ids = np.zeros((20000, 1), np.int32)
    ids[5, 0] = -3
    gpu_permute(ids, 8)
    assert B.kolibri_device_status() == B.KOLIBRI_ERR_DEVICE


# ------------------------------------------------ EQB, bit-exact

@pytest.mark.parametrize("N,E,K", [(4, 4, 2), (256, 384, 6), (999, 384, 6), (16384, 384, 6),
                                   (16385, 384, 6), (40000, 128, 8), (70001, 384, 6),
                                   (20011, 512, 16)])
def test_eqb_random(oracle_mod, N, E, K):
    z = workloads.random_logits(N, E, seed=N)
    z[:, : max(1, E // 48)] += np.float32(3.0)                # a few collapsed experts
    beta = workloads.random_logits(1, E, seed=1)[0] * np.float32(0.3)
    ids, alpha = _select_case(oracle_mod, z, beta, K)
    _eqb_case(oracle_mod, z, alpha, beta, K)
    _eqb_case(oracle_mod, z, None, beta, K)
    check_status()


def test_eqb_ties(oracle_mod):
    z = workloads.tied_logits(20000, 128, seed=5)
    _, alpha = _select_case(oracle_mod, z, None, 8)
    _eqb_case(oracle_mod, z, alpha, np.zeros(128, np.float32), 8)
    z2 = workloads.tied_logits(3000, 64, seed=6)
    _eqb_case(oracle_mod, z2, None, np.zeros(64, np.float32), 4)


def test_eqb_sample_misses_falls_back(oracle_mod):
    """Rows on the sampling stride carry values unlike the rest, so the
    bracket from the sample misses and every expert takes the full radix
    path -- the result must still be exact."""
    N, E, K = 65536 * 2, 64, 4
    z = workloads.random_logits(N, E, seed=9)
    stride = N // 16384
    z[::stride] += np.float32(25.0)           # the sample sees only huge values
    alpha = np.zeros(N, np.float32)
    _eqb_case(oracle_mod, z, alpha, np.zeros(E, np.float32), K)
    z2 = workloads.random_logits(N, E, seed=10)
    z2[::stride] -= np.float32(25.0)
    _eqb_case(oracle_mod, z2, alpha, np.zeros(E, np.float32), K)
    check_status()


def test_eqb_constant_columns(oracle_mod):
    N, E, K = 50000, 32, 2
    z = np.ones((N, E), np.float32) * np.arange(E, dtype=np.float32)[None, :]
    _eqb_case(oracle_mod, z, np.zeros(N, np.float32), np.zeros(E, np.float32), K)


# ------------------------------------------------ hygiene

def test_outputs_fully_written_and_deterministic(oracle_mod):
    N, E, K = 20000, 384, 6
    z = dev(workloads.random_logits(N, E, seed=31))
    beta = dev(workloads.random_logits(1, E, seed=32)[0])
    runs = []
    for poison in (0x7FC00000, 0x7F800001):
        ids = torch.full((N, K), -1, dtype=torch.int32, device="cuda")
        gates = torch.full((N, K), 0, dtype=torch.int32, device="cuda").fill_(poison).view(torch.float32)
        alpha = torch.empty(N, dtype=torch.int32, device="cuda").fill_(poison).view(torch.float32)
        B.kolibri_router_topk(z, beta, K, ids, gates, alpha)
        counts = torch.full((E,), -1, dtype=torch.int32, device="cuda")
        offsets = torch.full((E + 1,), -1, dtype=torch.int64, device="cuda")
        perm = torch.full((N * K,), -1, dtype=torch.int32, device="cuda")
        inv = torch.full((N * K,), -1, dtype=torch.int32, device="cuda")
        B.kolibri_expert_permute(ids, E, counts=counts, offsets=offsets, perm=perm, inv=inv)
        b = beta.clone()
        q = torch.empty(E, dtype=torch.int32, device="cuda").fill_(poison).view(torch.float32)
        B.kolibri_eqb_update(z, alpha, b, K, quantiles=q)
        runs.append([host(t).copy() for t in (ids, gates, alpha, counts, offsets, perm, inv, b, q)])
    for a, b in zip(*runs):
        assert_bit_equal(a, b, "run-to-run")
    ids, gates, alpha = runs[0][:3]
    assert (ids >= 0).all() and np.isfinite(gates).all() and np.isfinite(alpha).all()
    check_status()


# ------------------------------------------------ fused routing + EQB

@pytest.mark.parametrize("N,E,K", [(4, 4, 2), (300, 384, 6), (16384, 384, 6), (16385, 384, 6),
                                   (70001, 384, 6), (65536, 128, 8), (40000, 132, 3)])
def test_route_and_balance(oracle_mod, N, E, K):
    z = workloads.random_logits(N, E, seed=N + 3)
    z[:, : max(1, E // 48)] += np.float32(3.0)
    beta = workloads.random_logits(1, E, seed=2)[0] * np.float32(0.3)
    bt = dev(beta.copy())
    ids, gates, alpha, q = B.kolibri_route_and_balance(dev(z), bt, K)
    ids_o, gates_o, alpha_o = oracle_mod.select(z, beta, K)
    assert_bit_equal(host(ids), ids_o, "ids")
    assert_bit_equal(host(gates), gates_o, "gates")
    assert_bit_equal(host(alpha), alpha_o, "alpha")
    v_o = oracle_mod.column_quantiles(z, alpha_o, oracle_mod.eqb_target_rank(N, K, E))
    assert_bit_equal(host(q), v_o, "quantiles")
    assert_bit_equal(host(bt), oracle_mod.eqb_bias(v_o), "beta")
    check_status()


def test_route_and_balance_fallback_and_ties(oracle_mod):
    N, E, K = 131072, 64, 4
    z = workloads.random_logits(N, E, seed=19)
    z[:: N // 16384] += np.float32(25.0)      # the sample misleads the bracket
    z[:1000] = workloads.tied_logits(1000, E, seed=20)
    bt = dev(np.zeros(E, np.float32))
    ids, gates, alpha, q = B.kolibri_route_and_balance(dev(z), bt, K, want_alpha=False)
    ids_o, gates_o, alpha_o = oracle_mod.select(z, np.zeros(E, np.float32), K)
    assert_bit_equal(host(ids), ids_o, "ids")
    assert_bit_equal(host(gates), gates_o, "gates")
    v_o = oracle_mod.column_quantiles(z, alpha_o, oracle_mod.eqb_target_rank(N, K, E))
    assert_bit_equal(host(q), v_o, "quantiles")
    assert_bit_equal(host(bt), oracle_mod.eqb_bias(v_o), "beta")
    check_status()
