"""Pins for the CPU oracle: values the pages print, closed forms, invariants
and brute force on tiny inputs.  Each check is chosen so that a plausible
slip in the oracle (off-by-one rank, wrong sign, biased gate, missing
centring, reversed tie-break, dropped term) fails at least one of them.

Sources: "Kolibri Pre-Training from Scratch: UniBPE, Hybrid Attention and
Exact Quantile Balancing" sections 1, 6.1, 6.2, 7.1-7.3 and 9, through the
fixtures in tests/golden/.
"""
import itertools
import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest

from expert_load_balancing_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.fixture(scope="module")
def toy():
    return _golden("toy_router_e4k2.json")


@pytest.fixture(scope="module")
def qx():
    return _golden("quantile_examples.json")


# ----------------------------------------------------------- Q_m (section 1)

def test_q_worked_example(oracle_mod, qx):
    ex = qx["Q_example"]
    z = np.array(ex["values"], dtype=np.float32).reshape(-1, 1)
    v = oracle_mod.column_quantiles(z, None, ex["m"])
    assert v[0] == np.float32(ex["expected"])


def test_q_all_ranks_brute_force(oracle_mod):
    rng = np.random.default_rng(5)
    for n in range(1, 9):
        vals = rng.choice(np.array([-2.0, -0.5, 0.0, 0.5, 1.0, 3.0], np.float32), size=(n, 3))
        for m in range(n):
            v = oracle_mod.column_quantiles(vals, None, m)
            for e in range(3):
                assert v[e] == np.sort(vals[:, e])[::-1][m]


# ------------------------------------------------------- toy trace (6.1-7.2)

def test_toy_route_before_update(oracle_mod, toy):
    z = np.array(toy["logits_Z"], np.float32)
    ids, gates, alpha = oracle_mod.select(z, np.array(toy["beta0"], np.float32), toy["K"])
    assert [sorted(r) for r in ids.tolist()] == toy["top2_sets_beta0"]
    np.testing.assert_array_equal(alpha, np.array(toy["alpha"], np.float32))
    counts, offsets, perm, inv = oracle_mod.permute(ids, toy["E"])
    assert counts.tolist() == toy["loads_beta0"]
    assert oracle_mod.maxvio(counts, toy["T"], toy["K"]) == toy["maxvio_beta0"]


def test_toy_expert_update(oracle_mod, toy):
    z = np.array(toy["logits_Z"], np.float32)
    alpha = np.array(toy["alpha"], np.float32)
    cols = (z + alpha[:, None]).T
    np.testing.assert_array_equal(cols, np.array(toy["columns_plus_alpha"], np.float32))
    m = oracle_mod.eqb_target_rank(toy["T"], toy["K"], toy["E"])
    assert m == 2
    v = oracle_mod.column_quantiles(z, alpha, m)
    np.testing.assert_array_equal(-v, np.array(toy["beta_before_centring"], np.float32))
    # every column of Z + alpha + beta' has exactly r positives
    raw = -v
    shifted = z + alpha[:, None] + raw[None, :]
    assert ((shifted > 0).sum(axis=0) == toy["positives_per_column"]).all()
    np.testing.assert_array_equal(shifted[:, 0],
                                  np.array(toy["column_e1_plus_alpha_plus_beta"], np.float32))
    assert float(np.mean(raw.astype(np.float64))) == toy["mean_before_centring"]
    beta = oracle_mod.eqb_bias(v)
    np.testing.assert_array_equal(beta, np.array(toy["beta_centred"], np.float32))


def test_toy_reroute(oracle_mod, toy):
    z = np.array(toy["logits_Z"], np.float32)
    beta = np.array(toy["beta_centred"], np.float32)
    np.testing.assert_array_equal(z + beta[None, :],
                                  np.array(toy["biased_scores_after"], np.float32))
    ids, gates, _ = oracle_mod.select(z, beta, toy["K"])
    assert [sorted(r) for r in ids.tolist()] == toy["top2_sets_after"]
    # rank order: biased score descending
    assert ids.tolist() == [[0, 3], [1, 2], [1, 2], [0, 3]]
    counts, _, _, _ = oracle_mod.permute(ids, toy["E"])
    assert counts.tolist() == toy["loads_after"]
    assert oracle_mod.maxvio(counts, toy["T"], toy["K"]) == toy["maxvio_after"]
    g = toy["gates_t1_after_3dp"]
    assert round(float(gates[0, 0]), 3) == g["e1"]
    assert round(float(gates[0, 1]), 3) == g["e4"]
    assert round(float(gates[0, 0]) + float(gates[0, 1]), 3) == g["sum"]
    # gates come from the raw logits, not from B = Z + beta
    assert gates[0, 0] == oracle_mod.sigmoid_spec(2.0)
    assert gates[0, 1] == oracle_mod.sigmoid_spec(-1.0)
    ids_u, _, _ = oracle_mod.select(z, None, toy["K"])
    assert oracle_mod.intervention_rate(ids, ids_u) == toy["intervention_rate_after"]


# --------------------------------------------- intervention rate (section 9)

def test_intervention_random_closed_form(oracle_mod, qx):
    rng = np.random.default_rng(11)
    for K, E in ((2, 4), (6, 384), (8, 128)):
        N = 20000
        unb = np.tile(np.arange(K, dtype=np.int32), (N, 1))
        rnd = np.stack([rng.choice(E, size=K, replace=False) for _ in range(N)]).astype(np.int32)
        i = oracle_mod.intervention_rate(rnd, unb)
        expected = 1.0 - K / E
        # overlap ~ hypergeometric; its standard error over N tokens
        var = (K * (K / E) * (1 - K / E) * (E - K) / max(E - 1, 1)) / K**2
        assert abs(i - expected) < 5 * math.sqrt(var / N) + 1e-12
    kk = qx["kolibri_random_routing_intervention"]
    assert round(1 - kk["K"] / kk["E"], 3) == kk["value_3dp"]


# ---------------------------------------- exact quantile by radix (7.3)

def test_distributed_counter_example(oracle_mod, qx):
    d = qx["distributed"]
    a = np.array(d["rank_A"], np.float32).reshape(-1, 1)
    b = np.array(d["rank_B"], np.float32).reshape(-1, 1)
    qa = oracle_mod.column_quantiles(a, None, d["local_m"])[0]
    qb = oracle_mod.column_quantiles(b, None, d["local_m"])[0]
    assert [qa, qb] == d["local_quantiles"]
    assert (qa + qb) / 2 == d["mean_of_local"]
    union = np.concatenate([a, b])
    assert oracle_mod.column_quantiles(union, None, d["global_m"])[0] == d["global_quantile"]
    # summing per-rank histograms reaches the exact union quantile
    keys = np.array([oracle_mod.order_key(float(v)) for v in union.ravel()], np.uint64)
    k, _, _ = oracle_mod.radix_select(keys, d["global_m"], 256, 4, chunk_sizes=[2, 2])
    assert k == oracle_mod.order_key(d["global_quantile"])
    assert -d["global_quantile"] == d["beta1_exact"]
    assert -d["mean_of_local"] == d["beta1_from_mean"]


def test_two_digit_radix_analogue(oracle_mod, qx):
    r = qx["two_digit_radix"]
    k, hist, bins = oracle_mod.radix_select(np.array(r["keys"], np.uint64), r["m"],
                                            r["radix"], r["ndigits"])
    assert {str(i): int(c) for i, c in enumerate(hist[0]) if c} == r["pass1_hist"]
    assert bins.tolist() == [r["pass1_bin"], r["pass2_bin"]]
    assert k == r["result_key"]
    assert k / 10 == r["result_value"]


def test_allreduce_message_size(qx):
    a = qx["allreduce_bytes_E384"]
    assert a["bins"] * a["E"] * a["bytes_per_count"] == a["bytes"]


def test_radix_select_brute_force(oracle_mod):
    # every multiset of size <= 5 over {0..3}, base-2 digits, every rank
    for n in range(1, 6):
        for combo in itertools.combinations_with_replacement(range(4), n):
            keys = np.array(combo, np.uint64)
            for m in range(n):
                for split in ([n], [1, n - 1] if n > 1 else [n]):
                    k, _, _ = oracle_mod.radix_select(keys, m, 2, 2, chunk_sizes=split)
                    assert k == sorted(combo, reverse=True)[m]
    # fp32 keys, 4 passes of 8 bits, random chunking into "ranks"
    rng = np.random.default_rng(3)
    vals = np.concatenate([rng.standard_normal(300).astype(np.float32),
                           np.array([0.0, -0.0, 1.0, 1.0, -1.0], np.float32)])
    keys = oracle_mod.order_key_array(vals).astype(np.uint64)
    for m in (0, 1, 7, 150, 304):
        k, _, _ = oracle_mod.radix_select(keys, m, 256, 4, chunk_sizes=[100, 5, 200])
        assert k == np.sort(keys)[::-1][m]


# ---------------------------------------------------- order key

def test_order_key_monotone(oracle_mod):
    f = np.finfo(np.float32)
    tiny = np.float32(1e-45)
    vals = [-np.inf, -f.max, -1.0, -f.tiny, -tiny, -0.0, 0.0, tiny, f.tiny, 1.0, f.max, np.inf]
    keys = [oracle_mod.order_key(float(v)) for v in vals]
    assert all(a < b for a, b in zip(keys, keys[1:]))
    arr = oracle_mod.order_key_array(np.array(vals, np.float32))
    assert arr.tolist() == keys


# ---------------------------------------------------- exp and sigmoid

def test_exp_spec_accuracy(oracle_mod):
    assert oracle_mod.exp_spec(0.0) == 1.0
    xs = np.concatenate([np.linspace(-700, 700, 4001), np.linspace(-1, 1, 2001)])
    getcontext().prec = 40
    worst = 0.0
    for x in xs.tolist():
        ref = Decimal(x).exp()
        got = Decimal(oracle_mod.exp_spec(x))
        worst = max(worst, float(abs(got - ref) / ref))
    assert worst < 4.5e-16, worst


def _sigmoid_ref_f32(z):
    getcontext().prec = 40
    s = Decimal(1) / (Decimal(1) + Decimal(float(-np.float32(z))).exp())
    return np.float32(float(s))  # decimal -> nearest double -> nearest fp32


def test_sigmoid_spec_values(oracle_mod):
    assert oracle_mod.sigmoid_spec(0.0) == np.float32(0.5)
    assert round(float(oracle_mod.sigmoid_spec(2.0)), 3) == 0.881
    assert round(float(oracle_mod.sigmoid_spec(-1.0)), 3) == 0.269
    assert oracle_mod.sigmoid_spec(1000.0) == np.float32(1.0)
    assert oracle_mod.sigmoid_spec(-1000.0) == np.float32(0.0)
    assert oracle_mod.sigmoid_spec(-200.0) == np.float32(0.0)   # below fp32 range
    assert oracle_mod.sigmoid_spec(-90.0) > 0                    # subnormal fp32


def test_sigmoid_spec_within_one_ulp(oracle_mod):
    zs = np.concatenate([np.linspace(-30, 30, 6001, dtype=np.float32),
                         np.linspace(-1, 1, 4001, dtype=np.float32),
                         np.float32([-103.5, -88.0, -50.0, 17.0, 16.5, 40.0])])
    got = oracle_mod.sigmoid_spec_array(zs)
    bad = 0
    for z, g in zip(zs.tolist(), got.tolist()):
        r = _sigmoid_ref_f32(z)
        ulps = abs(int(np.float32(g).view(np.int32)) - int(r.view(np.int32)))
        assert ulps <= 1, (z, g, r)
        bad += ulps
    assert bad <= 2  # essentially always correctly rounded


# ---------------------------------------------------- router logits

def test_logits_one_hot_and_constant(oracle_mod):
    import torch
    E, d = 16, 128
    w = (torch.randn(E, d, generator=torch.Generator().manual_seed(0))).to(torch.bfloat16)
    x = torch.zeros(d, d, dtype=torch.bfloat16)
    x[torch.arange(d), torch.arange(d)] = 1.0
    z = oracle_mod.router_logits(workloads.bf16_bits(x), workloads.bf16_bits(w))
    np.testing.assert_array_equal(z, w.float().numpy().T)
    # constant rows: x = 0.5 everywhere, W row e = (e+1) * 2^-4 -> Z = d * 0.5 * (e+1)/16
    x2 = torch.full((3, d), 0.5, dtype=torch.bfloat16)
    w2 = ((torch.arange(E, dtype=torch.float32) + 1) / 16).repeat(d, 1).T.contiguous().to(torch.bfloat16)
    z2 = oracle_mod.router_logits(workloads.bf16_bits(x2), workloads.bf16_bits(w2))
    expect = np.float32(d * 0.5) * (np.arange(E, dtype=np.float32) + 1) / 16
    np.testing.assert_array_equal(z2, np.tile(expect, (3, 1)))


def test_logits_random_vs_float64_matmul(oracle_mod):
    import torch
    wl = workloads.Workload("t", 37, 256, 48, 4, offsets="collapsed8")
    x = workloads.make_x(wl)
    w = workloads.make_w(wl)
    z = oracle_mod.router_logits(workloads.bf16_bits(x), workloads.bf16_bits(w))
    ref = (x.double() @ w.double().T).float().numpy()
    ulps = np.abs(z.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1
    # the constant feature realises the offset: column shift of +3 on 8 experts
    o = workloads.expert_offsets(wl)
    assert (o == 3.0).sum() == 8 and (o == 0.0).sum() == wl.E - 8


# ---------------------------------------------------- selection

def _brute_topk(b_row, K):
    E = b_row.shape[0]
    keys = [int(k) for k in np.asarray(b_row, np.float32).view(np.uint32)]
    keys = [(~k & 0xFFFFFFFF) if k & 0x80000000 else (k | 0x80000000) for k in keys]
    rank = []
    for e in range(E):
        beats = sum(1 for f in range(E) if keys[f] > keys[e] or (keys[f] == keys[e] and f < e))
        rank.append(beats)
    order = sorted(range(E), key=lambda e: rank[e])
    return order[:K], order[K]


@pytest.mark.parametrize("tied", [False, True])
def test_select_brute_force(oracle_mod, tied):
    N, E, K = 40, 9, 3
    z = workloads.tied_logits(N, E, 1) if tied else workloads.random_logits(N, E, 1)
    beta = (workloads.tied_logits(1, E, 2)[0] * 0.5 if tied
            else workloads.random_logits(1, E, 2)[0] * 0.3)
    ids, gates, alpha = oracle_mod.select(z, beta, K)
    b = z + beta[None, :]
    for t in range(N):
        top, kth = _brute_topk(b[t], K)
        assert ids[t].tolist() == top
        assert len(set(ids[t].tolist())) == K
        assert alpha[t].view(np.uint32) == (-b[t, kth]).view(np.uint32)
        for k in range(K):
            assert gates[t, k] == oracle_mod.sigmoid_spec(z[t, ids[t, k]])


def test_select_tie_break_lower_id(oracle_mod):
    z = np.zeros((1, 6), np.float32)
    ids, _, alpha = oracle_mod.select(z, None, 4)
    assert ids.tolist() == [[0, 1, 2, 3]]
    assert alpha[0] == 0.0
    # +0.0 ranks above -0.0 in the total order
    z2 = np.array([[-0.0, 0.0, -0.0, 0.0]], np.float32)
    ids2, _, _ = oracle_mod.select(z2, None, 2)
    assert ids2.tolist() == [[1, 3]]


def test_gates_ignore_bias(oracle_mod):
    z = workloads.random_logits(200, 32, 4)
    b1 = workloads.random_logits(1, 32, 5)[0]
    b2 = workloads.random_logits(1, 32, 6)[0] * 3
    i1, g1, _ = oracle_mod.select(z, b1, 6)
    i2, g2, _ = oracle_mod.select(z, b2, 6)
    shared = 0
    for t in range(200):
        m1 = dict(zip(i1[t].tolist(), g1[t].tolist()))
        for e, g in zip(i2[t].tolist(), g2[t].tolist()):
            if e in m1:
                assert m1[e] == g
                shared += 1
    assert shared > 0


def test_alpha_leaves_k_positive(oracle_mod):
    z = workloads.random_logits(300, 40, 7)
    beta = workloads.random_logits(1, 40, 8)[0]
    _, _, alpha = oracle_mod.select(z, beta, 5)
    b = z + beta[None, :]
    pos = ((b + alpha[:, None]) > 0).sum(axis=1)
    assert (pos == 5).all()  # no ties in continuous data


# ---------------------------------------------------- permutation

def test_permute_against_stable_argsort(oracle_mod):
    z = workloads.random_logits(500, 24, 9)
    ids, _, _ = oracle_mod.select(z, None, 4)
    counts, offsets, perm, inv = oracle_mod.permute(ids, 24)
    flat = ids.ravel()
    assert counts.sum() == 500 * 4
    np.testing.assert_array_equal(counts, np.bincount(flat, minlength=24))
    np.testing.assert_array_equal(offsets[1:], np.cumsum(counts))
    assert offsets[0] == 0
    np.testing.assert_array_equal(perm, np.argsort(flat, kind="stable"))
    np.testing.assert_array_equal(inv[perm], np.arange(flat.shape[0]))
    for e in range(24):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert (flat[seg] == e).all() and (np.diff(seg) > 0).all()


# ---------------------------------------------------- column quantile + EQB

def test_column_quantile_invariant(oracle_mod):
    N, E, K = 1000, 16, 2
    z = workloads.random_logits(N, E, 12)
    _, _, alpha = oracle_mod.select(z, None, K)
    m = oracle_mod.eqb_target_rank(N, K, E)
    v = oracle_mod.column_quantiles(z, alpha, m)
    c = z + alpha[:, None]
    for e in range(E):
        assert (c[:, e] > v[e]).sum() <= m
        assert (c[:, e] >= v[e]).sum() >= m + 1
    # Each row's (K+1)-th entry of Z + alpha is exactly 0, so these columns
    # tie at 0 when the load equals m.  With a token bias free of ties,
    # subtracting v leaves exactly m positives in every column.
    a2 = workloads.random_logits(1, N, 16)[0]
    v2 = oracle_mod.column_quantiles(z, a2, m)
    c2 = z + a2[:, None]
    for e in range(E):
        assert (c2[:, e] - v2[e] > 0).sum() == m


def test_column_quantile_ties(oracle_mod):
    z = workloads.tied_logits(64, 8, 13)
    for m in (0, 5, 31, 63):
        v = oracle_mod.column_quantiles(z, None, m)
        for e in range(8):
            assert v[e].view(np.uint32) == np.float32(
                sorted(z[:, e].tolist(), key=oracle_mod.order_key, reverse=True)[m]).view(np.uint32)


def test_eqb_bias_centring(oracle_mod):
    v = workloads.random_logits(1, 384, 14)[0]
    beta = oracle_mod.eqb_bias(v)
    mean = np.float32(np.sum((-v).astype(np.float64)) / 384)
    np.testing.assert_array_equal(beta, (-v) - mean)
    assert abs(float(np.mean(beta.astype(np.float64)))) < 1e-6
    const = np.full(7, 2.5, np.float32)
    np.testing.assert_array_equal(oracle_mod.eqb_bias(const), np.zeros(7, np.float32))


def test_eqb_balances_collapsed_router(oracle_mod):
    """A collapsed router (+3 logit offset on a few experts) is re-balanced by
    repeated updates on the same batch: MaxVio falls from ~7 to a few percent
    (one update repairs the 4-token toy exactly; here the alternation needs
    a few steps, and each step must not undo the previous one)."""
    N, E, K = 4096, 32, 2
    z = workloads.random_logits(N, E, 15)
    z[:, :4] += 3.0
    beta = np.zeros(E, np.float32)
    mv = []
    for _ in range(6):
        ids, _, alpha = oracle_mod.select(z, beta, K)
        counts, _, _, _ = oracle_mod.permute(ids, E)
        mv.append(oracle_mod.maxvio(counts, N, K))
        v = oracle_mod.column_quantiles(z, alpha, oracle_mod.eqb_target_rank(N, K, E))
        beta = oracle_mod.eqb_bias(v)
    assert mv[0] > 6.0, mv
    assert mv[1] < mv[0] / 10, mv
    assert mv[3] < 0.1 and mv[5] < 0.1, mv


def test_maxvio_closed_form(oracle_mod):
    assert oracle_mod.maxvio(np.full(8, 5, np.int32), 20, 2) == 0.0
    assert oracle_mod.maxvio(np.array([10, 0, 0, 0], np.int32), 5, 2) == 3.0


# ------------------------------- intervention overlap count (section 9)

def test_intervention_overlap_pages_toy(oracle_mod, toy):
    """The toy re-routed after one EQB step keeps one of its own top-2 per
    token: 4 tokens x 1 shared expert, which is the rate 0.5 the pages give."""
    z = np.array(toy["logits_Z"], np.float32)
    beta = np.array(toy["beta_centred"], np.float32)
    ids, _, _ = oracle_mod.select(z, beta, toy["K"])
    ids_u, _, _ = oracle_mod.select(z, None, toy["K"])
    ovl = oracle_mod.intervention_overlap(ids, ids_u)
    assert ovl == 4
    assert 1.0 - ovl / (toy["T"] * toy["K"]) == toy["intervention_rate_after"]
    # before the update the router routes exactly its own choice
    assert oracle_mod.intervention_overlap(ids_u, ids_u) == toy["T"] * toy["K"]


def test_intervention_overlap_bruteforce(oracle_mod):
    rng = np.random.default_rng(5)
    for N, E, K in ((1, 4, 2), (50, 8, 3), (300, 64, 6), (200, 16, 8)):
        a = np.stack([rng.choice(E, K, replace=False) for _ in range(N)]).astype(np.int32)
        b = np.stack([rng.choice(E, K, replace=False) for _ in range(N)]).astype(np.int32)
        want = sum(len(set(x) & set(y)) for x, y in zip(a.tolist(), b.tolist()))
        assert oracle_mod.intervention_overlap(a, b) == want
        # order inside a token does not matter, the routed side and the
        # router's own side may be swapped
        assert oracle_mod.intervention_overlap(a[:, ::-1].copy(), b) == want
        assert oracle_mod.intervention_overlap(b, a) == want
        # disjoint halves of the experts share nothing
        lo = np.tile(np.arange(K, dtype=np.int32), (N, 1))
        assert oracle_mod.intervention_overlap(lo, lo + K) == 0
        # the rate is that count in one division, up to the rounding of the
        # rate's running mean
        r = oracle_mod.intervention_rate(a, b)
        assert abs(r - (1.0 - want / (N * K))) <= N * 2.0 ** -52


def test_intervention_overlap_random_routing_mean(oracle_mod):
    """Random routing against a fixed own choice: each token's overlap is
    hypergeometric with mean K^2 / E, so the total is N K^2 / E (section 9's
    closed form 1 - K/E for the rate)."""
    rng = np.random.default_rng(17)
    for K, E in ((2, 4), (6, 384), (8, 128)):
        N = 20000
        unb = np.tile(np.arange(K, dtype=np.int32), (N, 1))
        rnd = np.stack([rng.choice(E, size=K, replace=False) for _ in range(N)]).astype(np.int32)
        ovl = oracle_mod.intervention_overlap(rnd, unb)
        mean = K * K / E
        var = K * (K / E) * (1 - K / E) * (E - K) / max(E - 1, 1)
        assert abs(ovl - N * mean) < 5 * math.sqrt(N * var)
