"""The five Kolibri-shaped workloads end to end on the GPU, checked against
the oracle.  Stages after the GEMM are checked bit-exact on the GPU's own
logits; the GEMM within 1e-3 max(1,|Z|); end-to-end ids and biases against
oracle logits within the bounds their tolerances imply."""
import numpy as np
import pytest
import torch

from expert_load_balancing_b200 import binding as B
from expert_load_balancing_b200 import workloads

from gpu_helpers import (assert_bit_equal, assert_logits_close, check_status, dev, host)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(kolibri_lib):
    return kolibri_lib


def _forward(x, w, beta, K, E):
    # the call the benchmark times: logits with the selection in the epilogue
    z, ids, gates, alpha = B.kolibri_router_forward(x, w, beta, K)
    counts, offsets, perm, inv = B.kolibri_expert_permute(ids, E)
    return z, ids, gates, alpha, counts, offsets, perm, inv


def _check_route_exact(oracle_mod, z, beta, K, ids, gates, alpha, rows=None):
    z = host(z) if rows is None else host(z)[rows]
    ids_o, gates_o, alpha_o = oracle_mod.select(z, None if beta is None else host(beta), K)
    sel = slice(None) if rows is None else rows
    assert_bit_equal(host(ids)[sel], ids_o, "ids")
    assert_bit_equal(host(gates)[sel], gates_o, "gates")
    assert_bit_equal(host(alpha)[sel], alpha_o, "alpha")


def _check_end_to_end_ids(oracle_mod, z_ref, beta, K, ids_gpu, z_gpu):
    """Sets of ids agree except at tokens whose oracle top-K margin is within
    the logits tolerance (twice: both the K-th and (K+1)-th score may move)."""
    b = z_ref + (0 if beta is None else beta[None, :])
    srt = -np.sort(-b, axis=1)
    margin = srt[:, K - 1] - srt[:, K]
    tol = 2 * 1e-3 * np.maximum(1.0, np.abs(srt[:, K - 1]))
    ids_o, _, _ = oracle_mod.select(z_ref, beta, K)
    same = np.array([set(a) == set(c) for a, c in zip(ids_o.tolist(), ids_gpu.tolist())])
    near = margin <= tol
    assert (same | near).all(), np.nonzero(~(same | near))[0][:10]
    return int((~same).sum()), int(near.sum())


def _beta_bound(eps, v):
    ulp = np.spacing(np.float32(np.max(np.abs(v)) + 1.0))
    return 4 * eps + 8 * float(ulp)


# ------------------------------------------------------- small_n256

def test_small_n256(oracle_mod):
    wl = workloads.WORKLOADS["small_n256"]
    x, w, beta = workloads.make_x(wl), workloads.make_w(wl), workloads.make_beta(wl)
    z, ids, gates, alpha, counts, offsets, perm, inv = _forward(dev(x), dev(w), dev(beta), wl.K, wl.E)
    z_ref = oracle_mod.router_logits(workloads.bf16_bits(x), workloads.bf16_bits(w))
    eps = assert_logits_close(host(z), z_ref)
    _check_route_exact(oracle_mod, z, beta, wl.K, ids, gates, alpha)
    c_o, o_o, p_o, i_o = oracle_mod.permute(host(ids), wl.E)
    for g, o, n in ((counts, c_o, "counts"), (offsets, o_o, "offsets"), (perm, p_o, "perm"),
                    (inv, i_o, "inv")):
        assert_bit_equal(host(g), o, n)
    # EQB on the GPU logits: exact
    b = dev(beta.numpy().copy())
    _, q = B.kolibri_eqb_update(z, alpha, b, wl.K)
    v_o = oracle_mod.column_quantiles(host(z), host(alpha), wl.m)
    assert_bit_equal(host(q), v_o, "quantiles")
    assert_bit_equal(host(b), oracle_mod.eqb_bias(v_o), "beta")
    # end to end against the oracle's own logits
    _check_end_to_end_ids(oracle_mod, z_ref, beta.numpy(), wl.K, host(ids), host(z))
    _, _, a_ref = oracle_mod.select(z_ref, beta.numpy(), wl.K)
    b_ref = oracle_mod.eqb_bias(oracle_mod.column_quantiles(z_ref, a_ref, wl.m))
    assert np.abs(host(b) - b_ref).max() <= _beta_bound(eps, v_o)
    check_status()


# ------------------------------------------------------- collapsed_n16384

def test_collapsed_ten_updates(oracle_mod):
    """Collapsed router (+3 sigma on 8 experts), 10 EQB updates re-routing the
    same batch; every iteration bit-exact with the oracle on the same logits;
    MaxVio must fall."""
    wl = workloads.WORKLOADS["collapsed_n16384"]
    x, w = workloads.make_x(wl), workloads.make_w(wl)
    z = B.kolibri_router_logits(dev(x), dev(w))
    z_ref = oracle_mod.router_logits(workloads.bf16_bits(x), workloads.bf16_bits(w))
    assert_logits_close(host(z), z_ref)
    zh = host(z)
    beta_g = dev(workloads.make_beta(wl).numpy())
    beta_o = workloads.make_beta(wl).numpy()
    mv = []
    for it in range(wl.eqb_updates):
        ids, gates, alpha = B.kolibri_router_topk(z, beta_g, wl.K)
        counts, offsets, perm, inv = B.kolibri_expert_permute(ids, wl.E)
        ids_o, gates_o, alpha_o = oracle_mod.select(zh, beta_o, wl.K)
        assert_bit_equal(host(ids), ids_o, f"ids it{it}")
        assert_bit_equal(host(gates), gates_o, f"gates it{it}")
        assert_bit_equal(host(alpha), alpha_o, f"alpha it{it}")
        c_o, o_o, p_o, i_o = oracle_mod.permute(ids_o, wl.E)
        assert_bit_equal(host(counts), c_o, f"counts it{it}")
        assert_bit_equal(host(perm), p_o, f"perm it{it}")
        mv.append(oracle_mod.maxvio(c_o, wl.N, wl.K))
        B.kolibri_eqb_update(z, alpha, beta_g, wl.K)
        beta_o = oracle_mod.eqb_bias(oracle_mod.column_quantiles(zh, alpha_o, wl.m))
        assert_bit_equal(host(beta_g), beta_o, f"beta it{it}")
    assert mv[0] > 5.0 and mv[-1] < 0.2, mv
    check_status()


# ------------------------------------------------------- origin_n65536

def test_origin_shape(oracle_mod):
    wl = workloads.WORKLOADS["origin_n65536"]
    x, w, beta = workloads.make_x(wl), workloads.make_w(wl), workloads.make_beta(wl)
    z, ids, gates, alpha, counts, offsets, perm, inv = _forward(dev(x), dev(w), dev(beta), wl.K, wl.E)
    rows = np.random.default_rng(1).choice(wl.N, size=2048, replace=False)
    z_ref_rows = oracle_mod.router_logits(workloads.bf16_bits(x[rows]), workloads.bf16_bits(w))
    assert_logits_close(host(z)[rows], z_ref_rows)
    _check_route_exact(oracle_mod, z, beta, wl.K, ids, gates, alpha)
    c_o, o_o, p_o, i_o = oracle_mod.permute(host(ids), wl.E)
    assert_bit_equal(host(perm), p_o, "perm")
    assert_bit_equal(host(inv), i_o, "inv")
    assert_bit_equal(host(offsets), o_o, "offsets")
    b = dev(beta.numpy().copy())
    _, q = B.kolibri_eqb_update(z, alpha, b, wl.K)
    v_o = oracle_mod.column_quantiles(host(z), host(alpha), wl.m)
    assert_bit_equal(host(q), v_o, "quantiles")
    assert_bit_equal(host(b), oracle_mod.eqb_bias(v_o), "beta")
    check_status()


# ------------------------------------------------------- kolibri_n1m

@pytest.fixture(scope="module")
def n1m():
    wl = workloads.WORKLOADS["kolibri_n1m"]
    x = workloads.make_x(wl)
    w = workloads.make_w(wl)
    return wl, x, w


def test_kolibri_n1m(oracle_mod, n1m):
    """Full size: logits on sampled rows vs the oracle GEMM; selection on
    sampled rows and the permutation in full, bit-exact on the GPU logits;
    token biases, quantiles and biases exact over all rows and columns."""
    wl, x, w = n1m
    beta = workloads.make_beta(wl)
    xd, wd = dev(x), dev(w)
    z, ids, gates, alpha, counts, offsets, perm, inv = _forward(xd, wd, dev(beta), wl.K, wl.E)
    b = dev(beta.numpy().copy())
    _, q = B.kolibri_eqb_update(z, alpha, b, wl.K)
    check_status()
    del xd
    zh = host(z)
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([rng.choice(wl.N, size=512, replace=False),
                                     [0, 1, wl.N - 1, wl.N // 2]]))
    z_ref = oracle_mod.router_logits(workloads.bf16_bits(x[rows]), workloads.bf16_bits(w))
    assert_logits_close(zh[rows], z_ref)
    ids_o, gates_o, alpha_o = oracle_mod.select(zh, beta.numpy(), wl.K)
    assert_bit_equal(host(ids), ids_o, "ids")
    assert_bit_equal(host(gates), gates_o, "gates")
    assert_bit_equal(host(alpha), alpha_o, "alpha")
    c_o, o_o, p_o, i_o = oracle_mod.permute(ids_o, wl.E)
    assert_bit_equal(host(counts), c_o, "counts")
    assert_bit_equal(host(offsets), o_o, "offsets")
    assert_bit_equal(host(perm), p_o, "perm")
    assert_bit_equal(host(inv), i_o, "inv")
    v_o = oracle_mod.column_quantiles(zh, alpha_o, wl.m)
    assert_bit_equal(host(q), v_o, "quantiles")
    assert_bit_equal(host(b), oracle_mod.eqb_bias(v_o), "beta")
    # exactness property of the expert update at full size
    c = zh + alpha_o[:, None]
    above = (c > v_o[None, :]).sum(axis=0)
    at_least = (c >= v_o[None, :]).sum(axis=0)
    assert (above <= wl.m).all() and (at_least >= wl.m + 1).all()


# ------------------------------------------------------- decode sweep

@pytest.mark.parametrize("n_tokens", workloads.DECODE_TOKENS)
def test_decode_sweep(oracle_mod, n_tokens):
    wl = workloads.decode_workload(n_tokens)
    layers = range(wl.layers) if n_tokens <= 8 else range(0, wl.layers, 7)
    for layer in layers:
        x = workloads.make_x(wl, layer)
        w = workloads.make_w(wl, layer)
        beta = workloads.make_beta(wl, layer)
        z, ids, gates, alpha, counts, offsets, perm, inv = _forward(dev(x), dev(w), dev(beta),
                                                                     wl.K, wl.E)
        z_ref = oracle_mod.router_logits(workloads.bf16_bits(x), workloads.bf16_bits(w))
        assert_logits_close(host(z), z_ref)
        _check_route_exact(oracle_mod, z, beta, wl.K, ids, gates, alpha)
        c_o, o_o, p_o, i_o = oracle_mod.permute(host(ids), wl.E)
        assert_bit_equal(host(perm), p_o, "perm")
        assert_bit_equal(host(counts), c_o, "counts")
        _check_end_to_end_ids(oracle_mod, z_ref, beta.numpy(), wl.K, host(ids), host(z))
    check_status()
