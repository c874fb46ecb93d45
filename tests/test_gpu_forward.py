"""kolibri_router_forward (router GEMM with the selection in its epilogue).

Z must equal kolibri_router_logits's Z bit for bit (the same tensor-core
sums, the same order), and ids, gates and alpha must equal the oracle's
selection on that Z bit for bit ("Kolibri Pre-Training from Scratch" 6.1 and
7.1).  Covered: both column-group widths of the threshold, E that leaves
epilogue warps without columns, ragged token tails, several tiles per CTA,
heavy ties (rows finished by the row kernel) and the shapes that fall back
to the two separate kernels."""
import numpy as np
import pytest
import torch

from expert_load_balancing_b200 import binding as B
from expert_load_balancing_b200 import workloads

from gpu_helpers import assert_bit_equal, check_status, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(kolibri_lib):
    return kolibri_lib


def _poisoned(N, E, K):
    z = torch.full((N, E), float("nan"), device="cuda")
    ids = torch.full((N, K), -7, dtype=torch.int32, device="cuda")
    gates = torch.full((N, K), float("nan"), device="cuda")
    alpha = torch.full((N,), 12345.0, device="cuda")
    return z, ids, gates, alpha


def _check(oracle_mod, x, w, beta, K):
    N, E = x.shape[0], w.shape[0]
    xd, wd = x.cuda(), w.cuda()
    bd = None if beta is None else dev(beta)
    z, ids, gates, alpha = _poisoned(N, E, K)
    B.kolibri_router_forward(xd, wd, bd, K, z=z, ids=ids, gates=gates, alpha=alpha)
    z_ref = B.kolibri_router_logits(xd, wd)
    torch.cuda.synchronize()
    check_status()
    zf = host(z)
    assert_bit_equal(zf, host(z_ref), "z")
    oi, og, oa = oracle_mod.select(zf, beta, K)
    assert_bit_equal(host(ids), oi, "ids")
    assert_bit_equal(host(gates), og, "gates")
    assert_bit_equal(host(alpha), oa, "alpha")


CASES = [
    # N, d, E, K, logit offsets, beta
    (70001, 2560, 384, 6, "zipf1.1", "normal0.1"),   # Kolibri shape, ragged tail
    (4099, 2048, 128, 8, "none", "normal0.1"),       # Origin shape: groups of 8 columns
    (1000, 512, 384, 16, "collapsed8", "zeros"),     # largest K
    (777, 256, 64, 6, "none", "normal0.1"),          # groups of 8, one warp of columns
    (300, 640, 256, 2, "collapsed8", "normal0.1"),   # third column warp idle
    (257, 1024, 336, 6, "zipf1.1", "normal0.1"),     # E % 32 == 16
    (1, 2560, 384, 6, "none", "normal0.1"),
    (255, 128, 384, 1, "none", "zeros"),
    (77, 64, 16, 1, "none", "normal0.1"),           # smallest E: one 32-column TMEM block
]


@pytest.mark.parametrize("N,d,E,K,offsets,beta", CASES)
@pytest.mark.parametrize("with_bias", [True, False])
def test_forward_matches_logits_and_oracle(oracle_mod, N, d, E, K, offsets, beta, with_bias):
    wl = workloads.Workload("t", N, d, E, K, offsets=offsets, beta=beta)
    b = workloads.make_beta(wl).numpy() if with_bias else None
    _check(oracle_mod, workloads.make_x(wl), workloads.make_w(wl), b, K)


# decode batches: one clustered launch (16 tokens per cluster, E a multiple of
# 128, up to 96 tokens); 97 tokens and E = 512 at d = 2560 take the other paths
DECODE_CASES = [
    (1, 2560, 384, 6), (15, 2560, 384, 6), (16, 2560, 384, 6), (17, 2560, 384, 6),
    (33, 2560, 384, 6), (64, 2560, 384, 6), (95, 2560, 384, 6), (96, 2560, 384, 6), (97, 2560, 384, 6),
    (5, 2048, 128, 8), (40, 1024, 256, 16), (9, 1024, 512, 16), (3, 2560, 512, 6), (20, 64, 128, 1),
]


@pytest.mark.parametrize("N,d,E,K", DECODE_CASES)
@pytest.mark.parametrize("with_bias", [True, False])
def test_forward_decode_batches(oracle_mod, N, d, E, K, with_bias):
    wl = workloads.Workload("t", N, d, E, K, offsets="collapsed8", beta="normal0.1")
    b = workloads.make_beta(wl).numpy() if with_bias else None
    x, w = workloads.make_x(wl), workloads.make_w(wl)
    _check(oracle_mod, x, w, b, K)
    # and the logits against the oracle's sums
    from gpu_helpers import assert_logits_close
    z = B.kolibri_router_logits(x.cuda(), w.cuda())
    torch.cuda.synchronize()
    assert_logits_close(host(z), oracle_mod.router_logits(workloads.bf16_bits(x), workloads.bf16_bits(w)))


@pytest.mark.parametrize("N,d,E,K", [(1, 2560, 384, 6), (5, 2560, 384, 6), (16, 2560, 384, 6),
                                     (17, 2560, 384, 6), (64, 1024, 128, 8), (7, 1024, 512, 16),
                                     (300, 512, 384, 6), (5000, 256, 384, 6)])
@pytest.mark.parametrize("with_bias", [True, False])
def test_forward_permute_equals_the_two_calls(oracle_mod, N, d, E, K, with_bias):
    # up to 16 tokens the forward and the grouping come from one launch; every
    # output must equal the forward followed by the permutation, bit for bit
    wl = workloads.Workload("t", N, d, E, K, offsets="collapsed8", beta="normal0.1")
    b = dev(workloads.make_beta(wl).numpy()) if with_bias else None
    x, w = workloads.make_x(wl).cuda(), workloads.make_w(wl).cuda()
    got = B.kolibri_router_forward_permute(x, w, b, K)
    z, ids, gates, alpha = B.kolibri_router_forward(x, w, b, K)
    counts, offsets, perm, inv = B.kolibri_expert_permute(ids, E)
    torch.cuda.synchronize()
    check_status()
    for name, a, r in zip(("z", "ids", "gates", "alpha", "counts", "offsets", "perm", "inv"), got,
                          (z, ids, gates, alpha, counts, offsets, perm, inv)):
        assert_bit_equal(host(a), host(r), name)
    c_o, o_o, p_o, i_o = oracle_mod.permute(host(ids), E)
    assert_bit_equal(host(got[6]), p_o, "perm vs oracle")
    assert_bit_equal(host(got[4]), c_o, "counts vs oracle")


def _forward_permute_no_ws(x, w, b, K):
    """kolibri_router_forward_permute with ws = NULL: a decode batch then takes
    the clustered form."""
    N, d = x.shape
    E = w.shape[0]
    f32, i32 = torch.float32, torch.int32
    z, gates = torch.empty((N, E), dtype=f32, device="cuda"), torch.empty((N, K), dtype=f32, device="cuda")
    ids = torch.empty((N, K), dtype=i32, device="cuda")
    alpha = torch.empty((N,), dtype=f32, device="cuda")
    counts = torch.empty((E,), dtype=i32, device="cuda")
    offsets = torch.empty((E + 1,), dtype=torch.int64, device="cuda")
    perm, inv = torch.empty((N * K,), dtype=i32, device="cuda"), torch.empty((N * K,), dtype=i32, device="cuda")
    st = B.load().kolibri_router_forward_permute(
        B._ptr(x), B._ptr(w), B._ptr(b), B._ptr(z), N, d, E, K, B._ptr(ids), B._ptr(gates), B._ptr(alpha),
        B._ptr(counts), B._ptr(offsets), B._ptr(perm), B._ptr(inv), None, 0, B._stream(None))
    assert st == B.KOLIBRI_OK, B.status_string(st)
    return z, ids, gates, alpha, counts, offsets, perm, inv


@pytest.mark.parametrize("N,d,E,K", [(1, 2560, 384, 6), (8, 2560, 384, 6), (16, 2560, 384, 6),
                                     (3, 2048, 128, 8), (11, 1024, 256, 16), (16, 1024, 512, 16),
                                     (2, 4096, 128, 6), (3, 2560, 512, 6), (5, 2624, 384, 6)])
def test_forward_permute_decode_forms(oracle_mod, N, d, E, K):
    # up to 16 tokens: with a workspace, E/8 blocks and a counter (the last
    # block selects and groups); without, one 16-CTA cluster.  Both equal the
    # forward followed by the permutation bit for bit, over three calls on
    # one workspace (the counter goes back to zero after each).  The last two
    # shapes do not fit the cluster's shared memory: the forward takes the
    # small-batch kernels, and so does this call
    ws = B.workspace(B.KOLIBRI_OP_PERMUTE, N, E, K)
    for seed in range(3):
        wl = workloads.Workload("t", N, d, E, K, offsets="collapsed8", beta="normal0.1", seed=seed)
        b = dev(workloads.make_beta(wl).numpy()) if seed != 1 else None
        x, w = workloads.make_x(wl).cuda(), workloads.make_w(wl).cuda()
        got = B.kolibri_router_forward_permute(x, w, b, K, ws=ws)
        clustered = _forward_permute_no_ws(x, w, b, K)
        z, ids, gates, alpha = B.kolibri_router_forward(x, w, b, K)
        counts, offsets, perm, inv = B.kolibri_expert_permute(ids, E)
        torch.cuda.synchronize()
        check_status()
        names = ("z", "ids", "gates", "alpha", "counts", "offsets", "perm", "inv")
        for name, a, c, r in zip(names, got, clustered, (z, ids, gates, alpha, counts, offsets, perm, inv)):
            assert_bit_equal(host(a), host(r), name)
            assert_bit_equal(host(c), host(r), name + " (clustered)")
        ids_o, gates_o, alpha_o = oracle_mod.select(host(z), None if b is None else host(b), K)
        assert_bit_equal(host(got[1]), ids_o, "ids vs oracle")
        assert_bit_equal(host(got[2]), gates_o, "gates vs oracle")
        assert_bit_equal(host(got[3]), alpha_o, "alpha vs oracle")


def test_forward_permute_decode_counter_not_zero_is_reported():
    # a workspace whose counter was never zeroed: every block's ticket is out
    # of range, none selects, and the device status says so; zeroed, the same
    # workspace works
    N, d, E, K = 4, 1024, 384, 6
    wl = workloads.Workload("t", N, d, E, K, beta="normal0.1")
    x, w = workloads.make_x(wl).cuda(), workloads.make_w(wl).cuda()
    b = dev(workloads.make_beta(wl).numpy())
    ws = B.workspace(B.KOLIBRI_OP_PERMUTE, N, E, K)
    ws.fill_(0x7F)
    B.kolibri_router_forward_permute(x, w, b, K, ws=ws)
    torch.cuda.synchronize()
    assert B.kolibri_device_status() == B.KOLIBRI_ERR_DEVICE
    ws.zero_()
    got = B.kolibri_router_forward_permute(x, w, b, K, ws=ws)
    z, ids, gates, alpha = B.kolibri_router_forward(x, w, b, K)
    torch.cuda.synchronize()
    check_status()
    for name, a, r in zip(("z", "ids", "gates", "alpha"), got, (z, ids, gates, alpha)):
        assert_bit_equal(host(a), host(r), name)


def test_forward_decode_heavy_ties(oracle_mod):
    # identical router rows in a decode batch: the selection's slow path
    N, d, E, K = 40, 256, 384, 6
    g = torch.Generator().manual_seed(12)
    x = torch.randn(N, d, generator=g).to(torch.bfloat16)
    x[::4] = 0
    w = torch.randn(1, d, generator=g).repeat(E, 1)
    w[E // 2:] = torch.randn(E - E // 2, d, generator=g)
    w = (w / 16).to(torch.bfloat16)
    beta = np.zeros(E, np.float32)
    beta[::5] = 0.25
    _check(oracle_mod, x, w, beta, K)


def test_forward_many_tiles_per_cta(oracle_mod):
    # more 256-token tiles than SM pairs: every CTA pair loops, and the
    # per-row candidate counters are reused tile after tile
    wl = workloads.Workload("t", 148 * 256 * 3 + 77, 256, 384, 6, offsets="zipf1.1", beta="normal0.1")
    _check(oracle_mod, workloads.make_x(wl), workloads.make_w(wl), workloads.make_beta(wl).numpy(), 6)


@pytest.mark.parametrize("E,K", [(400, 6), (48, 6)])
def test_forward_fallback_shapes(oracle_mod, E, K):
    # E > 384, or too few column groups for a (K+1)-th group maximum: the
    # call runs the two kernels one after the other, with the same results
    wl = workloads.Workload("t", 513, 512, E, K, beta="normal0.1")
    _check(oracle_mod, workloads.make_x(wl), workloads.make_w(wl), workloads.make_beta(wl).numpy(), K)


@pytest.mark.parametrize("with_bias", [True, False])
def test_forward_heavy_ties(oracle_mod, with_bias):
    # identical router rows: every score of a token ties, far more candidates
    # than the epilogue's per-row buffer, so the row kernel finishes them;
    # zero tokens tie at exactly 0 (and +0 vs -0 never arises from sums)
    N, d, E, K = 1500, 256, 384, 6
    g = torch.Generator().manual_seed(11)
    x = torch.randn(N, d, generator=g).to(torch.bfloat16)
    x[::3] = 0
    w = torch.randn(1, d, generator=g).repeat(E, 1)
    w[E // 2:] = torch.randn(E - E // 2, d, generator=g)      # half the experts tie
    w = (w / 16).to(torch.bfloat16)
    beta = np.zeros(E, np.float32)
    if with_bias:
        beta[::5] = 0.25                                     # ties among biased scores too
    _check(oracle_mod, x, w, beta if with_bias else None, K)


def test_forward_rejects_bad_args():
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    lib = B.load()
    z = torch.empty((4, 16), device="cuda")
    ids = torch.empty((4, 2), dtype=torch.int32, device="cuda")
    g = torch.empty((4, 2), device="cuda")
    p = lambda t: None if t is None else t.data_ptr()
    st = lib.kolibri_router_forward(p(x), p(w), None, p(z), 4, 64, 16, 2, p(ids), p(g), None, None)
    assert st == B.KOLIBRI_ERR_INVALID_ARG          # alpha is required
    a = torch.empty((4,), device="cuda")
    st = lib.kolibri_router_forward(p(x), p(w), None, p(z), 4, 96, 16, 2, p(ids), p(g), p(a), None)
    assert st == B.KOLIBRI_ERR_UNSUPPORTED_SHAPE    # d % 64 != 0
