"""The synthetic input recipe (CPU): seeded, reproducible, and shaped as
stated -- x ~ N(0, 1) and W ~ N(0, 1/d) rounded to bf16, the per-expert logit
offsets carried by the constant feature 0, the collapsed router's +3 on eight
experts, the Zipf(1.1) offsets centred, and rows re-drawable block by block."""
import math

import numpy as np
import pytest
import torch

from expert_load_balancing_b200 import workloads as W


def test_named_workloads_have_the_pages_shapes():
    wl = W.WORKLOADS
    assert (wl["kolibri_n1m"].N, wl["kolibri_n1m"].d, wl["kolibri_n1m"].E, wl["kolibri_n1m"].K) == \
        (1 << 20, 2560, 384, 6)
    assert (wl["origin_n65536"].d, wl["origin_n65536"].E, wl["origin_n65536"].K) == (2048, 128, 8)
    assert wl["collapsed_n16384"].eqb_updates == 10
    assert [W.decode_workload(n).N for n in W.DECODE_TOKENS] == [1, 8, 64, 256]
    # EQB target ranks of the configs: 4, 256, 4096, 16384
    assert [wl[k].m for k in ("small_n256", "collapsed_n16384", "origin_n65536", "kolibri_n1m")] == \
        [4, 256, 4096, 16384]


def test_draws_are_seeded_and_distinct_per_layer():
    wl = W.Workload("t", 300, 256, 16, 2, beta="normal0.1")
    assert torch.equal(W.make_x(wl), W.make_x(wl))
    assert torch.equal(W.make_w(wl), W.make_w(wl))
    assert torch.equal(W.make_beta(wl), W.make_beta(wl))
    assert not torch.equal(W.make_w(wl, layer=0), W.make_w(wl, layer=1))
    assert not torch.equal(W.make_x(wl, layer=0), W.make_x(wl, layer=1))


def test_rows_redraw_block_by_block():
    wl = W.Workload("t", 3 * W.ROW_BLOCK + 123, 64, 16, 2, offsets="zipf1.1")
    x = W.make_x(wl)
    rows = np.array([0, 1, W.ROW_BLOCK - 1, W.ROW_BLOCK, 2 * W.ROW_BLOCK + 7, wl.N - 1])
    assert torch.equal(W.x_rows(wl, rows), x[torch.from_numpy(rows)])


def test_moments_of_x_and_w():
    wl = W.Workload("t", 8192, 2560, 384, 6)
    x = W.make_x(wl).float()
    w = W.make_w(wl).float()
    assert abs(float(x.mean())) < 0.01 and abs(float(x.var()) - 1.0) < 0.01
    # unit-variance logits: var(W) = 1 / d
    assert abs(float(w.var()) * wl.d - 1.0) < 0.02
    beta = W.make_beta(W.Workload("t", 1, 64, 4096, 2, beta="normal0.1"))
    assert abs(float(beta.var()) - 0.1) < 0.01


def test_collapsed_router_offsets():
    wl = W.Workload("t", 64, 256, 48, 4, offsets="collapsed8")
    o = W.expert_offsets(wl)
    assert (o == 3.0).sum() == 8 and (o == 0.0).sum() == wl.E - 8
    x, w = W.make_x(wl), W.make_w(wl)
    assert bool((x[:, 0].float() == 1.0).all())
    # 3.0 and 0.0 are bf16-exact: feature 0 adds exactly o_e to every logit of expert e
    assert np.array_equal(w[:, 0].float().numpy(), o)


@pytest.mark.parametrize("E", [128, 384])
def test_zipf_offsets(E):
    wl = W.Workload("t", 16, 256, E, 6, offsets="zipf1.1")
    o = W.expert_offsets(wl).astype(np.float64)
    assert abs(o.mean()) < 1e-6                       # centred
    # sorted descending they follow -1.1 ln(rank) up to the common shift
    s = np.sort(o)[::-1]
    ranks = np.arange(1, E + 1, dtype=np.float64)
    ref = -1.1 * np.log(ranks)
    np.testing.assert_allclose(s - s[0], ref - ref[0], atol=1e-5)
    # each expert's rank is a seeded permutation, not the identity
    assert not np.all(np.diff(o) <= 0)
    w = W.make_w(wl)
    # W[:, 0] carries bf16(o_e)
    np.testing.assert_array_equal(w[:, 0].float().numpy(),
                                  torch.from_numpy(o.astype(np.float32)).to(torch.bfloat16).float().numpy())
    assert math.isclose(float(W.make_x(wl)[:, 0].float().min()), 1.0)
