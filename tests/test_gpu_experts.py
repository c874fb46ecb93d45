"""The expert layer on the GPU against the oracle: y_t = f_shared(x_t) +
sum_k S_t,k f_e(x_t) ("Kolibri Pre-Training from Scratch" 6.1) with SwiGLU
experts ("Kolibri 1 im Detail": 2560 -> 2 x 512 -> 2560).

Bars (derived in the design notes):
- dispatch: bit-exact;
- h = bf16(SiLU(g) u): the GPU forms g and u in fp32 on the tensor cores,
  the oracle exactly; every h is within one bf16 step plus the fp32
  accumulation bound of g and u carried through SiLU(g) u (it matters where
  u or g nearly cancels), and nearly all are equal;
- y: |dy| <= 2^-10 * mag, mag the sum of the magnitudes of all products
  behind y (an h one step off moves a product by at most 2^-7 of itself);
- inputs whose every value is exact (the oracle's worked example, the
  rounding midpoint of h) must come out bit for bit."""
import math

import numpy as np
import pytest
import torch

from expert_load_balancing_b200 import binding as B

from gpu_helpers import check_status, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(kolibri_lib):
    return kolibri_lib


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _case(N, d, F, E, K, seed, shared=True, skew=False):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(N, d, generator=g).to(torch.bfloat16)
    wgu = (torch.randn(E, 2 * F, d, generator=g) / math.sqrt(d)).to(torch.bfloat16)
    wd = (torch.randn(E, d, F, generator=g) / math.sqrt(F)).to(torch.bfloat16)
    wgu_s = (torch.randn(2 * F, d, generator=g) / math.sqrt(d)).to(torch.bfloat16) if shared else None
    wd_s = (torch.randn(d, F, generator=g) / math.sqrt(F)).to(torch.bfloat16) if shared else None
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(N)]).astype(np.int32)
    if skew:                      # expert 0 in every token: several row blocks for one group
        for t in range(N):
            if 0 not in ids[t]:
                ids[t, 0] = 0
    gates = rng.uniform(0.05, 0.95, (N, K)).astype(np.float32)
    return x, wgu, wd, wgu_s, wd_s, ids, gates


def _oracle(o, x, wgu, wd, wgu_s, wd_s, ids, gates):
    return o.expert_ffn(_bits(x), ids, gates, _bits(wgu), _bits(wd),
                        None if wgu_s is None else _bits(wgu_s),
                        None if wd_s is None else _bits(wd_s), want_h=True)


def _gpu(x, wgu, wd, wgu_s, wd_s, ids, gates, o):
    E = wgu.shape[0]
    counts, offsets, perm, inv = o.permute(ids, E)
    xd = x.cuda()
    args = dict(perm=dev(perm.astype(np.int32)), offsets=dev(offsets.astype(np.int64)),
                inv=dev(inv.astype(np.int32)), gates=dev(gates))
    y = B.kolibri_expert_ffn(xd, args["perm"], args["offsets"], args["inv"], args["gates"],
                             wgu.cuda(), wd.cuda(), None if wgu_s is None else wgu_s.cuda(),
                             None if wd_s is None else wd_s.cuda())
    torch.cuda.synchronize()
    return y, args, perm


def _h_bound(a_rows, w_gate_up, group_of_row):
    """Per element of h: the fp32 accumulation bound of g and u carried
    through h = SiLU(g) u.  With g, u summed over d products in fp32,
    |dg| <= gamma Ag and |du| <= gamma Au (gamma = d 2^-24, Ag and Au the sums
    of the products' magnitudes), so |dh| <= gamma (1.1 |u| Ag + |SiLU(g)| Au)
    before the final rounding (|SiLU'| < 1.1); the rounding adds one step."""
    a = a_rows.float().numpy().astype(np.float64)
    w = w_gate_up.float().numpy().astype(np.float64)
    F = w.shape[1] // 2
    d = a.shape[1]
    out = np.empty((a.shape[0], F))
    for e in np.unique(group_of_row):
        r = np.nonzero(group_of_row == e)[0]
        wg, wu = w[e, :F], w[e, F:]
        g = a[r] @ wg.T
        u = a[r] @ wu.T
        ag = np.abs(a[r]) @ np.abs(wg).T
        au = np.abs(a[r]) @ np.abs(wu).T
        silu = g / (1.0 + np.exp(-np.clip(g, -700, 700)))
        out[r] = d * 2.0 ** -24 * (1.1 * np.abs(u) * ag + np.abs(silu) * au)
    return out


def _assert_h_close(h_gpu_bits, h_ref_bits, bound, min_equal=0.99):
    va = np.frombuffer((h_gpu_bits.astype(np.uint32) << 16).tobytes(), np.float32).reshape(h_gpu_bits.shape)
    vb = np.frombuffer((h_ref_bits.astype(np.uint32) << 16).tobytes(), np.float32).reshape(h_ref_bits.shape)
    # one bf16 step at the reference value (the spacing above |h|, 2^-133 at zero)
    step = np.spacing(np.abs(vb).astype(np.float32)) * np.float32(65536.0)
    step = np.maximum(step.astype(np.float64), 2.0 ** -133)
    err = np.abs(va.astype(np.float64) - vb.astype(np.float64))
    worst = float((err / (step + bound)).max())
    assert worst <= 1.0, ("h outside the accumulation bound", worst)
    eq = float((h_gpu_bits == h_ref_bits).mean())
    assert eq >= min_equal, eq
    return eq


def _assert_y_close(y, y_ref, mag):
    err = np.abs(y.astype(np.float64) - y_ref.astype(np.float64))
    bound = 2.0 ** -10 * mag + 1e-30
    worst = float((err / bound).max())
    assert worst <= 1.0, worst
    return worst


@pytest.mark.parametrize("N,d,F,E,K,shared,skew", [
    (37, 256, 256, 8, 2, True, False),
    (300, 256, 256, 16, 3, False, True),       # expert 0 spans several token blocks
    (700, 512, 256, 40, 4, True, True),       # three row blocks for one expert, empty experts
    (64, 2560, 512, 24, 6, True, False),      # the pages' d and F
])
def test_expert_ffn_matches_oracle(oracle_mod, N, d, F, E, K, shared, skew):
    x, wgu, wd, wgu_s, wd_s, ids, gates = _case(N, d, F, E, K, seed=N + E, shared=shared, skew=skew)
    y_ref, mag, h_ref, h_s_ref = _oracle(oracle_mod, x, wgu, wd, wgu_s, wd_s, ids, gates)
    y, args, perm = _gpu(x, wgu, wd, wgu_s, wd_s, ids, gates, oracle_mod)
    check_status()
    _assert_y_close(host(y), y_ref, mag)
    # the stages on their own: dispatch bit-exact, h within one bf16 step
    xp = B.kolibri_expert_dispatch(x.cuda(), args["perm"], K)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_bits(xp.cpu()), _bits(x)[perm // K])
    h = B.kolibri_expert_gate_up(xp, args["offsets"], wgu.cuda())
    torch.cuda.synchronize()
    group = ids.reshape(-1)[perm]
    _assert_h_close(_bits(h.cpu()), h_ref[perm], _h_bound(xp.cpu(), wgu, group))
    if shared:
        hs = B.kolibri_expert_gate_up(x.cuda(), None, wgu_s.cuda())
        torch.cuda.synchronize()
        _assert_h_close(_bits(hs.cpu()), h_s_ref,
                        _h_bound(x, wgu_s.unsqueeze(0), np.zeros(N, np.int64)))
    check_status()


def test_expert_ffn_pages_shape(oracle_mod):
    # E = 384 experts of 2560 -> 2 x 512 -> 2560 (3 GB of weights, drawn on the
    # device from a seeded generator); K = 6 plus the shared expert; the oracle
    # gets the slices of the experts these tokens use
    N, d, F, E, K = 48, 2560, 512, 384, 6
    g = torch.Generator(device="cuda").manual_seed(5)
    wgu = (torch.randn(E, 2 * F, d, generator=g, device="cuda") / math.sqrt(d)).to(torch.bfloat16)
    wd = (torch.randn(E, d, F, generator=g, device="cuda") / math.sqrt(F)).to(torch.bfloat16)
    wgu_s = (torch.randn(2 * F, d, generator=g, device="cuda") / math.sqrt(d)).to(torch.bfloat16)
    wd_s = (torch.randn(d, F, generator=g, device="cuda") / math.sqrt(F)).to(torch.bfloat16)
    x = torch.randn(N, d, generator=g, device="cuda").to(torch.bfloat16)
    rng = np.random.default_rng(5)
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(N)]).astype(np.int32)
    gates = rng.uniform(0.05, 0.95, (N, K)).astype(np.float32)
    used = np.unique(ids)
    remap = np.full(E, -1, np.int64)
    remap[used] = np.arange(len(used))
    y_ref, mag, _, _ = oracle_mod.expert_ffn(_bits(x.cpu()), remap[ids].astype(np.int32), gates,
                                             _bits(wgu[torch.from_numpy(used).cuda()].cpu()),
                                             _bits(wd[torch.from_numpy(used).cuda()].cpu()),
                                             _bits(wgu_s.cpu()), _bits(wd_s.cpu()), want_h=True)
    counts, offsets, perm, inv = oracle_mod.permute(ids, E)
    y = B.kolibri_expert_ffn(x, dev(perm.astype(np.int32)), dev(offsets.astype(np.int64)),
                             dev(inv.astype(np.int32)), dev(gates), wgu, wd, wgu_s, wd_s)
    torch.cuda.synchronize()
    check_status()
    _assert_y_close(host(y), y_ref, mag)
    # a second call repeats every bit (fixed summation orders throughout)
    y2 = B.kolibri_expert_ffn(x, dev(perm.astype(np.int32)), dev(offsets.astype(np.int64)),
                              dev(inv.astype(np.int32)), dev(gates), wgu, wd, wgu_s, wd_s)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(y2), host(y))


def _device_weights(E, d, F, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    wgu = (torch.randn(E, 2 * F, d, generator=g, device="cuda") / math.sqrt(d)).to(torch.bfloat16)
    wd = (torch.randn(E, d, F, generator=g, device="cuda") / math.sqrt(F)).to(torch.bfloat16)
    wgu_s = (torch.randn(2 * F, d, generator=g, device="cuda") / math.sqrt(d)).to(torch.bfloat16)
    wd_s = (torch.randn(d, F, generator=g, device="cuda") / math.sqrt(F)).to(torch.bfloat16)
    return wgu, wd, wgu_s, wd_s


def _oracle_on_tokens(o, rows, x, ids, gates, wgu, wd, wgu_s, wd_s):
    """The oracle on a subset of tokens (they are independent), with the
    slices of the experts those tokens use."""
    ids_r = ids[rows]
    used = np.unique(ids_r)
    remap = np.full(wgu.shape[0], -1, np.int64)
    remap[used] = np.arange(len(used))
    sl = torch.from_numpy(used).cuda()
    return o.expert_ffn(_bits(x[rows].cpu()), remap[ids_r].astype(np.int32), gates[rows],
                        _bits(wgu[sl].cpu()), _bits(wd[sl].cpu()), _bits(wgu_s.cpu()), _bits(wd_s.cpu()))


def test_expert_ffn_bench_size_sampled(oracle_mod):
    # the bench's microbatch: N = 16384 tokens, E = 384, K = 6, d = 2560, F = 512
    # plus the shared expert, the routing from the library's own permutation;
    # a sample of tokens (first, last, ragged and random) against the oracle
    N, d, F, E, K = 16384, 2560, 512, 384, 6
    wgu, wd, wgu_s, wd_s = _device_weights(E, d, F, 21)
    g = torch.Generator(device="cuda").manual_seed(22)
    x = torch.randn(N, d, generator=g, device="cuda").to(torch.bfloat16)
    rng = np.random.default_rng(22)
    ids = np.argsort(rng.random((N, E)), axis=1)[:, :K].astype(np.int32)
    gates = rng.uniform(0.05, 0.95, (N, K)).astype(np.float32)
    counts, offsets, perm, inv = B.kolibri_expert_permute(dev(ids), E)
    y = B.kolibri_expert_ffn(x, perm, offsets, inv, dev(gates), wgu, wd, wgu_s, wd_s)
    torch.cuda.synchronize()
    check_status()
    rows = np.unique(np.concatenate([[0, 1, N - 1, N - 256, 4095, 4096],
                                     rng.choice(N, 42, replace=False)]))
    y_ref, mag = _oracle_on_tokens(oracle_mod, rows, x, ids, gates, wgu, wd, wgu_s, wd_s)
    _assert_y_close(host(y)[rows], y_ref, mag)


@pytest.mark.parametrize("N,E,K,skew", [(1, 16, 1, False), (3, 8, 1, False), (2000, 4, 2, True)])
def test_expert_ffn_tiny_and_crowded(oracle_mod, N, E, K, skew):
    # one token, K = 1; and four experts that take hundreds of rows each (many
    # token blocks per group, both projections)
    d, F = 256, 256
    x, wgu, wd, wgu_s, wd_s, ids, gates = _case(N, d, F, E, K, seed=7 + N, shared=True, skew=skew)
    y_ref, mag, _, _ = _oracle(oracle_mod, x, wgu, wd, wgu_s, wd_s, ids, gates)
    y, _, _ = _gpu(x, wgu, wd, wgu_s, wd_s, ids, gates, oracle_mod)
    check_status()
    _assert_y_close(host(y), y_ref, mag)


def _pad(a, shape):
    out = np.zeros(shape, np.float32)
    out[tuple(slice(0, s) for s in a.shape)] = a
    return out


def test_expert_ffn_worked_example_exact(oracle_mod):
    # the oracle's hand-added example (d = 4, F = 2), zero-padded to d = 256,
    # F = 256: padded units have g = 0, SiLU(0) = 0, h = 0; every value is exact
    d, F, E = 256, 256, 3
    x = _pad(np.array([[1, 2, 4, 8], [8, 4, 2, 1]], np.float32), (2, d))
    wgu = np.zeros((E, 2 * F, d), np.float32)
    wd = np.zeros((E, d, F), np.float32)
    for e in range(E):
        wgu[e, :2, :4] = 4 * (e + 1)
        for j in range(2):
            wgu[e, F + j, (e + j) % 4] = 1 / 16
        for c in range(4):
            wd[e, c, 0] = c + 1
            wd[e, c, 1] = (c + 1) / 2
    wgu_s = np.zeros((2 * F, d), np.float32)
    wgu_s[:2, :4] = 8
    wd_s = np.zeros((d, F), np.float32)
    for j in range(2):
        wgu_s[F + j, j] = 1 / 8
        wd_s[j, j] = 1
    ids = np.array([[2, 0], [1, 2]], np.int32)
    gates = np.array([[0.5, 0.25], [1.0, 0.125]], np.float32)
    y, _, _ = _gpu(_bf16(x), _bf16(wgu), _bf16(wd), _bf16(wgu_s), _bf16(wd_s), ids, gates, oracle_mod)
    check_status()
    want = np.array([[61.875, 123.75, 140.625, 187.5],
                     [161.015625, 142.03125, 123.046875, 164.0625]], np.float32)
    np.testing.assert_array_equal(host(y)[:, :4], want)
    assert np.all(host(y)[:, 4:] == 0)
    y_ref, _, _, _ = _oracle(oracle_mod, _bf16(x), _bf16(wgu), _bf16(wd), _bf16(wgu_s), _bf16(wd_s),
                             ids, gates)
    np.testing.assert_array_equal(host(y), y_ref)


def test_gate_up_rounding_midpoint_exact():
    # g = 64 (SiLU(64) = 64 in fp32), u = 1 + 2^-8: h = 64.25, the midpoint of
    # bf16 64 and 64.5 -> 64 (even); u = 1 + 2^-8 + 2^-20 -> 64.5
    d, F = 256, 256
    wgu = np.zeros((1, 2 * F, d), np.float32)
    wgu[0, 0, :2] = 32
    wgu[0, F, :3] = [1, 2.0 ** -8, 2.0 ** -20]
    x = np.zeros((2, d), np.float32)
    x[0, :2] = 1
    x[1, :3] = 1
    h = B.kolibri_expert_gate_up(_bf16(x).cuda(), None, _bf16(wgu).cuda())
    torch.cuda.synchronize()
    hv = h.float().cpu().numpy()
    assert hv[0, 0] == 64.0 and hv[1, 0] == 64.5
    assert np.all(hv[:, 1:] == 0)


def test_combine_order_and_shared():
    # exact values: the fp32 multiply-adds in k order give the exact sum
    N, d, K = 5, 8, 3
    rng = np.random.default_rng(0)
    y_perm = rng.integers(-8, 8, (N * K, d)).astype(np.float32)
    y_sh = rng.integers(-8, 8, (N, d)).astype(np.float32)
    inv = rng.permutation(N * K).astype(np.int32)
    gates = np.array([0.5, 0.25, 2.0], np.float32)[None, :].repeat(N, 0)
    y = B.kolibri_expert_combine(dev(y_perm), dev(y_sh), dev(inv), dev(gates))
    torch.cuda.synchronize()
    want = y_sh + sum(gates[:, k:k + 1] * y_perm[inv.reshape(N, K)[:, k]] for k in range(K))
    np.testing.assert_array_equal(host(y), want)
    y0 = B.kolibri_expert_combine(dev(y_perm), None, dev(inv), dev(gates))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(y0), want - y_sh)


def test_expert_bad_perm_sets_device_status():
    N, d, K = 4, 256, 2
    x = torch.zeros(N, d, dtype=torch.bfloat16, device="cuda")
    perm = torch.tensor([0, 1, 2, 3, 4, 5, 6, 99], dtype=torch.int32, device="cuda")
    B.kolibri_expert_dispatch(x, perm, K)
    assert B.kolibri_device_status() == B.KOLIBRI_ERR_DEVICE
    assert B.kolibri_device_status() == B.KOLIBRI_OK


@pytest.mark.parametrize("offsets", [[0, 300, 100, 400], [0, 100, 200, 999], [5, 100, 200, 400]])
def test_expert_bad_offsets_flagged_and_nothing_written(offsets):
    # decreasing, past the rows, not starting at 0: the projection schedules
    # no tile, sets the device status, and leaves the output as it was
    rows, d, F, G = 400, 256, 256, 3
    a = torch.zeros(rows, d, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(G, 2 * F, d, dtype=torch.bfloat16, device="cuda")
    h = torch.full((rows, F), 7.0, dtype=torch.bfloat16, device="cuda")
    B.kolibri_expert_gate_up(a, dev(np.array(offsets, np.int64)), w, h)
    assert B.kolibri_device_status() == B.KOLIBRI_ERR_DEVICE
    assert bool((h == 7.0).all())
    assert B.kolibri_device_status() == B.KOLIBRI_OK


def test_expert_unsupported_shapes_rejected():
    a = torch.zeros(4, 192, dtype=torch.bfloat16, device="cuda")        # d not a multiple of 256
    w = torch.zeros(1, 256, 192, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.KolibriError) as ei:
        B.kolibri_expert_gate_up(a, None, w)
    assert ei.value.status == B.KOLIBRI_ERR_UNSUPPORTED_SHAPE
