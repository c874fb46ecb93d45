"""Pins of the oracle functions for the next rows of the path: the bf16-key
EQB quantile ("Kolibri Pre-Training from Scratch" 7.3), Load-Error Injection
(section 8) and its chain rule to the router logits.

Each function is checked against something other than itself: the pages'
printed values, brute force, the pages' own two-pass radix algorithm (run in
the oracle), closed forms and the bound the pages derive."""
import math
import struct

import numpy as np
import pytest


@pytest.fixture(scope="module")
def o(oracle_mod):
    return oracle_mod


def _f32_bits(v):
    return struct.unpack("<I", struct.pack("<f", np.float32(v)))[0]


def _bf16_value(b):
    return struct.unpack("<f", struct.pack("<I", (b & 0xffff) << 16))[0]


def _nearest_bf16_bruteforce(v):
    """The bf16 pattern nearest to the fp32 value v, ties to an even last
    bit, by comparing the two neighbours exactly in fp64."""
    u = _f32_bits(v)
    lo = u >> 16                     # truncation toward zero (same sign)
    hi = lo + 1                      # next pattern away from zero
    dl = abs(_bf16_value(lo) - float(np.float32(v)))
    hv = _bf16_value(hi)
    dh = abs(hv - float(np.float32(v))) if math.isfinite(hv) else math.inf
    if (hi & 0x7fff) == 0x7f80:      # the neighbour away from zero is infinity
        # IEEE overflow: round to inf when v is at or past the midpoint to
        # the next power of two beyond the largest finite bf16
        big = _bf16_value(lo) + (_bf16_value(lo) - _bf16_value(lo - 1)) / 2
        return hi if abs(float(np.float32(v))) >= abs(big) else lo
    if dl < dh:
        return lo
    if dh < dl:
        return hi
    return lo if (lo & 1) == 0 else hi


def test_bf16_round_matches_bruteforce(o):
    rng = np.random.default_rng(0)
    vals = list(rng.standard_normal(3000).astype(np.float32) * np.float32(7.0))
    vals += list((rng.standard_normal(500) * 1e-38).astype(np.float32))        # subnormals
    vals += [np.float32(x) for x in (0.0, -0.0, 1.0, -1.0, 3.0, 1.5, 0.5, 65504.0, 3.0e38)]
    # exact halfway cases: a bf16 value plus half of its last place
    for b in rng.integers(0x0080, 0x7f00, 300):
        base = _f32_bits(_bf16_value(int(b)))
        for sign in (0, 0x80000000):
            vals.append(struct.unpack("<f", struct.pack("<I", (base | 0x8000) ^ sign))[0])
    for v in vals:
        assert o.bf16_round(v) == _nearest_bf16_bruteforce(v), v


def test_bf16_key_orders_like_values(o):
    rng = np.random.default_rng(1)
    pats = list(rng.integers(0, 0x7f80, 2000)) + [int(p) | 0x8000 for p in rng.integers(0, 0x7f80, 2000)]
    pats += [0x0000, 0x8000]         # +0 and -0
    keys = [o.bf16_key(int(p)) for p in pats]
    vals = [_bf16_value(int(p)) for p in pats]
    for a in range(0, len(pats) - 1, 7):
        for b in range(a + 1, min(a + 40, len(pats))):
            va, vb = vals[a], vals[b]
            if va != vb:
                assert (keys[a] < keys[b]) == (va < vb)
    assert o.bf16_key(0x8000) < o.bf16_key(0x0000)      # -0 below +0, as for fp32


def test_bf16_quantile_pages_column(o):
    # 7.3: the column (3.0, 1.5, 0.5, 3.0); Q_2 = 1.5; all four values are exact in bf16
    col = np.array([[3.0], [1.5], [0.5], [3.0]], np.float32)
    assert o.column_quantiles_bf16(col, None, 2)[0] == np.float32(1.5)
    assert [o.column_quantiles_bf16(col, None, m)[0] for m in range(4)] == [3.0, 3.0, 1.5, 0.5]


def test_bf16_quantile_is_the_pages_two_pass_radix(o):
    # the pages' algorithm: 16-bit keys, two passes of 256-bin histograms of the
    # high then the low byte, histograms summed over ranks (chunks)
    rng = np.random.default_rng(2)
    N, E = 777, 5
    z = (rng.standard_normal((N, E)) * 2).astype(np.float32)
    a = (rng.standard_normal(N) * 0.3).astype(np.float32)
    for m in (0, 1, 31, 388, N - 1):
        v = o.column_quantiles_bf16(z, a, m)
        for e in range(E):
            keys = np.array([o.bf16_key(o.bf16_round(np.float32(z[t, e] + a[t]))) for t in range(N)],
                            dtype=np.uint64)
            k, _, _ = o.radix_select(keys, m, 256, 2, chunk_sizes=[300, 200, 277])
            b = (k & 0x7fff) if (k & 0x8000) else (~k & 0xffff)
            assert np.float32(_bf16_value(int(b))) == v[e], (m, e)


def test_bf16_quantile_commutes_with_rounding(o):
    # rounding to bf16 is monotone, so the (m+1)-th largest of the rounded
    # column is the rounding of the (m+1)-th largest fp32 value
    rng = np.random.default_rng(3)
    N, E = 1000, 7
    z = (rng.standard_normal((N, E)) * 3).astype(np.float32)
    a = (rng.standard_normal(N)).astype(np.float32)
    for m in (0, 5, 250, 999):
        v16 = o.column_quantiles_bf16(z, a, m)
        v32 = o.column_quantiles(z, a, m)
        for e in range(E):
            assert v16[e] == np.float32(_bf16_value(o.bf16_round(v32[e])))


def test_bf16_quantile_bruteforce_small(o):
    rng = np.random.default_rng(4)
    for trial in range(30):
        N = int(rng.integers(1, 9))
        col = rng.choice(np.array([-2.0, -0.0, 0.0, 0.5, 1.0, 1.0, 3.0, 1e-3], np.float32), N)
        z = col.reshape(N, 1).astype(np.float32)
        for m in range(N):
            want = sorted((_bf16_value(o.bf16_round(c)) for c in col), reverse=True)[m]
            assert o.column_quantiles_bf16(z, None, m)[0] == np.float32(want)


def test_tanh_spec(o):
    assert abs(o.tanh_spec(1.0) - 0.7616) < 5e-5                 # section 8 prints 0.7616
    # the spec forms 1 - e^(-2x): its error is a few units of the last place of
    # 1 (absolute), which only matters for small x
    for x in np.linspace(0.0, 40.0, 4001):
        t = o.tanh_spec(float(x))
        assert abs(t - math.tanh(x)) <= 4 * 2.0 ** -52 + 4 * math.ulp(math.tanh(x) + 1e-300)
    assert o.tanh_spec(1000.0) == 1.0


def test_lei_pages_example(o):
    # section 8: loads (4, 4, 0, 0) against a target of 2 -> rho = (1, 1, -1, -1),
    # xi = 1, tanh(1)/1 = 0.7616; every token receives lambda * 0.7616 * rho
    d = o.lei_delta(np.array([4, 4, 0, 0]), 4, 2)
    expect = np.float32(1e-5 * o.tanh_spec(1.0)) * np.array([1, 1, -1, -1], np.float32)
    np.testing.assert_array_equal(d, expect)
    assert abs(float(d[0]) - 1e-5 * 0.7616) < 1e-9
    g = np.zeros((4, 4), np.float32)
    out = o.lei_inject(np.array([4, 4, 0, 0]), g, 2)
    np.testing.assert_array_equal(out, np.tile(d, (4, 1)))


def test_lei_bound_and_small_imbalance(o):
    rng = np.random.default_rng(5)
    lam, tau = 1e-5, 1.0
    for trial in range(50):
        E, K, N = 64, 4, 1000
        counts = rng.multinomial(N * K, rng.dirichlet(np.full(E, 0.3 if trial % 2 else 50.0)))
        d = o.lei_delta(counts, N, K, lam, tau)
        # the pages' bound |delta| < lambda tau; rounding to fp32 is monotone,
        # so after it the bound holds with equality allowed at fp32(lambda tau)
        assert np.all(np.abs(d) <= np.float32(lam * tau))
        rho = counts / (K * N / E) - 1.0
        xi = np.abs(rho).max() / tau
        fac = 1.0 if xi == 0 else math.tanh(xi) / xi
        np.testing.assert_allclose(d, lam * fac * rho, rtol=1e-6, atol=1e-12)
    # balanced loads: rho = 0, the factor is 1 by continuity, delta = 0
    assert np.all(o.lei_delta(np.full(8, 50), 100, 4) == 0)
    # a small imbalance: tanh(xi)/xi ~ 1, the injection is ~ lambda * rho
    c = np.full(8, 50)
    c[0], c[1] = 51, 49
    d = o.lei_delta(c, 100, 4, lam, tau)
    np.testing.assert_allclose(d[:2], lam * np.array([0.02, -0.02]), rtol=2e-4)


def test_score_grad_to_logits(o):
    # section 8: sigma(2)(1 - sigma(2)) = 0.105
    g = o.score_grad_to_logits(np.array([2.0], np.float32), np.array([1.0], np.float32))
    assert abs(float(g[0]) - 0.105) < 5e-4
    z = np.linspace(-30, 30, 2001).astype(np.float32)
    gs = np.float32(1e-5 * 0.7616) * np.ones_like(z)
    got = o.score_grad_to_logits(z, gs)
    s = 1.0 / (1.0 + np.exp(-z.astype(np.float64)))
    want = (gs.astype(np.float64) * s * (1 - s)).astype(np.float32)
    assert np.all(np.abs(got.view(np.int32) - want.view(np.int32)) <= 1)   # within 1 fp32 ulp
    sat = o.score_grad_to_logits(np.array([800.0, -800.0], np.float32), np.array([1.0, 1.0], np.float32))
    np.testing.assert_array_equal(sat, np.zeros(2, np.float32))
