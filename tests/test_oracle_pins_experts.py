"""Pins of the oracle's expert layer: the layer output y_t = f_shared(x_t) +
sum_k S_t,k f_e(x_t) of "Kolibri Pre-Training from Scratch" 6.1 with SwiGLU
experts ("Kolibri 1 im Detail": two projections d -> F give SiLU(gate) x up,
then one F -> d).

Each function is checked against something other than itself: closed forms
of SiLU, the exact nearest bf16 by brute force, a worked example small
enough to add up by hand (every value in it is exact), the rounding point of
the activation, and invariants (token independence, order of the routed
experts, a zero up projection)."""
import math
import struct

import numpy as np
import pytest


@pytest.fixture(scope="module")
def o(oracle_mod):
    return oracle_mod


def _bf16_bits(v):
    """bf16 bits of an fp32-exact value with at most 8 significant bits."""
    u = struct.unpack("<I", struct.pack("<f", np.float32(v)))[0]
    assert u & 0xffff == 0, v
    return u >> 16


def _bf16_value(b):
    return struct.unpack("<f", struct.pack("<I", (int(b) & 0xffff) << 16))[0]


def _bits(a):
    a = np.asarray(a, np.float64)
    return np.vectorize(_bf16_bits, otypes=[np.uint16])(a)


# ------------------------------------------------------------------ SiLU

def test_silu_closed_forms(o):
    assert o.silu_spec(0.0) == 0.0
    # sigma(ln 3) = 1 / (1 + 1/3) = 3/4
    assert abs(o.silu_spec(math.log(3.0)) - 0.75 * math.log(3.0)) <= 2 * math.ulp(0.82)
    # sigma(-x) = 1 - sigma(x), so SiLU(x) - SiLU(-x) = x
    for x in np.linspace(0.01, 30.0, 301):
        assert abs(o.silu_spec(x) - o.silu_spec(-x) - x) <= 8 * math.ulp(x)
    # e^-40 < 2^-53: sigma(40) rounds to 1 and SiLU(40) is 40 exactly
    assert o.silu_spec(40.0) == 40.0
    assert o.silu_spec(-800.0) == 0.0
    # against the library exp, a different implementation
    for x in np.linspace(-50.0, 50.0, 2001):
        want = x / (1.0 + math.exp(-x))
        assert abs(o.silu_spec(x) - want) <= 4 * math.ulp(abs(want) + 1e-300) + 1e-300


# ----------------------------------------------------- rounding to bf16

def _nearest_bf16_f64(v):
    """The nearest bf16 to an fp64 value by comparing the two neighbours
    exactly (fractions), ties to the even pattern."""
    from fractions import Fraction
    fv = Fraction(v)
    # start from truncation of the fp32 pattern toward zero
    u = struct.unpack("<I", struct.pack("<f", np.float32(v)))[0] >> 16
    cands = [(u + k) & 0xffff for k in (-2, -1, 0, 1, 2)]
    best = None
    for b in cands:
        if (b & 0x7fff) >= 0x7f80:
            continue
        if (b >> 15) != (1 if v < 0 else 0) and _bf16_value(b) != 0.0:
            continue
        dist = abs(Fraction(_bf16_value(b)) - fv)
        key = (dist, b & 1)
        if best is None or key < best[0]:
            best = (key, b)
    return best[1]


def test_bf16_round_f64_bruteforce(o):
    rng = np.random.default_rng(0)
    vals = list(rng.standard_normal(2000) * 50.0)
    vals += list(rng.standard_normal(200) * 1e-3)
    # midpoints of bf16 neighbours, exactly and just off them
    for b in rng.integers(0x3000, 0x5000, 200):
        lo, hi = _bf16_value(int(b)), _bf16_value(int(b) + 1)
        mid = (lo + hi) / 2
        vals += [mid, math.nextafter(mid, math.inf), math.nextafter(mid, -math.inf)]
    for v in vals:
        assert o.bf16_round_f64(v) == _nearest_bf16_f64(v), v


def test_bf16_round_f64_is_one_rounding(o):
    # 1 + 2^-8 + 2^-30 lies above the midpoint 1 + 2^-8; rounding to fp32 first
    # would land on that midpoint and then on 1.0 (ties to even)
    v = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert o.bf16_round_f64(v) == 0x3f81                    # 1 + 2^-7
    assert o.bf16_round(np.float32(v)) == 0x3f80            # the double rounding
    assert o.bf16_round_f64(-0.0) == 0x8000 and o.bf16_round_f64(0.0) == 0
    for v in (1.5, -3.25, 2.0 ** -120, 65280.0):              # representable: unchanged
        assert _bf16_value(o.bf16_round_f64(v)) == v


# ------------------------------------------------------- the expert layer

def _worked_example():
    """d = 4, F = 2, E = 3, K = 2, N = 2.  Gate weights 4(e+1) everywhere so
    g_j = 60(e+1) >= 60 and SiLU(g) = g exactly (sigma rounds to 1); the up
    projection of expert e, unit j, picks x[(e+j) % 4] / 16; the down
    projection is Wd[c,j] = (c+1) (1 for j = 0, 1/2 for j = 1).  Shared
    expert: g = 120, u_j = x[j] / 8, Wd_s = identity on the first two rows."""
    d, F, E = 4, 2, 3
    x = np.array([[1, 2, 4, 8], [8, 4, 2, 1]], np.float64)
    wgu = np.zeros((E, 2 * F, d))
    wd = np.zeros((E, d, F))
    for e in range(E):
        wgu[e, :F, :] = 4 * (e + 1)
        for j in range(F):
            wgu[e, F + j, (e + j) % 4] = 1 / 16
        for c in range(d):
            wd[e, c, 0] = c + 1
            wd[e, c, 1] = (c + 1) / 2
    wgu_s = np.zeros((2 * F, d))
    wgu_s[:F, :] = 8
    wd_s = np.zeros((d, F))
    for j in range(F):
        wgu_s[F + j, j] = 1 / 8
        wd_s[j, j] = 1
    ids = np.array([[2, 0], [1, 2]], np.int32)
    gates = np.array([[0.5, 0.25], [1.0, 0.125]], np.float32)
    return x, ids, gates, wgu, wd, wgu_s, wd_s


def test_expert_ffn_worked_example(o):
    x, ids, gates, wgu, wd, wgu_s, wd_s = _worked_example()
    y, mag, h, h_s = o.expert_ffn(_bits(x), ids, gates, _bits(wgu), _bits(wd), _bits(wgu_s),
                                  _bits(wd_s), want_h=True)
    # token 0: expert 2 -> h = (180*4/16, 180*8/16) = (45, 90), Y = 90 (c+1);
    #          expert 0 -> h = (60*1/16, 60*2/16) = (3.75, 7.5), Y = 7.5 (c+1);
    #          shared  -> h = (120*1/8, 120*2/8) = (15, 30),  Y = (15, 30, 0, 0)
    #          y = 0.5 (90, 180, 270, 360) + 0.25 (7.5, 15, 22.5, 30) + (15, 30, 0, 0)
    # token 1: expert 1 -> h = (120*4/16, 120*2/16) = (30, 15), Y = 37.5 (c+1);
    #          expert 2 -> h = (180*2/16, 180*1/16) = (22.5, 11.25), Y = 28.125 (c+1);
    #          shared  -> h = (120*8/8, 120*4/8) = (120, 60), Y = (120, 60, 0, 0)
    #          y = (37.5, 75, 112.5, 150) + 0.125 (28.125, 56.25, 84.375, 112.5) + (120, 60, 0, 0)
    want = np.array([[61.875, 123.75, 140.625, 187.5],
                     [161.015625, 142.03125, 123.046875, 164.0625]], np.float32)
    np.testing.assert_array_equal(y, want)
    hv = np.vectorize(_bf16_value)(h)
    np.testing.assert_array_equal(hv, [[45, 90], [3.75, 7.5], [30, 15], [22.5, 11.25]])
    np.testing.assert_array_equal(np.vectorize(_bf16_value)(h_s), [[15, 30], [120, 60]])
    # every product is non-negative here, so the magnitude is the sum itself
    np.testing.assert_array_equal(mag.astype(np.float32), want)


def test_expert_ffn_rounding_point(o):
    # one expert, no shared one: g = 64 (SiLU(64) = 64); u = 1 + 2^-8 puts
    # h = 64.25 on the midpoint of bf16 64 and 64.5 -> 64 (even); one more
    # 2^-20 in u lifts it past the midpoint -> 64.5
    d, F = 4, 1
    wgu = np.zeros((1, 2, d))
    wgu[0, 0, :2] = 32
    wgu[0, 1, :3] = [1, 2.0 ** -8, 2.0 ** -20]
    wd = np.ones((1, d, F))
    ids = np.zeros((2, 1), np.int32)
    gates = np.ones((2, 1), np.float32)
    x = np.array([[1, 1, 0, 0], [1, 1, 1, 0]], np.float64)
    y, _, h, _ = o.expert_ffn(_bits(x), ids, gates, _bits(wgu), _bits(wd), want_h=True)
    assert _bf16_value(h[0, 0]) == 64.0 and _bf16_value(h[1, 0]) == 64.5
    np.testing.assert_array_equal(y, [[64.0] * 4, [64.5] * 4])


def _random_case(seed, N=5, d=64, F=16, E=6, K=3, shared=True):
    rng = np.random.default_rng(seed)
    to_bits = lambda a: (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    x = to_bits(rng.standard_normal((N, d)))
    wgu = to_bits(rng.standard_normal((E, 2 * F, d)) / math.sqrt(d))
    wd = to_bits(rng.standard_normal((E, d, F)) / math.sqrt(F))
    wgu_s = to_bits(rng.standard_normal((2 * F, d)) / math.sqrt(d)) if shared else None
    wd_s = to_bits(rng.standard_normal((d, F)) / math.sqrt(F)) if shared else None
    ids = np.stack([rng.choice(E, K, replace=False) for _ in range(N)]).astype(np.int32)
    gates = rng.uniform(0.05, 0.95, (N, K)).astype(np.float32)
    return x, ids, gates, wgu, wd, wgu_s, wd_s


def test_expert_ffn_tokens_are_independent(o):
    x, ids, gates, wgu, wd, wgu_s, wd_s = _random_case(1)
    y, _ = o.expert_ffn(x, ids, gates, wgu, wd, wgu_s, wd_s)
    for t in range(x.shape[0]):
        yt, _ = o.expert_ffn(x[t:t + 1], ids[t:t + 1], gates[t:t + 1], wgu, wd, wgu_s, wd_s)
        np.testing.assert_array_equal(yt[0], y[t])


def test_expert_ffn_routed_order_and_single_experts(o):
    x, ids, gates, wgu, wd, wgu_s, wd_s = _random_case(2)
    y, mag = o.expert_ffn(x, ids, gates, wgu, wd, wgu_s, wd_s)
    # reversing the K routed experts changes only the fp64 summation order
    y_rev, _ = o.expert_ffn(x, ids[:, ::-1], gates[:, ::-1], wgu, wd, wgu_s, wd_s)
    assert np.all(np.abs(y_rev.astype(np.float64) - y) <= 2.0 ** -23 * np.abs(y) + 1e-12 * mag)
    # the layer is the sum of its one-expert parts: shared alone, then each routed slot alone
    total = np.zeros(y.shape, np.float64)
    none_ids = np.zeros((x.shape[0], 1), np.int32)
    zero_g = np.zeros((x.shape[0], 1), np.float32)
    ys, _ = o.expert_ffn(x, none_ids, zero_g, wgu, wd, wgu_s, wd_s)   # gate 0: shared only
    total += ys
    for k in range(ids.shape[1]):
        yk, _ = o.expert_ffn(x, ids[:, k:k + 1], gates[:, k:k + 1], wgu, wd)
        total += yk
    assert np.all(np.abs(total - y) <= 1e-6 * mag + 1e-12)
    # a slot whose up projection is zero contributes nothing
    wgu0 = wgu.copy()
    wgu0[:, wgu.shape[1] // 2:, :] = 0
    y0, _ = o.expert_ffn(x, ids, gates, wgu0, wd)
    assert np.all(y0 == 0)


def test_expert_ffn_gate_scales_linearly(o):
    # doubling every gate doubles the routed part exactly (a power of two)
    x, ids, gates, wgu, wd, _, _ = _random_case(3, shared=False)
    y1, _ = o.expert_ffn(x, ids, gates, wgu, wd)
    y2, _ = o.expert_ffn(x, ids, gates * np.float32(2), wgu, wd)
    np.testing.assert_array_equal(y2, y1 * np.float32(2))


def test_expert_weight_count_matches_the_pages():
    # "Kolibri 1 im Detail": 3 x 2560 x 512 = 3,932,160 matrix weights per
    # expert; six routed plus the shared one touch about 27.5 million per token
    d, F = 2560, 512
    assert 2 * F * d + d * F == 3_932_160
    assert abs(7 * 3_932_160 - 27.5e6) < 0.05e6
