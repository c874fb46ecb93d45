"""Plain CPU oracle for the sigmoid router + Exact Quantile Balancing path.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are its only users.  The product package never imports it,
and it imports nothing from the product package.

The arithmetic lives in ``kolibri_oracle.c`` (plain C, compiled without
fast-math or FP contraction).  This module only compiles it, marshals numpy
arrays through ctypes and documents each call.  Every function follows the
page "Kolibri Pre-Training from Scratch: UniBPE, Hybrid Attention and Exact
Quantile Balancing" (sections 1, 6.1, 6.2, 7.1-7.3, 9); the C file names the
section each one restates.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kolibri_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "libkolibri_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/libkolibri_oracle.so``."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off",
           "-fno-finite-math-only", "-fopenmp", "-shared", "-fPIC",
           _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    i64, i32, f32, f64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_double
    lib.oracle_order_key.argtypes = [f32]
    lib.oracle_order_key.restype = ctypes.c_uint32
    lib.oracle_exp_spec.argtypes = [f64]
    lib.oracle_exp_spec.restype = f64
    lib.oracle_sigmoid_spec.argtypes = [f32]
    lib.oracle_sigmoid_spec.restype = f32
    lib.oracle_router_logits.argtypes = [P, P, P, i64, i32, i32]
    lib.oracle_select.argtypes = [P, P, i64, i32, i32, P, P, P]
    lib.oracle_permute.argtypes = [P, i64, i32, i32, P, P, P, P]
    lib.oracle_column_quantiles.argtypes = [P, P, i64, i32, i64, P]
    lib.oracle_eqb_bias.argtypes = [P, i32, P]
    lib.oracle_radix_select.argtypes = [P, P, i32, i64, i64, i32, P, P]
    lib.oracle_radix_select.restype = ctypes.c_uint64
    lib.oracle_maxvio.argtypes = [P, i32, i64, i32]
    lib.oracle_maxvio.restype = f64
    lib.oracle_intervention_rate.argtypes = [P, P, i64, i32]
    lib.oracle_intervention_rate.restype = f64
    lib.oracle_intervention_overlap.argtypes = [P, P, i64, i32]
    lib.oracle_intervention_overlap.restype = i64
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_bf16_round.argtypes = [f32]
    lib.oracle_bf16_round.restype = ctypes.c_uint16
    lib.oracle_bf16_key.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_key.restype = ctypes.c_uint16
    lib.oracle_column_quantiles_bf16.argtypes = [P, P, i64, i32, i64, P]
    lib.oracle_tanh_spec.argtypes = [f64]
    lib.oracle_tanh_spec.restype = f64
    lib.oracle_lei_delta.argtypes = [P, i64, i32, i32, f64, f64, P]
    lib.oracle_lei_inject.argtypes = [P, i64, i32, i32, f64, f64, P]
    lib.oracle_score_grad_to_logits.argtypes = [P, P, i64, P]
    lib.oracle_bf16_round_f64.argtypes = [f64]
    lib.oracle_bf16_round_f64.restype = ctypes.c_uint16
    lib.oracle_silu_spec.argtypes = [f64]
    lib.oracle_silu_spec.restype = f64
    lib.oracle_expert_ffn.argtypes = [P, P, P, P, P, P, P, i64, i32, i32, i32, i32, P, P, P, P]
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    """OpenMP threads the oracle uses (set OMP_NUM_THREADS to change)."""
    return int(_load().oracle_num_threads())


def order_key(v: float) -> int:
    """Order-preserving unsigned key of an fp32 value (the total order used
    for every comparison of scores)."""
    return int(_load().oracle_order_key(ctypes.c_float(v)))


def exp_spec(x: float) -> float:
    """fp64 exp used by the gate (Cody-Waite reduction + Taylor, |x| <= 700)."""
    return float(_load().oracle_exp_spec(float(x)))


def sigmoid_spec(z: float) -> np.float32:
    """Gate sigma(z) in fp64 rounded once to fp32 (section 6.1)."""
    return np.float32(_load().oracle_sigmoid_spec(ctypes.c_float(np.float32(z))))


def sigmoid_spec_array(z) -> np.ndarray:
    z = _c(z, np.float32).ravel()
    f = _load().oracle_sigmoid_spec
    return np.array([f(ctypes.c_float(v)) for v in z.tolist()], dtype=np.float32)


def router_logits(x_bf16_bits, w_bf16_bits) -> np.ndarray:
    """Z = x W^T with x [N,d], W [E,d] given as bf16 bit patterns (uint16);
    fp64 products and sum, rounded once to fp32 (section 6.1)."""
    x = _c(x_bf16_bits, np.uint16)
    w = _c(w_bf16_bits, np.uint16)
    N, d = x.shape
    E, d2 = w.shape
    assert d == d2
    z = np.empty((N, E), dtype=np.float32)
    _load().oracle_router_logits(_ptr(x), _ptr(w), _ptr(z), N, d, E)
    return z


def select(z, beta, K: int):
    """Bias add, top-K, gates and token bias (sections 6.1 and 7.1).

    Returns (ids [N,K] int32, gates [N,K] fp32, alpha [N] fp32).  ``beta``
    may be None (route on the raw logits)."""
    z = _c(z, np.float32)
    N, E = z.shape
    b = None if beta is None else _c(beta, np.float32)
    ids = np.empty((N, K), dtype=np.int32)
    gates = np.empty((N, K), dtype=np.float32)
    alpha = np.empty((N,), dtype=np.float32)
    _load().oracle_select(_ptr(z), _ptr(b), N, E, K, _ptr(ids), _ptr(gates), _ptr(alpha))
    return ids, gates, alpha


def permute(ids, E: int):
    """Expert loads and the stable grouping of the N*K routed slots.

    Returns (counts [E] int32, offsets [E+1] int64, perm [N*K] int32,
    inv [N*K] int32)."""
    ids = _c(ids, np.int32)
    N, K = ids.shape
    counts = np.empty((E,), dtype=np.int32)
    offsets = np.empty((E + 1,), dtype=np.int64)
    perm = np.empty((N * K,), dtype=np.int32)
    inv = np.empty((N * K,), dtype=np.int32)
    _load().oracle_permute(_ptr(ids), N, E, K, _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv))
    return counts, offsets, perm, inv


def column_quantiles(z, alpha, m: int) -> np.ndarray:
    """v_e = Q_m(Z[:,e] + alpha) by a full sort of each column (sections 1, 7.1).
    ``alpha`` may be None (quantiles of the plain columns)."""
    z = _c(z, np.float32)
    N, E = z.shape
    a = None if alpha is None else _c(alpha, np.float32)
    assert 0 <= m < N
    v = np.empty((E,), dtype=np.float32)
    _load().oracle_column_quantiles(_ptr(z), _ptr(a), N, E, int(m), _ptr(v))
    return v


def eqb_bias(v) -> np.ndarray:
    """beta = -v, centred (section 7.1; order of operations from 7.2)."""
    v = _c(v, np.float32)
    out = np.empty_like(v)
    _load().oracle_eqb_bias(_ptr(v), v.shape[0], _ptr(out))
    return out


def radix_select(keys, m: int, radix: int, ndigits: int, chunk_sizes=None):
    """The (m+1)-th largest key by digit-by-digit histograms (section 7.3).

    ``chunk_sizes`` splits ``keys`` into ranks whose histograms are summed.
    Returns (key, histograms [ndigits, radix], chosen bins [ndigits])."""
    keys = _c(keys, np.uint64)
    if chunk_sizes is None:
        chunk_sizes = [keys.shape[0]]
    cs = _c(chunk_sizes, np.int64)
    assert int(cs.sum()) == keys.shape[0] and 0 <= m < keys.shape[0]
    hist = np.zeros((ndigits, radix), dtype=np.int64)
    bins = np.zeros((ndigits,), dtype=np.int64)
    k = _load().oracle_radix_select(_ptr(keys), _ptr(cs), cs.shape[0], int(m), int(radix),
                                    int(ndigits), _ptr(hist), _ptr(bins))
    return int(k), hist, bins


def maxvio(counts, N: int, K: int) -> float:
    """MaxVio = max_e c_e / (K N / E) - 1 (section 6.2)."""
    c = _c(counts, np.int32)
    return float(_load().oracle_maxvio(_ptr(c), c.shape[0], N, K))


def intervention_rate(ids_routed, ids_unbiased) -> float:
    """Mean over tokens of 1 - |I^u_t and I_t| / K (section 9)."""
    a = _c(ids_routed, np.int32)
    b = _c(ids_unbiased, np.int32)
    N, K = a.shape
    return float(_load().oracle_intervention_rate(_ptr(a), _ptr(b), N, K))


def intervention_overlap(ids_routed, ids_unbiased) -> int:
    """Sum over tokens of |I^u_t and I_t| (section 9): the exact count behind
    the intervention rate, 1 - overlap / (N K)."""
    a = _c(ids_routed, np.int32)
    b = _c(ids_unbiased, np.int32)
    N, K = a.shape
    return int(_load().oracle_intervention_overlap(_ptr(a), _ptr(b), N, K))


def eqb_target_rank(N: int, K: int, E: int) -> int:
    """m = floor(N K / E): the reading of r = T K / E (section 7.1)."""
    return (N * K) // E


def order_key_array(v) -> np.ndarray:
    """Vectorised order key (same map as ``order_key``), for test bookkeeping."""
    u = _c(v, np.float32).view(np.uint32)
    neg = (u & np.uint32(0x80000000)) != 0
    return np.where(neg, ~u, u | np.uint32(0x80000000)).astype(np.uint32)


def bf16_round(v: float) -> int:
    """16-bit pattern of the bf16 value nearest to the fp32 value v (ties to even)."""
    return int(_load().oracle_bf16_round(ctypes.c_float(np.float32(v))))


def bf16_key(b: int) -> int:
    """Order-preserving 16-bit key of a bf16 pattern."""
    return int(_load().oracle_bf16_key(ctypes.c_uint16(b)))


def column_quantiles_bf16(z, alpha, m: int) -> np.ndarray:
    """v_e = the (m+1)-th largest of bf16(Z[:,e] + alpha), as float (section 7.3, bf16 keys)."""
    z = _c(z, np.float32)
    N, E = z.shape
    a = None if alpha is None else _c(alpha, np.float32)
    v = np.empty((E,), dtype=np.float32)
    _load().oracle_column_quantiles_bf16(_ptr(z), _ptr(a), N, E, int(m), _ptr(v))
    return v


def tanh_spec(x: float) -> float:
    return float(_load().oracle_tanh_spec(float(x)))


def lei_delta(counts, N: int, K: int, lam: float = 1e-5, tau: float = 1.0) -> np.ndarray:
    """Per-expert Load-Error Injection increment of section 8 (fp32)."""
    c = _c(counts, np.int32)
    out = np.empty((c.shape[0],), dtype=np.float32)
    _load().oracle_lei_delta(_ptr(c), int(N), c.shape[0], int(K), float(lam), float(tau), _ptr(out))
    return out


def lei_inject(counts, g, K: int, lam: float = 1e-5, tau: float = 1.0) -> np.ndarray:
    """G[t, e] + delta_e for every token of the microbatch (section 8)."""
    c = _c(counts, np.int32)
    g = np.array(g, dtype=np.float32, copy=True, order="C")
    N, E = g.shape
    _load().oracle_lei_inject(_ptr(c), N, E, int(K), float(lam), float(tau), _ptr(g))
    return g


def score_grad_to_logits(z, gs) -> np.ndarray:
    """dL/dZ = dL/dS * sigma(Z) (1 - sigma(Z)) (section 8, chain rule)."""
    z = _c(z, np.float32)
    gs = _c(gs, np.float32)
    out = np.empty_like(z)
    _load().oracle_score_grad_to_logits(_ptr(z), _ptr(gs), z.size, _ptr(out))
    return out


def bf16_round_f64(v: float) -> int:
    """bf16 bits of the nearest bf16 to the fp64 value v (one rounding)."""
    return int(_load().oracle_bf16_round_f64(float(v)))


def silu_spec(g: float) -> float:
    """SiLU(g) = g * sigma(g) in fp64 with the gate's exp."""
    return float(_load().oracle_silu_spec(float(g)))


def expert_ffn(x_bf16_bits, ids, gates, wgu_bf16_bits, wd_bf16_bits, wgu_s_bf16_bits=None,
               wd_s_bf16_bits=None, want_h=False):
    """The MoE layer output of section 6.1 with SwiGLU experts.

    x [N,d], wgu [E,2F,d] (gate rows then up rows), wd [E,d,F], optional
    shared expert wgu_s [2F,d], wd_s [d,F] (all bf16 bit patterns, uint16);
    ids [N,K] int32, gates [N,K] fp32.  Returns (y [N,d] fp32, mag [N,d] fp64)
    and, with want_h, also h [N*K,F] (slot order) and h_s [N,F] as uint16."""
    lib = _load()
    x = _c(x_bf16_bits, np.uint16)
    ids = _c(ids, np.int32)
    gates = _c(gates, np.float32)
    wgu = _c(wgu_bf16_bits, np.uint16)
    wd = _c(wd_bf16_bits, np.uint16)
    N, d = x.shape
    K = ids.shape[1]
    E, F2, d2 = wgu.shape
    F = F2 // 2
    assert d2 == d and wd.shape == (E, d, F) and gates.shape == ids.shape
    if wgu_s_bf16_bits is not None:
        wgu_s = _c(wgu_s_bf16_bits, np.uint16)
        wd_s = _c(wd_s_bf16_bits, np.uint16)
        assert wgu_s.shape == (2 * F, d) and wd_s.shape == (d, F)
    else:
        wgu_s = wd_s = None
    y = np.empty((N, d), np.float32)
    mag = np.empty((N, d), np.float64)
    h = np.empty((N * K, F), np.uint16) if want_h else None
    h_s = np.empty((N, F), np.uint16) if (want_h and wgu_s is not None) else None
    lib.oracle_expert_ffn(_ptr(x), _ptr(ids), _ptr(gates), _ptr(wgu), _ptr(wd),
                          None if wgu_s is None else _ptr(wgu_s),
                          None if wd_s is None else _ptr(wd_s), N, d, F, E, K,
                          None if h is None else _ptr(h), None if h_s is None else _ptr(h_s),
                          _ptr(y), _ptr(mag))
    if want_h:
        return y, mag, h, h_s
    return y, mag
