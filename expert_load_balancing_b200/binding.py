"""ctypes binding of ``libkolibri_router.so`` (include/kolibri_router.h).

Argument marshalling only: every step of the routing path runs in the
library's CUDA kernels.  PyTorch supplies device memory and the current
stream.  The library must have been built (``python -m
expert_load_balancing_b200.build``); loading fails loudly otherwise, and
there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkolibri_router.so")

KOLIBRI_OK = 0
KOLIBRI_ERR_INVALID_ARG = 1
KOLIBRI_ERR_UNSUPPORTED_SHAPE = 2
KOLIBRI_ERR_WORKSPACE_TOO_SMALL = 3
KOLIBRI_ERR_CUDA = 4
KOLIBRI_ERR_TIMEOUT = 5
KOLIBRI_ERR_DEVICE = 6
KOLIBRI_OP_PERMUTE = 1
KOLIBRI_OP_EQB = 2
KOLIBRI_OP_EQB_BF16 = 3

# every symbol the header declares, with (restype, argtypes)
_P, _I64, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
SIGNATURES = {
    "kolibri_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "kolibri_workspace_bytes": (_SZ, [ctypes.c_int, _I64, _I32, _I32]),
    "kolibri_router_logits": (ctypes.c_int, [_P, _P, _P, _I64, _I32, _I32, _P]),
    "kolibri_router_forward": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I32, _I32, _I32, _P, _P, _P, _P]),
    "kolibri_router_forward_eqb": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I32, _I32, _I32, _P, _P,
                                                  _P, _P, _P, _SZ, _P]),
    "kolibri_router_topk": (ctypes.c_int, [_P, _P, _I64, _I32, _I32, _P, _P, _P, _P]),
    "kolibri_eqb_update_bf16": (ctypes.c_int, [_P, _P, _P, _I64, _I32, _I32, _P, _P, _SZ, _P]),
    "kolibri_eqb_bf16_histogram": (ctypes.c_int, [_P, _P, _I64, _I32, _P, _P, _P]),
    "kolibri_eqb_bf16_digit": (ctypes.c_int, [_P, _I32, _P, _P, _P]),
    "kolibri_eqb_bf16_bias": (ctypes.c_int, [_P, _P, _I32, _P, _P, _P]),
    "kolibri_lei_inject": (ctypes.c_int, [_P, _I64, _I32, _I32, ctypes.c_double, ctypes.c_double, _P, _P]),
    "kolibri_score_grad_to_logits": (ctypes.c_int, [_P, _P, _I64, _P, _P]),
    "kolibri_intervention_rate": (ctypes.c_int, [_P, _P, _I64, _I32, _I32, _P, _P, _P]),
    "kolibri_expert_permute": (ctypes.c_int, [_P, _I64, _I32, _I32, _P, _P, _P, _P, _P, _SZ, _P]),
    "kolibri_expert_permute_noalloc": (ctypes.c_int, [_P, _I64, _I32, _I32, _P, _P, _P, _P, _P]),
    "kolibri_eqb_update": (ctypes.c_int, [_P, _P, _P, _I64, _I32, _I32, _P, _P, _SZ, _P]),
    "kolibri_route_and_balance": (ctypes.c_int, [_P, _P, _I64, _I32, _I32, _P, _P, _P, _P, _P,
                                                 _SZ, _P]),
    "kolibri_device_status": (ctypes.c_int, [_P]),
}


class KolibriError(RuntimeError):
    def __init__(self, call: str, status: int):
        self.status = status
        super().__init__(f"{call} failed: {status_string(status)} ({status})")


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once) and declare every entry point."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m expert_load_balancing_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().kolibri_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(name, st):
    if st != KOLIBRI_OK:
        raise KolibriError(name, st)


def _need(t, dtype, shape, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


def kolibri_workspace_bytes(op: int, N: int, E: int, K: int) -> int:
    return int(load().kolibri_workspace_bytes(op, N, E, K))


def workspace(op: int, N: int, E: int, K: int, device=None) -> torch.Tensor:
    """A device buffer large enough for ``op`` (uint8, 256-byte aligned)."""
    n = max(kolibri_workspace_bytes(op, N, E, K), 1)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def kolibri_router_logits(x: torch.Tensor, w: torch.Tensor, z: torch.Tensor | None = None,
                          stream=None) -> torch.Tensor:
    """Z = x W^T: x [N,d] bf16, w [E,d] bf16 -> z [N,E] fp32."""
    N, d = x.shape
    E = w.shape[0]
    _need(x, torch.bfloat16, (N, d), "x")
    _need(w, torch.bfloat16, (E, d), "w")
    if z is None:
        z = torch.empty((N, E), dtype=torch.float32, device=x.device)
    _need(z, torch.float32, (N, E), "z")
    _check("kolibri_router_logits",
           load().kolibri_router_logits(_ptr(x), _ptr(w), _ptr(z), N, d, E, _stream(stream)))
    return z


def kolibri_router_forward(x: torch.Tensor, w: torch.Tensor, bias: torch.Tensor | None, K: int,
                           z: torch.Tensor | None = None, ids: torch.Tensor | None = None,
                           gates: torch.Tensor | None = None, alpha: torch.Tensor | None = None,
                           stream=None):
    """Logits and selection in one call (the GEMM epilogue selects).

    Returns (z [N,E] fp32, ids [N,K] int32, gates [N,K] fp32, alpha [N] fp32)."""
    N, d = x.shape
    E = w.shape[0]
    _need(x, torch.bfloat16, (N, d), "x")
    _need(w, torch.bfloat16, (E, d), "w")
    if bias is not None:
        _need(bias, torch.float32, (E,), "bias")
    dev = x.device
    z = torch.empty((N, E), dtype=torch.float32, device=dev) if z is None else z
    ids = torch.empty((N, K), dtype=torch.int32, device=dev) if ids is None else ids
    gates = torch.empty((N, K), dtype=torch.float32, device=dev) if gates is None else gates
    alpha = torch.empty((N,), dtype=torch.float32, device=dev) if alpha is None else alpha
    _need(z, torch.float32, (N, E), "z")
    _need(ids, torch.int32, (N, K), "ids")
    _need(gates, torch.float32, (N, K), "gates")
    _need(alpha, torch.float32, (N,), "alpha")
    _check("kolibri_router_forward",
           load().kolibri_router_forward(_ptr(x), _ptr(w), _ptr(bias), _ptr(z), N, d, E, K,
                                         _ptr(ids), _ptr(gates), _ptr(alpha), _stream(stream)))
    return z, ids, gates, alpha


def kolibri_router_forward_eqb(x: torch.Tensor, w: torch.Tensor, bias: torch.Tensor, K: int,
                               ws: torch.Tensor | None = None, z: torch.Tensor | None = None,
                               ids: torch.Tensor | None = None, gates: torch.Tensor | None = None,
                               alpha: torch.Tensor | None = None,
                               quantiles: torch.Tensor | None = None, stream=None):
    """Logits, routing with ``bias`` and the EQB update of ``bias`` in place.

    Returns (z, ids, gates, alpha, quantiles)."""
    N, d = x.shape
    E = w.shape[0]
    _need(x, torch.bfloat16, (N, d), "x")
    _need(w, torch.bfloat16, (E, d), "w")
    _need(bias, torch.float32, (E,), "bias")
    dev = x.device
    if ws is None:
        ws = workspace(KOLIBRI_OP_EQB, N, E, K, dev)
    z = torch.empty((N, E), dtype=torch.float32, device=dev) if z is None else z
    ids = torch.empty((N, K), dtype=torch.int32, device=dev) if ids is None else ids
    gates = torch.empty((N, K), dtype=torch.float32, device=dev) if gates is None else gates
    alpha = torch.empty((N,), dtype=torch.float32, device=dev) if alpha is None else alpha
    quantiles = torch.empty((E,), dtype=torch.float32, device=dev) if quantiles is None else quantiles
    _need(z, torch.float32, (N, E), "z")
    _need(ids, torch.int32, (N, K), "ids")
    _need(gates, torch.float32, (N, K), "gates")
    _need(alpha, torch.float32, (N,), "alpha")
    _need(quantiles, torch.float32, (E,), "quantiles")
    _check("kolibri_router_forward_eqb",
           load().kolibri_router_forward_eqb(_ptr(x), _ptr(w), _ptr(bias), _ptr(z), N, d, E, K,
                                             _ptr(ids), _ptr(gates), _ptr(alpha), _ptr(quantiles),
                                             _ptr(ws), ws.numel(), _stream(stream)))
    return z, ids, gates, alpha, quantiles


def kolibri_router_topk(z: torch.Tensor, bias: torch.Tensor | None, K: int,
                        ids: torch.Tensor | None = None, gates: torch.Tensor | None = None,
                        alpha: torch.Tensor | None = None, want_alpha: bool = True, stream=None):
    """Bias add, top-K ids, sigmoid gates and token bias.

    Returns (ids [N,K] int32, gates [N,K] fp32, alpha [N] fp32 or None)."""
    N, E = z.shape
    _need(z, torch.float32, (N, E), "z")
    if bias is not None:
        _need(bias, torch.float32, (E,), "bias")
    if ids is None:
        ids = torch.empty((N, K), dtype=torch.int32, device=z.device)
    if gates is None:
        gates = torch.empty((N, K), dtype=torch.float32, device=z.device)
    if alpha is None and want_alpha:
        alpha = torch.empty((N,), dtype=torch.float32, device=z.device)
    _need(ids, torch.int32, (N, K), "ids")
    _need(gates, torch.float32, (N, K), "gates")
    if alpha is not None:
        _need(alpha, torch.float32, (N,), "alpha")
    _check("kolibri_router_topk",
           load().kolibri_router_topk(_ptr(z), _ptr(bias), N, E, K, _ptr(ids), _ptr(gates),
                                      _ptr(alpha), _stream(stream)))
    return ids, gates, alpha


def kolibri_expert_permute(ids: torch.Tensor, E: int, ws: torch.Tensor | None = None,
                           counts=None, offsets=None, perm=None, inv=None, want_inv: bool = True,
                           stream=None):
    """Expert loads and stable grouping of slots.

    Returns (counts [E] int32, offsets [E+1] int64, perm [N*K] int32, inv [N*K] int32 or None)."""
    N, K = ids.shape
    _need(ids, torch.int32, (N, K), "ids")
    dev = ids.device
    if ws is None:
        ws = workspace(KOLIBRI_OP_PERMUTE, N, E, K, dev)
    if counts is None:
        counts = torch.empty((E,), dtype=torch.int32, device=dev)
    if offsets is None:
        offsets = torch.empty((E + 1,), dtype=torch.int64, device=dev)
    if perm is None:
        perm = torch.empty((N * K,), dtype=torch.int32, device=dev)
    if inv is None and want_inv:
        inv = torch.empty((N * K,), dtype=torch.int32, device=dev)
    _check("kolibri_expert_permute",
           load().kolibri_expert_permute(_ptr(ids), N, E, K, _ptr(counts), _ptr(offsets),
                                         _ptr(perm), _ptr(inv), _ptr(ws), ws.numel(),
                                         _stream(stream)))
    return counts, offsets, perm, inv


def kolibri_expert_permute_noalloc(ids: torch.Tensor, E: int, counts=None, offsets=None,
                                   perm=None, inv=None, want_inv: bool = True, stream=None):
    """kolibri_expert_permute without a workspace (library-held scratch).

    For callers that cannot allocate device memory; see the header for the
    size limit and the rule that calls must not overlap on the GPU."""
    N, K = ids.shape
    _need(ids, torch.int32, (N, K), "ids")
    dev = ids.device
    if counts is None:
        counts = torch.empty((E,), dtype=torch.int32, device=dev)
    if offsets is None:
        offsets = torch.empty((E + 1,), dtype=torch.int64, device=dev)
    if perm is None:
        perm = torch.empty((N * K,), dtype=torch.int32, device=dev)
    if inv is None and want_inv:
        inv = torch.empty((N * K,), dtype=torch.int32, device=dev)
    _check("kolibri_expert_permute_noalloc",
           load().kolibri_expert_permute_noalloc(_ptr(ids), N, E, K, _ptr(counts), _ptr(offsets),
                                                 _ptr(perm), _ptr(inv), _stream(stream)))
    return counts, offsets, perm, inv


def kolibri_eqb_update(z: torch.Tensor, alpha: torch.Tensor | None, bias: torch.Tensor, K: int,
                       ws: torch.Tensor | None = None, quantiles: torch.Tensor | None = None,
                       want_quantiles: bool = True, stream=None):
    """Exact Quantile Balancing update, in place on ``bias``.

    Returns (bias, quantiles or None)."""
    N, E = z.shape
    _need(z, torch.float32, (N, E), "z")
    _need(bias, torch.float32, (E,), "bias")
    if alpha is not None:
        _need(alpha, torch.float32, (N,), "alpha")
    if ws is None:
        ws = workspace(KOLIBRI_OP_EQB, N, E, K, z.device)
    if quantiles is None and want_quantiles:
        quantiles = torch.empty((E,), dtype=torch.float32, device=z.device)
    _check("kolibri_eqb_update",
           load().kolibri_eqb_update(_ptr(z), _ptr(alpha), _ptr(bias), N, E, K, _ptr(quantiles),
                                     _ptr(ws), ws.numel(), _stream(stream)))
    return bias, quantiles


def kolibri_route_and_balance(z: torch.Tensor, bias: torch.Tensor, K: int,
                              ws: torch.Tensor | None = None, ids=None, gates=None, alpha=None,
                              quantiles=None, want_alpha: bool = True,
                              want_quantiles: bool = True, stream=None):
    """Routing with ``bias`` then the EQB update of ``bias`` in place.

    Returns (ids [N,K] int32, gates [N,K] fp32, alpha [N] or None, quantiles [E] or None)."""
    N, E = z.shape
    _need(z, torch.float32, (N, E), "z")
    _need(bias, torch.float32, (E,), "bias")
    dev = z.device
    if ws is None:
        ws = workspace(KOLIBRI_OP_EQB, N, E, K, dev)
    if ids is None:
        ids = torch.empty((N, K), dtype=torch.int32, device=dev)
    if gates is None:
        gates = torch.empty((N, K), dtype=torch.float32, device=dev)
    if alpha is None and want_alpha:
        alpha = torch.empty((N,), dtype=torch.float32, device=dev)
    if quantiles is None and want_quantiles:
        quantiles = torch.empty((E,), dtype=torch.float32, device=dev)
    _need(ids, torch.int32, (N, K), "ids")
    _need(gates, torch.float32, (N, K), "gates")
    _check("kolibri_route_and_balance",
           load().kolibri_route_and_balance(_ptr(z), _ptr(bias), N, E, K, _ptr(ids), _ptr(gates),
                                            _ptr(alpha), _ptr(quantiles), _ptr(ws), ws.numel(),
                                            _stream(stream)))
    return ids, gates, alpha, quantiles


def kolibri_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(load().kolibri_device_status(_stream(stream)))


# ------------------------------------------------ bf16-key EQB, LEI, intervention

def kolibri_eqb_update_bf16(z: torch.Tensor, alpha: torch.Tensor | None, bias: torch.Tensor, K: int,
                            quantiles: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                            stream=None):
    """EQB with bf16 keys (two 256-bin radix passes), in place on ``bias``.

    Returns (bias, quantiles)."""
    N, E = z.shape
    _need(z, torch.float32, (N, E), "z")
    _need(bias, torch.float32, (E,), "bias")
    if alpha is not None:
        _need(alpha, torch.float32, (N,), "alpha")
    if ws is None:
        ws = workspace(KOLIBRI_OP_EQB_BF16, N, E, K, z.device)
    if quantiles is None:
        quantiles = torch.empty((E,), dtype=torch.float32, device=z.device)
    _check("kolibri_eqb_update_bf16",
           load().kolibri_eqb_update_bf16(_ptr(z), _ptr(alpha), _ptr(bias), N, E, K, _ptr(quantiles),
                                          _ptr(ws), ws.numel(), _stream(stream)))
    return bias, quantiles


def kolibri_eqb_bf16_histogram(z, alpha, prefix, hist, stream=None):
    """Add this rank's bf16-key histogram (pass one: prefix None) into hist [E, 256] uint32."""
    N, E = z.shape
    _check("kolibri_eqb_bf16_histogram",
           load().kolibri_eqb_bf16_histogram(_ptr(z), _ptr(alpha), N, E, _ptr(prefix), _ptr(hist),
                                             _stream(stream)))
    return hist


def kolibri_eqb_bf16_digit(hist, rank, digit, stream=None):
    E = hist.shape[0]
    _check("kolibri_eqb_bf16_digit",
           load().kolibri_eqb_bf16_digit(_ptr(hist), E, _ptr(rank), _ptr(digit), _stream(stream)))
    return digit


def kolibri_eqb_bf16_bias(d_hi, d_lo, bias, quantiles, stream=None):
    E = bias.shape[0]
    _check("kolibri_eqb_bf16_bias",
           load().kolibri_eqb_bf16_bias(_ptr(d_hi), _ptr(d_lo), E, _ptr(bias), _ptr(quantiles),
                                        _stream(stream)))
    return bias, quantiles


def kolibri_lei_inject(counts: torch.Tensor, g: torch.Tensor, K: int, lam: float = 1e-5,
                       tau: float = 1.0, stream=None) -> torch.Tensor:
    """Load-Error Injection on the score gradient g [N, E] (in place)."""
    N, E = g.shape
    _need(g, torch.float32, (N, E), "g")
    _need(counts, torch.int32, (E,), "counts")
    _check("kolibri_lei_inject",
           load().kolibri_lei_inject(_ptr(counts), N, E, K, float(lam), float(tau), _ptr(g),
                                     _stream(stream)))
    return g


def kolibri_score_grad_to_logits(z: torch.Tensor, gs: torch.Tensor, gz: torch.Tensor | None = None,
                                 stream=None) -> torch.Tensor:
    """dL/dZ = dL/dS * sigma(Z) (1 - sigma(Z))."""
    _need(z, torch.float32, tuple(z.shape), "z")
    _need(gs, torch.float32, tuple(z.shape), "gs")
    if gz is None:
        gz = torch.empty_like(z)
    _check("kolibri_score_grad_to_logits",
           load().kolibri_score_grad_to_logits(_ptr(z), _ptr(gs), z.numel(), _ptr(gz), _stream(stream)))
    return gz


def kolibri_intervention_rate(z: torch.Tensor, ids: torch.Tensor, stream=None):
    """(rate [1] float64, overlaps [1] int64 as uint64 bits) on the device."""
    N, E = z.shape
    K = ids.shape[1]
    _need(z, torch.float32, (N, E), "z")
    _need(ids, torch.int32, (N, K), "ids")
    rate = torch.empty((1,), dtype=torch.float64, device=z.device)
    overlaps = torch.empty((1,), dtype=torch.int64, device=z.device)
    _check("kolibri_intervention_rate",
           load().kolibri_intervention_rate(_ptr(z), _ptr(ids), N, E, K, _ptr(rate), _ptr(overlaps),
                                            _stream(stream)))
    return rate, overlaps
