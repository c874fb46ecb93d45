"""ctypes binding of ``libkolibri_router.so`` (include/kolibri_router.h).

Argument marshalling only: every step of the routing path runs in the
library's CUDA kernels.  PyTorch supplies device memory and the current
stream.  The library must have been built (``python -m
expert_load_balancing_b200.build``); loading fails loudly otherwise, and
there is no CPU fallback.

The library launches on the current CUDA device: the tensors of a call must
live on it (inside ``torch.cuda.device(t.device)`` when several GPUs are in
use).  The wrappers check dtype, shape, contiguity and that tensors are on a
GPU, not which one, to keep the per-call host cost of small batches low.
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
# size of the library-held scratch of kolibri_expert_permute_noalloc (the header's macro)
KOLIBRI_NOALLOC_SCRATCH_BYTES = 2 << 20

# every symbol the header declares, with (restype, argtypes)
_P, _I64, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
SIGNATURES = {
    "kolibri_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "kolibri_workspace_bytes": (_SZ, [ctypes.c_int, _I64, _I32, _I32]),
    "kolibri_router_logits": (ctypes.c_int, [_P, _P, _P, _I64, _I32, _I32, _P]),
    "kolibri_router_forward": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I32, _I32, _I32, _P, _P, _P, _P]),
    "kolibri_router_forward_permute": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I32, _I32, _I32, _P, _P,
                                                      _P, _P, _P, _P, _P, _P, _SZ, _P]),
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
    "kolibri_eqb_key_histogram": (ctypes.c_int, [_P, _P, _I64, _I32, _I32, _P, _P, _P]),
    "kolibri_eqb_key_digit": (ctypes.c_int, [_P, _I32, _I32, _P, _P, _P]),
    "kolibri_eqb_key_bias": (ctypes.c_int, [_P, _I32, _P, _P, _P]),
    "kolibri_eqb_split_sample": (ctypes.c_int, [_P, _P, _I64, _I32, _I32, _I64, _P, _P]),
    "kolibri_eqb_split_brackets": (ctypes.c_int, [_P, _I32, _I64, _I32, _I64, _I32, _P, _P, _P, _P]),
    "kolibri_eqb_split_count": (ctypes.c_int, [_P, _P, _I64, _I32, _I32, _P, _P, _P, _P, _I64, _P]),
    "kolibri_eqb_split_rank": (ctypes.c_int, [_P, _I32, _I64, _I32, _P, _P, _P]),
    "kolibri_eqb_split_histogram": (ctypes.c_int, [_P, _P, _I64, _I32, _I32, _P, _P, _P]),
    "kolibri_expert_ffn_workspace_size": (_SZ, [_I64, _I32, _I32, _I32, _I32]),
    "kolibri_expert_ffn": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I32, _I32,
                                          _I32, _I32, _P, _SZ, _P]),
    "kolibri_expert_dispatch": (ctypes.c_int, [_P, _P, _I64, _I32, _I32, _P, _P]),
    "kolibri_expert_gate_up": (ctypes.c_int, [_P, _I64, _P, _I32, _P, _P, _I32, _I32, _P]),
    "kolibri_expert_down": (ctypes.c_int, [_P, _I64, _P, _I32, _P, _P, _I32, _I32, _P]),
    "kolibri_expert_combine": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I32, _I32, _P, _P]),
    "kolibri_device_status": (ctypes.c_int, [_P]),
    "kolibri_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_uint64, _P]),
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
    """A zero-filled device buffer large enough for ``op`` (uint8, 256-byte
    aligned).  Zero-filled because the decode form of
    kolibri_router_forward_permute keeps a counter in it that must start at
    zero; the calls leave it zero, so the buffer can be reused."""
    n = max(kolibri_workspace_bytes(op, N, E, K), 1)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


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


def kolibri_router_forward_permute(x: torch.Tensor, w: torch.Tensor, bias: torch.Tensor | None, K: int,
                                   z=None, ids=None, gates=None, alpha=None, counts=None, offsets=None,
                                   perm=None, inv=None, ws: torch.Tensor | None = None, want_inv: bool = True,
                                   stream=None):
    """The forward and the permutation of its ids in one call (one launch for
    decode batches of at most 16 tokens).  Returns (z, ids, gates, alpha,
    counts, offsets, perm, inv)."""
    N, d = x.shape
    E = w.shape[0]
    _need(x, torch.bfloat16, (N, d), "x")
    _need(w, torch.bfloat16, (E, d), "w")
    dev = x.device
    z = torch.empty((N, E), dtype=torch.float32, device=dev) if z is None else z
    ids = torch.empty((N, K), dtype=torch.int32, device=dev) if ids is None else ids
    gates = torch.empty((N, K), dtype=torch.float32, device=dev) if gates is None else gates
    alpha = torch.empty((N,), dtype=torch.float32, device=dev) if alpha is None else alpha
    counts = torch.empty((E,), dtype=torch.int32, device=dev) if counts is None else counts
    offsets = torch.empty((E + 1,), dtype=torch.int64, device=dev) if offsets is None else offsets
    perm = torch.empty((N * K,), dtype=torch.int32, device=dev) if perm is None else perm
    if inv is None and want_inv:
        inv = torch.empty((N * K,), dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace(KOLIBRI_OP_PERMUTE, N, E, K, dev)
    _check("kolibri_router_forward_permute",
           load().kolibri_router_forward_permute(
               _ptr(x), _ptr(w), _ptr(bias), _ptr(z), N, d, E, K, _ptr(ids), _ptr(gates), _ptr(alpha),
               _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv), _ptr(ws), ws.numel(), _stream(stream)))
    return z, ids, gates, alpha, counts, offsets, perm, inv


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


def kolibri_selftest_bounded_wait(limit_ns: int = 1_000_000, stream=None) -> None:
    """Enqueue a wait that runs out after about limit_ns; the next
    kolibri_device_status on that stream reports KOLIBRI_ERR_TIMEOUT."""
    _check("kolibri_selftest_bounded_wait", load().kolibri_selftest_bounded_wait(int(limit_ns), _stream(stream)))


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


def kolibri_eqb_key_histogram(z, alpha, pass_, prefix, hist, stream=None):
    """Add this rank's fp32-key histogram of digit pass pass_ (0..3) into hist [E, 256] uint32."""
    N, E = z.shape
    _check("kolibri_eqb_key_histogram",
           load().kolibri_eqb_key_histogram(_ptr(z), _ptr(alpha), N, E, int(pass_), _ptr(prefix),
                                            _ptr(hist), _stream(stream)))
    return hist


def kolibri_eqb_key_digit(hist, pass_, rank, prefix, stream=None):
    E = hist.shape[0]
    _check("kolibri_eqb_key_digit",
           load().kolibri_eqb_key_digit(_ptr(hist), E, int(pass_), _ptr(rank), _ptr(prefix),
                                        _stream(stream)))
    return prefix


def kolibri_eqb_key_bias(key, bias, quantiles, stream=None):
    E = bias.shape[0]
    _check("kolibri_eqb_key_bias",
           load().kolibri_eqb_key_bias(_ptr(key), E, _ptr(bias), _ptr(quantiles), _stream(stream)))
    return bias, quantiles


def kolibri_eqb_split_sample(z, alpha, K, S, sample, stream=None):
    """Keys of this rank's z + alpha at S strided rows into sample [E, S] uint32."""
    N, E = z.shape
    _check("kolibri_eqb_split_sample",
           load().kolibri_eqb_split_sample(_ptr(z), _ptr(alpha), N, E, int(K), int(S), _ptr(sample),
                                           _stream(stream)))
    return sample


def kolibri_eqb_split_brackets(sample, n_total, K, scratch, lo, hi, stream=None):
    """Brackets lo, hi [E] uint32 from the gathered samples [R, E, S];
    scratch [E, ld] uint32 with ld = R S rounded up to a multiple of 4."""
    R, E, S = sample.shape
    ld = (R * S + 3) // 4 * 4
    _need(scratch, scratch.dtype, (E, ld), "scratch")
    _check("kolibri_eqb_split_brackets",
           load().kolibri_eqb_split_brackets(_ptr(sample), R, S, E, int(n_total), int(K),
                                             _ptr(scratch), _ptr(lo), _ptr(hi), _stream(stream)))
    return lo, hi


def kolibri_eqb_split_count(z, alpha, K, lo, hi, counts, cand, stream=None):
    """One pass over this rank's z + alpha: counts [3, E] uint32, cand [E, cap] uint32."""
    N, E = z.shape
    cap = cand.shape[1]
    _check("kolibri_eqb_split_count",
           load().kolibri_eqb_split_count(_ptr(z), _ptr(alpha), N, E, int(K), _ptr(lo), _ptr(hi),
                                          _ptr(counts), _ptr(cand), cap, _stream(stream)))
    return counts, cand


def kolibri_eqb_split_rank(counts_sum, n_total, K, rank, flag, stream=None):
    """rank [E] int64 and flag [E] uint32 from the counts summed over ranks."""
    E = counts_sum.shape[1]
    _check("kolibri_eqb_split_rank",
           load().kolibri_eqb_split_rank(_ptr(counts_sum), E, int(n_total), int(K), _ptr(rank),
                                         _ptr(flag), _stream(stream)))
    return rank, flag


def kolibri_eqb_split_histogram(cand, counts, pass_, prefix, hist, stream=None):
    """Add this rank's histogram of its bracketed keys, digit pass pass_, into hist [E, 256]."""
    E, cap = cand.shape
    _check("kolibri_eqb_split_histogram",
           load().kolibri_eqb_split_histogram(_ptr(cand), _ptr(counts), cap, E, int(pass_),
                                              _ptr(prefix), _ptr(hist), _stream(stream)))
    return hist


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


# ---------------------------------------------------------------- the experts

def expert_ffn_workspace(N: int, d: int, F: int, K: int, shared: bool, device=None) -> torch.Tensor:
    """Device workspace for kolibri_expert_ffn."""
    n = int(load().kolibri_expert_ffn_workspace_size(N, d, F, K, 1 if shared else 0))
    return torch.empty((max(n, 1),), dtype=torch.uint8, device=device or "cuda")


def kolibri_expert_ffn(x: torch.Tensor, perm: torch.Tensor, offsets: torch.Tensor, inv: torch.Tensor,
                       gates: torch.Tensor, w_gate_up: torch.Tensor, w_down: torch.Tensor,
                       ws_gate_up: torch.Tensor | None = None, ws_down: torch.Tensor | None = None,
                       y: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """y [N, d] fp32 = shared expert + sum_k gates[t,k] expert_{ids[t,k]}(x_t) (SwiGLU experts)."""
    N, d = x.shape
    K = gates.shape[1]
    E, F2, _ = w_gate_up.shape
    F = F2 // 2
    _need(x, torch.bfloat16, (N, d), "x")
    _need(perm, torch.int32, (N * K,), "perm")
    _need(offsets, torch.int64, (E + 1,), "offsets")
    _need(inv, torch.int32, (N * K,), "inv")
    _need(gates, torch.float32, (N, K), "gates")
    _need(w_gate_up, torch.bfloat16, (E, 2 * F, d), "w_gate_up")
    _need(w_down, torch.bfloat16, (E, d, F), "w_down")
    if ws_gate_up is not None:
        _need(ws_gate_up, torch.bfloat16, (2 * F, d), "ws_gate_up")
        _need(ws_down, torch.bfloat16, (d, F), "ws_down")
    if y is None:
        y = torch.empty((N, d), dtype=torch.float32, device=x.device)
    _need(y, torch.float32, (N, d), "y")
    if ws is None:
        ws = expert_ffn_workspace(N, d, F, K, ws_gate_up is not None, x.device)
    _check("kolibri_expert_ffn",
           load().kolibri_expert_ffn(_ptr(x), _ptr(perm), _ptr(offsets), _ptr(inv), _ptr(gates),
                                     _ptr(w_gate_up), _ptr(w_down), _ptr(ws_gate_up), _ptr(ws_down),
                                     _ptr(y), N, d, F, E, K, _ptr(ws), ws.numel(), _stream(stream)))
    return y


def kolibri_expert_dispatch(x: torch.Tensor, perm: torch.Tensor, K: int,
                            x_perm: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """x_perm [N*K, d] with x_perm[p] = x[perm[p] // K]."""
    N, d = x.shape
    _need(x, torch.bfloat16, (N, d), "x")
    _need(perm, torch.int32, (N * K,), "perm")
    if x_perm is None:
        x_perm = torch.empty((N * K, d), dtype=torch.bfloat16, device=x.device)
    _need(x_perm, torch.bfloat16, (N * K, d), "x_perm")
    _check("kolibri_expert_dispatch",
           load().kolibri_expert_dispatch(_ptr(x), _ptr(perm), N, d, K, _ptr(x_perm), _stream(stream)))
    return x_perm


def kolibri_expert_gate_up(a: torch.Tensor, offsets: torch.Tensor | None, w_gate_up: torch.Tensor,
                           h: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """h [rows, F] bf16 = bf16(SiLU(a Wg^T) * (a Wu^T)), expert g on rows [offsets[g], offsets[g+1])."""
    rows, d = a.shape
    if w_gate_up.dim() == 2:
        w_gate_up = w_gate_up.unsqueeze(0)
    G, F2, _ = w_gate_up.shape
    F = F2 // 2
    _need(a, torch.bfloat16, (rows, d), "a")
    _need(w_gate_up, torch.bfloat16, (G, 2 * F, d), "w_gate_up")
    if offsets is not None:
        _need(offsets, torch.int64, (G + 1,), "offsets")
    if h is None:
        h = torch.empty((rows, F), dtype=torch.bfloat16, device=a.device)
    _need(h, torch.bfloat16, (rows, F), "h")
    _check("kolibri_expert_gate_up",
           load().kolibri_expert_gate_up(_ptr(a), rows, _ptr(offsets), G, _ptr(w_gate_up), _ptr(h),
                                         d, F, _stream(stream)))
    return h


def kolibri_expert_down(h: torch.Tensor, offsets: torch.Tensor | None, w_down: torch.Tensor,
                        y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y [rows, d] fp32 = h Wd_g^T per group."""
    rows, F = h.shape
    if w_down.dim() == 2:
        w_down = w_down.unsqueeze(0)
    G, d, _ = w_down.shape
    _need(h, torch.bfloat16, (rows, F), "h")
    _need(w_down, torch.bfloat16, (G, d, F), "w_down")
    if offsets is not None:
        _need(offsets, torch.int64, (G + 1,), "offsets")
    if y is None:
        y = torch.empty((rows, d), dtype=torch.float32, device=h.device)
    _need(y, torch.float32, (rows, d), "y")
    _check("kolibri_expert_down",
           load().kolibri_expert_down(_ptr(h), rows, _ptr(offsets), G, _ptr(w_down), _ptr(y), d, F,
                                      _stream(stream)))
    return y


def kolibri_expert_combine(y_perm: torch.Tensor, y_shared: torch.Tensor | None, inv: torch.Tensor,
                           gates: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y [N, d] = y_shared + sum_k gates[t,k] y_perm[inv[t*K+k]] (fp32, k ascending)."""
    N, K = gates.shape
    d = y_perm.shape[1]
    _need(y_perm, torch.float32, (N * K, d), "y_perm")
    if y_shared is not None:
        _need(y_shared, torch.float32, (N, d), "y_shared")
    _need(inv, torch.int32, (N * K,), "inv")
    _need(gates, torch.float32, (N, K), "gates")
    if y is None:
        y = torch.empty((N, d), dtype=torch.float32, device=y_perm.device)
    _need(y, torch.float32, (N, d), "y")
    _check("kolibri_expert_combine",
           load().kolibri_expert_combine(_ptr(y_perm), _ptr(y_shared), _ptr(inv), _ptr(gates), N, d, K,
                                         _ptr(y), _stream(stream)))
    return y
