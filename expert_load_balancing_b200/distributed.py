"""EQB over a batch split across ranks ("Kolibri Pre-Training from Scratch"
7.3): each rank histograms its own keys, the 256-bin histograms of all
experts are summed with one all-reduce per pass, and every rank then picks
the same digit, so all ranks end with the same exact quantile and the same
bias.  Two forms: the pages' bf16 keys (two passes,
``eqb_update_bf16_distributed``), and the fp32 keys of the main update (four
passes, ``eqb_update_distributed``; on one rank it equals
kolibri_eqb_update).  The kernels are the library's; torch.distributed (NCCL
on GPUs) carries the sums.

``ops`` replaces the library calls (same signatures) where no GPU is
present, e.g. for a gloo test of the exchange on CPU ranks."""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding as B


class _LibraryOps:
    histogram = staticmethod(B.kolibri_eqb_bf16_histogram)
    digit = staticmethod(B.kolibri_eqb_bf16_digit)
    bias = staticmethod(B.kolibri_eqb_bf16_bias)


class _LibraryKeyOps:
    histogram = staticmethod(B.kolibri_eqb_key_histogram)
    digit = staticmethod(B.kolibri_eqb_key_digit)
    bias = staticmethod(B.kolibri_eqb_key_bias)


def eqb_update_bf16_distributed(z: torch.Tensor, alpha: torch.Tensor | None, bias: torch.Tensor,
                                K: int, n_total: int, group=None, quantiles=None, ops=None):
    """One EQB update of ``bias`` (in place, identical on every rank).

    z [n_local, E] and alpha [n_local] are this rank's tokens; n_total is the
    number of tokens over all ranks (the target rank is floor(n_total K / E)).
    Returns (bias, quantiles)."""
    ops = ops or _LibraryOps
    E = z.shape[1]
    dev = z.device
    hist = torch.zeros((E, 256), dtype=torch.int32, device=dev)
    rank = torch.full((E,), (int(n_total) * int(K)) // E, dtype=torch.int64, device=dev)
    d_hi = torch.empty((E,), dtype=torch.int32, device=dev)
    d_lo = torch.empty((E,), dtype=torch.int32, device=dev)
    if quantiles is None:
        quantiles = torch.empty((E,), dtype=torch.float32, device=dev)
    distributed = dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1
    # pass one: high byte of every key
    ops.histogram(z, alpha, None, hist)
    if distributed:
        dist.all_reduce(hist, op=dist.ReduceOp.SUM, group=group)
    ops.digit(hist, rank, d_hi)
    # pass two: low byte of the keys inside the chosen high bin
    hist.zero_()
    ops.histogram(z, alpha, d_hi, hist)
    if distributed:
        dist.all_reduce(hist, op=dist.ReduceOp.SUM, group=group)
    ops.digit(hist, rank, d_lo)
    ops.bias(d_hi, d_lo, bias, quantiles)
    return bias, quantiles


def eqb_update_distributed(z: torch.Tensor, alpha: torch.Tensor | None, bias: torch.Tensor,
                           K: int, n_total: int, group=None, quantiles=None, ops=None):
    """One EQB update of ``bias`` from the exact fp32 quantile of the union
    (in place, identical on every rank): four passes of 8-bit digits of the
    order key of Z + alpha, one all-reduce of the [E, 256] histogram each.

    z [n_local, E] and alpha [n_local] are this rank's tokens; n_total is the
    number of tokens over all ranks.  Returns (bias, quantiles)."""
    ops = ops or _LibraryKeyOps
    E = z.shape[1]
    dev = z.device
    hist = torch.zeros((E, 256), dtype=torch.int32, device=dev)
    rank = torch.full((E,), (int(n_total) * int(K)) // E, dtype=torch.int64, device=dev)
    prefix = torch.zeros((E,), dtype=torch.int32, device=dev)
    if quantiles is None:
        quantiles = torch.empty((E,), dtype=torch.float32, device=dev)
    distributed = dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1
    for p in range(4):
        if p:
            hist.zero_()
        ops.histogram(z, alpha, p, prefix, hist)
        if distributed:
            dist.all_reduce(hist, op=dist.ReduceOp.SUM, group=group)
        ops.digit(hist, p, rank, prefix)
    ops.bias(prefix, bias, quantiles)
    return bias, quantiles
