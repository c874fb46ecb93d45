"""EQB over a batch split across ranks ("Kolibri Pre-Training from Scratch"
7.3): each rank holds its own tokens, only counts cross ranks, and every rank
ends with the same exact quantile of the union and the same bias.  Three
forms, all built from the library's kernels, with torch.distributed carrying
the exchange:

* ``eqb_update_split``: the one-GPU design of kolibri_eqb_update (a sample
  brackets the target, one full pass gathers the keys inside the bracket,
  radix selection over those) with the pages' exchange between its steps:
  one all-gather of the samples, one all-reduce of 3 E counts, four
  all-reduces of the [E, 256] histograms of the gathered keys.  Z is read
  once per rank.  If the sample misleads (the target falls outside the
  bracket on the union), it finishes with the four-pass form.
* ``eqb_update_distributed``: four passes of 8-bit digits of the fp32 order
  key over Z, one all-reduce of the [E, 256] histogram each (Z read four
  times per rank).
* ``eqb_update_bf16_distributed``: the pages' bf16 keys, two passes.

On one rank each equals the one-call update bit for bit.  ``ops`` replaces
the library calls (same signatures) where no GPU is present, e.g. for a gloo
test of the exchange on CPU ranks; ``comm`` chooses how tensors cross ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import binding as B

SAMPLE_ROWS = 16384      # sample rows over all ranks, as one GPU's update takes
CAND_CAP = 65536         # bracketed keys a rank gathers per expert


class _LibraryOps:
    histogram = staticmethod(B.kolibri_eqb_bf16_histogram)
    digit = staticmethod(B.kolibri_eqb_bf16_digit)
    bias = staticmethod(B.kolibri_eqb_bf16_bias)


class _LibraryKeyOps:
    histogram = staticmethod(B.kolibri_eqb_key_histogram)
    digit = staticmethod(B.kolibri_eqb_key_digit)
    bias = staticmethod(B.kolibri_eqb_key_bias)


class _LibrarySplitOps:
    sample = staticmethod(B.kolibri_eqb_split_sample)
    brackets = staticmethod(B.kolibri_eqb_split_brackets)
    count = staticmethod(B.kolibri_eqb_split_count)
    rank = staticmethod(B.kolibri_eqb_split_rank)
    histogram = staticmethod(B.kolibri_eqb_split_histogram)
    digit = staticmethod(B.kolibri_eqb_key_digit)
    bias = staticmethod(B.kolibri_eqb_key_bias)


class DeviceComm:
    """Collectives on the tensors where they live (NCCL for GPU tensors, gloo
    for CPU tensors).  One rank, or no process group: nothing crosses."""

    def __init__(self, group=None):
        self.group = group

    def world(self) -> int:
        if not (dist.is_available() and dist.is_initialized()):
            return 1
        return dist.get_world_size(self.group)

    def all_reduce(self, t: torch.Tensor, op=None):
        if self.world() > 1:
            dist.all_reduce(t, op=op or dist.ReduceOp.SUM, group=self.group)
        return t

    def all_gather(self, out: torch.Tensor, t: torch.Tensor):
        """out [R, *t.shape] = every rank's t, rank-major."""
        if self.world() > 1:
            # concatenated along dim 0: rank r's t is rows [r n, (r+1) n)
            dist.all_gather_into_tensor(out.view(-1, *t.shape[1:]), t.contiguous(), group=self.group)
        else:
            out[0].copy_(t)
        return out


class HostComm(DeviceComm):
    """Collectives through host memory: a device tensor is copied to the CPU,
    the collective runs there (a gloo process group), and the result is
    copied back.  For ranks whose process group has no device backend."""

    def all_reduce(self, t, op=None):
        if self.world() > 1:
            h = t.cpu()
            dist.all_reduce(h, op=op or dist.ReduceOp.SUM, group=self.group)
            t.copy_(h)
        return t

    def all_gather(self, out, t):
        if self.world() > 1:
            parts = [torch.empty_like(t, device="cpu") for _ in range(self.world())]
            dist.all_gather(parts, t.cpu().contiguous(), group=self.group)
            out.copy_(torch.stack(parts))
        else:
            out[0].copy_(t)
        return out


def eqb_update_bf16_distributed(z: torch.Tensor, alpha: torch.Tensor | None, bias: torch.Tensor,
                                K: int, n_total: int, group=None, quantiles=None, ops=None,
                                comm=None):
    """One EQB update of ``bias`` (in place, identical on every rank).

    z [n_local, E] and alpha [n_local] are this rank's tokens; n_total is the
    number of tokens over all ranks (the target rank is floor(n_total K / E)).
    Returns (bias, quantiles)."""
    ops = ops or _LibraryOps
    comm = comm or DeviceComm(group)
    E = z.shape[1]
    dev = z.device
    hist = torch.zeros((E, 256), dtype=torch.int32, device=dev)
    rank = torch.full((E,), (int(n_total) * int(K)) // E, dtype=torch.int64, device=dev)
    d_hi = torch.empty((E,), dtype=torch.int32, device=dev)
    d_lo = torch.empty((E,), dtype=torch.int32, device=dev)
    if quantiles is None:
        quantiles = torch.empty((E,), dtype=torch.float32, device=dev)
    # pass one: high byte of every key
    ops.histogram(z, alpha, None, hist)
    comm.all_reduce(hist)
    ops.digit(hist, rank, d_hi)
    # pass two: low byte of the keys inside the chosen high bin
    hist.zero_()
    ops.histogram(z, alpha, d_hi, hist)
    comm.all_reduce(hist)
    ops.digit(hist, rank, d_lo)
    ops.bias(d_hi, d_lo, bias, quantiles)
    return bias, quantiles


def eqb_update_distributed(z: torch.Tensor, alpha: torch.Tensor | None, bias: torch.Tensor,
                           K: int, n_total: int, group=None, quantiles=None, ops=None, comm=None):
    """One EQB update of ``bias`` from the exact fp32 quantile of the union
    (in place, identical on every rank): four passes of 8-bit digits of the
    order key of Z + alpha, one all-reduce of the [E, 256] histogram each.

    z [n_local, E] and alpha [n_local] are this rank's tokens; n_total is the
    number of tokens over all ranks.  Returns (bias, quantiles)."""
    ops = ops or _LibraryKeyOps
    comm = comm or DeviceComm(group)
    E = z.shape[1]
    dev = z.device
    hist = torch.zeros((E, 256), dtype=torch.int32, device=dev)
    rank = torch.full((E,), (int(n_total) * int(K)) // E, dtype=torch.int64, device=dev)
    prefix = torch.zeros((E,), dtype=torch.int32, device=dev)
    if quantiles is None:
        quantiles = torch.empty((E,), dtype=torch.float32, device=dev)
    for p in range(4):
        if p:
            hist.zero_()
        ops.histogram(z, alpha, p, prefix, hist)
        comm.all_reduce(hist)
        ops.digit(hist, p, rank, prefix)
    ops.bias(prefix, bias, quantiles)
    return bias, quantiles


class SplitBuffers:
    """Device buffers of eqb_update_split for one shape (reused across calls)."""

    def __init__(self, E: int, S: int, R: int, cap: int, device):
        i32 = dict(dtype=torch.int32, device=device)
        self.sample = torch.empty((E, S), **i32)
        self.gathered = torch.empty((R, E, S), **i32)
        self.expert_major = torch.empty((E, (R * S + 3) // 4 * 4), **i32)
        self.lo = torch.empty((E,), **i32)
        self.hi = torch.empty((E,), **i32)
        self.counts = torch.empty((3, E), **i32)
        self.counts_sum = torch.empty((3, E), **i32)
        self.cand = torch.empty((E, cap), **i32)
        self.rank = torch.empty((E,), dtype=torch.int64, device=device)
        self.flag = torch.empty((E,), **i32)
        self.prefix = torch.zeros((E,), **i32)
        self.hist = torch.zeros((E, 256), **i32)


def split_sample_rows(n_local_min: int, world: int, sample_rows: int = SAMPLE_ROWS) -> int:
    """Rows each rank samples: the one-GPU sample size shared out over the
    ranks, at most the smallest rank's batch (every rank gives the same
    count, so the samples gather into one [R, E, S] buffer)."""
    return max(1, min(sample_rows // world, n_local_min))


def eqb_update_split(z: torch.Tensor, alpha: torch.Tensor, bias: torch.Tensor, K: int,
                     n_total: int, group=None, quantiles=None, ops=None, comm=None,
                     bufs: SplitBuffers | None = None, n_local_min: int | None = None,
                     cap: int = CAND_CAP, fallback_ops=None):
    """One EQB update of ``bias`` (in place, identical on every rank) from the
    exact fp32 quantile of the union, by the sampled-bracket design:

      1. every rank samples the keys of its z + alpha at S strided rows; the
         samples are gathered (all-gather), and every rank takes the same
         bracket [lo, hi] per expert from them;
      2. one pass over each rank's z + alpha counts the keys above hi and
         gathers the keys inside the bracket; the counts are summed
         (all-reduce) and give the target's rank among the bracketed keys;
      3. four radix passes over the gathered keys, their [E, 256] histograms
         summed (all-reduce) before every rank picks the same digit;
      4. bias = -v, centred.

    Where the summed counts show the target outside the bracket (the sample
    misled), every rank sees it and the update finishes with the four-pass
    form over z.  z [n_local, E], alpha [n_local]; n_total = tokens over all
    ranks; n_local_min = the smallest rank's n_local (found by an all-reduce
    when not given).  Returns (bias, quantiles)."""
    ops = ops or _LibrarySplitOps
    comm = comm or DeviceComm(group)
    R = comm.world()
    n_local, E = z.shape
    dev = z.device
    if quantiles is None:
        quantiles = torch.empty((E,), dtype=torch.float32, device=dev)
    if n_local_min is None:
        t = torch.tensor([n_local], dtype=torch.int64, device=dev)
        comm.all_reduce(t, op=dist.ReduceOp.MIN)
        n_local_min = int(t.item())
    S = split_sample_rows(n_local_min, R)
    if bufs is None:
        bufs = SplitBuffers(E, S, R, cap, dev)
    ops.sample(z, alpha, K, S, bufs.sample)
    comm.all_gather(bufs.gathered, bufs.sample)
    ops.brackets(bufs.gathered, n_total, K, bufs.expert_major, bufs.lo, bufs.hi)
    ops.count(z, alpha, K, bufs.lo, bufs.hi, bufs.counts, bufs.cand)
    bufs.counts_sum.copy_(bufs.counts)
    comm.all_reduce(bufs.counts_sum)
    ops.rank(bufs.counts_sum, n_total, K, bufs.rank, bufs.flag)
    if bool(bufs.flag.any()):      # the same on every rank: it comes from the summed counts
        return eqb_update_distributed(z, alpha, bias, K, n_total, group=group,
                                      quantiles=quantiles, ops=fallback_ops, comm=comm)
    for p in range(4):
        bufs.hist.zero_()
        ops.histogram(bufs.cand, bufs.counts, p, bufs.prefix, bufs.hist)
        comm.all_reduce(bufs.hist)
        ops.digit(bufs.hist, p, bufs.rank, bufs.prefix)
    ops.bias(bufs.prefix, bias, quantiles)
    return bias, quantiles
