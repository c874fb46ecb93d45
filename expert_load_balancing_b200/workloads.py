"""Seeded synthetic inputs shaped like the Kolibri router's workloads.

This module only draws random numbers and lays them out; it holds none of the
routing or balancing arithmetic.  The test suite feeds the same arrays to the
CUDA library and to the CPU oracle, and the benchmark uses the same recipes.

Shapes come from the model table of "Kolibri Pre-Training from Scratch"
(section 2: width 2560, 384 routed experts, top-6; Kolibri Origin width 2048,
128 experts, top-8) and from the router interface of "Kolibri 1 im Detail"
(bf16 router, tokens [N, 2560], fp32 logits [N, 384]).

Recipe (all draws seeded; "N(0, s)" is mean 0 and VARIANCE s):
  x      ~ N(0, 1) in fp32, rounded to bf16 (round to nearest even).
  W      ~ N(0, 1/d) in fp32, rounded to bf16, so logits have unit variance.
  offsets: a per-expert logit offset o_e is realised inside the GEMM by a
         constant feature: x[:, 0] = 1 and W[e, 0] = bf16(o_e).  Feature 0
         then carries no noise and every logit of expert e shifts by o_e.
         - collapsed router: o_e = +3 (three logit standard deviations) on
           the first 8 experts of a seeded permutation, 0 elsewhere;
         - Zipf(1.1): o_e = -1.1 ln(rank_e), rank a seeded permutation of
           1..E, centred to zero mean before rounding.
  beta   zeros, or ~ N(0, 0.1) in fp32 where a config fixes biases.

x is drawn in blocks of ``ROW_BLOCK`` rows, block b from its own generator,
so any block can be re-drawn on its own (the tests check sampled rows of the
million-token batch without holding a second copy).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

ROW_BLOCK = 4096

# stream ids keep the draws for x, W, beta and offsets independent
_STREAM_X, _STREAM_W, _STREAM_BETA, _STREAM_OFFSETS = 1, 2, 3, 4


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int
    d: int
    E: int
    K: int
    offsets: str = "none"        # "none" | "collapsed8" | "zipf1.1"
    beta: str = "zeros"          # "zeros" | "normal0.1"
    eqb_updates: int = 1
    layers: int = 1
    seed: int = 0

    @property
    def m(self) -> int:
        """EQB target rank floor(N K / E)."""
        return (self.N * self.K) // self.E


# The five workloads: the small case, the collapsed router re-routed by ten
# updates, the Origin shape, the million-token batch, and the decode sweep.
WORKLOADS = {
    "small_n256": Workload("small_n256", 256, 2560, 384, 6),
    "collapsed_n16384": Workload("collapsed_n16384", 16384, 2560, 384, 6,
                                 offsets="collapsed8", eqb_updates=10),
    "origin_n65536": Workload("origin_n65536", 65536, 2048, 128, 8, beta="normal0.1"),
    "kolibri_n1m": Workload("kolibri_n1m", 1 << 20, 2560, 384, 6, offsets="zipf1.1"),
}
DECODE_TOKENS = (1, 8, 64, 256)
DECODE_LAYERS = 50


def decode_workload(n_tokens: int) -> Workload:
    return Workload(f"decode_n{n_tokens}", n_tokens, 2560, 384, 6, beta="normal0.1",
                    layers=DECODE_LAYERS, eqb_updates=0)


def _gen(seed: int, stream: int, index: int = 0) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed((seed * 1_000_003 + stream) * 1_000_033 + index)
    return g


def _rng(seed: int, stream: int, index: int = 0) -> np.random.Generator:
    return np.random.default_rng([seed, stream, index])


def expert_offsets(wl: Workload, layer: int = 0) -> np.ndarray | None:
    """Per-expert logit offsets o_e (fp32) or None."""
    if wl.offsets == "none":
        return None
    rng = _rng(wl.seed, _STREAM_OFFSETS, layer)
    order = rng.permutation(wl.E)
    o = np.zeros(wl.E, dtype=np.float64)
    if wl.offsets == "collapsed8":
        o[order[:8]] = 3.0
    elif wl.offsets == "zipf1.1":
        rank = np.empty(wl.E, dtype=np.float64)
        rank[order] = np.arange(1, wl.E + 1, dtype=np.float64)
        o = -1.1 * np.log(rank)
        o = o - o.mean()
    else:
        raise ValueError(wl.offsets)
    return o.astype(np.float32)


def x_block(wl: Workload, block: int, layer: int = 0) -> torch.Tensor:
    """Rows [block*ROW_BLOCK, ...) of x as a bf16 CPU tensor."""
    r0 = block * ROW_BLOCK
    rows = min(ROW_BLOCK, wl.N - r0)
    g = _gen(wl.seed, _STREAM_X, layer * 1_000_000 + block)
    x = torch.randn(rows, wl.d, generator=g, dtype=torch.float32)
    if wl.offsets != "none":
        x[:, 0] = 1.0
    return x.to(torch.bfloat16)


def make_x(wl: Workload, layer: int = 0, out: torch.Tensor | None = None) -> torch.Tensor:
    """The whole x [N, d] bf16 on the CPU (optionally into ``out``)."""
    if out is None:
        out = torch.empty((wl.N, wl.d), dtype=torch.bfloat16)
    nblocks = (wl.N + ROW_BLOCK - 1) // ROW_BLOCK
    for b in range(nblocks):
        r0 = b * ROW_BLOCK
        blk = x_block(wl, b, layer)
        out[r0:r0 + blk.shape[0]].copy_(blk)
    return out


def x_rows(wl: Workload, rows, layer: int = 0) -> torch.Tensor:
    """Selected rows of x (re-drawn block by block)."""
    rows = np.asarray(rows, dtype=np.int64)
    out = torch.empty((rows.shape[0], wl.d), dtype=torch.bfloat16)
    for b in np.unique(rows // ROW_BLOCK):
        blk = x_block(wl, int(b), layer)
        sel = np.nonzero(rows // ROW_BLOCK == b)[0]
        out[torch.from_numpy(sel)] = blk[torch.from_numpy(rows[sel] - b * ROW_BLOCK)]
    return out


def make_w(wl: Workload, layer: int = 0) -> torch.Tensor:
    """Router weight W [E, d] bf16 on the CPU."""
    g = _gen(wl.seed, _STREAM_W, layer)
    w = torch.randn(wl.E, wl.d, generator=g, dtype=torch.float32) * (1.0 / math.sqrt(wl.d))
    o = expert_offsets(wl, layer)
    if o is not None:
        w[:, 0] = torch.from_numpy(o)
    return w.to(torch.bfloat16)


def make_beta(wl: Workload, layer: int = 0) -> torch.Tensor:
    """Initial selection bias beta [E] fp32 on the CPU."""
    if wl.beta == "zeros":
        return torch.zeros(wl.E, dtype=torch.float32)
    if wl.beta == "normal0.1":
        g = _gen(wl.seed, _STREAM_BETA, layer)
        return torch.randn(wl.E, generator=g, dtype=torch.float32) * math.sqrt(0.1)
    raise ValueError(wl.beta)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 tensor (for the oracle's C interface)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def random_logits(N: int, E: int, seed: int, scale: float = 1.0) -> np.ndarray:
    """fp32 logits ~ N(0, scale^2) for tests that start from given logits."""
    return (_rng(seed, 9).standard_normal((N, E), dtype=np.float32) * np.float32(scale))


def tied_logits(N: int, E: int, seed: int, levels: int = 4) -> np.ndarray:
    """fp32 logits drawn from a few values only, so rows and columns carry
    many exact ties (including +0.0 and -0.0)."""
    vals = np.array([-1.5, -0.0, 0.0, 0.75, 2.0, 3.25][:max(2, levels)], dtype=np.float32)
    idx = _rng(seed, 10).integers(0, vals.shape[0], size=(N, E))
    return vals[idx]
