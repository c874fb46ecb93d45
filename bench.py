"""Routing throughput of the B200 sigmoid router + Exact Quantile Balancing.

One step = the whole hot path over one batch: router logits (tcgen05 GEMM),
bias add + top-K + sigmoid gates + token bias, expert counts + stable
permutation, and one exact EQB bias update.  Default workload: the
million-token Kolibri-shaped batch (N = 1,048,576, d = 2560, E = 384, K = 6,
Zipf(1.1) expert offsets), inputs resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): data parallel, weak scaling.  Each
rank routes its own batch of N tokens (logits, selection, permutation stay
local) and the EQB update is the exact quantile of the union of all ranks'
tokens ("Kolibri Pre-Training from Scratch" 7.3), by the sampled-bracket
form over NCCL (distributed.eqb_update_split: an all-gather of the samples,
an all-reduce of 3 E counts, four all-reduces of [E, 256] histograms).  The
reported value is all ranks' tokens over the slowest rank's device time.
``--eqb split`` runs that form on one GPU too (no exchange), to time it.

``--impl reference`` times the CPU oracle on the host cores (bounded sample
of the same workload per step); it is the slow baseline, not a target.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from expert_load_balancing_b200 import binding as B  # noqa: E402
from expert_load_balancing_b200 import workloads  # noqa: E402

METRIC = "routed tokens/sec (GEMM+top-K+permute+EQB) at N=1M, E=384, K=6; % of roofline"
UNIT = "routed tokens/s"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---------------------------------------------------------------- algorithmic work

def algorithmic_work(N, d, E, K, updates=1):
    """FLOPs and bytes a perfect implementation must spend per step.

    GEMM 2 N d E FLOP.  Bytes: x read (2Nd), Z written once (4NE), W once
    (2Ed); then per routing + EQB update: Z read once (4NE), ids+gates
    written (8NK), perm+inv written (8NK), alpha (4N).  counts/offsets/beta
    are negligible.  `updates` > 1 re-routes the same Z with each new bias
    (the collapsed-router loop)."""
    flops = 2.0 * N * d * E
    bytes_ = (2.0 * N * d + 4.0 * N * E + 2.0 * E * d
              + updates * (4.0 * N * E + 16.0 * N * K + 4.0 * N))
    return flops, bytes_


def gemm_bytes(N, d, E):
    """Algorithmic bytes of the logits GEMM alone: x in, Z out, W once."""
    return 2.0 * N * d + 4.0 * N * E + 2.0 * E * d


def launches_per_step(N, E, K, updates=1, split=False):
    """Kernels of ours per step: logits + selection 2 (the fused GEMM and the
    check for rows it left to the row kernel, or the small-batch logits and
    the row kernel); EQB update 2 (N <= 16384: sample, exact select ending
    in the bias update) or 4 (sample, bracket, bracketed pass, and one grid
    for the select, any column fallback and the bias update), or over a
    split batch 15 (sample, brackets, bracketed pass and its finish, rank,
    four histogram + digit passes, key value, bias); permutation 1 or 3.
    Each further update re-routes (1) first."""
    eqb = 15 if split else (2 if N <= 16384 else 4)
    permute = 1 if N * K <= 4096 else 3
    return 2 + eqb + permute + (updates - 1) * (1 + eqb + permute)


def choose_bf16_peak(peaks, clocks, timed_s):
    """The bf16 peak a tensor-bound fraction is taken against: the burst
    figure when the timed region is short (under 0.5 s) or the clock record
    shows no sw_power_cap under load, the sustained one otherwise."""
    capped = "sw_power_cap" in ((clocks or {}).get("reasons") or [])
    if timed_s < 0.5 or not capped:
        return peaks["bf16_tflops"], "burst"
    return peaks["bf16_tflops_sustained"], "sustained"


def reduce_max_over_ranks(value: float, device) -> float:
    """The slowest rank's value (device time per step); identity on one rank."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return value
    if torch.distributed.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling during the timed region (SM clock, reasons)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- our path

class RouterStep:
    """Buffers and the four calls of one step, all on one stream."""

    def __init__(self, wl, device, seed=0, split_eqb=False, world=1):
        self.wl = wl
        # the EQB update over the union of all ranks' tokens (sampled-bracket form)
        self.split_eqb = split_eqb
        self.n_total = wl.N * world
        self.split_bufs = None
        N, d, E, K = wl.N, wl.d, wl.E, wl.K
        g = torch.Generator(device=device)
        g.manual_seed(1234 + seed)
        self.x = torch.empty((N, d), dtype=torch.bfloat16, device=device)
        rows = 65536
        for r0 in range(0, N, rows):
            r1 = min(N, r0 + rows)
            self.x[r0:r1] = torch.randn((r1 - r0, d), generator=g, device=device).to(torch.bfloat16)
        if wl.offsets != "none":
            self.x[:, 0] = 1.0
        self.w = workloads.make_w(wl).to(device)
        self.beta0 = workloads.make_beta(wl).to(device)
        self.beta = self.beta0.clone()
        self.z = torch.empty((N, E), dtype=torch.float32, device=device)
        self.ids = torch.empty((N, K), dtype=torch.int32, device=device)
        self.gates = torch.empty((N, K), dtype=torch.float32, device=device)
        self.alpha = torch.empty((N,), dtype=torch.float32, device=device)
        self.counts = torch.empty((E,), dtype=torch.int32, device=device)
        self.offsets = torch.empty((E + 1,), dtype=torch.int64, device=device)
        self.perm = torch.empty((N * K,), dtype=torch.int32, device=device)
        self.inv = torch.empty((N * K,), dtype=torch.int32, device=device)
        self.q = torch.empty((E,), dtype=torch.float32, device=device)
        self.ws_perm = B.workspace(B.KOLIBRI_OP_PERMUTE, N, E, K, device)
        self.ws_eqb = B.workspace(B.KOLIBRI_OP_EQB, N, E, K, device)
        # the permutation needs only ids: it runs on a second stream while
        # the EQB update runs on the first
        self.side = torch.cuda.Stream(device)
        self.fork = torch.cuda.Event()
        self.join = torch.cuda.Event()

    def run(self, stream, events=None):
        """logits + routing (selection in the GEMM epilogue), then on two
        streams: the EQB update of beta from that alpha (one bracketed read
        of Z) and the permutation.  events (6, optional): start, forward
        done, EQB done, permutation start and end (second stream), step end."""
        wl = self.wl
        if wl.eqb_updates > 1:
            self._run_loop(stream, events)
            return
        if events:
            events[0].record(stream)
        B.kolibri_router_forward(self.x, self.w, self.beta, wl.K, z=self.z, ids=self.ids,
                                 gates=self.gates, alpha=self.alpha, stream=stream)
        fork = events[1] if events else self.fork
        fork.record(stream)
        self.side.wait_event(fork)
        if events:
            events[3].record(self.side)
        B.kolibri_expert_permute(self.ids, wl.E, self.ws_perm, self.counts, self.offsets,
                                 self.perm, self.inv, stream=self.side)
        join = events[4] if events else self.join
        join.record(self.side)
        if self.split_eqb:
            self._split_update(stream)
        else:
            B.kolibri_eqb_update(self.z, self.alpha, self.beta, wl.K, self.ws_eqb, self.q,
                                 stream=stream)
        if events:
            events[2].record(stream)
        stream.wait_event(join)
        if events:
            events[5].record(stream)


    def _split_update(self, stream):
        """The EQB update over every rank's tokens, sampled-bracket form."""
        from expert_load_balancing_b200 import distributed as D
        wl = self.wl
        if self.split_bufs is None:
            R = D.DeviceComm().world()
            S = D.split_sample_rows(wl.N, R)
            self.split_bufs = D.SplitBuffers(wl.E, S, R, D.CAND_CAP, self.z.device)
        with torch.cuda.stream(stream):
            D.eqb_update_split(self.z, self.alpha, self.beta, wl.K, self.n_total,
                               quantiles=self.q, bufs=self.split_bufs, n_local_min=wl.N)

    def _run_loop(self, stream, events=None):
        """The collapsed-router loop: the same batch re-routed after every
        update ("Kolibri Pre-Training from Scratch" 7.2 repairs a collapsed
        router in one update; this configuration applies ten).  Logits +
        routing with the initial bias, its permutation and the first update;
        then per further update the routing with the new bias together with
        the update (kolibri_route_and_balance) and its permutation.  One
        stream: each routing's ids feed its permutation.  events as in run();
        EQB done marks the end of the loop, the permutation events bracket
        the first permutation."""
        wl = self.wl
        ev = events
        if ev:
            ev[0].record(stream)
        with torch.cuda.stream(stream):
            self.beta.copy_(self.beta0, non_blocking=True)   # every step repairs the collapse anew
        B.kolibri_router_forward(self.x, self.w, self.beta, wl.K, z=self.z, ids=self.ids,
                                 gates=self.gates, alpha=self.alpha, stream=stream)
        if ev:
            ev[1].record(stream)
            ev[3].record(stream)
        B.kolibri_expert_permute(self.ids, wl.E, self.ws_perm, self.counts, self.offsets,
                                 self.perm, self.inv, stream=stream)
        if ev:
            ev[4].record(stream)
        B.kolibri_eqb_update(self.z, self.alpha, self.beta, wl.K, self.ws_eqb, self.q,
                             stream=stream)
        for _ in range(wl.eqb_updates - 1):
            B.kolibri_route_and_balance(self.z, self.beta, wl.K, self.ws_eqb, ids=self.ids,
                                        gates=self.gates, alpha=self.alpha, quantiles=self.q,
                                        stream=stream)
            B.kolibri_expert_permute(self.ids, wl.E, self.ws_perm, self.counts, self.offsets,
                                     self.perm, self.inv, stream=stream)
        if ev:
            ev[2].record(stream)
            ev[5].record(stream)


def maxvio(counts, wl):
    """MaxVio of one routing ("Kolibri Pre-Training from Scratch" 6.2): the
    largest expert load over the mean load N K / E, minus one."""
    return float(counts.max().item()) / (wl.N * wl.K / wl.E) - 1.0


def rerouted_maxvio(step, stream):
    """MaxVio of the batch routed again with the bias the last timed step's
    EQB update produced (outside the timed region)."""
    wl = step.wl
    B.kolibri_router_forward(step.x, step.w, step.beta, wl.K, z=step.z, ids=step.ids,
                             gates=step.gates, alpha=step.alpha, stream=stream)
    B.kolibri_expert_permute(step.ids, wl.E, step.ws_perm, step.counts, step.offsets, step.perm,
                             step.inv, stream=stream)
    stream.synchronize()
    return maxvio(step.counts, wl)


def run_ours(args, rank, world, local_rank):
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    B.load()
    wl = workloads.WORKLOADS[args.workload]
    if args.tokens:
        import dataclasses
        wl = dataclasses.replace(wl, N=args.tokens)
    N, d, E, K = wl.N, wl.d, wl.E, wl.K
    split_eqb = world > 1 or args.eqb == "split"
    if split_eqb and wl.eqb_updates > 1:
        raise SystemExit("the split-batch EQB update runs the one-update step only")
    step = RouterStep(wl, device, seed=rank, split_eqb=split_eqb, world=world)
    stream = torch.cuda.Stream(device)
    balance = {}
    with torch.cuda.stream(stream):
        # the loads of the first routing, with the workload's initial bias
        B.kolibri_router_forward(step.x, step.w, step.beta, wl.K, z=step.z, ids=step.ids,
                                 gates=step.gates, alpha=step.alpha, stream=stream)
        B.kolibri_expert_permute(step.ids, wl.E, step.ws_perm, step.counts, step.offsets,
                                 step.perm, step.inv, stream=stream)
        stream.synchronize()
        balance["maxvio_initial_bias"] = maxvio(step.counts, wl)
        for i in range(args.warmup):
            step.run(stream)
    stream.synchronize()
    st = B.kolibri_device_status(stream)
    if st != B.KOLIBRI_OK:
        raise RuntimeError(f"device status after warm-up: {B.status_string(st)}")

    # ---- timed region: device time, CUDA events on the launching stream
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    visible = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    gpu_id = visible.split(",")[local_rank] if visible else str(local_rank)
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.3)
    t0.record(stream)
    for i in range(args.steps):
        step.run(stream, ev[i])
    t1.record(stream)
    t1.synchronize()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    total_ms = t0.elapsed_time(t1)
    stage_ms = np.array([[ev[i][0].elapsed_time(ev[i][1]), ev[i][1].elapsed_time(ev[i][2]),
                          ev[i][3].elapsed_time(ev[i][4])]
                         for i in range(args.steps)]).mean(axis=0)
    st = B.kolibri_device_status(stream)
    if st != B.KOLIBRI_OK:
        raise RuntimeError(f"device status after timing: {B.status_string(st)}")

    total_ms = reduce_max_over_ranks(total_ms, device)
    ms_per_step = total_ms / args.steps
    # balance of the routing, outside the timed region: the last timed step's
    # loads (bias before its update) and a re-route with the updated bias
    balance["maxvio_last_step"] = maxvio(step.counts, wl)
    with torch.cuda.stream(stream):
        balance["maxvio_rerouted"] = rerouted_maxvio(step, stream)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, step, stream, device, world)

    if rank != 0:
        return None
    timed_s = total_ms * 1e-3
    line = result_line(wl, world, args, ms_per_step, stage_ms, clocks, timed_s, split_eqb)
    if split_eqb:
        line["config"]["parallelism"] = (f"dp{world}: tokens split by rank, EQB over the union "
                                         f"({world * N} tokens), sampled-bracket form")
    line["e2e"] = e2e
    line["balance"] = balance
    line["gpu_name"] = torch.cuda.get_device_name(device)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    return line


def result_line(wl, world, args, ms_per_step, stage_ms, clocks, timed_s, split=False):
    """The JSON line of one routing-step run: throughput, the fused
    kernel's roofline (tensor-bound), the EQB update's (HBM-bound), the
    whole step's against max(FLOP / bf16 peak, bytes / HBM peak)."""
    N, d, E, K, U = wl.N, wl.d, wl.E, wl.K, wl.eqb_updates
    peaks = _peaks()
    peak_t, peak_kind = choose_bf16_peak(peaks, clocks, timed_s)
    flops, bytes_ = algorithmic_work(N, d, E, K, U)
    roof_ms = max(flops / (peak_t * 1e12), bytes_ / (peaks["hbm_gbs"] * 1e9)) * 1e3
    gemm_ms = float(stage_ms[0])   # the fused GEMM + selection, and the row check after it
    gemm_tflops = 2.0 * N * d * E / (gemm_ms * 1e-3) / 1e12
    # the profiled DRAM bytes per token scale with N only where x and Z stream
    # through HBM (at and above the 131,072-token capture)
    traffic = _traffic_from_profile(N) if (d, E) == (2560, 384) and N >= 131072 else None
    routed = N * U
    line = {
        "metric": METRIC,
        "value": world * routed / (ms_per_step * 1e-3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16/fp32",
        "data": "synthetic",
        "config": {"workload": wl.name, "N": N, "d": d, "E": E, "K": K, "offsets": wl.offsets,
                   "beta0": wl.beta, "eqb_updates": U,
                   "parallelism": f"replicas{world}",
                   "l2": ("inputs larger than L2 (x %.2f GB, Z %.2f GB)" if 2 * N * d > 126e6 else
                          "inputs fit in L2 (x %.3f GB, Z %.3f GB); warm, stated so")
                         % (2 * N * d / 1e9, 4 * N * E / 1e9)},
        "roofline": {"bound": "tensor", "kernel": "router_forward_kernel" if N > 1024 else
                     "small_logits_kernel + route_rows_kernel",
                     "achieved": gemm_tflops, "peak": peak_t, "unit": "TFLOP/s",
                     "frac": gemm_tflops / peak_t, "traffic": traffic,
                     "peak_kind": f"bf16 {peak_kind} (cuBLAS), of {peaks['source']}: "
                                  f"timed region {timed_s:.3f} s",
                     "burst_frac": gemm_tflops / peaks["bf16_tflops"],
                     "sustained_frac": gemm_tflops / peaks["bf16_tflops_sustained"]},
        "path_roofline": {"roofline_ms": roof_ms, "frac": roof_ms / ms_per_step,
                          "flops": flops, "bytes": bytes_,
                          "peaks": f"bf16 {peak_kind} {peak_t} TF/s, HBM {peaks['hbm_gbs']} GB/s, "
                                   f"of {peaks['source']}"},
        "stages_ms": {"logits_and_routing": gemm_ms},
        "gpu_launches": launches_per_step(N, E, K, U, split) * args.steps,
        "clocks": clocks,
    }
    if U == 1:
        eqb_ms = float(stage_ms[1])
        eqb_bytes = 4.0 * N * E + 4.0 * N        # Z and alpha read once
        line["stages_ms"]["eqb_update"] = eqb_ms
        line["stages_ms"]["permute_concurrent"] = float(stage_ms[2])
        line["eqb_roofline"] = {"bound": "hbm", "achieved": eqb_bytes / (eqb_ms * 1e-3) / 1e9,
                                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                "frac": eqb_bytes / (eqb_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                "algorithmic": "4E + 4 B per token (Z and alpha read once)"}
    else:
        line["stages_ms"]["update_loop"] = float(stage_ms[1])
        line["stages_ms"]["first_permute"] = float(stage_ms[2])
        line["config"]["routed"] = f"{U} routings of the same N tokens per step (value counts each)"
    return line


GEMM_PROFILE = os.path.join(ROOT, "profiles", "router_forward_kolibri.md")
GEMM_SOURCES = [os.path.join(ROOT, "expert_load_balancing_b200", "csrc", f)
                for f in ("router_forward.cu", "gemm_pair.cuh", "common.cuh")]


def kernel_source_digest():
    """sha256 over the fused kernel's source files, in a fixed order."""
    import hashlib
    h = hashlib.sha256()
    for p in GEMM_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _traffic_from_profile(N):
    """DRAM bytes per GEMM launch (read + write) from the committed ncu
    summary, scaled to N tokens; None if the kernel source changed since the
    counters were taken."""
    try:
        text = open(GEMM_PROFILE).read()
        digest = kernel_source_digest()
    except OSError:
        return None
    fields = {}
    for line in text.splitlines():
        if ":" in line and line.startswith("- "):
            k, v = line[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("source_sha256") != digest:
        return None
    try:
        per_token = float(fields["dram_bytes_per_token"])
    except (KeyError, ValueError):
        return None
    return per_token * N


def run_e2e(args, step, stream, device, world):
    """Same step through the public API with the step's inputs copied in
    from pinned host memory and its routing result read back, every step."""
    wl = step.wl
    N, d, E, K = wl.N, wl.d, wl.E, wl.K
    x_h = torch.empty((N, d), dtype=torch.bfloat16, pin_memory=True)
    x_h.copy_(step.x, non_blocking=False)
    w_h = step.w.cpu().pin_memory()
    b_h = step.beta0.cpu().pin_memory()
    ids_h = torch.empty((N, K), dtype=torch.int32, pin_memory=True)
    gates_h = torch.empty((N, K), dtype=torch.float32, pin_memory=True)
    counts_h = torch.empty((E,), dtype=torch.int32, pin_memory=True)
    beta_h = torch.empty((E,), dtype=torch.float32, pin_memory=True)
    h2d = x_h.numel() * 2 + w_h.numel() * 2 + b_h.numel() * 4
    d2h = ids_h.numel() * 4 + gates_h.numel() * 4 + counts_h.numel() * 4 + beta_h.numel() * 4

    def one():
        with torch.cuda.stream(stream):
            step.x.copy_(x_h, non_blocking=True)
            step.w.copy_(w_h, non_blocking=True)
            step.beta.copy_(b_h, non_blocking=True)
            step.run(stream)
            ids_h.copy_(step.ids, non_blocking=True)
            gates_h.copy_(step.gates, non_blocking=True)
            counts_h.copy_(step.counts, non_blocking=True)
            beta_h.copy_(step.beta, non_blocking=True)

    for _ in range(max(1, min(args.warmup, 2))):
        one()
    stream.synchronize()
    n = args.e2e_steps
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(n):
        one()
    b.record(stream)
    b.synchronize()
    ms = a.elapsed_time(b) / n
    ms = reduce_max_over_ranks(ms, device)
    return {"value": world * N / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms, "steps": n,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}


# ---------------------------------------------------------------- the oracle

def _oracle_step(oracle, wl, n_rows, beta):
    """One oracle pass of the whole path over the first n_rows tokens."""
    x = workloads.bf16_bits(workloads.x_rows(wl, np.arange(n_rows)))
    w = workloads.bf16_bits(workloads.make_w(wl))
    t = time.perf_counter()
    z = oracle.router_logits(x, w)
    b = beta
    for _ in range(wl.eqb_updates):      # re-routing with each new bias (collapsed loop)
        ids, gates, alpha = oracle.select(z, b, wl.K)
        oracle.permute(ids, wl.E)
        v = oracle.column_quantiles(z, alpha, oracle.eqb_target_rank(n_rows, wl.K, wl.E))
        b = oracle.eqb_bias(v)
    return time.perf_counter() - t


def cpu_baseline(wl, seconds):
    import oracle
    oracle.build()
    beta = workloads.make_beta(wl).numpy()
    t_cal = _oracle_step(oracle, wl, 256, beta)
    n_rows = int(max(256, min(wl.N, 256 * seconds / max(t_cal, 1e-3))))
    n_rows = (n_rows // 256) * 256
    t = _oracle_step(oracle, wl, n_rows, beta)
    return {"value": n_rows * wl.eqb_updates / t, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"first {n_rows} tokens of {wl.name} (full d, E, K), one pass of logits, then "
                      f"{wl.eqb_updates} x (top-K, permutation, EQB update) over that sample; {t:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle
    oracle.build()
    wl = workloads.WORKLOADS[args.workload]
    beta = workloads.make_beta(wl).numpy()
    t_cal = _oracle_step(oracle, wl, 256, beta)
    # size each step so the whole run takes a few minutes at most
    total_steps = args.warmup + args.steps
    per_step = min(20.0, 150.0 / max(total_steps, 1))
    n_rows = int(max(256, min(wl.N, 256 * per_step / max(t_cal, 1e-3))))
    n_rows = (n_rows // 256) * 256
    for _ in range(args.warmup):
        _oracle_step(oracle, wl, 256, beta)
    times = [_oracle_step(oracle, wl, n_rows, beta) for _ in range(args.steps)]
    ms = 1e3 * sum(times) / len(times)
    value = n_rows * wl.eqb_updates / (ms * 1e-3)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64/fp32",
        "data": "synthetic",
        "config": {"workload": wl.name, "N": wl.N, "d": wl.d, "E": wl.E, "K": wl.K,
                   "parallelism": "host cores", "sample_tokens_per_step": n_rows},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"first {n_rows} tokens of {wl.name} per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------- the balancing pieces

PARTS = {
    # name: (what, algorithmic bytes per token as a function of (E, K), note)
    "eqb_bf16": ("EQB update with bf16 keys (one GPU: exact fp32 quantile, rounded)",
                 lambda E, K: 4 * E + 4, "Z and alpha read once"),
    "eqb_bf16_split": ("EQB with bf16 keys, the two histogram passes of the multi-rank form, one rank",
                       lambda E, K: 8 * E + 8, "Z and alpha read twice"),
    "eqb_fp32_split": ("EQB with fp32 keys, the four histogram passes of the multi-rank form, one rank",
                       lambda E, K: 16 * E + 16, "Z and alpha read four times"),
    "lei": ("Load-Error Injection on the [N, E] score gradient",
            lambda E, K: 8 * E, "G read and written"),
    "score_grad": ("chain rule from the score gradient to the logits",
                   lambda E, K: 12 * E, "Z and dS read, dZ written"),
    "intervention": ("intervention rate (own top-K vs routed ids)",
                     lambda E, K: 4 * E + 4 * K, "Z and ids read"),
    "topk": ("selection alone: bias add, top-K ids, sigmoid gates, alpha (kolibri_router_topk)",
             lambda E, K: 4 * E + 8 * K + 4, "Z read; ids, gates and alpha written"),
}


def run_part(args):
    """One of the balancing pieces on the kolibri_n1m shape, timed like the
    step (CUDA events, clock samples), with its HBM roofline and the oracle
    on a sample of the same data beside it."""
    import oracle
    from expert_load_balancing_b200 import distributed as D
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    wl = workloads.WORKLOADS[args.workload]
    if args.tokens:
        import dataclasses
        wl = dataclasses.replace(wl, N=args.tokens)
    N, d, E, K = wl.N, wl.d, wl.E, wl.K
    step = RouterStep(wl, device)
    stream = torch.cuda.Stream(device)
    # a few routing steps first, as the step's warm-up does: the workload's
    # initial bias is far from balanced, and the pieces are timed on the
    # routing they meet in steady state (Z, ids and alpha of the last step)
    with torch.cuda.stream(stream):
        for _ in range(5):
            step.run(stream)
    stream.synchronize()
    g = torch.Generator(device=device)
    g.manual_seed(7)
    gs = torch.randn((N, E), generator=g, device=device) * 1e-4 if args.part in ("lei", "score_grad") else None
    gz = torch.empty_like(gs) if gs is not None else None
    ws16 = B.workspace(B.KOLIBRI_OP_EQB_BF16, N, E, K, device)
    ids_t = torch.empty((N, K), dtype=torch.int32, device=device) if args.part == "topk" else None
    gates_t = torch.empty((N, K), dtype=torch.float32, device=device) if args.part == "topk" else None
    alpha_t = torch.empty((N,), dtype=torch.float32, device=device) if args.part == "topk" else None
    beta0 = step.beta.clone()
    q = torch.empty((E,), dtype=torch.float32, device=device)

    def once():
        if args.part == "eqb_bf16":
            step.beta.copy_(beta0)
            B.kolibri_eqb_update_bf16(step.z, step.alpha, step.beta, K, q, ws16, stream=stream)
        elif args.part == "eqb_bf16_split":
            step.beta.copy_(beta0)
            with torch.cuda.stream(stream):
                D.eqb_update_bf16_distributed(step.z, step.alpha, step.beta, K, N, quantiles=q)
        elif args.part == "eqb_fp32_split":
            step.beta.copy_(beta0)
            with torch.cuda.stream(stream):
                D.eqb_update_distributed(step.z, step.alpha, step.beta, K, N, quantiles=q)
        elif args.part == "lei":
            B.kolibri_lei_inject(step.counts, gs, K, stream=stream)
        elif args.part == "score_grad":
            B.kolibri_score_grad_to_logits(step.z, gs, gz, stream=stream)
        elif args.part == "topk":
            B.kolibri_router_topk(step.z, step.beta, K, ids_t, gates_t, alpha_t, stream=stream)
        else:
            B.kolibri_intervention_rate(step.z, step.ids, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            once()
    stream.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0] or "0")
    sampler.start()
    time.sleep(0.3)
    t0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            once()
    t1.record(stream)
    t1.synchronize()
    clocks = sampler.stop()
    st = B.kolibri_device_status(stream)
    if st != B.KOLIBRI_OK:
        raise RuntimeError(f"device status: {B.status_string(st)}")
    ms = t0.elapsed_time(t1) / args.steps
    what, bpt, note = PARTS[args.part]
    peaks = _peaks()
    bytes_ = bpt(E, K) * N
    achieved = bytes_ / (ms * 1e-3) / 1e9
    # the oracle on the first rows of the same data
    n = min(N, 4096 if args.part.startswith("eqb") else 2048)
    zh = step.z[:n].cpu().numpy()
    t = time.time()
    if args.part == "eqb_fp32_split":
        oracle.column_quantiles(zh, step.alpha[:n].cpu().numpy(), (n * K) // E)
    elif args.part in ("eqb_bf16", "eqb_bf16_split"):
        oracle.column_quantiles_bf16(zh, step.alpha[:n].cpu().numpy(), (n * K) // E)
    elif args.part == "lei":
        oracle.lei_inject(step.counts.cpu().numpy(), gs[:n].cpu().numpy(), K)
    elif args.part == "score_grad":
        oracle.score_grad_to_logits(zh, gs[:n].cpu().numpy())
    elif args.part == "topk":
        oracle.select(zh, step.beta.cpu().numpy(), K)
    else:
        ids_u, _, _ = oracle.select(zh, None, K)
        oracle.intervention_rate(step.ids[:n].cpu().numpy(), ids_u)
    reps = 1
    cpu_s = time.time() - t
    while cpu_s < 2.0:                 # repeat the sample to about 2 s of CPU work
        t = time.time()
        if args.part == "eqb_fp32_split":
            oracle.column_quantiles(zh, step.alpha[:n].cpu().numpy(), (n * K) // E)
        elif args.part in ("eqb_bf16", "eqb_bf16_split"):
            oracle.column_quantiles_bf16(zh, step.alpha[:n].cpu().numpy(), (n * K) // E)
        elif args.part == "lei":
            oracle.lei_inject(step.counts.cpu().numpy(), gs[:n].cpu().numpy(), K)
        elif args.part == "score_grad":
            oracle.score_grad_to_logits(zh, gs[:n].cpu().numpy())
        elif args.part == "topk":
            oracle.select(zh, step.beta.cpu().numpy(), K)
        else:
            ids_u, _, _ = oracle.select(zh, None, K)
            oracle.intervention_rate(step.ids[:n].cpu().numpy(), ids_u)
        cpu_s += time.time() - t
        reps += 1
    return {
        "metric": f"{what}: tokens/s at N={N}, E={E}, K={K}", "part": args.part,
        "value": N / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "dtype": "fp32/f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "N": N, "E": E, "K": K,
                   "inputs": "the step's own Z, ids, alpha, counts after five routing steps"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                     "algorithmic": f"{bpt(E, K)} B per token ({note})",
                     "peak_kind": f"HBM copy, of {peaks['source']}"},
        "clocks": clocks,
        "cpu_baseline": {"value": n * reps / cpu_s, "unit": "tokens/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": f"first {n} tokens, {reps} times, {cpu_s:.1f} s"},
    }


# ---------------------------------------------------------------- the experts

def run_experts(args):
    """The expert layer after the router on one microbatch of N = 16384 tokens
    (d = 2560, E = 384 routed experts of 2560 -> 2 x 512 -> 2560, K = 6, plus
    the shared expert): dispatch, the grouped gate/up and down projections,
    combine.  The routing is our own: logits, one EQB update, re-routing with
    the new bias, permutation.  Timed region: kolibri_expert_ffn alone, inputs
    resident.  Roofline: the layer's FLOPs against the measured bf16 peak (the
    run is short, so the burst figure applies); the algorithmic bytes (every
    weight once, x in, y out) would take less time at the HBM peak."""
    import oracle
    oracle.build()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    B.load()
    N, d, F, E, K = args.tokens or 16384, 2560, 512, args.experts or 384, 6
    g = torch.Generator(device=device)
    g.manual_seed(11)
    wgu = (torch.randn(E, 2 * F, d, generator=g, device=device) / math.sqrt(d)).to(torch.bfloat16)
    wd = (torch.randn(E, d, F, generator=g, device=device) / math.sqrt(F)).to(torch.bfloat16)
    wgu_s = (torch.randn(2 * F, d, generator=g, device=device) / math.sqrt(d)).to(torch.bfloat16)
    wd_s = (torch.randn(d, F, generator=g, device=device) / math.sqrt(F)).to(torch.bfloat16)
    wl = workloads.Workload("experts", N, d, E, K)
    x = torch.randn(N, d, generator=g, device=device).to(torch.bfloat16)
    w_router = workloads.make_w(wl).to(device)
    beta = torch.zeros(E, dtype=torch.float32, device=device)
    z = torch.empty((N, E), dtype=torch.float32, device=device)
    ids = torch.empty((N, K), dtype=torch.int32, device=device)
    gates = torch.empty((N, K), dtype=torch.float32, device=device)
    alpha = torch.empty((N,), dtype=torch.float32, device=device)
    B.kolibri_router_forward(x, w_router, beta, K, z=z, ids=ids, gates=gates, alpha=alpha)
    B.kolibri_eqb_update(z, alpha, beta, K, B.workspace(B.KOLIBRI_OP_EQB, N, E, K, device))
    B.kolibri_router_forward(x, w_router, beta, K, z=z, ids=ids, gates=gates, alpha=alpha)
    counts = torch.empty((E,), dtype=torch.int32, device=device)
    offsets = torch.empty((E + 1,), dtype=torch.int64, device=device)
    perm = torch.empty((N * K,), dtype=torch.int32, device=device)
    inv = torch.empty((N * K,), dtype=torch.int32, device=device)
    B.kolibri_expert_permute(ids, E, B.workspace(B.KOLIBRI_OP_PERMUTE, N, E, K, device), counts,
                             offsets, perm, inv)
    ws = B.expert_ffn_workspace(N, d, F, K, True, device)
    y = torch.empty((N, d), dtype=torch.float32, device=device)
    stream = torch.cuda.Stream(device)

    def once():
        B.kolibri_expert_ffn(x, perm, offsets, inv, gates, wgu, wd, wgu_s, wd_s, y=y, ws=ws,
                             stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            once()
    stream.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0] or "0")
    sampler.start()
    time.sleep(0.3)
    t0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            once()
    t1.record(stream)
    t1.synchronize()
    clocks = sampler.stop()
    st = B.kolibri_device_status(stream)
    if st != B.KOLIBRI_OK:
        raise RuntimeError(f"device status: {B.status_string(st)}")
    ms = t0.elapsed_time(t1) / args.steps
    c = counts.cpu().numpy()
    flops = 6.0 * d * F * N * (K + 1)
    bytes_alg = 2.0 * 3 * d * F * (E + 1) + 2.0 * N * d + 4.0 * N * d + 16.0 * N * K
    peaks = _peaks()
    achieved = flops / (ms * 1e-3) / 1e12
    # the oracle on a bounded sample: the first tokens of the same microbatch
    n = 8
    xs = x[:n].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    ids_h = ids[:n].cpu().numpy()
    used = np.unique(ids_h)
    remap = np.full(E, -1, np.int64)
    remap[used] = np.arange(len(used))
    sl = torch.from_numpy(used).to(device)
    wgu_h = wgu[sl].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    wd_h = wd[sl].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    wgu_sh = wgu_s.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    wd_sh = wd_s.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    gates_h = gates[:n].cpu().numpy()
    reps, cpu_s = 0, 0.0
    while cpu_s < 2.0:
        t = time.time()
        oracle.expert_ffn(xs, remap[ids_h].astype(np.int32), gates_h, wgu_h, wd_h, wgu_sh, wd_sh)
        cpu_s += time.time() - t
        reps += 1
    return {
        "metric": "expert layer (dispatch + grouped SwiGLU gate/up + down + combine, shared + 6 routed "
                  f"experts of 2560 -> 2x512 -> 2560, E={E}): tokens/s at N={N}",
        "part": "experts", "value": N / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "dtype": "bf16 in, fp32 accumulate", "data": "synthetic",
        "config": {"workload": "experts", "N": N, "d": d, "F": F, "E": E, "K": K,
                   "routing": "own forward after one EQB update",
                   "load_min_max": [int(c.min()), int(c.max())]},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": None,
                     "algorithmic": f"{flops / 1e12:.3f} TFLOP per layer (6 d F per token-expert); "
                                    f"{bytes_alg / 1e9:.2f} GB of weights, x and y "
                                    f"({bytes_alg / peaks['hbm_gbs'] / 1e6:.3f} ms at the HBM peak)",
                     "peak_kind": f"bf16 burst, of {peaks['source']}"},
        "clocks": clocks,
        "gpu_launches": 7,
        "cpu_baseline": {"value": n * reps / cpu_s, "unit": "tokens/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": f"first {n} tokens, {reps} times, {cpu_s:.1f} s"},
    }


# ---------------------------------------------------------------- decode

def _decode_oracle(oracle, wl, layers, xs, ws, betas):
    t = time.perf_counter()
    for l in layers:
        z = oracle.router_logits(xs[l], ws[l])
        ids, _, _ = oracle.select(z, betas[l], wl.K)
        oracle.permute(ids, wl.E)
    return time.perf_counter() - t


def _decode_e2e(args, wl, xs, ws, betas, stream, a, b):
    """The decode step through the public API with host buffers: every
    layer's tokens copied in from pinned host memory, the forward + grouping
    call per layer, and every layer's ids and gates read back, each step."""
    L, N, d, E, K = wl.layers, wl.N, wl.d, wl.E, wl.K
    dev = xs[0].device
    x_h = torch.stack([x.cpu() for x in xs]).pin_memory()
    ids = torch.empty((L, N, K), dtype=torch.int32, device=dev)
    gates = torch.empty((L, N, K), dtype=torch.float32, device=dev)
    ids_h = torch.empty((L, N, K), dtype=torch.int32, pin_memory=True)
    gates_h = torch.empty((L, N, K), dtype=torch.float32, pin_memory=True)
    z = torch.empty((N, E), dtype=torch.float32, device=dev)
    alpha = torch.empty((N,), dtype=torch.float32, device=dev)
    counts = torch.empty((E,), dtype=torch.int32, device=dev)
    offsets = torch.empty((E + 1,), dtype=torch.int64, device=dev)
    perm = torch.empty((N * K,), dtype=torch.int32, device=dev)
    inv = torch.empty((N * K,), dtype=torch.int32, device=dev)
    wsp = B.workspace(B.KOLIBRI_OP_PERMUTE, N, E, K, dev)

    def one():
        with torch.cuda.stream(stream):
            for l in range(L):
                xs[l].copy_(x_h[l], non_blocking=True)
                B.kolibri_router_forward_permute(xs[l], ws[l], betas[l], K, z=z, ids=ids[l],
                                                 gates=gates[l], alpha=alpha, counts=counts,
                                                 offsets=offsets, perm=perm, inv=inv, ws=wsp,
                                                 stream=stream)
            ids_h.copy_(ids, non_blocking=True)
            gates_h.copy_(gates, non_blocking=True)

    for _ in range(max(3, args.warmup)):
        one()
    stream.synchronize()
    a.record(stream)
    for _ in range(args.steps):
        one()
    b.record(stream)
    b.synchronize()
    us = a.elapsed_time(b) * 1e3 / args.steps
    return {"us_per_step": us, "unit": "us/step", "tokens": N, "path": "eager, one call per layer",
            "h2d_bytes_per_step": int(x_h.numel() * 2),
            "d2h_bytes_per_step": int(ids_h.numel() * 4 + gates_h.numel() * 4)}


def run_decode(args):
    """The decode sweep: per step, 50 layers of logits + top-K + gates + alpha
    + counts + stable permutation (kolibri_router_forward_permute) for N in
    (1, 8, 64, 256) tokens, every layer with its own x, W and beta.  Timed eager (one call per kernel per layer)
    and as one CUDA graph per step; the forward alone and the logits alone are
    timed the same way to show where the step goes.  The roofline is W
    streamed once from HBM per layer (1.97 MB)."""
    import oracle
    oracle.build()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    B.load()
    stream = torch.cuda.Stream(device)
    peaks = _peaks()
    per_n = {}
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0] or "0")
    sampler.start()
    for n_tok in workloads.DECODE_TOKENS:
        wl = workloads.decode_workload(n_tok)
        L, N, d, E, K = wl.layers, wl.N, wl.d, wl.E, wl.K
        xs = [workloads.make_x(wl, l).to(device) for l in range(L)]
        ws = [workloads.make_w(wl, l).to(device) for l in range(L)]
        betas = [workloads.make_beta(wl, l).to(device) for l in range(L)]
        z = torch.empty((N, E), dtype=torch.float32, device=device)
        ids = torch.empty((N, K), dtype=torch.int32, device=device)
        gates = torch.empty((N, K), dtype=torch.float32, device=device)
        alpha = torch.empty((N,), dtype=torch.float32, device=device)
        counts = torch.empty((E,), dtype=torch.int32, device=device)
        offsets = torch.empty((E + 1,), dtype=torch.int64, device=device)
        perm = torch.empty((N * K,), dtype=torch.int32, device=device)
        inv = torch.empty((N * K,), dtype=torch.int32, device=device)
        wsp = B.workspace(B.KOLIBRI_OP_PERMUTE, N, E, K, device)

        def step(part="step"):
            for l in range(L):
                if part == "logits":
                    B.kolibri_router_logits(xs[l], ws[l], z=z, stream=stream)
                    continue
                if part == "step":
                    B.kolibri_router_forward_permute(xs[l], ws[l], betas[l], K, z=z, ids=ids, gates=gates,
                                                     alpha=alpha, counts=counts, offsets=offsets,
                                                     perm=perm, inv=inv, ws=wsp, stream=stream)
                else:
                    B.kolibri_router_forward(xs[l], ws[l], betas[l], K, z=z, ids=ids, gates=gates,
                                             alpha=alpha, stream=stream)

        def timed(fn, reps):
            for _ in range(args.warmup):
                fn()
            stream.synchronize()
            a.record(stream)
            for _ in range(reps):
                fn()
            b.record(stream)
            b.synchronize()
            return a.elapsed_time(b) * 1e3 / reps

        res = {}
        with torch.cuda.stream(stream):
            res["eager_us"] = timed(step, args.steps)
            for part in ("step", "forward", "logits"):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=stream):
                    step(part)
                res[f"graph_us" if part == "step" else f"graph_{part}_us"] = timed(gr.replay, args.steps)
                del gr
        st = B.kolibri_device_status(stream)
        if st != B.KOLIBRI_OK:
            raise RuntimeError(f"device status: {B.status_string(st)}")
        res["graph_us_per_layer"] = res["graph_us"] / L
        if n_tok == workloads.DECODE_TOKENS[-1]:
            e2e = _decode_e2e(args, wl, xs, ws, betas, stream, a, b)
        # per layer: one launch up to 16 tokens (forward and grouping); else the forward (one launch
        # up to 96 tokens, else logits + selection) and the permutation
        res["gpu_launches"] = (1 if N <= 16 else 2 if N <= 96 else 3) * L
        res["w_bytes_per_step"] = 2 * E * d * L
        per_n[str(n_tok)] = res
    clocks = sampler.stop()
    # the oracle: one whole decode step at N = 8 (all 50 layers)
    wl = workloads.decode_workload(8)
    xs = [workloads.bf16_bits(workloads.make_x(wl, l)) for l in range(wl.layers)]
    wh = [workloads.bf16_bits(workloads.make_w(wl, l)) for l in range(wl.layers)]
    bh = [workloads.make_beta(wl, l).numpy() for l in range(wl.layers)]
    cpu_s = _decode_oracle(oracle, wl, range(wl.layers), xs, wh, bh)
    top = per_n[str(workloads.DECODE_TOKENS[-1])]
    e2e["value"] = e2e.pop("us_per_step")
    w_bytes = top["w_bytes_per_step"]
    achieved = w_bytes / (top["graph_us"] * 1e-6) / 1e9
    return {
        "metric": "decode step latency, 50 layers of logits + top-K + gates + permutation "
                  f"(d=2560, E=384, K=6), N={workloads.DECODE_TOKENS[-1]} tokens, CUDA graph",
        "part": "decode", "value": top["graph_us"], "unit": "us/step", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": top["graph_us"] * 1e-3,
        "higher_is_better": False, "dtype": "bf16 in, fp32 accumulate", "data": "synthetic",
        "config": {"workload": "decode", "layers": workloads.DECODE_LAYERS,
                   "tokens": list(workloads.DECODE_TOKENS), "d": 2560, "E": 384, "K": 6,
                   "inputs": "distinct x, W, beta per layer (98 MB of W per step, under L2 size)"},
        "per_n": per_n,
        "e2e": e2e,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                     "algorithmic": "W read once per layer: 2 E d bytes",
                     "peak_kind": f"HBM copy, of {peaks['source']}"},
        "clocks": clocks,
        "cpu_baseline": {"value": cpu_s * 1e6, "unit": "us/step", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": "one whole step at N=8 (50 layers)"},
    }


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)   # ~1 s timed: clock samples fall inside it
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="kolibri_n1m", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--tokens", type=int, default=0,
                    help="override N (smaller captures for the profiler only)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override E for --part experts (smaller captures for the profiler only)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--eqb", choices=["one", "split"], default="one",
                    help="split: the EQB update by the split-batch form even on one GPU")
    ap.add_argument("--decode", action="store_true",
                    help="time the decode sweep (50 layers, N = 1, 8, 64, 256; one GPU)")
    ap.add_argument("--part", choices=sorted(PARTS) + ["experts"], default=None,
                    help="time one balancing piece instead of the routing step (one GPU)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.decode and args.impl == "ours":
        print(json.dumps(run_decode(args)), flush=True)
        return
    if args.part == "experts" and args.impl == "ours":
        print(json.dumps(run_experts(args)), flush=True)
        return
    if args.part and args.impl == "ours":
        print(json.dumps(run_part(args)), flush=True)
        return
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
