"""The cross-rank plumbing of bench.py's multi-GPU path: the barrier, the
max-over-ranks reduction of device times, and the reference arm that runs on
rank 0 only.  (Its data-path exchange, the EQB update over the union of the
ranks' tokens, is distributed.eqb_update_split: tests/test_multirank_eqb.py
on gloo ranks, tests/test_gpu_multirank_eqb.py with the library's kernels.)
Checked here with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        got = bench.reduce_max_over_ranks(1.5 + rank, torch.device("cpu"))
        dist.barrier()
        # the reference arm runs on rank 0 only; other ranks return without work
        class A:
            workload, steps, warmup = "small_n256", 1, 0
        ref = bench.run_reference(A, rank, world) if rank != 0 else "skipped"
        out[rank] = (got, ref)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_reduction_and_reference_arm():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0][0] == pytest.approx(2.5) and out[1][0] == pytest.approx(2.5)
    assert out[1][1] is None


def test_single_process_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max_over_ranks(3.25, torch.device("cpu")) == 3.25
