"""EQB over a batch split across ranks with the library's own kernels in
every rank ("Kolibri Pre-Training from Scratch" 7.3): two processes on one
GPU, each holding half of the tokens, run the sampled-bracket form
(distributed.eqb_update_split) and the four-pass form
(distributed.eqb_update_distributed).  Their counts and samples cross ranks
through a gloo process group on host copies (HostComm): the kernels of the
two processes never wait on one another, only the host exchange does.
Every rank must end with the oracle's exact quantile of the union, which is
also what kolibri_eqb_update gives on the whole batch on one GPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from gpu_helpers import dev, host

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, z_parts, a_parts, K, cap, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        torch.cuda.set_device(0)
        from expert_load_balancing_b200 import binding as B
        from expert_load_balancing_b200 import distributed as D
        B.load()
        z = torch.from_numpy(z_parts[rank]).cuda()
        a = torch.from_numpy(a_parts[rank]).cuda()
        n_total = sum(p.shape[0] for p in z_parts)
        comm = D.HostComm()
        res = {}
        bias = torch.zeros(z.shape[1], device="cuda")
        _, q = D.eqb_update_split(z, a, bias, K, n_total, comm=comm, cap=cap)
        torch.cuda.synchronize()
        res["split"] = (q.cpu().numpy().copy(), bias.cpu().numpy().copy())
        bias = torch.zeros(z.shape[1], device="cuda")
        _, q = D.eqb_update_distributed(z, a, bias, K, n_total, comm=comm)
        torch.cuda.synchronize()
        res["four_pass"] = (q.cpu().numpy().copy(), bias.cpu().numpy().copy())
        res["status"] = B.kolibri_device_status()
        out[rank] = res
    finally:
        dist.destroy_process_group()


def _run(z_parts, a_parts, K, cap):
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    world = len(z_parts)
    procs = [ctx.Process(target=_worker, args=(r, world, port, z_parts, a_parts, K, cap, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not end")
        assert p.exitcode == 0
    return [out[r] for r in range(world)]


def _check(oracle_mod, res, z_parts, a_parts, K):
    from expert_load_balancing_b200 import binding as B
    z = np.concatenate(z_parts)
    a = np.concatenate(a_parts)
    m = (z.shape[0] * K) // z.shape[1]
    v = oracle_mod.column_quantiles(z, a, m)
    b = oracle_mod.eqb_bias(v)
    # the one-GPU update on the whole batch gives the same
    bias1 = torch.zeros(z.shape[1], device="cuda")
    _, q1 = B.kolibri_eqb_update(dev(z), dev(a), bias1, K)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(q1).view(np.uint32), v.view(np.uint32))
    for r in res:
        assert r["status"] == B.KOLIBRI_OK
        for form in ("split", "four_pass"):
            q, bb = r[form]
            np.testing.assert_array_equal(q.view(np.uint32), v.view(np.uint32), err_msg=form)
            np.testing.assert_array_equal(bb.view(np.uint32), b.view(np.uint32), err_msg=form)


def test_two_ranks_pages_counter_example(oracle_mod):
    # 7.3: column e1 + alpha is (3.0, 1.5) on rank A and (0.5, 3.0) on rank B;
    # the exact Q_2 of the union is 1.5 (averaging local quantiles gives 1.0)
    E = 4
    za = np.zeros((2, E), np.float32)
    zb = np.zeros((2, E), np.float32)
    za[:, 0] = (3.0, 1.5)
    zb[:, 0] = (0.5, 3.0)
    zero = np.zeros(2, np.float32)
    res = _run([za, zb], [zero, zero], K=2, cap=64)          # N = 4, E = 4, K = 2: m = 2
    for r in res:
        assert r["split"][0][0] == np.float32(1.5)
        assert r["four_pass"][0][0] == np.float32(1.5)
    _check(oracle_mod, res, [za, zb], [zero, zero], K=2)


@pytest.mark.parametrize("cap", [65536, 16])   # 16: every gather overflows, four-pass fallback
def test_two_ranks_kolibri_shape(oracle_mod, cap):
    from expert_load_balancing_b200 import workloads
    E, K, n = 384, 6, 40000
    z = workloads.random_logits(2 * n, E, seed=21)
    z[:, 5] = np.where(z[:, 5] > 0, np.float32(0.0), np.float32(-0.0))     # signed zeros
    z[: n // 2, 9] = np.float32(0.25)                                     # ties across ranks
    a = (np.random.default_rng(22).standard_normal(2 * n) * 0.5 - 2.0).astype(np.float32)
    z_parts, a_parts = [z[:n], z[n:]], [a[:n], a[n:]]
    res = _run(z_parts, a_parts, K, cap)
    _check(oracle_mod, res, z_parts, a_parts, K)
