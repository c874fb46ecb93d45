"""EQB over a batch split across ranks ("Kolibri Pre-Training from Scratch"
7.3): expert_load_balancing_b200.distributed sums the per-rank 256-bin
histograms with an all-reduce between the passes (two for the pages' bf16
keys, four for the fp32 keys of the main update).  Run here with
two and three gloo ranks on the CPU; the three library calls are replaced by
CPU stand-ins built from the oracle's bf16 rounding and key (the GPU kernels
behind them are checked against the oracle in test_gpu_balance.py).  Every
rank must end with the exact quantile of the union and the same bias; the
pages' counter-example shows that averaging per-rank quantiles would not.
A rank that exits or stalls between steps makes the survivor's next
all-reduce end with an error, not wait for good."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _CpuOps:
    """The three per-rank calls on the CPU (test stand-ins)."""

    def __init__(self, oracle):
        self.o = oracle

    def _keys(self, z, alpha):
        zz = z.numpy()
        a = np.zeros(zz.shape[0], np.float32) if alpha is None else alpha.numpy()
        keys = np.empty(zz.shape, np.int64)
        for t in range(zz.shape[0]):
            for e in range(zz.shape[1]):
                keys[t, e] = self.o.bf16_key(self.o.bf16_round(np.float32(zz[t, e] + a[t])))
        return keys

    def histogram(self, z, alpha, prefix, hist):
        keys = self._keys(z, alpha)
        for e in range(keys.shape[1]):
            k = keys[:, e]
            if prefix is None:
                b = k >> 8
            else:
                b = (k & 0xff)[(k >> 8) == int(prefix[e])]
            hist[e] += torch.from_numpy(np.bincount(b, minlength=256).astype(np.int32))
        return hist

    def digit(self, hist, rank, digit):
        for e in range(hist.shape[0]):
            r = int(rank[e])
            above = 0
            for b in range(255, -1, -1):
                c = int(hist[e, b])
                if above + c > r:
                    digit[e] = b
                    rank[e] = r - above
                    break
                above += c
        return digit

    def bias(self, d_hi, d_lo, bias, quantiles):
        v = np.empty(bias.shape[0], np.float32)
        for e in range(bias.shape[0]):
            k = (int(d_hi[e]) << 8) | int(d_lo[e])
            b = (k & 0x7fff) if (k & 0x8000) else (~k & 0xffff)
            v[e] = np.frombuffer(np.uint32(b << 16).tobytes(), np.float32)[0]
        quantiles.copy_(torch.from_numpy(v))
        bias.copy_(torch.from_numpy(self.o.eqb_bias(v)))
        return bias, quantiles


class _CpuKeyOps:
    """The three per-rank calls of the fp32-key passes on the CPU (test stand-ins)."""

    def __init__(self, oracle):
        self.o = oracle

    def histogram(self, z, alpha, p, prefix, hist):
        zz = z.numpy()
        a = np.zeros(zz.shape[0], np.float32) if alpha is None else alpha.numpy()
        keys = self.o.order_key_array((zz + a[:, None]).astype(np.float32)).astype(np.int64)
        shift = 24 - 8 * p
        for e in range(keys.shape[1]):
            k = keys[:, e]
            if p:
                hi = (0xffffffff << (shift + 8)) & 0xffffffff
                k = k[(k & hi) == (int(prefix[e]) & 0xffffffff & hi)]
            hist[e] += torch.from_numpy(np.bincount((k >> shift) & 0xff, minlength=256).astype(np.int32))
        return hist

    def digit(self, hist, p, rank, prefix):
        shift = 24 - 8 * p
        for e in range(hist.shape[0]):
            r = int(rank[e])
            above = 0
            for b in range(255, -1, -1):
                c = int(hist[e, b])
                if above + c > r:
                    keep = 0 if p == 0 else (int(prefix[e]) & 0xffffffff) & ((0xffffffff << (shift + 8)) & 0xffffffff)
                    prefix[e] = np.int64(keep | (b << shift)).astype(np.uint32).view(np.int32)
                    rank[e] = r - above
                    break
                above += c
        return prefix

    def bias(self, key, bias, quantiles):
        k = key.numpy().view(np.uint32)
        u = np.where(k & 0x80000000, k & 0x7fffffff, ~k & 0xffffffff).astype(np.uint32)
        v = u.view(np.float32)
        quantiles.copy_(torch.from_numpy(v.copy()))
        bias.copy_(torch.from_numpy(self.o.eqb_bias(v)))
        return bias, quantiles


class _CpuSplitOps:
    """The per-rank calls of the sampled-bracket form on the CPU (test
    stand-ins).  miss=True brackets every expert away from its target, so
    the update has to take its four-pass fallback."""

    def __init__(self, oracle, miss=False):
        self.o = oracle
        self.miss = miss
        self.key_ops = _CpuKeyOps(oracle)

    def _keys(self, z, alpha):
        zz, a = z.numpy(), alpha.numpy()
        return self.o.order_key_array((zz + a[:, None]).astype(np.float32)).astype(np.int64)

    def sample(self, z, alpha, K, S, sample):
        N = z.shape[0]
        keys = self._keys(z, alpha)[np.arange(S) * (N // S)]
        sample.copy_(torch.from_numpy(keys.T.astype(np.uint32).view(np.int32).copy()))
        return sample

    def brackets(self, gathered, n_total, K, scratch, lo, hi):
        R, E, S = gathered.shape
        m = (n_total * K) // E
        q = (m + 1) / n_total
        c = q * R * S
        margin = int(np.ceil(6 * np.sqrt(c * (1 - q)))) + 8
        r_hi = max(0, int(np.floor(c)) - margin)
        r_lo = min(R * S - 1, int(np.ceil(c)) + margin)
        for e in range(E):
            k = np.sort(gathered[:, e, :].numpy().view(np.uint32).reshape(-1).astype(np.int64))[::-1]
            if self.miss:          # a bracket above every key: the target is never inside
                a = b = int(k[0])
            else:
                a, b = int(k[r_hi]), int(k[r_lo])
            hi[e] = np.int64(a).astype(np.uint32).view(np.int32)
            lo[e] = np.int64(b).astype(np.uint32).view(np.int32)
        return lo, hi

    def count(self, z, alpha, K, lo, hi, counts, cand):
        keys = self._keys(z, alpha)
        E, cap = cand.shape
        for e in range(E):
            l_, h_ = int(lo[e]) & 0xffffffff, int(hi[e]) & 0xffffffff
            k = keys[:, e]
            inside = k[(k >= l_) & (k <= h_)]
            counts[0, e] = int((k > h_).sum())
            counts[1, e] = int(inside.shape[0])
            counts[2, e] = 1 if inside.shape[0] > cap else 0
            n = min(cap, inside.shape[0])
            cand[e, :n] = torch.from_numpy(inside[:n].astype(np.uint32).view(np.int32).copy())
        return counts, cand

    def rank(self, counts_sum, n_total, K, rank, flag):
        E = counts_sum.shape[1]
        m = (n_total * K) // E
        for e in range(E):
            above, inside, over = (int(counts_sum[i, e]) for i in range(3))
            ok = over == 0 and above <= m < above + inside
            rank[e] = m - above if ok else 0
            flag[e] = 0 if ok else 1
        return rank, flag

    def histogram(self, cand, counts, p, prefix, hist):
        shift = 24 - 8 * p
        E, cap = cand.shape
        for e in range(E):
            k = cand[e, :min(cap, int(counts[1, e]))].numpy().view(np.uint32).astype(np.int64)
            if p:
                hi = (0xffffffff << (shift + 8)) & 0xffffffff
                k = k[(k & hi) == (int(prefix[e]) & 0xffffffff & hi)]
            hist[e] += torch.from_numpy(np.bincount((k >> shift) & 0xff, minlength=256).astype(np.int32))
        return hist

    def digit(self, hist, p, rank, prefix):
        return self.key_ops.digit(hist, p, rank, prefix)

    def bias(self, key, bias, quantiles):
        return self.key_ops.bias(key, bias, quantiles)


class _CountingKeyOps(_CpuKeyOps):
    """The four-pass stand-ins, counting how often the fallback runs."""
    calls = 0

    def histogram(self, *a):
        type(self).calls += 1
        return super().histogram(*a)


def _worker(rank, world, port, z_parts, a_parts, K, out, fp32=False, split=None):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from expert_load_balancing_b200 import distributed as D
        z = torch.from_numpy(z_parts[rank])
        a = torch.from_numpy(a_parts[rank])
        n_total = sum(p.shape[0] for p in z_parts)
        bias = torch.zeros(z.shape[1])
        fell_back = 0
        if split is not None:
            _CountingKeyOps.calls = 0
            _, q = D.eqb_update_split(z, a, bias, K, n_total,
                                      ops=_CpuSplitOps(oracle, miss=split.get("miss", False)),
                                      cap=split.get("cap", 64), fallback_ops=_CountingKeyOps(oracle))
            fell_back = _CountingKeyOps.calls
        elif fp32:
            _, q = D.eqb_update_distributed(z, a, bias, K, n_total, ops=_CpuKeyOps(oracle))
        else:
            _, q = D.eqb_update_bf16_distributed(z, a, bias, K, n_total, ops=_CpuOps(oracle))
        out[rank] = (q.numpy().copy(), bias.numpy().copy(), fell_back)
    finally:
        dist.destroy_process_group()


def _run(z_parts, a_parts, K, fp32=False, split=None):
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    world = len(z_parts)
    procs = [ctx.Process(target=_worker, args=(r, world, port, z_parts, a_parts, K, out, fp32, split))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    return [out[r] for r in range(world)]


def test_pages_counter_example_two_ranks(oracle_mod):
    # 7.3: column e1 + alpha is (3.0, 1.5) on rank A and (0.5, 3.0) on rank B;
    # the exact Q_2 of the union is 1.5, the average of local quantiles 1.0
    za = np.array([[3.0, 0.0], [1.5, 0.0]], np.float32)
    zb = np.array([[0.5, 0.0], [3.0, 0.0]], np.float32)
    zero = np.zeros(2, np.float32)
    res = _run([za, zb], [zero, zero], K=1)        # N = 4, E = 2, K = 1: m = 2
    for q, b, _ in res:
        assert q[0] == np.float32(1.5)
    np.testing.assert_array_equal(res[0][1], res[1][1])
    local = [oracle_mod.column_quantiles_bf16(p, None, 1)[0] for p in (za, zb)]   # r = 1 each
    assert np.mean(local) == 1.0 != 1.5


def test_three_ranks_equal_the_union(oracle_mod):
    rng = np.random.default_rng(0)
    E, K = 6, 2
    sizes = [17, 30, 9]
    z_parts = [(rng.standard_normal((n, E)) * 2).astype(np.float32) for n in sizes]
    z_parts[1][:, 2] = 0.5                         # ties across ranks
    a_parts = [(rng.standard_normal(n) * 0.3).astype(np.float32) for n in sizes]
    res = _run(z_parts, a_parts, K)
    z = np.concatenate(z_parts)
    a = np.concatenate(a_parts)
    m = (z.shape[0] * K) // E
    v = oracle_mod.column_quantiles_bf16(z, a, m)
    for q, b, _ in res:
        np.testing.assert_array_equal(q, v)
        np.testing.assert_array_equal(b, oracle_mod.eqb_bias(v))


def test_fp32_keys_pages_counter_example(oracle_mod):
    # the same counter-example through the fp32-key passes of the main update
    za = np.array([[3.0, 0.0], [1.5, 0.0]], np.float32)
    zb = np.array([[0.5, 0.0], [3.0, 0.0]], np.float32)
    zero = np.zeros(2, np.float32)
    res = _run([za, zb], [zero, zero], K=1, fp32=True)
    for q, b, _ in res:
        assert q[0] == np.float32(1.5)
    np.testing.assert_array_equal(res[0][1], res[1][1])


def test_fp32_keys_three_ranks_equal_the_union(oracle_mod):
    rng = np.random.default_rng(1)
    E, K = 8, 3
    sizes = [23, 11, 40]
    z_parts = [(rng.standard_normal((n, E)) * 2).astype(np.float32) for n in sizes]
    z_parts[0][:, 1] = -0.0                           # signed zeros and ties across ranks
    z_parts[2][:5, 1] = 0.0
    z_parts[1][:, 4] = 0.75
    a_parts = [(rng.standard_normal(n) * 0.3).astype(np.float32) for n in sizes]
    a_parts[0][:] = 0.0
    res = _run(z_parts, a_parts, K, fp32=True)
    z = np.concatenate(z_parts)
    a = np.concatenate(a_parts)
    m = (z.shape[0] * K) // E
    v = oracle_mod.column_quantiles(z, a, m)
    for q, b, _ in res:
        np.testing.assert_array_equal(q, v)
        np.testing.assert_array_equal(b, oracle_mod.eqb_bias(v))



# ------------------------------------------- the sampled-bracket split form

def test_split_pages_counter_example(oracle_mod):
    # the counter-example through the sampled-bracket form: exact 1.5 on both
    # ranks, where averaging the local quantiles gives 1.0
    za = np.array([[3.0, 0.0], [1.5, 0.0]], np.float32)
    zb = np.array([[0.5, 0.0], [3.0, 0.0]], np.float32)
    zero = np.zeros(2, np.float32)
    res = _run([za, zb], [zero, zero], K=1, split={})
    for q, b, fell_back in res:
        assert q[0] == np.float32(1.5)
        assert fell_back == 0
    np.testing.assert_array_equal(res[0][1], res[1][1])


def _split_parts(seed, sizes, E):
    rng = np.random.default_rng(seed)
    z_parts = [(rng.standard_normal((n, E)) * 2).astype(np.float32) for n in sizes]
    z_parts[0][:, 1] = -0.0                           # signed zeros and ties across ranks
    z_parts[2][:7, 1] = 0.0
    z_parts[1][:, 4] = 0.75
    a_parts = [(rng.standard_normal(n) * 0.3).astype(np.float32) for n in sizes]
    return z_parts, a_parts


@pytest.mark.parametrize("case", ["bracket", "miss", "overflow"])
def test_split_three_ranks_equal_the_union(oracle_mod, case):
    """Three ranks of unequal size: every rank ends with the oracle's exact
    quantile of the union and its bias.  "bracket": the sampled bracket holds
    the target (no fallback); "miss": the bracket misses every target;
    "overflow": a rank's gather buffer is too small; both finish by the
    four-pass form, with the same exact result."""
    E, K = 8, 3
    z_parts, a_parts = _split_parts(2, [300, 120, 257], E)
    split = {"bracket": {"cap": 4096}, "miss": {"miss": True, "cap": 4096},
             "overflow": {"cap": 3}}[case]
    res = _run(z_parts, a_parts, K, split=split)
    z = np.concatenate(z_parts)
    a = np.concatenate(a_parts)
    m = (z.shape[0] * K) // E
    v = oracle_mod.column_quantiles(z, a, m)
    for q, b, fell_back in res:
        np.testing.assert_array_equal(q, v)
        np.testing.assert_array_equal(b, oracle_mod.eqb_bias(v))
        assert (fell_back > 0) == (case != "bracket")


def _worker_peer_lost(rank, world, port, out, mode):
    """Rank 1 fails right after joining: it exits ("exit") or stays alive
    without entering any collective ("stall").  Rank 0 then runs the update,
    whose first histogram all-reduce must end in an error, not wait for good."""
    import sys
    import time
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        out[1] = "left"
        if mode == "stall":
            time.sleep(15)
        os._exit(0)            # no destroy, no collective: the peer is gone
    import oracle
    from expert_load_balancing_b200 import distributed as D
    rng = np.random.default_rng(5)
    z = torch.from_numpy((rng.standard_normal((12, 4)) * 2).astype(np.float32))
    a = torch.zeros(12)
    bias = torch.zeros(4)
    t = time.time()
    try:
        D.eqb_update_distributed(z, a, bias, 2, 24, ops=_CpuKeyOps(oracle))
        out[0] = ("finished", time.time() - t)
    except Exception as e:          # the collective reports the lost peer
        out[0] = ("error", time.time() - t, type(e).__name__)
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


@pytest.mark.parametrize("mode", ["exit", "stall"])
def test_lost_rank_ends_the_update_with_an_error(mode):
    # host-side failure between steps: a rank that exits, or one that never
    # joins the next collective; the survivor's all-reduce fails (at once, or
    # after the process group's 5 s timeout) instead of hanging
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker_peer_lost, args=(r, 2, port, out, mode)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not end")
    assert out[1] == "left"
    res = out[0]
    assert res[0] == "error", res
    assert res[1] < 14.0, res          # ended by the error, before the stalled rank left
