"""Shared helpers of the GPU parity tests: run the CUDA path through the C
ABI and compare with the oracle."""
import numpy as np
import torch

from expert_load_balancing_b200 import binding as B


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)) if isinstance(a, np.ndarray) else a
    if dtype is not None:
        t = t.to(dtype)
    return t.contiguous().cuda()


def host(t):
    return t.detach().cpu().numpy()


def bits(a):
    a = np.ascontiguousarray(a)
    return a.view(np.uint32) if a.dtype == np.float32 else a


def assert_bit_equal(got, want, what):
    got, want = np.asarray(got), np.asarray(want)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    g, w = bits(got), bits(want)
    bad = np.nonzero(g != w)
    if bad[0].size:
        idx = tuple(b[0] for b in bad)
        raise AssertionError(f"{what}: {bad[0].size} mismatches, first at {idx}: "
                             f"got {got[idx]!r} want {want[idx]!r}")


def logits_tol(z_ref):
    """Router logits contract: |dZ| <= 1e-3 * max(1, |Z|) (bf16 inputs, fp32 sums)."""
    return 1e-3 * np.maximum(1.0, np.abs(z_ref))


def assert_logits_close(z_gpu, z_ref):
    err = np.abs(z_gpu.astype(np.float64) - z_ref.astype(np.float64))
    tol = logits_tol(z_ref)
    assert (err <= tol).all(), f"max |dZ| = {err.max()} (tol at worst {tol.flat[np.argmax(err - tol)]})"
    return float(err.max())


def gpu_select(z, beta, K):
    zt = dev(z)
    bt = None if beta is None else dev(beta)
    ids, gates, alpha = B.kolibri_router_topk(zt, bt, K)
    return host(ids), host(gates), host(alpha)


def gpu_permute(ids, E):
    counts, offsets, perm, inv = B.kolibri_expert_permute(dev(ids), E)
    return host(counts), host(offsets), host(perm), host(inv)


def gpu_eqb(z, alpha, beta_in, K):
    zt = dev(z)
    at = None if alpha is None else dev(alpha)
    bt = dev(beta_in.copy())
    bias, q = B.kolibri_eqb_update(zt, at, bt, K)
    return host(bias), host(q)


def check_status():
    st = B.kolibri_device_status()
    assert st == B.KOLIBRI_OK, B.status_string(st)
