"""kolibri_expert_permute_noalloc: the permutation for callers that may not
allocate device memory (servers that pre-reserve the whole GPU for their own
pool, plugins inside another runtime's memory budget).  It must give exactly
what kolibri_expert_permute gives with a caller workspace, call after call,
and refuse sizes whose scratch would not fit the library's fixed array.

This file is named to run last, so a failure here does not hide the rest of
the suite; it also passes when run alone in a fresh process."""
import numpy as np
import pytest
import torch

from expert_load_balancing_b200 import binding as B

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(kolibri_lib):
    return kolibri_lib


def _ids(N, E, K, seed):
    rng = np.random.default_rng(seed)
    ids = np.argsort(rng.random((N, E)), axis=1)[:, :K].astype(np.int32)
    return torch.from_numpy(ids).cuda()


@pytest.mark.parametrize("N,E,K", [(300000, 384, 6), (65536, 128, 8), (500, 384, 6)])
def test_noalloc_matches_workspace_version_twice(N, E, K):
    for call, seed in enumerate((1, 2)):          # two calls in a row, different inputs
        ids = _ids(N, E, K, seed + N)
        want = B.kolibri_expert_permute(ids, E)
        got = B.kolibri_expert_permute_noalloc(ids, E)
        torch.cuda.synchronize()
        for g, w, name in zip(got, want, ("counts", "offsets", "perm", "inv")):
            assert torch.equal(g, w), f"call {call}: {name} differs"
    assert B.kolibri_device_status() == B.KOLIBRI_OK


def test_noalloc_refuses_oversized():
    """One slot beyond the fixed array is refused before anything is enqueued.
    Every buffer has the size the arguments imply (ids, perm and inv of N*K
    entries), so even a call that got past the size check would stay inside
    the caller's buffers."""
    import ctypes
    E, K = 384, 1
    N = 11_173_888 + 1                            # the header's limit, plus one slot
    ids = torch.zeros((N, K), dtype=torch.int32, device="cuda")
    counts = torch.empty((E,), dtype=torch.int32, device="cuda")
    offsets = torch.empty((E + 1,), dtype=torch.int64, device="cuda")
    perm = torch.empty((N * K,), dtype=torch.int32, device="cuda")
    inv = torch.empty((N * K,), dtype=torch.int32, device="cuda")
    st = B.load().kolibri_expert_permute_noalloc(
        ctypes.c_void_p(ids.data_ptr()), N, E, K, ctypes.c_void_p(counts.data_ptr()),
        ctypes.c_void_p(offsets.data_ptr()), ctypes.c_void_p(perm.data_ptr()),
        ctypes.c_void_p(inv.data_ptr()), None)
    assert st == B.KOLIBRI_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    assert B.kolibri_device_status() == B.KOLIBRI_OK
