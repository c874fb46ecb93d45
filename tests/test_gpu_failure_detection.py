"""Device-side failure detection, exercised without a fault: a bounded wait
that runs out (on a barrier nothing arrives at) records KOLIBRI_ERR_TIMEOUT,
its kernel returns, the status is read and cleared on the host, and the
context stays usable: the next call runs and is bit-exact."""
import time

import numpy as np
import pytest
import torch

from expert_load_balancing_b200 import binding as B

from gpu_helpers import assert_bit_equal, check_status, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(kolibri_lib):
    return kolibri_lib


@pytest.mark.parametrize("limit_ns", [1_000, 1_000_000, 50_000_000])
def test_bounded_wait_runs_out_and_reports_timeout(oracle_mod, limit_ns):
    torch.cuda.synchronize()
    assert B.kolibri_device_status() == B.KOLIBRI_OK
    t = time.perf_counter()
    B.kolibri_selftest_bounded_wait(limit_ns)
    st = B.kolibri_device_status()          # synchronises the stream
    waited = time.perf_counter() - t
    assert st == B.KOLIBRI_ERR_TIMEOUT, B.status_string(st)
    assert waited >= limit_ns * 1e-9         # it waited out its limit
    assert waited < limit_ns * 1e-9 + 1.0    # and then gave up
    assert B.kolibri_device_status() == B.KOLIBRI_OK       # read and cleared
    # the context still works: a routing call right after is exact
    rng = np.random.default_rng(limit_ns % 97)
    z = rng.standard_normal((300, 128)).astype(np.float32)
    beta = (0.1 * rng.standard_normal(128)).astype(np.float32)
    ids, gates, alpha = B.kolibri_router_topk(dev(z), dev(beta), 6)
    torch.cuda.synchronize()
    check_status()
    ids_o, gates_o, alpha_o = oracle_mod.select(z, beta, 6)
    assert_bit_equal(host(ids), ids_o, "ids")
    assert_bit_equal(host(gates), gates_o, "gates")
    assert_bit_equal(host(alpha), alpha_o, "alpha")


def test_timeout_on_a_side_stream_is_reported_there(oracle_mod):
    s = torch.cuda.Stream()
    B.kolibri_selftest_bounded_wait(2_000_000, stream=s)
    assert B.kolibri_device_status(s) == B.KOLIBRI_ERR_TIMEOUT
    assert B.kolibri_device_status() == B.KOLIBRI_OK
