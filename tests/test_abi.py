"""The C ABI loads, exports every declared symbol, and rejects bad arguments
on the host before anything reaches a GPU (no device needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kolibri_router.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"KOLIBRI_API\s+[\w\s\*]+?\b(kolibri_\w+)\s*\(", src)))


def test_header_declares_the_four_calls():
    names = _declared_functions()
    for n in ("kolibri_router_logits", "kolibri_router_topk", "kolibri_expert_permute",
              "kolibri_eqb_update"):
        assert n in names


def test_every_declared_symbol_is_exported(kolibri_lib):
    from expert_load_balancing_b200 import binding
    names = _declared_functions()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(kolibri_lib, n), n
        assert n in binding.SIGNATURES, n


def test_status_strings(kolibri_lib):
    from expert_load_balancing_b200 import binding
    assert binding.status_string(0) == "KOLIBRI_OK"
    assert binding.status_string(3) == "KOLIBRI_ERR_WORKSPACE_TOO_SMALL"
    assert binding.status_string(99) == "KOLIBRI_ERR_UNKNOWN"


def test_workspace_sizes(kolibri_lib):
    from expert_load_balancing_b200 import binding as B
    assert B.kolibri_workspace_bytes(B.KOLIBRI_OP_EQB, 0, 384, 6) == 0
    assert B.kolibri_workspace_bytes(B.KOLIBRI_OP_EQB, 16, 384, 384) == 0      # K >= E
    assert B.kolibri_workspace_bytes(99, 16, 384, 6) == 0
    small = B.kolibri_workspace_bytes(B.KOLIBRI_OP_EQB, 256, 384, 6)
    big = B.kolibri_workspace_bytes(B.KOLIBRI_OP_EQB, 1 << 20, 384, 6)
    assert 0 < small < big
    # large batches: sample keys + gather buffer + token bias, well under 1 GB
    assert big < (1 << 30)
    assert B.kolibri_workspace_bytes(B.KOLIBRI_OP_PERMUTE, 1 << 20, 384, 6) > 0


def test_binding_workspace_is_zero_filled(kolibri_lib):
    # the decode form of kolibri_router_forward_permute keeps a counter in the
    # permutation workspace that must be zero on first use: the binding's
    # buffers start zeroed, and a decode batch still gets a workspace
    from expert_load_balancing_b200 import binding as B
    for N in (1, 16, 4096):
        need = B.kolibri_workspace_bytes(B.KOLIBRI_OP_PERMUTE, N, 384, 6)
        assert need > 0
        ws = B.workspace(B.KOLIBRI_OP_PERMUTE, N, 384, 6, device="cpu")
        assert ws.numel() >= need and ws.dtype.itemsize == 1
        assert int(ws.count_nonzero()) == 0


def _call(lib, name, *args):
    return getattr(lib, name)(*args)


def test_host_validation_rejects_before_launch(kolibri_lib):
    lib = kolibri_lib
    P = ctypes.c_void_p
    fake = P(0x10000)       # aligned, never dereferenced: validation fails first
    odd = P(0x10004)
    # null pointers
    assert _call(lib, "kolibri_router_logits", None, fake, fake, 128, 2560, 384, None) == 1
    assert _call(lib, "kolibri_router_topk", None, None, 128, 384, 6, fake, fake, None, None) == 1
    # misaligned
    assert _call(lib, "kolibri_router_logits", odd, fake, fake, 128, 2560, 384, None) == 1
    # K >= E, K > 16, E % 4, E too large
    assert _call(lib, "kolibri_router_topk", fake, None, 128, 8, 8, fake, fake, None, None) == 1
    assert _call(lib, "kolibri_router_topk", fake, None, 128, 384, 17, fake, fake, None, None) == 2
    assert _call(lib, "kolibri_router_topk", fake, None, 128, 386, 6, fake, fake, None, None) == 2
    assert _call(lib, "kolibri_router_topk", fake, None, 128, 1024, 6, fake, fake, None, None) == 2
    # d not a multiple of 64, E not a multiple of 16
    assert _call(lib, "kolibri_router_logits", fake, fake, fake, 128, 2500, 384, None) == 2
    assert _call(lib, "kolibri_router_logits", fake, fake, fake, 128, 2560, 388, None) == 2
    # N < 1
    assert _call(lib, "kolibri_router_topk", fake, None, 0, 384, 6, fake, fake, None, None) == 1
    # N*K beyond int32 slot indices
    assert _call(lib, "kolibri_router_topk", fake, None, 1 << 29, 384, 6, fake, fake, None, None) == 2
    # workspace too small
    need = lib.kolibri_workspace_bytes(2, 1 << 20, 384, 6)
    assert _call(lib, "kolibri_eqb_update", fake, None, fake, 1 << 20, 384, 6, None, fake,
                 need - 1, None) == 3
    needp = lib.kolibri_workspace_bytes(1, 1 << 20, 384, 6)
    assert _call(lib, "kolibri_expert_permute", fake, 1 << 20, 384, 6, fake, fake, fake, None,
                 fake, needp - 1, None) == 3


def test_package_has_no_oracle_dependency():
    """The product package never imports the oracle (and vice versa)."""
    pkg = os.path.join(ROOT, "expert_load_balancing_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "kolibri_oracle" not in text, f
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith((".py", ".c")):
            text = open(os.path.join(ROOT, "oracle", f)).read()
            assert "expert_load_balancing_b200" not in text, f
            assert "kolibri_router.h" not in text, f


def test_library_refuses_to_run_without_extension(tmp_path):
    from expert_load_balancing_b200 import binding
    with pytest.raises(RuntimeError):
        binding._lib = None
        try:
            binding.load(str(tmp_path / "missing.so"))
        finally:
            binding._lib = None


def _noalloc_header_limit():
    src = open(HEADER).read()
    m = re.search(r"up to ([\d,]+) routed slots N\*K fit", src)
    assert m, "the header states the no-allocation limit"
    return int(m.group(1).replace(",", ""))


def test_noalloc_limit_is_the_largest_size_that_fits(kolibri_lib):
    """The figure the header gives for E = 384 is exactly the boundary of the
    fixed scratch array: that many slots fit, one more does not (host-side
    layout sizes only; K = 1 so that every slot count can be formed)."""
    from expert_load_balancing_b200 import binding as B
    limit = _noalloc_header_limit()
    cap = B.KOLIBRI_NOALLOC_SCRATCH_BYTES
    assert B.kolibri_workspace_bytes(B.KOLIBRI_OP_PERMUTE, limit, 384, 1) <= cap
    assert B.kolibri_workspace_bytes(B.KOLIBRI_OP_PERMUTE, limit + 1, 384, 1) > cap
    # the figure does not depend on how the slots split into tokens and ranks
    assert B.kolibri_workspace_bytes(B.KOLIBRI_OP_PERMUTE, limit // 8, 384, 8) <= cap


def test_noalloc_refuses_oversized_on_the_host(kolibri_lib):
    """The size check runs before any CUDA call, so with placeholder pointers
    an oversized call is refused without a device.  Skipped where a GPU is
    present: there the GPU test checks the refusal with real buffers."""
    from conftest import gpu_available
    if gpu_available():
        pytest.skip("covered with real buffers by the GPU test")
    from expert_load_balancing_b200 import binding as B
    limit = _noalloc_header_limit()
    fake = ctypes.c_void_p(0x1000)
    st = kolibri_lib.kolibri_expert_permute_noalloc(fake, limit + 1, 384, 1, fake, fake, fake,
                                                    None, None)
    assert st == B.KOLIBRI_ERR_WORKSPACE_TOO_SMALL
