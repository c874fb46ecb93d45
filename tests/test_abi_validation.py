"""Host-side argument checks of every entry point beyond the four core calls
(no device needed: each case fails validation before anything is enqueued,
so no CUDA call is made).  Status codes: 1 invalid argument, 2 unsupported
shape, 3 workspace too small."""
import pytest

INVALID, SHAPE, SMALL = 1, 2, 3
F = 0x10000        # a 16-byte aligned address that is never dereferenced
ODD = 0x10004      # a misaligned one


@pytest.fixture(scope="module")
def lib(kolibri_lib):
    return kolibri_lib


def test_forward_permute_checks(lib):
    f = lib.kolibri_router_forward_permute
    #            x  w  bias z  N    d     E    K  ids gates alpha counts offsets perm inv ws ws_bytes stream
    assert f(F, F, None, F, 128, 2560, 384, 6, F, F, F, None, F, F, None, F, 1 << 30, None) == INVALID
    assert f(ODD, F, None, F, 128, 2560, 384, 6, F, F, F, F, F, F, None, F, 1 << 30, None) == INVALID
    assert f(F, F, None, F, 128, 2500, 384, 6, F, F, F, F, F, F, None, F, 1 << 30, None) == SHAPE
    assert f(F, F, None, F, 128, 2560, 384, 384, F, F, F, F, F, F, None, F, 1 << 30, None) == INVALID
    # a batch too large for the one-block grouping needs a workspace of the permutation's size
    n = 1 << 20
    need = lib.kolibri_workspace_bytes(1, n, 384, 6)
    assert need > 0
    assert f(F, F, None, F, n, 2560, 384, 6, F, F, F, F, F, F, None, None, 0, None) == INVALID
    assert f(F, F, None, F, n, 2560, 384, 6, F, F, F, F, F, F, None, F, need - 1, None) == SMALL


def test_forward_eqb_and_route_balance_checks(lib):
    need = lib.kolibri_workspace_bytes(2, 4096, 384, 6)
    f = lib.kolibri_router_forward_eqb
    #            x  w  bias  z  N     d     E    K  ids gates alpha q  ws ws_bytes stream
    assert f(F, F, None, F, 4096, 2560, 384, 6, F, F, None, None, F, need, None) == INVALID   # bias is in/out
    assert f(F, F, F, F, 4096, 2560, 384, 6, F, F, None, None, None, need, None) == INVALID
    assert f(F, F, F, F, 4096, 2560, 390, 6, F, F, None, None, F, need, None) == SHAPE
    assert f(F, F, F, F, 4096, 2560, 384, 6, F, F, None, None, F, need - 1, None) == SMALL
    g = lib.kolibri_route_and_balance
    #            z  bias N     E    K  ids gates alpha q   ws ws_bytes stream
    assert g(F, F, 4096, 384, 6, None, F, None, None, F, need, None) == INVALID
    assert g(F, ODD, 4096, 384, 6, F, F, None, None, F, need, None) == INVALID
    assert g(F, F, 4096, 384, 17, F, F, None, None, F, need, None) == SHAPE
    assert g(F, F, 4096, 384, 6, F, F, None, None, F, need - 1, None) == SMALL


def test_bf16_eqb_checks(lib):
    need = lib.kolibri_workspace_bytes(3, 4096, 384, 6)
    assert need > 0
    f = lib.kolibri_eqb_update_bf16
    #            z  alpha bias N     E    K  q     ws ws_bytes stream
    assert f(F, None, F, 4096, 384, 6, None, F, need - 1, None) == SMALL
    assert f(F, None, None, 4096, 384, 6, None, F, need, None) == INVALID
    assert f(ODD, None, F, 4096, 384, 6, None, F, need, None) == INVALID
    h = lib.kolibri_eqb_bf16_histogram
    #            z  alpha N    E    prefix hist stream
    assert h(F, None, 0, 384, None, F, None) == INVALID
    assert h(F, None, 64, 6, None, F, None) == SHAPE
    assert h(F, None, 64, 516, None, F, None) == SHAPE
    assert h(ODD, None, 64, 384, None, F, None) == INVALID
    assert h(F, None, 64, 384, None, None, None) == INVALID
    assert lib.kolibri_eqb_bf16_digit(F, 0, F, F, None) == SHAPE
    assert lib.kolibri_eqb_bf16_digit(F, 384, None, F, None) == INVALID
    assert lib.kolibri_eqb_bf16_bias(F, F, 384, F, None, None) == INVALID
    assert lib.kolibri_eqb_bf16_bias(F, F, 513, F, F, None) == SHAPE


def test_fp32_key_passes_checks(lib):
    h = lib.kolibri_eqb_key_histogram
    #            z  alpha N    E    pass prefix hist stream
    assert h(F, None, 64, 384, 4, F, F, None) == INVALID
    assert h(F, None, 64, 384, -1, F, F, None) == INVALID
    assert h(F, None, 64, 384, 1, None, F, None) == INVALID        # passes 1-3 need the prefix
    assert h(F, None, 64, 10, 0, None, F, None) == SHAPE
    assert h(F, None, 0, 384, 0, None, F, None) == INVALID
    assert lib.kolibri_eqb_key_digit(F, 384, 4, F, F, None) == INVALID
    assert lib.kolibri_eqb_key_digit(F, 384, 0, F, None, None) == INVALID
    assert lib.kolibri_eqb_key_digit(F, 600, 0, F, F, None) == SHAPE
    assert lib.kolibri_eqb_key_bias(None, 384, F, F, None) == INVALID
    assert lib.kolibri_eqb_key_bias(F, 0, F, F, None) == SHAPE


def test_split_eqb_checks(lib):
    # the sampled-bracket form over a split batch: every argument error is
    # refused on the host before anything is enqueued
    smp = lib.kolibri_eqb_split_sample
    #            z  alpha N    E    K  S     sample stream
    assert smp(F, F, 1000, 384, 6, 0, F, None) == INVALID
    assert smp(F, F, 1000, 384, 6, 1001, F, None) == INVALID       # S > N
    assert smp(F, None, 1000, 384, 6, 100, F, None) == INVALID     # alpha is required
    assert smp(ODD, F, 1000, 384, 6, 100, F, None) == INVALID
    assert smp(F, F, 1000, 386, 6, 100, F, None) == SHAPE          # E % 4
    br = lib.kolibri_eqb_split_brackets
    #           sample R  S    E    N_total K scratch lo hi stream
    assert br(F, 0, 100, 384, 1000, 6, F, F, F, None) == INVALID
    assert br(F, 4, 300, 384, 1000, 6, F, F, F, None) == INVALID      # R S > N_total
    assert br(F, 2, 100, 384, 1000, 6, F, F, None, None) == INVALID
    assert br(F, 2, 100, 384, 1000, 6, ODD, F, F, None) == INVALID    # scratch 16-byte aligned
    assert br(F, 2, 100, 384, 1000, 400, F, F, F, None) == INVALID    # K >= E
    cnt = lib.kolibri_eqb_split_count
    #            z  alpha N    E    K  lo hi counts cand cap stream
    assert cnt(F, F, 1000, 384, 6, F, F, F, F, 0, None) == INVALID
    assert cnt(F, F, 1000, 384, 6, F, None, F, F, 64, None) == INVALID
    assert cnt(ODD, F, 1000, 384, 6, F, F, F, F, 64, None) == INVALID
    rk = lib.kolibri_eqb_split_rank
    #           counts E    N_total K rank flag stream
    assert rk(F, 384, 0, 6, F, F, None) == INVALID
    assert rk(F, 384, 1000, 6, None, F, None) == INVALID
    h = lib.kolibri_eqb_split_histogram
    #          cand counts cap E    pass prefix hist stream
    assert h(F, F, 64, 384, 4, F, F, None) == INVALID               # pass 0..3
    assert h(F, F, 64, 384, 1, None, F, None) == INVALID            # prefix from pass 1 on
    assert h(F, F, 0, 384, 0, None, F, None) == INVALID
    assert h(F, F, 64, 600, 0, None, F, None) == SHAPE


def test_balance_metric_checks(lib):
    lei = lib.kolibri_lei_inject
    #              counts N   E    K  lambda tau  g    stream
    assert lei(F, 128, 384, 6, 1e-5, 0.0, F, None) == INVALID            # tau must be positive
    assert lei(F, 128, 384, 6, 1e-5, 1.0, ODD, None) == INVALID
    assert lei(None, 128, 384, 6, 1e-5, 1.0, F, None) == INVALID
    assert lei(F, 128, 384, 400, 1e-5, 1.0, F, None) == INVALID           # K >= E
    assert lib.kolibri_score_grad_to_logits(F, F, 0, F, None) == INVALID
    assert lib.kolibri_score_grad_to_logits(F, None, 16, F, None) == INVALID
    ir = lib.kolibri_intervention_rate
    #             z  ids N    E    K  rate overlaps stream
    assert ir(F, F, 128, 384, 6, None, F, None) == INVALID
    assert ir(ODD, F, 128, 384, 6, F, F, None) == INVALID
    assert ir(F, F, 128, 384, 20, F, F, None) == SHAPE


def test_expert_layer_checks(lib):
    ws_size = lib.kolibri_expert_ffn_workspace_size
    assert ws_size(0, 2560, 512, 6, 1) == 0
    n, d, Fh, E, K = 4096, 2560, 512, 384, 6
    need = ws_size(n, d, Fh, K, 1)
    # x_perm (bf16) + h (bf16) + routed rows (fp32) + the shared expert's h and rows
    assert need >= n * K * (2 * d + 2 * Fh + 4 * d) + n * (2 * Fh + 4 * d)
    assert ws_size(n, d, Fh, K, 0) < need
    f = lib.kolibri_expert_ffn
    #          x  perm offs inv gates wgu wd  wgu_s wd_s y  N  d  F   E  K  ws ws_bytes stream
    assert f(F, F, F, F, F, F, F, F, F, F, n, d, Fh, E, K, F, need - 1, None) == SMALL
    assert f(F, F, F, F, F, F, F, F, None, F, n, d, Fh, E, K, F, need, None) == INVALID   # shared: both or neither
    assert f(F, F, F, None, F, F, F, F, F, F, n, d, Fh, E, K, F, need, None) == INVALID
    assert f(F, F, F, F, F, F, F, F, F, ODD, n, d, Fh, E, K, F, need, None) == INVALID
    assert f(F, F, F, F, F, F, F, F, F, F, n, 2500, Fh, E, K, F, need, None) == SHAPE    # d % 256
    assert f(F, F, F, F, F, F, F, F, F, F, n, d, 384, E, K, F, need, None) == SHAPE     # F % 256
    assert f(F, F, F, F, F, F, F, F, F, F, n, d, Fh, 600, K, F, need, None) == SHAPE    # E > 512
    assert f(F, F, F, F, F, F, F, F, F, F, n, d, Fh, E, 33, F, need, None) == INVALID
    disp = lib.kolibri_expert_dispatch
    #             x  perm N  d     K  x_perm stream
    assert disp(F, F, n, 2564, K, F, None) == SHAPE
    assert disp(F, F, n, 8200, K, F, None) == SHAPE
    assert disp(F, F, 0, d, K, F, None) == INVALID
    assert disp(ODD, F, n, d, K, F, None) == INVALID
    gu = lib.kolibri_expert_gate_up
    #           a  rows offs G  w  h  d  F   stream
    assert gu(F, n, None, 3, F, F, d, Fh, None) == INVALID        # no offsets: one group
    assert gu(F, n, F, 3, F, F, d, 128, None) == SHAPE
    assert gu(F, 0, F, 3, F, F, d, Fh, None) == INVALID
    dn = lib.kolibri_expert_down
    assert dn(F, n, None, 2, F, F, d, Fh, None) == INVALID
    assert dn(F, n, F, 2, F, F, 9000, Fh, None) == SHAPE
    cb = lib.kolibri_expert_combine
    #           y_perm y_sh inv gates N  d  K  y  stream
    assert cb(F, None, F, F, n, 2562, K, F, None) == SHAPE
    assert cb(F, None, F, F, n, d, 40, F, None) == INVALID
    assert cb(F, ODD, F, F, n, d, K, F, None) == INVALID
    assert cb(None, None, F, F, n, d, K, F, None) == INVALID


def test_selftest_limits(lib):
    # the diagnostic wait takes 1 us to 1 s; anything else is refused on the host
    assert lib.kolibri_selftest_bounded_wait(0, None) == INVALID
    assert lib.kolibri_selftest_bounded_wait(999, None) == INVALID
    assert lib.kolibri_selftest_bounded_wait(1_000_000_001, None) == INVALID
