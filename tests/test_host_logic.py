"""Host-side logic that needs no GPU: the split-KV heuristic and workspace
sizes of the C-ABI library, argument validation of the newer entry points
(rejected before any launch), and the FLOP accounting the benchmark uses."""
import ctypes
import math

import pytest

from exact_io_aware_57_b200 import workloads


def _lib():
    from exact_io_aware_57_b200 import attn

    return attn, attn.lib()


def _fill(ctas, t):
    n = ctas * t
    return n / (math.ceil(n / 148) * 148)


@pytest.mark.parametrize("b,h,nq,nk", [(1, 32, 512, 65536), (1, 4, 128, 4000), (1, 8, 256, 8192),
                                       (2, 32, 8192, 8192), (1, 1, 128, 100000), (1, 2, 64, 300)])
def test_split_count_fills_the_last_wave(b, h, nq, nk):
    attn, lib = _lib()
    t = attn.attn_splitkv_num_splits(b, h, nq, nk)
    ctas = math.ceil(nq / 256) * h * b  # one forward CTA per 256 query rows
    kv_tiles = math.ceil(nk / 128)
    assert 1 <= t <= 64
    assert t == 1 or t <= max(1, kv_tiles // 4)
    # no count up to the cap fills the last wave better by more than the 5 % margin
    cap = max(1, min(64, kv_tiles // 4))
    assert all(_fill(ctas, u) <= _fill(ctas, t) + 0.05 + 1e-12 for u in range(1, cap + 1))
    if ctas >= 148 and _fill(ctas, 1) > 0.95:
        assert t == 1


def test_split_workspace_size():
    attn, lib = _lib()
    lib.attn_splitkv_workspace_size.restype = ctypes.c_size_t
    rows = 1 * 512 * 32
    a256 = lambda x: (x + 255) // 256 * 256
    assert lib.attn_splitkv_workspace_size(1, 32, 512, 128, 8) == a256(rows * 128 * 8 * 4) + a256(rows * 8 * 4)
    assert lib.attn_splitkv_workspace_size(1, 32, 512, 128, 0) == 0


@pytest.mark.parametrize("entry", ["fwd_local", "bwd_local", "fwd_alibi_null", "splitkv_f32", "merge_dim",
                                   "merge_null", "bwd_varlen_null", "bwd_varlen_maxlen", "grid_heads",
                                   "grid_batch_splits", "selftest_limit", "grid_seqs"])
def test_new_entry_points_validate_before_launch(entry):
    attn, lib = _lib()
    p = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    fp = ctypes.cast(p, ctypes.POINTER(ctypes.c_float))
    ip = ctypes.cast(p, ctypes.POINTER(ctypes.c_int))
    before = attn.attn_launch_count()
    if entry == "fwd_local":      # h_q not a multiple of h_kv
        rc = lib.attn_fwd_local(p, p, p, None, p, fp, 1, 4, 3, 64, 64, 128, 0.1, 1, 16, -1, 0, None)
        want = attn.ATTN_ERR_INVALID
    elif entry == "bwd_local":    # head dim 96
        rc = lib.attn_bwd_local(p, p, p, None, p, fp, p, p, p, p, p, 1 << 20, 1, 4, 4, 64, 64, 96, 0.1, 1, 16, -1,
                                0, None)
        want = attn.ATTN_ERR_UNSUPPORTED
    elif entry == "fwd_alibi_null":
        rc = lib.attn_fwd_alibi(p, p, p, None, p, fp, 1, 4, 4, 64, 64, 128, 0.1, 1, 0, None)
        want = attn.ATTN_ERR_INVALID
    elif entry == "splitkv_f32":
        rc = lib.attn_fwd_splitkv(p, p, p, p, fp, 1, 4, 4, 64, 4096, 128, 0.1, 0, 4, p, 1 << 20, 1, None)
        want = attn.ATTN_ERR_UNSUPPORTED
    elif entry == "merge_dim":
        rc = lib.attn_merge_partials(fp, fp, 3, p, fp, 1, 4, 64, 96, 0, None)
        want = attn.ATTN_ERR_UNSUPPORTED
    elif entry == "merge_null":
        rc = lib.attn_merge_partials(None, fp, 3, p, fp, 1, 4, 64, 128, 0, None)
        want = attn.ATTN_ERR_INVALID
    elif entry == "bwd_varlen_null":
        rc = lib.attn_bwd_varlen(p, p, p, p, fp, p, p, p, p, None, ip, 2, 64, 64, 128, 128, 4, 4, 128, 0.1, 1, p,
                                 1 << 20, 0, None)
        want = attn.ATTN_ERR_INVALID
    elif entry == "bwd_varlen_maxlen":  # longest sequence longer than the packed total
        rc = lib.attn_bwd_varlen(p, p, p, p, fp, p, p, p, p, ip, ip, 2, 200, 64, 128, 128, 4, 4, 128, 0.1, 1, p,
                                 1 << 20, 0, None)
        want = attn.ATTN_ERR_INVALID
    elif entry == "grid_heads":   # more heads than the grid's y extent
        rc = lib.attn_fwd(p, p, p, None, 0, p, fp, 1, 70000, 70000, 64, 64, 128, 0.1, 0, 0, None)
        want = attn.ATTN_ERR_UNSUPPORTED
    elif entry == "grid_seqs":    # more packed sequences than the grid's z extent
        rc = lib.attn_fwd_varlen(p, p, p, p, fp, ip, ip, 70000, 64, 64, 1 << 20, 1 << 20, 4, 4, 128, 0.1, 1, 0,
                                 None)
        want = attn.ATTN_ERR_UNSUPPORTED
    elif entry == "selftest_limit":  # wait limit below the accepted range
        rc = lib.attn_selftest_wait_timeout(10, None)
        want = attn.ATTN_ERR_INVALID
    else:                         # batch x key splits beyond the grid's z extent
        rc = lib.attn_fwd_splitkv(p, p, p, p, fp, 20000, 1, 1, 64, 4096, 128, 0.1, 0, 8, p, 1 << 40, 0, None)
        want = attn.ATTN_ERR_UNSUPPORTED
    assert rc == want
    assert attn.attn_launch_count() == before


def test_window_pairs_match_brute_force():
    for n, w in ((10, 3), (5, 4), (5, 10), (1, 0), (257, 128), (8192, 1024)):
        assert workloads.window_pairs(n, w) == sum(min(i + 1, w + 1) for i in range(n))


def test_flops_of_each_workload():
    W = workloads.WORKLOADS
    # causal N = 8192, d = 128, 2 x 32 heads: forward 4 * N^2 * d / 2 per head, backward 2.5x more
    f = 4.0 * 8192 * 8192 * 128 * 0.5 * 2 * 32
    assert workloads.flops(W["c3"], backward=False) == f
    assert workloads.flops(W["c3"]) == 3.5 * f
    # exact visible pairs for a query block at the end of a longer key sequence
    nq, nk = 512, 65536
    pairs = sum(i + (nk - nq) + 1 for i in range(nq))
    assert workloads.flops(W["kv1"]) == 4.0 * 128 * pairs * 32
    # a causal window counts 4 d per visible pair
    assert workloads.flops(W["c3"], backward=False, window=1024) == \
        4.0 * 128 * workloads.window_pairs(8192, 1024) * 2 * 32
