"""The oracle against what the pages and mathematics fix (CPU only).

Parity status per oracle function:
  fwd          pinned: merge_every_split, constant_scores, single_key, causal_prefix,
               permutation, shift, library_softmax
  fwd_stream   pinned: stream_equals_oneshot (against the one-shot definition)
  fwd_rows     pinned through fwd (rows_match_full below)
  fwd_varlen   pinned through fwd (varlen_matches_dense below)
  bwd          pinned: backward_fd, gqa_sum
  merge        pinned: merge_every_split
  byte model   pinned: the storage figures printed on the pages (tests/golden)
The pages print no worked numeric attention example, so no value-level golden
vector exists for fwd/bwd beyond these closed forms.
"""
from pathlib import Path

import numpy as np
import pytest

import oracle
from oracle_pins import ALL_PINS

GOLDEN = Path(__file__).parent / "golden"


@pytest.mark.parametrize("name", sorted(ALL_PINS))
def test_pin(orc, name):
    ok, detail = ALL_PINS[name](orc)
    assert ok, f"{name}: {detail}"


def test_byte_model_matches_pages():
    rows = [l.split() for l in (GOLDEN / "score_storage.txt").read_text().splitlines()
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for tq, tk, s, entries, nbytes, _src in rows:
        assert oracle.score_matrix_entries(int(tq)) == int(entries)
        assert oracle.score_matrix_bytes(int(tq), int(tk), int(s)) == int(nbytes)
    # the quoted unit conversions
    assert oracle.score_matrix_bytes(8192, 8192, 2) == 128 * 2**20
    assert oracle.score_matrix_bytes(4096, 4096, 4) == 64 * 2**20
    assert oracle.score_matrix_bytes(4096, 4096, 2) == 32 * 2**20


def test_rows_match_full(orc):
    rng = np.random.default_rng(3)
    B, n, hq, hkv, d = 2, 37, 4, 2, 16
    q = rng.standard_normal((B, n, hq, d))
    k = rng.standard_normal((B, n, hkv, d))
    v = rng.standard_normal((B, n, hkv, d))
    bias = rng.standard_normal((hq, n, n))
    o, lse = orc.fwd(q, k, v, bias=bias, causal=True)
    rows = [0, 1, 17, 36]
    for b, h in ((0, 0), (1, 3)):
        o_r, l_r = orc.fwd_rows(q[b, rows, h], k[b, :, h // 2], v[b, :, h // 2], rows, n,
                                bias_rows=bias[h, rows], causal=True)
        np.testing.assert_allclose(o_r, o[b, rows, h], rtol=0, atol=1e-14)
        np.testing.assert_allclose(l_r, lse[b, h, rows], rtol=0, atol=1e-13)


def test_varlen_matches_dense(orc):
    rng = np.random.default_rng(4)
    lens = [5, 1, 12, 8]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, hq, hkv, d = cu[-1], 4, 2, 8
    q = rng.standard_normal((T, hq, d))
    k = rng.standard_normal((T, hkv, d))
    v = rng.standard_normal((T, hkv, d))
    for causal, window in ((False, None), (True, None), (True, (3, None)), (False, (2, 1))):
        o, lse = orc.fwd_varlen(q, k, v, cu, cu, causal=causal, window=window)
        for z in range(len(lens)):
            a, b = cu[z], cu[z + 1]
            o_d, l_d = orc.fwd(q[None, a:b], k[None, a:b], v[None, a:b], causal=causal, window=window)
            np.testing.assert_allclose(o[a:b], o_d[0], rtol=0, atol=1e-14)
            np.testing.assert_allclose(lse[:, a:b], l_d[0], rtol=0, atol=1e-13)


def test_fully_masked_rows(orc):
    """Causal with Nq > Nk (bottom-right aligned): the first Nq-Nk rows see no
    key -> o = 0, LSE = -inf, zero gradients; a row whose bias is all -inf too."""
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 6, 1, 4))
    k = rng.standard_normal((1, 3, 1, 4))
    v = rng.standard_normal((1, 3, 1, 4))
    o, lse = orc.fwd(q, k, v, causal=True)
    assert np.all(o[0, :3] == 0) and np.all(np.isneginf(lse[0, 0, :3]))
    assert np.all(np.isfinite(lse[0, 0, 3:]))
    # row 3 sees key 0 only
    np.testing.assert_allclose(o[0, 3, 0], v[0, 0, 0], rtol=0, atol=1e-15)
    dq, dk, dv = orc.bwd(q, k, v, rng.standard_normal(q.shape), causal=True)
    assert np.all(dq[0, :3] == 0)
    bias = np.zeros((1, 6, 3))
    bias[0, 4, :] = -np.inf
    o2, l2 = orc.fwd(q, k, v, bias=bias, causal=True)
    assert np.all(o2[0, 4] == 0) and np.isneginf(l2[0, 0, 4])


def test_peaked_rows_force_rescales(orc):
    """Q,K ~ N(0, 3^2) at d=128 (the causal fwd+bwd workload's distribution):
    the streaming replay with 128-key blocks does rescale, and its jumps are
    the regime the lab's score-spread slider shows."""
    rng = np.random.default_rng(6)
    n, d = 1024, 128
    q = rng.standard_normal((1, n, 1, d)) * 3
    k = rng.standard_normal((1, n, 1, d)) * 3
    v = rng.standard_normal((1, n, 1, d))
    o1, l1 = orc.fwd(q, k, v, causal=True)
    o2, l2, rescales = orc.fwd_stream(q, k, v, causal=True, block=128)
    assert rescales > 0
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-11)
