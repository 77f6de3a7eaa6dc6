"""Parity of local (sliding-window) attention: attn_fwd_local / attn_bwd_local
against the fp64 oracle with the same window.  With a = i + Nk - Nq, key j is
visible from row i iff a - left <= j <= a + right (negative: unbounded; causal
caps the right side at a).  Windows are chosen to end inside, on and across
128-key tiles, with Nq != Nk shifts and rows that see no key at all."""
import pytest
import torch

from exact_io_aware_57_b200 import synth
from parity import (TOL_F32, TOL_GRAD_BF16, TOL_LSE_BF16, TOL_O_BF16, check_fwd_sampled, check_grad,
                    guarded_empty, guards_intact, max_abs, rel_fro, sample_rows)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

BF16, F32 = torch.bfloat16, torch.float32

CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal, window, alibi, dtype
    (1, 2, 2, 1000, 1000, 128, True, (256, -1), False, BF16),
    (1, 2, 1, 700, 700, 64, True, (100, -1), False, BF16),
    (2, 4, 2, 513, 513, 128, False, (200, 50), False, BF16),
    (1, 2, 2, 300, 900, 128, True, (130, -1), False, BF16),
    (1, 2, 2, 900, 300, 64, True, (60, -1), False, BF16),     # rows before the first key see nothing
    (1, 2, 2, 400, 400, 128, False, (-1, 0), False, BF16),    # right side 0 == causal
    (1, 2, 2, 400, 400, 128, False, (0, 0), False, BF16),     # the aligned key only
    (1, 2, 2, 400, 400, 64, False, (5, 300), False, BF16),
    (2, 4, 2, 600, 600, 128, True, (200, -1), True, BF16),    # window and ALiBi slopes together
    (1, 2, 1, 150, 150, 128, True, (40, -1), False, F32),
    (1, 2, 2, 97, 97, 64, False, (10, 20), True, F32),
]


def _ids(c):
    return f"B{c[0]}h{c[1]}-{c[2]}n{c[3]}x{c[4]}d{c[5]}{'c' if c[6] else ''}w{c[7][0]}_{c[7][1]}" + \
        ("alibi" if c[8] else "") + ("f32" if c[9] == F32 else "")


def _run(inp, causal, window, slopes, backward):
    from exact_io_aware_57_b200 import attn

    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    sl = None if slopes is None else slopes.cuda()
    B, Nq, Hq, d = q.shape
    ob, o = guarded_empty(q.shape, q.dtype)
    lb, lse = guarded_empty((B, Hq, Nq), torch.float32)
    attn.attn_fwd(q, k, v, causal=causal, alibi_slopes=sl, window=window, out=o, lse=lse)
    out = [o, lse]
    bufs = []
    if backward:
        bufs = [guarded_empty(t.shape, t.dtype) for t in (q, k, v)]
        attn.attn_bwd(q, k, v, o, lse, inp.dout.cuda(), causal=causal, alibi_slopes=sl, window=window,
                      dq=bufs[0][1], dk=bufs[1][1], dv=bufs[2][1])
        out += [b[1] for b in bufs]
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    assert guards_intact(ob) and guards_intact(lb) and all(guards_intact(b[0]) for b in bufs)
    return [t.cpu() for t in out]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,window,alibi,dtype", CASES, ids=[_ids(c) for c in CASES])
def test_local_fwd(orc, B, Hq, Hkv, Nq, Nk, d, causal, window, alibi, dtype):
    inp = synth.make_dense(B, Hq, Hkv, Nq, Nk, d, dtype=dtype, with_dout=False)
    slopes = synth.alibi_like_slopes(Hq) * 10 if alibi else None
    o, lse = _run(inp, causal, window, slopes, False)
    bias = None if slopes is None else synth.bias_from_slopes(slopes, Nq, Nk)
    o_ref, lse_ref = orc.fwd(inp.q, inp.k, inp.v, bias=bias, causal=causal, window=window)
    tol_o, tol_l = (TOL_O_BF16, TOL_LSE_BF16) if dtype == BF16 else (TOL_F32, TOL_F32)
    eo, el = max_abs(o.double().numpy(), o_ref), max_abs(lse.double().numpy(), lse_ref)
    assert eo <= tol_o and el <= tol_l, (eo, el)


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,window,alibi,dtype", CASES, ids=[_ids(c) for c in CASES])
def test_local_bwd(orc, B, Hq, Hkv, Nq, Nk, d, causal, window, alibi, dtype):
    inp = synth.make_dense(B, Hq, Hkv, Nq, Nk, d, dtype=dtype)
    slopes = synth.alibi_like_slopes(Hq) * 10 if alibi else None
    _, _, dq, dk, dv = _run(inp, causal, window, slopes, True)
    bias = None if slopes is None else synth.bias_from_slopes(slopes, Nq, Nk)
    dq_r, dk_r, dv_r = orc.bwd(inp.q, inp.k, inp.v, inp.dout, bias=bias, causal=causal, window=window)
    for name, a, r in (("dq", dq, dq_r), ("dk", dk, dk_r), ("dv", dv, dv_r)):
        check_grad(name, a.double().numpy(), r, dtype)


def test_window_wider_than_sequence_is_bitwise_plain():
    """A window that reaches past both ends takes the same tiles and the same
    arithmetic as the plain causal path, so the results are bit-identical."""
    from exact_io_aware_57_b200 import attn

    inp = synth.make_dense(1, 4, 2, 777, 777, 128)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.dout))
    o1, l1 = attn.attn_fwd(q, k, v, causal=True)
    o2, l2 = attn.attn_fwd(q, k, v, causal=True, window=(5000, None))
    g1 = attn.attn_bwd(q, k, v, o1, l1, do, causal=True)
    g2 = attn.attn_bwd(q, k, v, o2, l2, do, causal=True, window=(5000, None))
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert all(torch.equal(a, b) for a, b in zip(g1, g2))


def test_local_full_size_long_sequence(orc):
    """One sequence of 32768 tokens, 16 heads, d=128, causal with a 4096-key
    window: sampled forward rows on three heads against the oracle, and the
    full dQ/dK/dV of one head on its first 12288 positions (the window makes
    them independent of the rest: a row's keys lie inside [i - 4096, i])."""
    N, H, d, W = 32768, 16, 128, 4096
    inp = synth.make_dense(1, H, H, N, N, d)
    o, lse, dq, dk, dv = _run(inp, True, (W, -1), None, True)
    eo, el = check_fwd_sampled(orc, inp.q, inp.k, inp.v, o, lse, True, [(0, 0), (0, 7), (0, 15)], sample_rows(N),
                               window=(W, -1))
    assert eo <= TOL_O_BF16 and el <= TOL_LSE_BF16, (eo, el)
    n, h = 12288, 9
    # rows < n see only keys < n, and keys < n - W are seen only by rows < n: on the
    # first n positions dQ is complete, and so are dK/dV of the keys below n - W
    sl = lambda t: t[:, :n, h:h + 1].contiguous()
    dq_r, dk_r, dv_r = orc.bwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.dout), causal=True, window=(W, -1))
    kk = n - W
    for name, a, r in (("dq", sl(dq), dq_r), ("dk", sl(dk)[:, :kk], dk_r[:, :kk]),
                       ("dv", sl(dv)[:, :kk], dv_r[:, :kk])):
        e = rel_fro(a.double().numpy(), r)
        assert e <= TOL_GRAD_BF16, f"{name} rel Frobenius {e:.3e}"
