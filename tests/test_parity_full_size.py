"""Oracle parity of the workloads at their full sizes, launched exactly as the
benchmark launches them (same generators, seeds, shapes and entry points).

Forward rows are independent, so a seeded sample of rows -- every sequence's
first and last row, rows on both sides of tile boundaries, random rows -- is
compared with the oracle one row at a time.  Gradients are compared in full
for one KV group (all of its query heads), which the oracle computes on its
own because groups do not interact.

  * packed: 16 sequences with lengths uniform in [512, 8192] from the seed,
    32 heads, d=128, causal (attn_fwd_varlen);
  * long: one sequence of 32768 tokens, 16 heads, d=128, causal, no window:
    the last rows walk all 256 key tiles;
  * grouped: batch 4, 32 query / 8 KV heads, N=4096, d=128, causal, with the
    dense fp32 bias tensor B[h, i, j] = -0.05 |i - j| (h + 1) / 32 (2.1 GB).
"""
import numpy as np
import pytest
import torch

from exact_io_aware_57_b200 import synth
from parity import (TOL_GRAD_BF16, TOL_LSE_BF16, TOL_O_BF16, check_fwd_sampled, guarded_empty, guards_intact,
                    max_abs, rel_fro, sample_rows)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_packed_sixteen_sequences_full_size(orc):
    from exact_io_aware_57_b200 import attn

    H, d = 32, 128
    lengths = synth.varlen_lengths(16, 512, 8192, seed=0)
    inp = synth.make_packed(lengths, H, H, d, seed=0)
    cu = inp.cu_seqlens
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    T = q.shape[0]
    ob, o = guarded_empty((T, H, d), torch.bfloat16)
    lb, lse = guarded_empty((H, T), torch.float32)
    mx = int(max(lengths))
    attn.attn_fwd_varlen(q, k, v, cu.cuda(), cu.cuda(), mx, mx, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    assert guards_intact(ob) and guards_intact(lb)
    o, lse = o.cpu(), lse.cpu()
    rng = np.random.default_rng(0)
    worst_o = worst_l = 0.0
    for z in range(16):
        a, b = int(cu[z]), int(cu[z + 1])
        L = b - a
        rows = sorted({0, L - 1, 127, 128, 255, 256, L // 2, *rng.integers(0, L, size=3).tolist()})
        rows = [r for r in rows if 0 <= r < L]
        for h in (z % H, (7 * z + 3) % H):
            o_ref, l_ref = orc.fwd_rows(inp.q[a:b][rows, h], inp.k[a:b, h], inp.v[a:b, h], rows, L, causal=True)
            worst_o = max(worst_o, max_abs(o[a:b][rows, h].double().numpy(), o_ref))
            worst_l = max(worst_l, max_abs(lse[h, a:b][rows].double().numpy(), l_ref))
    assert worst_o <= TOL_O_BF16 and worst_l <= TOL_LSE_BF16, (worst_o, worst_l)


def test_long_sequence_causal_full_size(orc):
    from exact_io_aware_57_b200 import attn

    N, H, d = 32768, 16, 128
    inp = synth.make_dense(1, H, H, N, N, d, with_dout=False)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    ob, o = guarded_empty(q.shape, torch.bfloat16)
    lb, lse = guarded_empty((1, H, N), torch.float32)
    attn.attn_fwd(q, k, v, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    assert guards_intact(ob) and guards_intact(lb)
    rows = sorted(set(sample_rows(N)) | {N - 129, N - 128, N - 2})
    eo, el = check_fwd_sampled(orc, inp.q, inp.k, inp.v, o.cpu(), lse.cpu(), True, [(0, 0), (0, 6), (0, 15)], rows)
    assert eo <= TOL_O_BF16 and el <= TOL_LSE_BF16, (eo, el)


def test_grouped_dense_bias_full_size(orc):
    from exact_io_aware_57_b200 import attn

    B, Hq, Hkv, N, d = 4, 32, 8, 4096, 128
    inp = synth.make_dense(B, Hq, Hkv, N, N, d)
    bias = synth.alibi_like_bias(Hq, N, N)  # [32, 4096, 4096] fp32, broadcast over the batch
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.dout))
    bd = bias.cuda()
    o, lse = attn.attn_fwd(q, k, v, bias=bd, causal=True)
    bufs = [guarded_empty(t.shape, t.dtype) for t in (q, k, v)]
    dq, dk, dv = attn.attn_bwd(q, k, v, o, lse, do, bias=bd, causal=True, dq=bufs[0][1], dk=bufs[1][1],
                               dv=bufs[2][1])
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    assert all(guards_intact(b[0]) for b in bufs)
    o, lse, dq, dk, dv = (t.cpu() for t in (o, lse, dq, dk, dv))
    del bd
    rows = sample_rows(N)
    eo, el = check_fwd_sampled(orc, inp.q, inp.k, inp.v, o, lse, True, [(0, 0), (1, 9), (3, 31)], rows,
                               bias_fn=lambda h, r: bias[h, r])
    assert eo <= TOL_O_BF16 and el <= TOL_LSE_BF16, (eo, el)
    b, hk = 2, 6
    qs = slice(4 * hk, 4 * hk + 4)
    sq = lambda t: t[b:b + 1, :, qs].contiguous()
    sk = lambda t: t[b:b + 1, :, hk:hk + 1].contiguous()
    dq_r, dk_r, dv_r = orc.bwd(sq(inp.q), sk(inp.k), sk(inp.v), sq(inp.dout), bias=bias[qs], causal=True)
    for name, a, r in (("dq", sq(dq), dq_r), ("dk", sk(dk), dk_r), ("dv", sk(dv), dv_r)):
        e = rel_fro(a.double().numpy(), r)
        assert e <= TOL_GRAD_BF16, f"{name} rel Frobenius {e:.3e}"
