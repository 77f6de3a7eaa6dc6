"""Parity of the in-kernel ALiBi position bias: attn_fwd_alibi / attn_bwd_alibi
form B[h, i, j] = -slope_h * |j - (i + Nk - Nq)| in registers; the oracle gets
the same bias as a dense fp32 tensor built on the CPU from the slopes.  For
Nq == Nk with slopes (h + 1) * 0.05 / 32 this is the grouped-query workload's
bias -0.05 * |i - j| * (h + 1) / 32."""
import numpy as np
import pytest
import torch

from exact_io_aware_57_b200 import synth
from parity import (TOL_F32, TOL_GRAD_BF16, TOL_LSE_BF16, TOL_O_BF16, check_fwd_sampled, gpu_fwd, gpu_fwd_bwd,
                    max_abs, rel_fro, sample_rows)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _slopes(Hq, steep=False):
    s = synth.alibi_like_slopes(Hq)
    return s * 40.0 if steep else s


CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal, dtype, steep
    (2, 4, 2, 257, 257, 128, True, torch.bfloat16, False),
    (1, 2, 1, 190, 190, 64, False, torch.bfloat16, False),
    (1, 4, 4, 300, 500, 128, True, torch.bfloat16, False),
    (1, 2, 2, 500, 300, 64, True, torch.bfloat16, False),   # rows above the first key: fully masked
    (1, 2, 2, 130, 1000, 128, False, torch.bfloat16, True),  # steep slopes: only nearby keys matter
    (2, 4, 2, 150, 150, 128, True, torch.float32, False),
    (1, 2, 1, 97, 97, 64, False, torch.float32, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,dtype,steep", CASES)
def test_alibi_fwd(orc, B, Hq, Hkv, Nq, Nk, d, causal, dtype, steep):
    inp = synth.make_dense(B, Hq, Hkv, Nq, Nk, d, dtype=dtype, with_dout=False)
    sl = _slopes(Hq, steep)
    o, lse = gpu_fwd(inp, causal, alibi=sl)
    o_ref, lse_ref = orc.fwd(inp.q, inp.k, inp.v, bias=synth.bias_from_slopes(sl, Nq, Nk), causal=causal)
    tol_o, tol_l = (TOL_O_BF16, TOL_LSE_BF16) if dtype == torch.bfloat16 else (TOL_F32, TOL_F32)
    eo = max_abs(o.double().numpy(), o_ref)
    el = max_abs(lse.double().numpy(), lse_ref)
    assert eo <= tol_o and el <= tol_l, (eo, el)


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,dtype,steep", CASES)
def test_alibi_bwd(orc, B, Hq, Hkv, Nq, Nk, d, causal, dtype, steep):
    inp = synth.make_dense(B, Hq, Hkv, Nq, Nk, d, dtype=dtype)
    sl = _slopes(Hq, steep)
    o, lse, dq, dk, dv = gpu_fwd_bwd(inp, causal, alibi=sl)
    dense = synth.bias_from_slopes(sl, Nq, Nk)
    dq_r, dk_r, dv_r = orc.bwd(inp.q, inp.k, inp.v, inp.dout, bias=dense, causal=causal)
    for name, a, r in (("dq", dq, dq_r), ("dk", dk, dk_r), ("dv", dv, dv_r)):
        if dtype == torch.float32:
            e = max_abs(a.double().numpy(), r)
            assert e <= TOL_F32, f"{name} max-abs {e:.3e}"
        else:
            e = rel_fro(a.double().numpy(), r)
            assert e <= TOL_GRAD_BF16, f"{name} rel Frobenius {e:.3e}"


def test_alibi_matches_dense_bias_path():
    """Both bias routes of the tensor-core kernels give the same attention (they
    differ only in how the bias value is rounded)."""
    from exact_io_aware_57_b200 import attn

    inp = synth.make_dense(2, 8, 2, 640, 640, 128, with_dout=False)
    sl = synth.alibi_like_slopes(8)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    o1, l1 = attn.attn_fwd(q, k, v, bias=synth.alibi_like_bias(8, 640, 640).cuda(), causal=True)
    o2, l2 = attn.attn_fwd(q, k, v, alibi_slopes=sl.cuda(), causal=True)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l1 - l2).abs().max().item() <= 1e-3


def test_alibi_rejects_bias_and_slopes_together():
    from exact_io_aware_57_b200 import attn

    inp = synth.make_dense(1, 2, 2, 64, 64, 64, with_dout=False)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    with pytest.raises(attn.AttnError):
        attn.attn_fwd(q, k, v, bias=torch.zeros(2, 64, 64, device="cuda"),
                      alibi_slopes=torch.zeros(2, device="cuda"))
    with pytest.raises(attn.AttnError):
        attn.attn_fwd(q, k, v, alibi_slopes=torch.zeros(3, device="cuda"))


def test_alibi_full_size_grouped(orc):
    """The grouped-query workload at full size (batch 4, 32 query / 8 KV heads,
    N=4096, d=128, causal) with the bias formed in the kernel: sampled forward
    rows on three heads, and the full gradients of one KV group (its 4 query
    heads) against the oracle."""
    B, Hq, Hkv, N, d = 4, 32, 8, 4096, 128
    inp = synth.make_dense(B, Hq, Hkv, N, N, d)
    sl = synth.alibi_like_slopes(Hq)
    o, lse, dq, dk, dv = gpu_fwd_bwd(inp, True, alibi=sl)
    rows = sample_rows(N)
    bias_fn = lambda h, r: synth.alibi_like_bias(Hq, N, N, rows=r, heads=[h])[0]
    eo, el = check_fwd_sampled(orc, inp.q, inp.k, inp.v, o, lse, True, [(0, 0), (2, 13), (3, 31)], rows,
                               bias_fn=bias_fn)
    assert eo <= TOL_O_BF16 and el <= TOL_LSE_BF16, (eo, el)
    b, hk = 3, 5
    qs = slice(4 * hk, 4 * hk + 4)
    sq = lambda t: t[b:b + 1, :, qs].contiguous()
    sk = lambda t: t[b:b + 1, :, hk:hk + 1].contiguous()
    dense = synth.bias_from_slopes(sl[qs], N, N)
    dq_r, dk_r, dv_r = orc.bwd(sq(inp.q), sk(inp.k), sk(inp.v), sq(inp.dout), bias=dense, causal=True)
    for name, a, r in (("dq", sq(dq), dq_r), ("dk", sk(dk), dk_r), ("dv", sk(dv), dv_r)):
        e = rel_fro(a.double().numpy(), r)
        assert e <= TOL_GRAD_BF16, f"{name} rel Frobenius {e:.3e}"
