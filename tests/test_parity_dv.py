"""Forward with a value width d_v different from the query/key width d
(attn_fwd_dv), against the fp64 oracle given the same V."""
import pytest
import torch

from parity import TOL_LSE_BF16, TOL_O_BF16, guarded_empty, guards_intact, max_abs

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,dv,causal", [
    (1, 4, 2, 300, 300, 128, 64, True),
    (2, 2, 2, 129, 700, 128, 64, False),
    (1, 4, 1, 257, 257, 64, 128, True),
    (1, 2, 2, 500, 200, 64, 128, True),     # rows before the first key see nothing
    (1, 2, 2, 64, 64, 128, 128, False),     # d_v == d: the plain path
])
def test_fwd_value_width(orc, B, Hq, Hkv, Nq, Nk, d, dv, causal):
    from exact_io_aware_57_b200 import attn

    g = torch.Generator().manual_seed(7)
    q = torch.randn(B, Nq, Hq, d, generator=g).bfloat16()
    k = torch.randn(B, Nk, Hkv, d, generator=g).bfloat16()
    v = torch.randn(B, Nk, Hkv, dv, generator=g).bfloat16()
    ob, o = guarded_empty((B, Nq, Hq, dv), torch.bfloat16)
    lb, lse = guarded_empty((B, Hq, Nq), torch.float32)
    attn.attn_fwd_dv(q.cuda(), k.cuda(), v.cuda(), causal=causal, out=o, lse=lse)
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    assert guards_intact(ob) and guards_intact(lb)
    o_ref, lse_ref = orc.fwd(q, k, v, causal=causal)
    eo = max_abs(o.cpu().double().numpy(), o_ref)
    el = max_abs(lse.cpu().double().numpy(), lse_ref)
    assert eo <= TOL_O_BF16 and el <= TOL_LSE_BF16, (eo, el)


def test_fwd_value_width_rejects_fp32():
    from exact_io_aware_57_b200 import attn

    q = torch.zeros(1, 64, 2, 128, device="cuda")
    v = torch.zeros(1, 64, 2, 64, device="cuda")
    with pytest.raises(attn.AttnError):
        attn.attn_fwd_dv(q, q, v)


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,dv,causal", [
    (1, 4, 2, 300, 300, 128, 64, True),
    (2, 2, 2, 129, 700, 128, 64, False),
    (1, 4, 1, 257, 257, 64, 128, True),
    (1, 2, 2, 500, 200, 64, 128, True),     # rows before the first key see nothing
    (1, 4, 4, 1100, 1100, 128, 64, True),   # several steps through both staging stages
])
def test_bwd_value_width(orc, B, Hq, Hkv, Nq, Nk, d, dv, causal):
    """attn_bwd_dv: the fp32 dQ tile (width d) is staged beside a value width of its own."""
    from exact_io_aware_57_b200 import attn
    from parity import check_grad

    g = torch.Generator().manual_seed(8)
    q = torch.randn(B, Nq, Hq, d, generator=g).bfloat16()
    k = torch.randn(B, Nk, Hkv, d, generator=g).bfloat16()
    v = torch.randn(B, Nk, Hkv, dv, generator=g).bfloat16()
    do = torch.randn(B, Nq, Hq, dv, generator=g).bfloat16()
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = attn.attn_fwd_dv(qd, kd, vd, causal=causal)
    bufs = [guarded_empty(t.shape, t.dtype) for t in (qd, kd, vd)]
    attn.attn_bwd_dv(qd, kd, vd, o, lse, dod, causal=causal, dq=bufs[0][1], dk=bufs[1][1], dv=bufs[2][1])
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    assert all(guards_intact(b[0]) for b in bufs)
    dq_r, dk_r, dv_r = orc.bwd(q, k, v, do, causal=causal)
    for name, a, r in zip(("dq", "dk", "dv"), (b[1] for b in bufs), (dq_r, dk_r, dv_r)):
        check_grad(name, a.cpu().double().numpy(), r)
