"""Packed-sequence offsets are checked on the device before any access.

Each case passes cu_seqlens that the kernels must reject (an offset past the
total, decreasing offsets, a length above max_seqlen).  The offsets are chosen
so that the check catches them before a single row is read or written: the
call returns normally, attn_device_status reports ATTN_ERR_INVALID, the valid
sequences are still computed, and the guard bands around every output hold.
"""
import pytest
import torch

from exact_io_aware_57_b200 import synth
from parity import TOL_F32, TOL_LSE_BF16, TOL_O_BF16, guarded_empty, guards_intact, max_abs

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

BF16, F32 = torch.bfloat16, torch.float32
T, H, d = 600, 2, 128

# (offsets, max_seqlen, index of the one valid sequence or None)
BAD = [
    ([0, 200, T + 300], 400, 0),       # the last offset lies past the total
    ([0, 300, 200, T], 400, None),     # decreasing: sequence 1 has a negative length
    ([0, 100, T], 300, 0),             # sequence 1 (500 rows) is longer than max_seqlen
    ([-64, 100, T], 600, 1),           # a negative first offset
]


def _inputs(dtype):
    g = torch.Generator().manual_seed(11)
    mk = lambda *s: torch.randn(*s, generator=g).to(dtype)
    return mk(T, H, d), mk(T, H, d), mk(T, H, d), mk(T, H, d)


@pytest.mark.parametrize("dtype", [BF16, F32])
@pytest.mark.parametrize("cu,mx,valid", BAD)
def test_bad_offsets_are_rejected_on_device(orc, dtype, cu, mx, valid):
    from exact_io_aware_57_b200 import attn

    q, k, v, do = _inputs(dtype)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    cud = torch.tensor(cu, dtype=torch.int32, device="cuda")
    assert attn.attn_device_status() == 0
    ob, o = guarded_empty((T, H, d), dtype)
    lb, lse = guarded_empty((H, T), torch.float32)
    attn.attn_fwd_varlen(qd, kd, vd, cud, cud, mx, mx, causal=True, out=o, lse=lse)
    assert attn.attn_device_status() == attn.ATTN_ERR_INVALID
    assert guards_intact(ob) and guards_intact(lb)
    if valid is not None:  # the valid sequence is computed as usual
        a, b = cu[valid], cu[valid + 1]
        o_ref, l_ref = orc.fwd(q[None, a:b], k[None, a:b], v[None, a:b], causal=True)
        tol_o, tol_l = (TOL_O_BF16, TOL_LSE_BF16) if dtype == BF16 else (TOL_F32, TOL_F32)
        assert max_abs(o[a:b].cpu().double().numpy(), o_ref[0]) <= tol_o
        assert max_abs(lse[:, a:b].cpu().double().numpy(), l_ref[0]) <= tol_l
    bufs = [guarded_empty((T, H, d), dtype) for _ in range(3)]
    attn.attn_bwd_varlen(qd, kd, vd, torch.zeros_like(qd), torch.zeros(H, T, device="cuda"), dod, cud, cud, mx, mx,
                         causal=True, dq=bufs[0][1], dk=bufs[1][1], dv=bufs[2][1])
    assert attn.attn_device_status() == attn.ATTN_ERR_INVALID
    assert all(guards_intact(b[0]) for b in bufs)
    # the status word was cleared by the read: a valid call reports ATTN_OK again
    good = torch.tensor([0, 250, T], dtype=torch.int32, device="cuda")
    attn.attn_fwd_varlen(qd, kd, vd, good, good, 350, 350, causal=True)
    assert attn.attn_device_status() == 0
