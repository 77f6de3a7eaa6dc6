"""Backward of the packed variable-length forward, against the fp64 oracle.

Packed sequences are independent problems, so each sequence's slice of
dQ / dK / dV is compared with the dense oracle backward of that sequence alone
(the oracle's packed forward is pinned to the dense one the same way)."""
import pytest
import torch

from exact_io_aware_57_b200 import synth
from parity import check_grad, guarded_empty, guards_intact

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _packed(lens_q, lens_k, Hq, Hkv, d, dtype, seed=0):
    g = torch.Generator().manual_seed(seed)
    cq, ck = synth.cu_seqlens_of(lens_q), synth.cu_seqlens_of(lens_k)
    Tq, Tk = int(cq[-1]), int(ck[-1])
    mk = lambda *s: torch.randn(*s, generator=g).to(dtype)
    return mk(Tq, Hq, d), mk(Tk, Hkv, d), mk(Tk, Hkv, d), mk(Tq, Hq, d), cq, ck


def _run(q, k, v, do, cq, ck, causal):
    from exact_io_aware_57_b200 import attn

    q, k, v, do = (t.cuda() for t in (q, k, v, do))
    cqd, ckd = cq.cuda(), ck.cuda()
    mq, mk = int((cq[1:] - cq[:-1]).max()), int((ck[1:] - ck[:-1]).max())
    o, lse = attn.attn_fwd_varlen(q, k, v, cqd, ckd, mq, mk, causal=causal)
    bufs = [guarded_empty(t.shape, t.dtype) for t in (q, k, v)]
    attn.attn_bwd_varlen(q, k, v, o, lse, do, cqd, ckd, mq, mk, causal=causal, dq=bufs[0][1], dk=bufs[1][1],
                         dv=bufs[2][1])
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    assert all(guards_intact(b[0]) for b in bufs), "backward wrote outside its outputs"
    return [b[1].cpu() for b in bufs]


def _check(orc, q, k, v, do, cq, ck, causal, grads, dtype):
    for z in range(len(cq) - 1):
        a, b_ = int(cq[z]), int(cq[z + 1])
        c, e = int(ck[z]), int(ck[z + 1])
        if b_ == a or e == c:
            continue
        ref = orc.bwd(q[None, a:b_], k[None, c:e], v[None, c:e], do[None, a:b_], causal=causal)
        got = (grads[0][None, a:b_], grads[1][None, c:e], grads[2][None, c:e])
        for name, g_, r in zip(("dq", "dk", "dv"), got, ref):
            check_grad(f"seq {z} {name}", g_.double().numpy(), r, dtype)


@pytest.mark.parametrize("lens_q,lens_k,Hq,Hkv,d,causal,dtype", [
    ([130, 1, 257, 64, 500], None, 4, 2, 128, True, torch.bfloat16),
    ([130, 1, 257, 64, 500], None, 2, 2, 64, False, torch.bfloat16),
    ([100, 300, 129], [250, 300, 128], 4, 1, 128, True, torch.bfloat16),   # per-sequence Nq != Nk
    ([300, 40], [100, 200], 2, 2, 64, True, torch.bfloat16),               # rows that see no key
    ([70, 33, 150], None, 2, 1, 128, True, torch.float32),
])
def test_varlen_bwd(orc, lens_q, lens_k, Hq, Hkv, d, causal, dtype):
    lens_k = lens_q if lens_k is None else lens_k
    q, k, v, do, cq, ck = _packed(lens_q, lens_k, Hq, Hkv, d, dtype)
    grads = _run(q, k, v, do, cq, ck, causal)
    _check(orc, q, k, v, do, cq, ck, causal, grads, dtype)


def test_varlen_bwd_mixed_lengths_large(orc):
    """Six sequences drawn like the packed workload's (uniform lengths from the
    seed, here in [512, 3000]), 8 query / 4 KV heads, causal."""
    lens = synth.varlen_lengths(6, 512, 3000, seed=3)
    q, k, v, do, cq, ck = _packed(lens, lens, 8, 4, 128, torch.bfloat16, seed=3)
    grads = _run(q, k, v, do, cq, ck, True)
    _check(orc, q, k, v, do, cq, ck, True, grads, torch.bfloat16)
