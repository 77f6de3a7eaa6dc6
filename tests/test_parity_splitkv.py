"""Split-KV forward and the merge of partial results, against the fp64 oracle.

attn_fwd_splitkv computes the same function as attn_fwd over several key
ranges and merges them; attn_merge_partials is checked on its own against the
oracle's merge of the same fp32 partials (which the oracle pins against the
one-shot softmax at every split point)."""
import numpy as np
import pytest
import torch

from exact_io_aware_57_b200 import synth
from parity import TOL_LSE_BF16, TOL_O_BF16, guarded_empty, guards_intact, max_abs

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,splits", [
    (1, 4, 2, 128, 4000, 128, False, 0),    # automatic split count
    (1, 4, 2, 128, 4000, 128, False, 3),
    (1, 2, 1, 100, 2900, 64, False, 7),     # ragged last split and ragged query tile
    (1, 4, 4, 300, 2000, 128, True, 4),     # bottom-right causal: late splits hold keys only late rows see
    (2, 2, 2, 257, 257, 128, True, 2),
    (1, 2, 2, 64, 1000, 128, False, 100),   # more splits than key tiles: capped, none empty
    (1, 2, 2, 500, 300, 64, True, 3),       # rows that see no key at all
])
def test_splitkv_fwd(orc, B, Hq, Hkv, Nq, Nk, d, causal, splits):
    from exact_io_aware_57_b200 import attn

    inp = synth.make_dense(B, Hq, Hkv, Nq, Nk, d, with_dout=False)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    ob, o = guarded_empty(q.shape, q.dtype)
    lb, lse = guarded_empty((B, Hq, Nq), torch.float32)
    attn.attn_fwd_splitkv(q, k, v, causal=causal, num_splits=splits, out=o, lse=lse)
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    assert guards_intact(ob) and guards_intact(lb)
    o_ref, lse_ref = orc.fwd(inp.q, inp.k, inp.v, causal=causal)
    eo = max_abs(o.cpu().double().numpy(), o_ref)
    el = max_abs(lse.cpu().double().numpy(), lse_ref)
    assert eo <= TOL_O_BF16 and el <= TOL_LSE_BF16, (eo, el)


def test_splitkv_long_keys(orc):
    """256 queries at the end of 8192 keys (bottom-right causal), 8 splits and
    the automatic choice, against the oracle; the single-pass forward on the
    same inputs stays within the same tolerance (the two round P to bf16
    against different running maxima, so they agree only to bf16 precision)."""
    from exact_io_aware_57_b200 import attn

    inp = synth.make_dense(1, 8, 2, 256, 8192, 128, with_dout=False, sigma_qk=2.0)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    o_ref, lse_ref = orc.fwd(inp.q, inp.k, inp.v, causal=True)
    for o, lse in (attn.attn_fwd_splitkv(q, k, v, causal=True, num_splits=8),
                   attn.attn_fwd_splitkv(q, k, v, causal=True),
                   attn.attn_fwd(q, k, v, causal=True)):
        torch.cuda.synchronize()
        eo = max_abs(o.cpu().double().numpy(), o_ref)
        el = max_abs(lse.cpu().double().numpy(), lse_ref)
        assert eo <= TOL_O_BF16 and el <= TOL_LSE_BF16, (eo, el)


@pytest.mark.parametrize("d,out", [(128, torch.bfloat16), (64, torch.float32)])
def test_merge_partials(orc, d, out):
    """Random fp32 partials, including partials with LSE_t = -inf (no key in that
    range) and rows where every partial is -inf."""
    from exact_io_aware_57_b200 import attn

    rng = np.random.default_rng(5)
    T, B, Nq, Hq = 5, 2, 70, 3
    o_parts = rng.standard_normal((T, B, Nq, Hq, d)).astype(np.float32)
    lse_parts = (rng.standard_normal((T, B, Hq, Nq)) * 4).astype(np.float32)
    lse_parts[1, 0, 1, :30] = -np.inf
    lse_parts[:, 1, 2, 5] = -np.inf
    o, lse = attn.attn_merge_partials(torch.from_numpy(o_parts).cuda(), torch.from_numpy(lse_parts).cuda(),
                                      out_dtype=out)
    torch.cuda.synchronize()
    # oracle: rows in (b, i, h) order of o, partials [T, R, d] / [T, R]
    op = o_parts.reshape(T, B * Nq * Hq, d)
    lp = lse_parts.transpose(0, 1, 3, 2).reshape(T, B * Nq * Hq)
    o_ref, lse_ref = orc.merge_partials(op, lp)
    tol = TOL_O_BF16 if out == torch.bfloat16 else 1e-5
    eo = max_abs(o.cpu().double().numpy().reshape(-1, d), o_ref)
    el = max_abs(lse.cpu().double().numpy().transpose(0, 2, 1).reshape(-1), lse_ref)
    assert eo <= tol and el <= 1e-5, (eo, el)
    assert np.all(o.cpu().float().numpy()[1, 5, 2] == 0)


def test_splitkv_rejects_fp32_and_small_workspace():
    from exact_io_aware_57_b200 import attn

    inp = synth.make_dense(1, 2, 2, 64, 2048, 64, with_dout=False, dtype=torch.float32)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    with pytest.raises(attn.AttnError):
        attn.attn_fwd_splitkv(q, k, v, num_splits=4)
    qb, kb, vb = (t.bfloat16() for t in (q, k, v))
    with pytest.raises(attn.AttnError):
        attn.attn_fwd_splitkv(qb, kb, vb, num_splits=4, workspace=torch.empty(256, dtype=torch.uint8, device="cuda"))
