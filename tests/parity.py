"""Helpers for the GPU-vs-oracle parity tests: run a case through the C-ABI
binding on cuda:0 and through the fp64 oracle on the same (bf16 or fp32)
inputs, and compare with the stated tolerances.

Tolerances (fixed by the method's stated targets):
  bf16 I/O, fp32 accumulation: forward max-abs <= 2e-2, LSE max-abs <= 5e-3,
  gradients relative Frobenius <= 2e-2;  fp32 path: max-abs <= 1e-4.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from exact_io_aware_57_b200 import synth

TOL_O_BF16, TOL_LSE_BF16, TOL_GRAD_BF16 = 2e-2, 5e-3, 2e-2
TOL_F32 = 1e-4
GUARD = 4096  # elements of sentinel on each side of an output buffer


def guarded_empty(shape, dtype, device="cuda"):
    """An output tensor embedded in a buffer whose guard bands hold a sentinel."""
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * GUARD,), 1234.5, dtype=dtype, device=device)
    return buf, buf[GUARD:GUARD + n].view(*shape)


def guards_intact(buf) -> bool:
    head, tail = buf[:GUARD], buf[-GUARD:]
    return bool(torch.all(head == 1234.5).item() and torch.all(tail == 1234.5).item())


def max_abs(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    fa, fb = np.isneginf(a), np.isneginf(b)
    assert np.array_equal(fa, fb), "-inf pattern (fully masked rows) differs"
    if (~fa).sum() == 0:
        return 0.0
    return float(np.max(np.abs(a[~fa] - b[~fb])))


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(1e-30, np.linalg.norm(b)))


def check_grad(name, got, ref, dtype=torch.bfloat16):
    """One gradient against the oracle: max-abs for fp32, relative Frobenius for
    bf16.  A gradient that vanishes exactly in the definition (one visible key
    per row: P = 1, so dS = P (dP - D) = 0 and dQ = dK = 0) has no relative
    error to speak of; there only rounding noise may remain (max-abs 1e-3)."""
    got = np.asarray(got, dtype=np.float64)
    if dtype == torch.float32:
        e = max_abs(got, ref)
        assert e <= TOL_F32, f"{name} max-abs {e:.3e} > {TOL_F32}"
    elif not np.asarray(ref).any():
        e = max_abs(got, ref)
        assert e <= 1e-3, f"{name} should vanish, max-abs {e:.3e}"
    else:
        e = rel_fro(got, ref)
        assert e <= TOL_GRAD_BF16, f"{name} rel Frobenius {e:.3e} > {TOL_GRAD_BF16}"
    return e


def gpu_fwd(inp, causal, scale=None, bias=None, alibi=None):
    from exact_io_aware_57_b200 import attn

    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    B, Nq, Hq, d = q.shape
    ob, o = guarded_empty((B, Nq, Hq, d), q.dtype)
    lb, lse = guarded_empty((B, Hq, Nq), torch.float32)
    attn.attn_fwd(q, k, v, bias=None if bias is None else bias.cuda(), causal=causal, scale=scale, out=o, lse=lse,
                  alibi_slopes=None if alibi is None else alibi.cuda())
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    assert guards_intact(ob) and guards_intact(lb), "kernel wrote outside its output"
    return o.cpu(), lse.cpu()


def check_fwd(orc, B, Hq, Hkv, Nq, Nk, d, causal, *, dtype=torch.bfloat16, sigma=1.0, bias=False, seed=0,
              per_batch_bias=False):
    inp = synth.make_dense(B, Hq, Hkv, Nq, Nk, d, dtype=dtype, seed=seed, sigma_qk=sigma, with_dout=False)
    b = None
    if bias:
        b = synth.alibi_like_bias(Hq, Nq, Nk)
        if per_batch_bias:
            b = torch.stack([b * (1.0 + 0.5 * i) for i in range(B)])
    o, lse = gpu_fwd(inp, causal, bias=b)
    o_ref, lse_ref = orc.fwd(inp.q, inp.k, inp.v, bias=b, causal=causal)
    tol_o, tol_l = (TOL_O_BF16, TOL_LSE_BF16) if dtype == torch.bfloat16 else (TOL_F32, TOL_F32)
    eo = max_abs(o.double().numpy(), o_ref)
    el = max_abs(lse.double().numpy(), lse_ref)
    assert eo <= tol_o, f"O max-abs {eo:.3e} > {tol_o}"
    assert el <= tol_l, f"LSE max-abs {el:.3e} > {tol_l}"
    return eo, el


def sample_rows(n: int, tile: int = 128, extra: int = 6, seed: int = 0):
    """Row 0, the last row, rows on both sides of every few tile boundaries, and random rows."""
    rng = np.random.default_rng(seed)
    rows = {0, n - 1}
    for t in range(tile, n, max(tile, (n // 8) // tile * tile)):
        rows.update({t - 1, t})
    rows.update(rng.integers(0, n, size=extra).tolist())
    return sorted(r for r in rows if 0 <= r < n)


def check_fwd_sampled(orc, q, k, v, o, lse, causal, heads, rows, bias_fn=None, scale=None, window=None):
    """Compare sampled outputs of a full-size launch (CPU copies) with the oracle,
    one (batch, head) at a time.  bias_fn(h, rows) -> [R, Nk] fp32 or None."""
    B, Nq, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    worst_o = worst_l = 0.0
    for (b, h) in heads:
        br = bias_fn(h, rows) if bias_fn else None
        o_ref, l_ref = orc.fwd_rows(q[b, rows, h], k[b, :, h // G], v[b, :, h // G], rows, Nq, bias_rows=br,
                                    causal=causal, scale=scale, window=window)
        worst_o = max(worst_o, max_abs(o[b, rows, h].double().numpy(), o_ref))
        worst_l = max(worst_l, max_abs(lse[b, h, rows].double().numpy(), l_ref))
    return worst_o, worst_l


def gpu_fwd_bwd(inp, causal, bias=None, scale=None, alibi=None):
    """Forward then backward through the C-ABI on cuda:0; returns CPU tensors.
    ``alibi``: fp32 per-head slopes for the in-kernel position bias."""
    from exact_io_aware_57_b200 import attn

    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.dout))
    bd = None if bias is None else bias.cuda()
    sd = None if alibi is None else alibi.cuda()
    o, lse = attn.attn_fwd(q, k, v, bias=bd, causal=causal, scale=scale, alibi_slopes=sd)
    bufs = [guarded_empty(t.shape, t.dtype) for t in (q, k, v)]
    dq, dk, dv = attn.attn_bwd(q, k, v, o, lse, do, bias=bd, causal=causal, scale=scale,
                               dq=bufs[0][1], dk=bufs[1][1], dv=bufs[2][1], alibi_slopes=sd)
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    assert all(guards_intact(b[0]) for b in bufs), "backward wrote outside its outputs"
    return o.cpu(), lse.cpu(), dq.cpu(), dk.cpu(), dv.cpu()


def check_bwd(orc, B, Hq, Hkv, Nq, Nk, d, causal, *, dtype=torch.bfloat16, sigma=1.0, bias=False, seed=0):
    inp = synth.make_dense(B, Hq, Hkv, Nq, Nk, d, dtype=dtype, seed=seed, sigma_qk=sigma)
    b = synth.alibi_like_bias(Hq, Nq, Nk) if bias else None
    o, lse, dq, dk, dv = gpu_fwd_bwd(inp, causal, bias=b)
    o_ref, _ = orc.fwd(inp.q, inp.k, inp.v, bias=b, causal=causal)
    dq_r, dk_r, dv_r = orc.bwd(inp.q, inp.k, inp.v, inp.dout, bias=b, causal=causal)
    errs = {}
    if dtype == torch.float32:
        for name, a, r in (("o", o, o_ref), ("dq", dq, dq_r), ("dk", dk, dk_r), ("dv", dv, dv_r)):
            errs[name] = max_abs(a.double().numpy(), r)
            assert errs[name] <= TOL_F32, f"{name} max-abs {errs[name]:.3e} > {TOL_F32}"
    else:
        for name, a, r in (("dq", dq, dq_r), ("dk", dk, dk_r), ("dv", dv, dv_r)):
            errs[name] = rel_fro(a.double().numpy(), r)
            assert errs[name] <= TOL_GRAD_BF16, f"{name} rel Frobenius {errs[name]:.3e} > {TOL_GRAD_BF16}"
    return errs
