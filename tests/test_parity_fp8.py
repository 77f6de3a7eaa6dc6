"""FP8 forward against the fp64 oracle.

The reference of an FP8 forward is the exact attention of the dequantised
inputs: the oracle quantises Q and K itself (per (batch, head) scale
amax / 448, codes decided on the fp32 quotient as the kernel decides them) and
computes softmax(scale Q' K'^T) V in fp64; the kernel's output must meet the
bf16 bounds against that.  The quantiser itself must produce exactly the
oracle's codes and scales.  The error that quantisation adds against the
unquantised attention is reported separately, not folded into the bounds."""
import numpy as np
import pytest
import torch

from exact_io_aware_57_b200 import synth
from parity import TOL_LSE_BF16, TOL_O_BF16, check_fwd_sampled, guarded_empty, guards_intact, max_abs, sample_rows

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _run(inp, causal):
    from exact_io_aware_57_b200 import attn

    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    q8, qs = attn.attn_quantize_e4m3(q)
    k8, ks = attn.attn_quantize_e4m3(k)
    B, Nq, Hq, d = q.shape
    ob, o = guarded_empty((B, Nq, Hq, d), torch.bfloat16)
    lb, lse = guarded_empty((B, Hq, Nq), torch.float32)
    attn.attn_fwd_fp8(q8, qs, k8, ks, v, causal=causal, out=o, lse=lse)
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    assert guards_intact(ob) and guards_intact(lb)
    return o.cpu(), lse.cpu(), (q8.cpu(), qs.cpu(), k8.cpu(), ks.cpu())


def _dequant(x8, s):
    return x8.view(torch.float8_e4m3fn).double() * s.double()[:, None, :, None]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,causal,sigma", [
    (2, 4, 2, 300, 300, True, 1.0),
    (1, 2, 2, 517, 517, False, 1.0),
    (1, 4, 1, 200, 700, True, 3.0),     # peaked scores, bottom-right causal, MQA
    (2, 2, 2, 129, 129, True, 3.0),
])
def test_fp8_forward_matches_oracle_on_dequantised_inputs(orc, B, Hq, Hkv, Nq, Nk, causal, sigma):
    inp = synth.make_dense(B, Hq, Hkv, Nq, Nk, 128, sigma_qk=sigma, with_dout=False, seed=4)
    o, lse, (q8, qs, k8, ks) = _run(inp, causal)
    qd, qsc = orc.quantize_e4m3_heads(inp.q)
    kd, ksc = orc.quantize_e4m3_heads(inp.k)
    # the quantiser: the oracle's codes and scales exactly
    assert np.array_equal(qs.double().numpy(), qsc) and np.array_equal(ks.double().numpy(), ksc)
    assert np.array_equal(_dequant(q8, qs).numpy(), qd) and np.array_equal(_dequant(k8, ks).numpy(), kd)
    o_ref, lse_ref = orc.fwd(qd, kd, inp.v, causal=causal)
    eo, el = max_abs(o.double().numpy(), o_ref), max_abs(lse.double().numpy(), lse_ref)
    assert eo <= TOL_O_BF16 and el <= TOL_LSE_BF16, (eo, el)
    # reported: what quantisation itself costs against the unquantised attention
    o_full, _ = orc.fwd(inp.q, inp.k, inp.v, causal=causal)
    print(f"quantisation error (max-abs O vs unquantised oracle): {max_abs(o.double().numpy(), o_full):.3e}")


def test_fp8_forward_causal_full_size(orc):
    """The causal workload's shape (batch 2, 32 heads, N=8192, d=128, Q/K std 3):
    sampled rows of three heads against the oracle on the dequantised inputs."""
    N, H = 8192, 32
    inp = synth.make_dense(2, H, H, N, N, 128, sigma_qk=3.0, with_dout=False)
    o, lse, _ = _run(inp, True)
    qd, _ = orc.quantize_e4m3_heads(inp.q)
    kd, _ = orc.quantize_e4m3_heads(inp.k)
    eo, el = check_fwd_sampled(orc, torch.from_numpy(qd), torch.from_numpy(kd), inp.v, o, lse, True,
                               [(0, 0), (1, 17), (1, 31)], sample_rows(N))
    assert eo <= TOL_O_BF16 and el <= TOL_LSE_BF16, (eo, el)


def test_fp8_rejects_what_it_does_not_cover():
    from exact_io_aware_57_b200 import attn

    inp = synth.make_dense(1, 2, 2, 64, 64, 64, with_dout=False)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    q8, qs = attn.attn_quantize_e4m3(q)     # d = 64 quantises
    k8, ks = attn.attn_quantize_e4m3(k)
    with pytest.raises(attn.AttnError):      # but the FP8 forward takes d = 128 only
        attn.attn_fwd_fp8(q8, qs, k8, ks, v)
