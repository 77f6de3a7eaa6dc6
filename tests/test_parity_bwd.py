"""Backward parity: dQ, dK, dV through the C-ABI against the fp64 oracle's exact
gradient on the same seeded inputs."""
import numpy as np
import pytest
import torch

from exact_io_aware_57_b200 import synth
from parity import (TOL_GRAD_BF16, TOL_LSE_BF16, TOL_O_BF16, check_bwd, check_fwd_sampled, gpu_fwd_bwd, max_abs,
                    rel_fro, sample_rows)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_bwd_f32_single_head(orc):
    """The fp32 workload: batch 1, 1 head, N=128, d=64, non-causal, fwd+bwd, max-abs <= 1e-4."""
    check_bwd(orc, 1, 1, 1, 128, 128, 64, False, dtype=torch.float32)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_f32_general(orc, causal):
    check_bwd(orc, 2, 4, 2, 150, 150, 128, causal, dtype=torch.float32, bias=True)


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", [
    (1, 2, 2, 128, 64, False),
    (1, 2, 2, 128, 128, True),
    (1, 2, 1, 1, 64, False),
    (1, 2, 1, 7, 64, True),
    (1, 2, 2, 129, 128, False),
    (2, 2, 2, 200, 128, True),
    (1, 4, 2, 1000, 128, True),
    (1, 4, 1, 333, 64, False),
])
def test_bwd_bf16_shapes(orc, B, Hq, Hkv, N, d, causal):
    check_bwd(orc, B, Hq, Hkv, N, N, d, causal)


def test_bwd_bf16_ragged_head_groups(orc):
    """Six (batch, KV head) pairs: the grid interleaves the key tiles of groups of
    four pairs, so the last group holds two; four key tiles, the last ragged."""
    check_bwd(orc, 3, 4, 2, 400, 400, 128, True, seed=12)


@pytest.mark.parametrize("Nq,Nk", [(300, 500), (500, 300)])
def test_bwd_bf16_unequal_lengths(orc, Nq, Nk):
    check_bwd(orc, 1, 2, 1, Nq, Nk, 128, True)


def test_bwd_bf16_peaked(orc):
    check_bwd(orc, 1, 2, 2, 1024, 1024, 128, True, sigma=3.0)


def test_bwd_bf16_bias_gqa(orc):
    """Causal GQA 4:2 with the ALiBi-like fp32 bias (the grouped workload's features)."""
    check_bwd(orc, 2, 4, 2, 257, 257, 128, True, bias=True)


@pytest.mark.parametrize("Nq,Nk", [(300, 500), (500, 300)])
def test_bwd_bf16_bias_unequal_lengths(orc, Nq, Nk):
    """Dense bias with bottom-right aligned causal lengths (bias values loaded a
    step ahead, clamped at the last row)."""
    check_bwd(orc, 1, 4, 2, Nq, Nk, 128, True, bias=True, seed=15)


def test_bwd_bf16_bias_shared_three_batches(orc):
    """A bias shared by three batch elements: their CTAs run side by side
    (batch-innermost grid); rows of 388 keys with a ragged last tile."""
    check_bwd(orc, 3, 4, 2, 388, 388, 128, True, bias=True)


def test_fwd_bwd_full_size_causal_d128(orc):
    """The causal workload at full size (batch 2, 32 heads, N=8192, d=128, Q/K std 3),
    launched exactly as the benchmark launches it: sampled forward rows on three
    heads, and full-length dQ/dK/dV of one (batch, head) against the oracle."""
    inp = synth.make_dense(2, 32, 32, 8192, 8192, 128, sigma_qk=3.0)
    o, lse, dq, dk, dv = gpu_fwd_bwd(inp, True)
    eo, el = check_fwd_sampled(orc, inp.q, inp.k, inp.v, o, lse, True, [(0, 0), (1, 17), (1, 31)],
                               sample_rows(8192))
    assert eo <= TOL_O_BF16 and el <= TOL_LSE_BF16, (eo, el)
    b, h = 1, 17
    sl = lambda t: t[b:b + 1, :, h:h + 1].contiguous()
    dq_r, dk_r, dv_r = orc.bwd(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.dout), causal=True)
    for name, a, r in (("dq", sl(dq), dq_r), ("dk", sl(dk), dk_r), ("dv", sl(dv), dv_r)):
        e = rel_fro(a.double().numpy(), r)
        assert e <= TOL_GRAD_BF16, f"{name} rel Frobenius {e:.3e}"


def test_bwd_bf16_per_batch_bias(orc):
    """A bias of its own per batch element [B, Hq, N, N]: the usual grid order."""
    inp = synth.make_dense(2, 4, 2, 300, 300, 128, seed=5)
    b = synth.alibi_like_bias(4, 300, 300)
    b = torch.stack([b, 0.5 * b])
    _, _, dq, dk, dv = gpu_fwd_bwd(inp, True, bias=b)
    dq_r, dk_r, dv_r = orc.bwd(inp.q, inp.k, inp.v, inp.dout, bias=b, causal=True)
    for name, a, r in (("dq", dq, dq_r), ("dk", dk, dk_r), ("dv", dv, dv_r)):
        e = rel_fro(a.double().numpy(), r)
        assert e <= TOL_GRAD_BF16, f"{name} rel Frobenius {e:.3e}"


def test_bwd_bf16_shared_bias_noncausal(orc):
    """A shared dense bias over three batch elements (batch-innermost grid),
    non-causal: every key tile of every step is unmasked except the ragged one."""
    check_bwd(orc, 3, 4, 2, 388, 388, 128, False, bias=True)
