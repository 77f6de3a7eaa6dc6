"""Forward parity: the CUDA path through the C-ABI against the fp64 oracle on
the same seeded inputs (bf16 tensor-core path and fp32 CUDA-core path)."""
import numpy as np
import pytest
import torch

from exact_io_aware_57_b200 import synth
from parity import (TOL_LSE_BF16, TOL_O_BF16, check_fwd, check_fwd_sampled, max_abs, sample_rows)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", [
    (1, 2, 2, 128, 64, False),
    (1, 2, 2, 128, 128, True),
    (1, 4, 1, 1, 64, False),   # single row, single key, MQA
    (1, 2, 2, 7, 128, True),
    (1, 2, 2, 63, 64, True),
    (1, 2, 2, 129, 128, False),
    (2, 2, 2, 200, 128, True),
    (2, 4, 2, 1000, 128, True),
    (1, 3, 3, 777, 64, False),
])
def test_fwd_bf16_shapes(orc, B, Hq, Hkv, N, d, causal):
    check_fwd(orc, B, Hq, Hkv, N, N, d, causal)


@pytest.mark.parametrize("Nq,Nk,causal", [(300, 500, True), (500, 300, True), (130, 1000, False), (1, 257, True)])
def test_fwd_bf16_unequal_lengths(orc, Nq, Nk, causal):
    """Bottom-right aligned causal mask; Nq > Nk leaves the first rows with no key
    (O = 0, LSE = -inf)."""
    check_fwd(orc, 1, 2, 1, Nq, Nk, 128, causal)


def test_fwd_bf16_ragged_head_groups(orc):
    """Twelve (batch, head) pairs: the grid interleaves the row blocks of groups
    of eight pairs, so the last group holds four; three row blocks, the last ragged."""
    check_fwd(orc, 3, 4, 2, 600, 600, 128, True, seed=11)


def test_fwd_bf16_tail_wave_single_tiles(orc):
    """52 heads x 3 row blocks = 156 equal units on 148 SMs: the last 8 run as
    single 128-row tiles, two CTAs each, among them the ragged last row block
    (one of its CTAs has no rows at all)."""
    check_fwd(orc, 1, 52, 4, 600, 600, 64, False, seed=13)


def test_fwd_bf16_peaked_scores(orc):
    """Q, K ~ N(0, 3^2): frequent running-max rescales (the causal fwd+bwd workload's regime)."""
    check_fwd(orc, 1, 2, 2, 1024, 1024, 128, True, sigma=3.0)


@pytest.mark.parametrize("per_batch", [False, True])
def test_fwd_bf16_bias_gqa(orc, per_batch):
    """ALiBi-like additive fp32 bias with GQA 4:2, causal (the grouped workload's features)."""
    check_fwd(orc, 2, 4, 2, 257, 257, 128, True, bias=True, per_batch_bias=per_batch)


@pytest.mark.parametrize("Nq,Nk", [(300, 500), (500, 300)])
def test_fwd_bf16_bias_unequal_lengths(orc, Nq, Nk):
    """Dense bias (rows of Nk = 0 mod 4 floats: staged by TMA) with bottom-right
    aligned causal lengths: a ragged last key tile and, for Nq > Nk, rows with no key."""
    check_fwd(orc, 2, 4, 2, Nq, Nk, 128, True, bias=True, seed=14)


def test_fwd_bf16_bias_noncausal_d64(orc):
    check_fwd(orc, 1, 2, 1, 190, 190, 64, False, bias=True)


@pytest.mark.parametrize("per_batch", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_fwd_bf16_bias_rows_of_vectors(orc, per_batch, d):
    """Rows of 388 keys (a multiple of 4: whole key tiles are read as 16-byte
    vectors) with a ragged last tile (read element by element); with a shared
    bias the three batch elements run side by side, with a per-batch one in the
    usual order."""
    check_fwd(orc, 3, 4, 2, 388, 388, d, True, bias=True, per_batch_bias=per_batch)


def test_fwd_bf16_bias_unaligned_view(orc):
    """A bias view that starts 4 bytes into its allocation: the rows are not
    16-byte aligned, so every tile is read element by element."""
    from parity import gpu_fwd

    inp = synth.make_dense(2, 2, 2, 256, 256, 128, seed=3, with_dout=False)
    b = synth.alibi_like_bias(2, 256, 256)
    store = torch.empty(b.numel() + 1, dtype=torch.float32, device="cuda")
    view = store[1:].view(b.shape)
    view.copy_(b.cuda())
    assert view.data_ptr() % 16 != 0
    o, lse = gpu_fwd(inp, True, bias=view)
    o_ref, lse_ref = orc.fwd(inp.q, inp.k, inp.v, bias=b, causal=True)
    assert max_abs(o.double().numpy(), o_ref) <= TOL_O_BF16
    assert max_abs(lse.double().numpy(), lse_ref) <= TOL_LSE_BF16


def test_fwd_f32_single_head(orc):
    """The fp32 workload: batch 1, 1 head, N=128, d=64, non-causal."""
    check_fwd(orc, 1, 1, 1, 128, 128, 64, False, dtype=torch.float32)


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_f32_general(orc, causal):
    check_fwd(orc, 2, 4, 2, 150, 150, 128, causal, dtype=torch.float32, bias=True)


@pytest.mark.parametrize("causal", [False, True])
def test_fwd_varlen(orc, causal):
    from exact_io_aware_57_b200 import attn

    lens = [5, 130, 1, 257, 64, 128]
    inp = synth.make_packed(lens, 4, 2, 128, seed=3)
    cu = inp.cu_seqlens.cuda()
    o, lse = attn.attn_fwd_varlen(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), cu, cu, max(lens), max(lens),
                                  causal=causal)
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    o_ref, l_ref = orc.fwd_varlen(inp.q, inp.k, inp.v, inp.cu_seqlens, inp.cu_seqlens, causal=causal)
    assert max_abs(o.cpu().double().numpy(), o_ref) <= TOL_O_BF16
    assert max_abs(lse.cpu().double().numpy(), l_ref) <= TOL_LSE_BF16


def test_fwd_full_size_mha_d64(orc):
    """Batch 4, 16 heads, N=2048, d=64, non-causal, at full size; sampled rows."""
    from exact_io_aware_57_b200 import attn

    inp = synth.make_dense(4, 16, 16, 2048, 2048, 64, with_dout=False)
    o, lse = attn.attn_fwd(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), causal=False)
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    eo, el = check_fwd_sampled(orc, inp.q, inp.k, inp.v, o.cpu(), lse.cpu(), False,
                               [(0, 0), (1, 7), (3, 15)], sample_rows(2048))
    assert eo <= TOL_O_BF16 and el <= TOL_LSE_BF16, (eo, el)


@pytest.mark.parametrize("d,causal", [(128, True), (64, False)])
def test_fwd_naive_comparator(orc, d, causal):
    """The materialising three-kernel comparator computes the same function."""
    from exact_io_aware_57_b200 import attn

    inp = synth.make_dense(2, 4, 2, 300, 300, d, with_dout=False, seed=9)
    o, lse = attn.attn_fwd_naive(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), causal=causal)
    torch.cuda.synchronize()
    o_ref, l_ref = orc.fwd(inp.q, inp.k, inp.v, causal=causal)
    assert max_abs(o.cpu().double().numpy(), o_ref) <= TOL_O_BF16
    assert max_abs(lse.cpu().double().numpy(), l_ref) <= TOL_LSE_BF16
