"""No score-sized allocation: a forward and a backward at N = 8192 raise the
torch allocator's peak by the outputs and the linear workspace only, far
below one head's N x N fp32 score matrix (the library itself allocates
nothing; the binding allocates outputs and the O(N) workspace)."""
import pytest
import torch

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_peak_allocation_is_linear_in_n():
    from exact_io_aware_57_b200 import attn

    B, H, N, d = 1, 4, 8192, 128
    g = torch.Generator(device="cuda").manual_seed(0)
    q, k, v, do = (torch.randn(B, N, H, d, device="cuda", generator=g).bfloat16() for _ in range(4))
    torch.cuda.synchronize()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    o, lse = attn.attn_fwd(q, k, v, causal=True)
    dq, dk, dv = attn.attn_bwd(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    assert attn.attn_device_status() == 0
    grown = torch.cuda.max_memory_allocated() - base
    linear = 4 * q.numel() * q.element_size() + attn.attn_bwd_workspace_size(B, H, N, d) + B * H * N * 4
    score_matrix = N * N * 4                      # one head's fp32 scores
    assert grown <= linear + (1 << 20), (grown, linear)
    assert grown < score_matrix // 4
