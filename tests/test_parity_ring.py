"""Key-sharded forward through libattn's kernels on one GPU: the ring of
ranks is emulated in one process (each virtual rank's exchange hands it the
chunk the ring would bring), so the per-block partials (attn_fwd_partial) and
their merge (attn_merge_partials) run exactly as on several GPUs, and every
rank's rows are compared with the fp64 oracle on the whole sequence.  Chunks
of 640 rows end inside key tiles; GQA 4:2."""
import pytest
import torch

from exact_io_aware_57_b200 import synth
from exact_io_aware_57_b200.ring import chunk_rows, ring_attention_fwd
from parity import TOL_LSE_BF16, TOL_O_BF16, max_abs

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def virtual_exchange(chunks, rank, world):
    """The ring transfer of rank `rank`, served from the chunks in memory."""
    state = {"s": 0}

    def post(k, v):
        state["s"] += 1
        c = (rank - state["s"]) % world

        class _Handle:
            def wait(self):
                return chunks[c]

        return _Handle()

    return post


@pytest.mark.parametrize("world,causal,d", [(4, True, 128), (4, False, 128), (3, True, 64), (2, False, 64)])
def test_ring_forward_matches_oracle(orc, world, causal, d):
    C = 640
    N = C * world
    inp = synth.make_dense(1, 4, 2, N, N, d, with_dout=False, seed=9)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    chunks = [(k[:, chunk_rows(N, world, r)].contiguous(), v[:, chunk_rows(N, world, r)].contiguous())
              for r in range(world)]
    o_ref, lse_ref = orc.fwd(inp.q, inp.k, inp.v, causal=causal)
    for r in range(world):
        rows = chunk_rows(N, world, r)
        o, lse = ring_attention_fwd(q[:, rows].contiguous(), *chunks[r], rank=r, world=world, causal=causal,
                                    exchange=virtual_exchange(chunks, r, world))
        torch.cuda.synchronize()
        eo = max_abs(o.cpu().double().numpy(), o_ref[:, rows])
        el = max_abs(lse.cpu().double().numpy(), lse_ref[:, :, rows])
        assert eo <= TOL_O_BF16 and el <= TOL_LSE_BF16, (r, eo, el)


def test_partial_over_whole_sequence_is_the_forward(orc):
    """One block holding every key: the partial result, merged alone, is attn_fwd."""
    from exact_io_aware_57_b200 import attn

    inp = synth.make_dense(2, 4, 4, 300, 300, 128, with_dout=False, seed=2)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    op, lp = attn.attn_fwd_partial(q, k, v, causal=True)
    o_ref, lse_ref = orc.fwd(inp.q, inp.k, inp.v, causal=True)
    torch.cuda.synchronize()
    assert max_abs(op.cpu().double().numpy(), o_ref) <= TOL_O_BF16
    assert max_abs(lp.cpu().double().numpy(), lse_ref) <= TOL_LSE_BF16
