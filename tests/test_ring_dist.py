"""Key-sharded forward across ranks (exact_io_aware_57_b200.ring), host side:
2 and 3 gloo ranks on CPU, each holding one chunk of the sequence, pass the
key/value chunks around the ring with point-to-point sends.  The per-block
step and the merge are injected here as the fp64 oracle's (the product's are
libattn's kernels, checked on the GPU in test_parity_ring.py), so this checks
the schedule: which chunks each rank attends to, the causal diagonal, the
exchange, and that the merged rows equal the one-shot oracle on the whole
sequence."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from exact_io_aware_57_b200 import synth
from exact_io_aware_57_b200.ring import Block, blocks_for, chunk_rows, p2p_exchange, ring_attention_fwd


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def oracle_block(orc):
    def block(q, k, v, causal, scale):
        return orc.fwd(q, k, v, causal=causal, scale=scale)
    return block


def oracle_merge(orc):
    def merge(parts):
        B, C, H, d = parts[0][0].shape
        o_parts = np.stack([p[0].reshape(-1, d) for p in parts])                   # rows (b, i, h)
        lse_parts = np.stack([p[1].transpose(0, 2, 1).reshape(-1) for p in parts])  # same row order
        o, lse = orc.merge_partials(o_parts, lse_parts)
        return o.reshape(B, C, H, d), lse.reshape(B, C, H).transpose(0, 2, 1)
    return merge


def _worker(rank, world, port, causal, out):
    import torch.distributed as dist

    import oracle

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    orc = oracle.get()
    inp = synth.make_dense(2, 4, 2, 96 * world, 96 * world, 16, dtype=torch.float32, seed=7, with_dout=False)
    rows = chunk_rows(96 * world, world, rank)
    q, k, v = (t[:, rows].contiguous() for t in (inp.q, inp.k, inp.v))
    o, lse = ring_attention_fwd(q, k, v, rank=rank, world=world, causal=causal, exchange=p2p_exchange(),
                                block_fn=oracle_block(orc), merge_fn=oracle_merge(orc))
    o_ref, lse_ref = orc.fwd(inp.q, inp.k, inp.v, causal=causal)
    out[rank] = (float(np.max(np.abs(o - o_ref[:, rows]))), float(np.max(np.abs(lse - lse_ref[:, :, rows]))))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_forward_equals_one_shot(world, causal):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), causal, out), nprocs=world, join=True)
    for r in range(world):
        eo, el = out[r]
        assert eo <= 1e-12 and el <= 1e-12, (r, eo, el)


def test_blocks_for_schedule():
    # non-causal: every chunk, own chunk first, then the ring order
    assert [b.owner for b in blocks_for(1, 4, False)] == [1, 0, 3, 2]
    assert not any(b.causal for b in blocks_for(1, 4, False))
    # causal: own chunk (diagonal) at step 0, then the earlier chunks only
    assert blocks_for(2, 4, True) == [Block(0, 2, True), Block(1, 1, False), Block(2, 0, False)]
    assert blocks_for(0, 4, True) == [Block(0, 0, True)]
    # over all ranks every (query chunk, key chunk) pair is visited once
    for causal in (False, True):
        pairs = {(r, b.owner) for r in range(5) for b in blocks_for(r, 5, causal)}
        expect = {(r, c) for r in range(5) for c in range(5) if not causal or c <= r}
        assert pairs == expect


def test_chunk_rows_need_even_split():
    assert chunk_rows(12, 3, 2) == slice(8, 12)
    with pytest.raises(ValueError):
        chunk_rows(10, 3, 0)
