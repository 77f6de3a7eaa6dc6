"""Key-sharded (context-parallel) forward: one sequence cut into equal chunks
across ranks, one process per GPU.

Rank r owns query, key and value rows [r C, (r + 1) C) of every batch element
and head (C = N / world).  Its output rows need every key they can see, and
those live on other ranks.  The key/value chunks therefore travel around a
ring: at step s rank r holds chunk c = (r - s) mod world, attends to it with
``attn_fwd_partial`` (its own query rows against that chunk only, an exact
partial result O_t, LSE_t), and meanwhile passes the chunk on to rank r + 1
and receives the next one from rank r - 1 with point-to-point sends into a
local buffer.  After world steps the partials merge exactly with
``attn_merge_partials`` ("Softmax does not need the matrix", "Carry the
Normalizer": the carried (m, l, a) state resumes the softmax over a new block
of keys, so the order of the blocks does not matter).

Causal masking by chunks: a chunk before the rank's own is fully visible, the
rank's own chunk is causal on its diagonal, a later chunk is invisible and is
skipped (its partial is never computed), but every rank still forwards every
chunk, so all ranks take the same exchange steps in the same order.

Every kernel reads only memory of its own device: received chunks land in
local buffers before any kernel touches them.  The compute and the merge run
in libattn's kernels; this module only schedules them and the exchange.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Block:
    step: int      # ring step at which this rank holds the chunk
    owner: int     # rank whose rows the chunk holds
    causal: bool   # True on the diagonal block (causal inside the chunk)


def blocks_for(rank: int, world: int, causal: bool) -> list[Block]:
    """Key chunks that rank ``rank`` attends to, in the order the ring brings them."""
    if not (0 <= rank < world):
        raise ValueError("rank out of range")
    out = []
    for s in range(world):
        c = (rank - s) % world
        if causal and c > rank:
            continue  # every key of a later chunk lies after every query row of this rank
        out.append(Block(s, c, causal and c == rank))
    return out


def chunk_rows(n: int, world: int, rank: int) -> slice:
    """Rows of a length-n sequence held by ``rank`` (n must divide evenly)."""
    if n % world:
        raise ValueError(f"sequence length {n} does not split into {world} equal chunks")
    c = n // world
    return slice(rank * c, (rank + 1) * c)


def p2p_exchange(group=None):
    """Ring exchange over torch.distributed: send (k, v) to rank + 1 and receive
    the next chunk from rank - 1 into fresh local buffers.  Returns a function
    that posts the transfers and returns a handle whose wait() yields the
    received (k, v)."""
    import torch
    import torch.distributed as dist

    def post(k, v):
        world = dist.get_world_size(group)
        rank = dist.get_rank(group)
        nxt, prv = (rank + 1) % world, (rank - 1) % world
        nk, nv = torch.empty_like(k), torch.empty_like(v)
        ops = [dist.P2POp(dist.isend, k.contiguous(), nxt, group), dist.P2POp(dist.isend, v.contiguous(), nxt, group),
               dist.P2POp(dist.irecv, nk, prv, group), dist.P2POp(dist.irecv, nv, prv, group)]
        reqs = dist.batch_isend_irecv(ops)

        class _Handle:
            def wait(self):
                for r in reqs:
                    r.wait()
                return nk, nv

        return _Handle()

    return post


def _gpu_block(q, k, v, causal, scale):
    from . import attn

    return attn.attn_fwd_partial(q, k, v, causal=causal, scale=scale)


def _gpu_merge(parts, out_dtype):
    import torch

    from . import attn

    o_parts = torch.stack([p[0] for p in parts])
    lse_parts = torch.stack([p[1] for p in parts])
    return attn.attn_merge_partials(o_parts, lse_parts, out_dtype=out_dtype)


def ring_attention_fwd(q, k, v, *, rank: int, world: int, causal: bool = False, scale=None, exchange=None,
                       block_fn=None, merge_fn=None):
    """Forward of this rank's query rows against the whole sequence.

    q, k, v: this rank's chunk, [B, C, Hq, d] and [B, C, Hkv, d] (bf16, on this
    rank's GPU).  exchange: a function posting the ring transfer (default:
    ``p2p_exchange()`` over the default process group).  block_fn(q, k, v,
    causal, scale) -> (O_t, LSE_t) and merge_fn(list of partials) -> (O, LSE)
    default to libattn's attn_fwd_partial and attn_merge_partials.
    Returns O [B, C, Hq, d] (q's dtype) and LSE [B, Hq, C] (fp32)."""
    if world == 1:
        exchange = exchange or (lambda k_, v_: None)
    exchange = exchange or p2p_exchange()
    block_fn = block_fn or _gpu_block
    merge_fn = merge_fn or (lambda parts: _gpu_merge(parts, q.dtype))
    visible = {b.step: b for b in blocks_for(rank, world, causal)}
    parts = []
    cur_k, cur_v = k, v
    for s in range(world):
        pending = exchange(cur_k, cur_v) if s + 1 < world else None  # overlaps the block's compute
        b = visible.get(s)
        if b is not None:
            parts.append(block_fn(q, cur_k, cur_v, b.causal, scale))
        if pending is not None:
            cur_k, cur_v = pending.wait()
    return merge_fn(parts)
