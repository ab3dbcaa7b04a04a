"""Context-parallel pair-biased attention over a 1D ring of ranks.

"Fold-CP: A Context Parallelism Framework for Biomolecular Modeling",
Figure 2(c): the keys, values and pair bias of the attention move around a
one-dimensional ring of ranks and the per-step partials are combined by a
tiled-softmax merge; Table 1's caption adds that each ring takes P steps with
the next transfer overlapped.  Rank r of P holds the query rows of block r, the
key/value rows of block r, and its own rows of the pair bias against every
key (the row sharding of "Design-CP: Context Parallelism for Design of
Protein Nanoparticles"), so only the key/value blocks travel around the ring.
At step s rank r holds the key block (r - s) mod P; it computes the
online-softmax partial of its queries against that block with
``pba_partial`` while the block moves on to rank r + 1 and block
(r - s - 1) mod P arrives from rank r - 1.  After P steps ``softmax_merge``
combines the P partials into the exact softmax.

Every arithmetic step runs in the library's kernels; this module only orders
them and moves the blocks with ``torch.distributed`` point-to-point calls
(NCCL between GPUs).  ``partial_fn`` and ``merge_fn`` can be replaced, which
the CPU tests of the ring schedule use.
"""
from __future__ import annotations

from typing import Callable, Iterator, Sequence

import torch


def ring_block_order(world: int, rank: int) -> list[int]:
    """Key blocks rank ``rank`` works on, step by step: rank, rank-1, ... (mod world)."""
    return [(rank - s) % world for s in range(world)]


def _partials(q, bias_rows, key_mask, block_len: int, blocks: Iterator, softmax_scale, partial_fn, stream):
    """Partials of q against the key blocks the iterator yields as (block, k, v)."""
    parts = []
    for blk, k, v in blocks:
        cols = slice(blk * block_len, (blk + 1) * block_len)
        km = None if key_mask is None else key_mask[:, cols]
        parts.append(partial_fn(q, k, v, bias_rows[..., cols], km, softmax_scale=softmax_scale, stream=stream))
    return parts


def _merge(parts, out_dtype, merge_fn, stream):
    o = torch.stack([p[0] for p in parts])
    m = torch.stack([p[1] for p in parts])
    l = torch.stack([p[2] for p in parts])
    return merge_fn(o, m, l, out_dtype=out_dtype, stream=stream)


def ring_attention(q, k, v, bias_rows, key_mask=None, group=None, softmax_scale=None,
                   partial_fn: Callable | None = None, merge_fn: Callable | None = None, stream=None):
    """Pair-biased attention of this rank's queries against all ranks' keys.

    q [B,H,n,D]: this rank's query rows.  k, v [B,H,L,D]: this rank's key
    block (block index = rank; every rank holds L keys).  bias_rows
    [B|1,H|1,n,P*L]: this rank's bias rows against all keys, with a row stride
    of a multiple of 8 and L a multiple of 8 (the key blocks are column views
    of it).  key_mask [B,P*L] uint8 or None.  Returns out [B,H,n,D] in q's
    dtype and the natural log-sum-exp [B,H,n] (fp32)."""
    import torch.distributed as dist

    from . import pba_partial, softmax_merge

    partial_fn = partial_fn or pba_partial
    merge_fn = merge_fn or softmax_merge
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    L = k.shape[2]
    send_to, recv_from = (rank + 1) % world, (rank - 1) % world
    # global ranks of the ring neighbours, as the point-to-point calls want them
    if group is not None:
        send_to = dist.get_global_rank(group, send_to)
        recv_from = dist.get_global_rank(group, recv_from)

    def blocks():
        cur_k, cur_v = k.contiguous(), v.contiguous()
        for s, blk in enumerate(ring_block_order(world, rank)):
            reqs = []
            if s + 1 < world:
                # double buffering: the next block is in flight during this step
                nxt_k, nxt_v = torch.empty_like(cur_k), torch.empty_like(cur_v)
                ops = [dist.P2POp(dist.isend, cur_k, send_to, group), dist.P2POp(dist.isend, cur_v, send_to, group),
                       dist.P2POp(dist.irecv, nxt_k, recv_from, group), dist.P2POp(dist.irecv, nxt_v, recv_from, group)]
                reqs = dist.batch_isend_irecv(ops)
            yield blk, cur_k, cur_v
            for rq in reqs:
                rq.wait()
            if s + 1 < world:
                cur_k, cur_v = nxt_k, nxt_v

    parts = _partials(q, bias_rows, key_mask, L, blocks(), softmax_scale, partial_fn, stream)
    return _merge(parts, q.dtype, merge_fn, stream)


def ring_attention_emulated(q_blocks: Sequence, k_blocks: Sequence, v_blocks: Sequence, bias_rows: Sequence,
                            key_mask=None, softmax_scale=None, partial_fn: Callable | None = None,
                            merge_fn: Callable | None = None, stream=None):
    """The same schedule for P ranks in one process (no exchange): rank r's
    partials visit the key blocks in ``ring_block_order(P, r)``.  Returns the
    per-rank (out, lse).  Used to check the ring on one GPU."""
    from . import pba_partial, softmax_merge

    partial_fn = partial_fn or pba_partial
    merge_fn = merge_fn or softmax_merge
    P = len(q_blocks)
    L = k_blocks[0].shape[2]
    res = []
    for r in range(P):
        order = ring_block_order(P, r)
        blocks = ((b, k_blocks[b], v_blocks[b]) for b in order)
        parts = _partials(q_blocks[r], bias_rows[r], key_mask, L, blocks, softmax_scale, partial_fn, stream)
        res.append(_merge(parts, q_blocks[r].dtype, merge_fn, stream))
    return res
