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
them and moves the blocks.  The partials go straight into the slots of one
[P, B, H, n, D] buffer that ``softmax_merge`` reads as it is, and the two
key/value receive buffers are allocated once per call (or passed in, for
reuse across calls), so a step allocates nothing.  ``exchange`` moves one
block between ranks (default: ``torch.distributed`` point-to-point calls, NCCL
between GPUs); ``host_staged_exchange`` stages device blocks through host
memory for backends that move host tensors only (gloo).  ``partial_fn`` and
``merge_fn`` can be replaced, which the CPU tests of the schedule use.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch


def ring_block_order(world: int, rank: int) -> list[int]:
    """Key blocks rank ``rank`` works on, step by step: rank, rank-1, ... (mod world)."""
    return [(rank - s) % world for s in range(world)]


class _Requests:
    def __init__(self, reqs, after=None):
        self.reqs, self.after = reqs, after

    def wait(self):
        for r in self.reqs:
            r.wait()
        if self.after is not None:
            self.after()


def p2p_exchange(send: Sequence[torch.Tensor], recv: Sequence[torch.Tensor], dst: int, src: int, group=None):
    """Sends ``send`` to global rank ``dst`` and receives ``recv`` from global
    rank ``src`` with one batch of point-to-point calls; returns a handle whose
    ``wait()`` returns once ``recv`` holds the data."""
    import torch.distributed as dist

    ops = [dist.P2POp(dist.isend, t, dst, group) for t in send] + \
          [dist.P2POp(dist.irecv, t, src, group) for t in recv]
    return _Requests(dist.batch_isend_irecv(ops))


def host_staged_exchange(send, recv, dst: int, src: int, group=None):
    """As ``p2p_exchange`` for a backend that moves host tensors only: the
    device blocks are copied to host memory, sent and received there, and the
    received blocks are copied back to ``recv`` in ``wait()``."""
    import torch.distributed as dist

    hs = [t.to("cpu") for t in send]
    hr = [torch.empty(t.shape, dtype=t.dtype) for t in recv]
    reqs = [dist.isend(t, dst, group) for t in hs] + [dist.irecv(t, src, group) for t in hr]

    def copy_back():
        for d, h in zip(recv, hr):
            d.copy_(h)

    return _Requests(reqs, copy_back)


def alloc_partials(P: int, q: torch.Tensor):
    """The [P, B, H, n, D] O_p buffer and the [P, B, H, n] m_p, l_p buffers
    that the P partials of q fill and softmax_merge reads: fp32, as the
    kernels write them (fp64 for fp64 queries, which only a CPU replay of the
    schedule uses)."""
    B, H, n, D = q.shape
    dt = torch.float64 if q.dtype == torch.float64 else torch.float32
    o = torch.empty((P, B, H, n, D), dtype=dt, device=q.device)
    m = torch.empty((P, B, H, n), dtype=dt, device=q.device)
    return o, m, torch.empty_like(m)


def ring_attention(q, k, v, bias_rows, key_mask=None, group=None, softmax_scale=None,
                   partial_fn: Callable | None = None, merge_fn: Callable | None = None, stream=None,
                   exchange: Callable | None = None, workspace: dict | None = None):
    """Pair-biased attention of this rank's queries against all ranks' keys.

    q [B,H,n,D]: this rank's query rows.  k, v [B,H,L,D]: this rank's key
    block (block index = rank; every rank holds L keys).  bias_rows
    [B|1,H|1,n,P*L]: this rank's bias rows against all keys, with a row stride
    of a multiple of 8 and L a multiple of 8 (the key blocks are column views
    of it).  key_mask [B,P*L] uint8 or None.  ``workspace`` (a dict, filled on
    first use) keeps the partial and receive buffers for the next call of the
    same shapes.  Returns out [B,H,n,D] in q's dtype and the natural
    log-sum-exp [B,H,n] (fp32)."""
    import torch.distributed as dist

    from . import pba_partial, softmax_merge

    partial_fn = partial_fn or pba_partial
    merge_fn = merge_fn or softmax_merge
    exchange = exchange or p2p_exchange
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    L = k.shape[2]
    send_to, recv_from = (rank + 1) % world, (rank - 1) % world
    # global ranks of the ring neighbours, as the point-to-point calls want them
    if group is not None:
        send_to = dist.get_global_rank(group, send_to)
        recv_from = dist.get_global_rank(group, recv_from)
    ws = {} if workspace is None else workspace
    key = (tuple(q.shape), tuple(k.shape), q.dtype, k.dtype, q.device, world)
    if ws.get("key") != key:
        ws.clear()
        ws["key"] = key
        ws["parts"] = alloc_partials(world, q)
        ws["kv"] = [(torch.empty_like(k, memory_format=torch.contiguous_format),
                     torch.empty_like(v, memory_format=torch.contiguous_format)) for _ in range(2)]
    o_parts, m_parts, l_parts = ws["parts"]
    bufs = ws["kv"]
    bufs[0][0].copy_(k)
    bufs[0][1].copy_(v)
    for s, blk in enumerate(ring_block_order(world, rank)):
        cur_k, cur_v = bufs[s % 2]
        handle = None
        if s + 1 < world:
            # double buffering: the next block is in flight while this step's partial runs
            nxt_k, nxt_v = bufs[(s + 1) % 2]
            handle = exchange((cur_k, cur_v), (nxt_k, nxt_v), send_to, recv_from, group)
        cols = slice(blk * L, (blk + 1) * L)
        km = None if key_mask is None else key_mask[:, cols]
        partial_fn(q, cur_k, cur_v, bias_rows[..., cols], km, o_parts[s], m_parts[s], l_parts[s],
                   softmax_scale=softmax_scale, stream=stream)
        if handle is not None:
            # the next step receives into the buffer this step sent and read:
            # the send has read it once wait() returns, and the next receive is
            # ordered after this step's partial on the stream (NCCL waits on the
            # current stream; the host-staged copy back is issued on it)
            handle.wait()
    return merge_fn(o_parts, m_parts, l_parts, out_dtype=q.dtype, stream=stream)


def ring_attention_emulated(q_blocks: Sequence, k_blocks: Sequence, v_blocks: Sequence, bias_rows: Sequence,
                            key_mask=None, softmax_scale=None, partial_fn: Callable | None = None,
                            merge_fn: Callable | None = None, stream=None):
    """The same schedule for P ranks in one process (no exchange): rank r's
    partials visit the key blocks in ``ring_block_order(P, r)``, each into its
    slot of rank r's [P, ...] buffer.  Returns the per-rank (out, lse).  Used
    to check the ring on one GPU."""
    from . import pba_partial, softmax_merge

    partial_fn = partial_fn or pba_partial
    merge_fn = merge_fn or softmax_merge
    P = len(q_blocks)
    L = k_blocks[0].shape[2]
    res = []
    for r in range(P):
        o_parts, m_parts, l_parts = alloc_partials(P, q_blocks[r])
        for s, blk in enumerate(ring_block_order(P, r)):
            cols = slice(blk * L, (blk + 1) * L)
            km = None if key_mask is None else key_mask[:, cols]
            partial_fn(q_blocks[r], k_blocks[blk], v_blocks[blk], bias_rows[r][..., cols], km, o_parts[s],
                       m_parts[s], l_parts[s], softmax_scale=softmax_scale, stream=stream)
        res.append(merge_fn(o_parts, m_parts, l_parts, out_dtype=q_blocks[r].dtype, stream=stream))
    return res
