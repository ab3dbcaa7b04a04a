"""The benchmark's multi-rank plumbing on CPU (gloo, world size 2): each rank
runs the same workload, the job time is the maximum over ranks and the rate
counts every rank's work.  The kernels are not involved: the path has no
data-path collective (replicas of independent problems)."""
import os

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _init(rank, world, rendezvous):
    # a file rendezvous: no TCP port to collide with other processes; the
    # ranks' own gloo sockets on the loopback interface, whatever the host
    # name resolves to
    os.environ.setdefault("GLOO_SOCKET_IFNAME", "lo")
    dist.init_process_group("gloo", init_method=f"file://{rendezvous}", rank=rank, world_size=world)


def _rank_main(rank, world, rendezvous, times_ms, out):
    _init(rank, world, rendezvous)
    try:
        t = bench.max_over_ranks(times_ms[rank], True, device="cpu")
        out[rank] = t
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_job_time_is_max_over_ranks(world, tmp_path):
    times = [3.0, 7.5][:world]
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, str(tmp_path / "rdv"), times, out), nprocs=world, join=True,
                       start_method="spawn")
    assert [out[r] for r in range(world)] == [max(times)] * world


def test_job_throughput_counts_every_rank():
    # 2 ranks x 1e12 flop per step x 10 steps in 20 ms (slowest rank) = 1e15 flop/s
    assert bench.job_throughput(2, 1e12, 10, 20.0) == pytest.approx(1e15)
    assert bench.job_throughput(1, 1e12, 10, 20.0) == pytest.approx(5e14)


def test_single_rank_needs_no_group():
    assert bench.max_over_ranks(4.2, False) == 4.2


# ---------------------------------------------------------------- ring attention schedule (gloo, CPU)
def _oracle_partial(q, k, v, bias, key_mask, o_part, m_part, l_part, softmax_scale=None, stream=None):
    import oracle
    r = oracle.pba_partial(q, k, v, bias, key_mask, softmax_scale)
    for dst, n in ((o_part, "o"), (m_part, "m"), (l_part, "l")):
        dst.copy_(torch.from_numpy(r[n]))
    return o_part, m_part, l_part


def _oracle_merge(o, m, l, out_dtype=None, stream=None):
    import oracle
    r = oracle.merge(o, m, l)
    return torch.from_numpy(r["o"]), torch.from_numpy(r["lse"])


def _ring_problem(P, B=1, H=2, L=24, D=8, seed=0):
    g = torch.Generator().manual_seed(seed)
    N = P * L
    q = torch.randn(B, H, N, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, H, N, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, H, N, D, generator=g, dtype=torch.float64)
    bias = torch.randn(B, H, N, N, generator=g, dtype=torch.float64)
    mask = (torch.rand(B, N, generator=g) > 0.2).to(torch.uint8)
    return q, k, v, bias, mask


def _ring_rank(rank, world, rendezvous, out):
    from pair_biased_attention_b200 import ring
    _init(rank, world, rendezvous)
    try:
        q, k, v, bias, mask = _ring_problem(world)
        L = k.shape[2] // world
        rows = slice(rank * L, (rank + 1) * L)
        o, lse = ring.ring_attention(q[:, :, rows], k[:, :, rows], v[:, :, rows], bias[:, :, rows], mask,
                                     partial_fn=_oracle_partial, merge_fn=_oracle_merge)
        out[rank] = (o.numpy(), lse.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ring_attention_schedule_equals_full_attention(world, tmp_path):
    """The distributed ring (point-to-point rotation of the key/value blocks,
    one partial per step, tiled-softmax merge) gives each rank the attention
    of its rows against all keys."""
    import oracle
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_ring_rank, args=(world, str(tmp_path / "rdv"), out), nprocs=world, join=True,
                       start_method="spawn")
    q, k, v, bias, mask = _ring_problem(world)
    ref = oracle.pba(q, k, v, bias, mask)
    L = k.shape[2] // world
    for r in range(world):
        o, lse = out[r]
        assert abs(o - ref["o"][:, :, r * L:(r + 1) * L]).max() < 1e-12
        assert abs(lse - ref["lse"][:, :, r * L:(r + 1) * L]).max() < 1e-12


def test_ring_block_order():
    from pair_biased_attention_b200 import ring
    assert ring.ring_block_order(4, 0) == [0, 3, 2, 1]
    assert ring.ring_block_order(4, 2) == [2, 1, 0, 3]
    for P in (1, 2, 5):
        for r in range(P):
            assert sorted(ring.ring_block_order(P, r)) == list(range(P))
