"""The ring schedule of context-parallel attention (pair_biased_attention_b200.ring)
on one GPU: P ranks emulated in one process, each computing pba_partial
against the key blocks in ring order and merging with softmax_merge, compared
with pba_forward of the same rows and with the fp64 oracle; and ring_attention
itself, its exchange loop included, as two processes sharing the GPU."""
import numpy as np
import pytest
import torch

import oracle
import pair_biased_attention_b200 as pba
import workloads as W
from pair_biased_attention_b200 import ring

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("P,N,D,mask_frac", [(4, 1024, 64, 0.1), (3, 768, 32, 0.0), (8, 1024, 64, 0.3)])
def test_emulated_ring_matches_forward_and_oracle(cuda_device, P, N, D, mask_frac):
    q, k, v, bias, mask = W.random_attn(1, 4, N, N, D, seed=P * 10 + D, device=cuda_device, mask_frac=mask_frac)
    L = N // P
    rows = [slice(r * L, (r + 1) * L) for r in range(P)]
    res = ring.ring_attention_emulated([q[:, :, s] for s in rows], [k[:, :, s].contiguous() for s in rows],
                                       [v[:, :, s].contiguous() for s in rows], [bias[:, :, s] for s in rows], mask)
    full_o, full_l = pba.pba_forward(q, k, v, bias, mask)
    ref = oracle.pba(q[:, :, :64], k, v, bias[:, :, :64], mask)  # rows of rank 0, checked against fp64
    for r, (o, lse) in enumerate(res):
        assert (o.float() - full_o[:, :, rows[r]].float()).abs().max().item() <= 1e-2
        assert (lse - full_l[:, :, rows[r]]).abs().max().item() <= 1e-4
    o0 = res[0][0][:, :, :64].double().cpu().numpy()
    assert np.abs(o0 - ref["o"]).max() <= 1e-2 + 2.0 ** -8 * np.abs(ref["o"]).max()


# ---------------------------------------------------------------- the ring itself, two processes
def _ring_rank_gpu(rank, world, rendezvous, out):
    """One rank of ring_attention with the real kernels: each process drives
    cuda:0, the key/value blocks travel through host memory over gloo while
    this rank's pba_partial of the current block runs on the GPU."""
    import datetime
    import os

    import torch.distributed as dist

    os.environ.setdefault("GLOO_SOCKET_IFNAME", "lo")
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"file://{rendezvous}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        pba.load_library()
        dev = torch.device("cuda:0")
        N, H, D = 512 * world, 4, 64
        q, k, v, bias, mask = W.random_attn(1, H, N, N, D, seed=77, device=dev, mask_frac=0.1)
        L = N // world
        rows = slice(rank * L, (rank + 1) * L)
        qr, br = q[:, :, rows], bias[:, :, rows]
        kb, vb = k[:, :, rows].contiguous(), v[:, :, rows].contiguous()
        ws = {}
        res = [ring.ring_attention(qr, kb, vb, br, mask, exchange=ring.host_staged_exchange, workspace=ws)
               for _ in range(2)]  # the second call reuses the partial and receive buffers
        fo, fl = pba.pba_forward(qr, k, v, br, mask)
        torch.cuda.synchronize()
        sample = [0, 1, 127, 128, L - 1]
        st = torch.as_tensor(sample, device=dev)
        ref = oracle.pba(qr.index_select(2, st), k, v, br.index_select(2, st), mask)
        o_s = res[1][0].index_select(2, st).double().cpu().numpy()
        out[rank] = {
            "fwd_o": max((o.float() - fo.float()).abs().max().item() for o, _ in res),
            "fwd_lse": max((lse - fl).abs().max().item() for _, lse in res),
            "oracle_excess": float((np.abs(o_s - ref["o"]) - (1e-2 + 2.0 ** -8 * np.abs(ref["o"]))).max()),
            "oracle_lse": float(np.abs(res[1][1].index_select(2, st).double().cpu().numpy() - ref["lse"]).max()),
            "same_twice": bool(torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])),
            "deverr": pba.pba_last_device_error(),
        }
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ring_attention_two_processes_real_kernels(cuda_device, tmp_path):
    """ring_attention's exchange loop itself (double-buffered point-to-point
    rotation of the key/value blocks, partials into one preallocated buffer,
    softmax_merge) with the real kernels: two ranks as two processes on one
    GPU, gloo moving host-staged copies of the blocks.  Each rank's rows match
    pba_forward of the same rows against all keys and the fp64 oracle."""
    import torch.multiprocessing as mp

    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_ring_rank_gpu, args=(world, str(tmp_path / "rdv"), out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        res = out[r]
        assert res["deverr"] == pba.PBA_OK
        assert res["fwd_o"] <= 1e-2 and res["fwd_lse"] <= 1e-4, res
        assert res["oracle_excess"] <= 0 and res["oracle_lse"] <= 1e-3, res
        assert res["same_twice"], res
