"""The ring schedule of context-parallel attention (pair_biased_attention_b200.ring)
on one GPU: P ranks emulated in one process, each computing pba_partial
against the key blocks in ring order and merging with softmax_merge, compared
with pba_forward of the same rows and with the fp64 oracle."""
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
