"""GPU parity of the output projection of triangle attention
(tri_out_proj_forward, through the C ABI) against the fp64 oracle.

The kernel sums bf16 products in fp32 and rounds once to bf16, so every
output is within half a bf16 unit in the last place of the exact value plus
the fp32 summation error: |out - ref| <= 2^-8 |ref| + 1e-4 (values are
O(1)).  Almost all outputs equal the exact value rounded to bf16.
"""
import numpy as np
import pytest
import torch

import oracle
import pair_biased_attention_b200 as pba

pytestmark = pytest.mark.gpu

REL = 2.0 ** -8
ABS = 1e-4


def _bf16_np(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


def _inputs(N, H, D, c, seed, device):
    g = torch.Generator(device.type).manual_seed(seed)
    o = torch.randn((N, N, H, D), generator=g, device=device).to(torch.bfloat16)
    w_o = (torch.randn((H * D, c), generator=g, device=device) / (H * D) ** 0.5).to(torch.bfloat16)
    return o, w_o


def _run(N, H, D, c, seed, device, rows=None):
    o, w_o = _inputs(N, H, D, c, seed, device)
    out = pba.tri_out_proj_forward(o, w_o)
    torch.cuda.synchronize()
    assert pba.pba_last_device_error() == pba.PBA_OK
    assert out.shape == (N, N, c)
    ref = oracle.tri_out_proj(o, w_o, rows=rows)
    got = out.reshape(N * N, c)
    if rows is not None:
        got = got[torch.as_tensor(rows, device=device)]
    got = got.double().cpu().numpy()
    excess = (np.abs(got - ref) - (REL * np.abs(ref) + ABS)).max()
    assert excess <= 0, f"N={N} H={H} D={D} c={c}: error exceeds its bound by {excess:.3e}"
    exact = np.mean(got == _bf16_np(ref))
    assert exact >= 0.99, f"N={N} c={c}: only {exact:.4f} of outputs equal the rounded exact value"


@pytest.mark.parametrize("N,H,D,c", [
    (64, 4, 32, 128),   # 32 whole tiles
    (64, 2, 64, 64),    # c = 64: one weight slab, two output chunks
    (100, 4, 32, 128),  # 10000 rows: a ragged last tile
    (37, 1, 128, 64),   # odd N, one head of 128
])
def test_shapes(cuda_device, N, H, D, c):
    _run(N, H, D, c, seed=N + c, device=cuda_device)


def test_tri1024_sampled_rows(cuda_device):
    """The bench's size: 8 tiles per CTA at 148 CTAs; sampled rows, tile edges included."""
    N = 1024
    rng = np.random.default_rng(9)
    rows = np.unique(np.concatenate([[0, 127, 128, 129, N * N - 129, N * N - 128, N * N - 1],
                                     rng.integers(0, N * N, 3000)]))
    _run(N, 4, 32, 128, seed=11, device=cuda_device, rows=rows)


def test_after_triangle_attention(cuda_device):
    """The attention output feeds the projection as it is laid out."""
    N, H, D, c = 48, 4, 32, 64
    g = torch.Generator(cuda_device.type).manual_seed(5)
    q, k, v, gate = (torch.randn((N, N, H, D), generator=g, device=cuda_device).to(torch.bfloat16) for _ in range(4))
    bias = torch.randn((H, N, N), generator=g, device=cuda_device).to(torch.bfloat16)
    o = torch.empty_like(q)
    pba.tri_attn_forward(q, k, v, bias, gate, None, "starting", o, None)
    w_o = (torch.randn((H * D, c), generator=g, device=cuda_device) / (H * D) ** 0.5).to(torch.bfloat16)
    out = pba.tri_out_proj_forward(o, w_o)
    torch.cuda.synchronize()
    ref = oracle.tri_out_proj(o, w_o)
    got = out.reshape(N * N, c).double().cpu().numpy()
    assert (np.abs(got - ref) - (REL * np.abs(ref) + ABS)).max() <= 0


def test_zero_size(cuda_device):
    o = torch.zeros((0, 0, 4, 32), dtype=torch.bfloat16, device=cuda_device)
    w_o = torch.zeros((128, 64), dtype=torch.bfloat16, device=cuda_device)
    assert pba.tri_out_proj_forward(o, w_o).numel() == 0
