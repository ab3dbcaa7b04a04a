"""GPU parity of the triangle projections (tri_proj_forward, through the C
ABI) against the fp64 oracle.

The kernel sums bf16 products in fp32 and rounds once to bf16, so every
output is within half a bf16 unit in the last place of the exact value plus
the fp32 summation error: |out - ref| <= 2^-8 |ref| + 1e-4 (values are
O(1)).  Almost all outputs equal the exact value rounded to bf16; the rest
differ by one bf16 unit, where the fp32 sum landed on the other side of a
rounding boundary.
"""
import numpy as np
import pytest
import torch

import oracle
import pair_biased_attention_b200 as pba
import workloads as W

pytestmark = pytest.mark.gpu

REL = 2.0 ** -8
ABS = 1e-4


def _bf16_np(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


def _check(name, got, ref):
    got = got.double().cpu().numpy()
    err = np.abs(got - ref)
    excess = (err - (REL * np.abs(ref) + ABS)).max()
    assert excess <= 0, f"{name}: error exceeds its bound by {excess:.3e}"
    exact = np.mean(got == _bf16_np(ref))
    assert exact >= 0.99, f"{name}: only {exact:.4f} of outputs equal the rounded exact value"


def _run(N, c, H, D, seed, device, rows=None):
    cfg = W.TriConfig("p", N=N, c=c, H=H, D=D, seed=seed)
    z, w, wb = W.tri_pair_inputs(cfg, device)
    q, k, v, g, bias = pba.tri_proj_forward(z, w, wb, H)
    torch.cuda.synchronize()
    assert pba.pba_last_device_error() == pba.PBA_OK
    ref = oracle.tri_proj(z, w, wb, rows=rows)
    sel = slice(None) if rows is None else torch.as_tensor(rows, device=device)
    F = 4 * H * D
    flat = [x.reshape(N * N, H * D) for x in (q, k, v, g)]
    for i, (name, x) in enumerate(zip("qkvg", flat)):
        _check(f"{name} N={N} c={c} H={H}", x[sel], ref["out"][:, i * H * D:(i + 1) * H * D])
    _check(f"bias N={N} c={c} H={H}", bias.reshape(H, N * N)[:, sel], ref["bias"])
    assert F == w.shape[1]
    return q, k, v, g, bias


def test_tri512_sampled_rows(cuda_device):
    N = 512
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([[0, 127, 128, 129, 255, N * N - 129, N * N - 128, N * N - 1],
                                     rng.integers(0, N * N, 2000)]))
    _run(N, 128, 4, 32, seed=2, device=cuda_device, rows=rows)


@pytest.mark.parametrize("N,c,H,D", [
    (8, 128, 4, 32),     # 64 rows: one partial tile
    (24, 128, 4, 32),    # 576 rows: four tiles and a ragged one
    (40, 64, 4, 32),     # c = 64
    (32, 128, 8, 16),    # H = 8
    (32, 128, 2, 64),    # H = 2
    (16, 128, 1, 128),   # H = 1
    (136, 128, 4, 32),   # more tiles than SMs: several tiles per CTA
])
def test_shapes_full(cuda_device, N, c, H, D):
    _run(N, c, H, D, seed=N + c + H, device=cuda_device)


def test_zero_size(cuda_device):
    z = torch.zeros((0, 0, 128), dtype=torch.bfloat16, device=cuda_device)
    w = torch.zeros((128, 512), dtype=torch.bfloat16, device=cuda_device)
    wb = torch.zeros((128, 4), dtype=torch.bfloat16, device=cuda_device)
    q, k, v, g, bias = pba.tri_proj_forward(z, w, wb, 4)
    assert q.numel() == 0 and bias.numel() == 0


def test_projections_feed_triangle_attention(cuda_device):
    """The projected tensors are what tri_attn_forward takes: the attention of
    kernel-projected inputs equals the oracle's attention of the same inputs."""
    q, k, v, g, bias = _run(64, 128, 4, 32, seed=11, device=cuda_device)
    out, lse = pba.tri_attn_forward(q, k, v, bias, g, None, "starting")
    lines = [0, 31, 63]
    ref = oracle.tri_attn(q, k, v, bias, g, None, ending=False, lines=lines)
    o = out[lines].double().cpu().numpy()
    assert np.abs(o - ref["o"]).max() <= 1e-2 + REL * np.abs(ref["o"]).max()
