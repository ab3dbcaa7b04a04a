"""GPU parity of the backward (pba_backward, through the C ABI) against the
fp64 oracle, element by element.

The kernels recompute P from the forward's log-sum-exp in fp32, round P and
dS to bf16 for the tensor-core products and accumulate in fp32; dbias is
written in bf16.  Bounds: |g - ref| <= 1e-2 * max|ref| + 2^-7 |ref| per
element for dq, dk, dv, dbias, and a relative L2 error <= 1e-2.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import pair_biased_attention_b200 as pba
import workloads as W

pytestmark = pytest.mark.gpu


def _cmp(name, got, ref):
    g = got.double().cpu().numpy()
    scale = np.abs(ref).max() if ref.size else 0.0
    excess = (np.abs(g - ref) - (1e-2 * scale + 2.0 ** -7 * np.abs(ref))).max() if g.size else -1
    assert excess <= 0, f"{name}: error exceeds its bound by {excess:.3e} (scale {scale:.3e})"
    den = np.linalg.norm(ref)
    if den > 0:
        rel = np.linalg.norm(g - ref) / den
        assert rel <= 1e-2, f"{name}: relative L2 error {rel:.3e}"


def _run(name, q, k, v, bias, mask, seed=0, scale=None):
    out, lse = pba.pba_forward(q, k, v, bias, mask, softmax_scale=scale)
    g = torch.Generator(q.device.type).manual_seed(seed + 100)
    dout = torch.randn(q.shape, generator=g, device=q.device).to(torch.bfloat16)
    dq, dk, dv, dbias, delta = pba.pba_backward(q, k, v, bias, mask, out, lse, dout, softmax_scale=scale)
    torch.cuda.synchronize()
    assert pba.pba_last_device_error() == pba.PBA_OK
    ref = oracle.pba_backward(q, k, v, bias, dout, mask, softmax_scale=scale)
    for n in ("dq", "dk", "dv", "dbias"):
        _cmp(f"{name} {n}", {"dq": dq, "dk": dk, "dv": dv, "dbias": dbias}[n], ref[n])
    d_ref = (dout.double() * out.double()).sum(-1).cpu().numpy()
    assert np.abs(delta.double().cpu().numpy() - d_ref).max() <= 1e-3 * max(1.0, np.abs(d_ref).max())


@pytest.mark.parametrize("B,H,Nq,Nk,D,mask_frac", [
    (1, 2, 128, 128, 64, 0.0),     # one tile each way
    (2, 3, 200, 264, 64, 0.1),     # ragged query and key tiles, mask
    (1, 2, 384, 256, 32, 0.2),     # D = 32, several tiles
    (1, 1, 64, 512, 64, 0.5),      # half the keys masked
])
def test_backward_shapes(cuda_device, B, H, Nq, Nk, D, mask_frac):
    q, k, v, bias, mask = W.random_attn(B, H, Nq, Nk, D, seed=Nq + Nk + D, device=cuda_device, mask_frac=mask_frac)
    _run(f"bwd {B}x{H}x{Nq}x{Nk}x{D}", q, k, v, bias, mask, seed=Nq)


def test_backward_apb2k_head_slice(cuda_device):
    """The apb2k workload's shapes (N=2048, D=64, key padding), two heads."""
    cfg = W.APB2K
    q, k, v, bias, mask = W.attn_inputs(cfg, cuda_device)
    sl = lambda x: x[:, :2].contiguous()
    _run("bwd apb2k[:2]", sl(q), sl(k), sl(v), sl(bias), mask)


def test_backward_broadcast_bias_and_scale(cuda_device):
    q, k, v, bias, mask = W.random_attn(2, 2, 136, 136, 64, seed=3, device=cuda_device, mask_frac=0.1)
    b1 = bias[:1, :1]
    out, lse = pba.pba_forward(q, k, v, b1, mask, softmax_scale=0.2)
    dout = torch.randn(q.shape, generator=torch.Generator("cuda").manual_seed(9), device=q.device).to(torch.bfloat16)
    dq, dk, dv, dbias, _ = pba.pba_backward(q, k, v, b1, mask, out, lse, dout, softmax_scale=0.2)
    ref = oracle.pba_backward(q, k, v, b1.expand(2, 2, -1, -1), dout, mask, softmax_scale=0.2)
    for n, x in (("dq", dq), ("dk", dk), ("dv", dv), ("dbias", dbias)):
        _cmp(f"broadcast {n}", x, ref[n])


def test_backward_minus_inf_bias(cuda_device):
    q, k, v, bias, _ = W.random_attn(1, 2, 136, 264, 64, seed=4, device=cuda_device)
    full = torch.zeros((1, 2, 136, 264), dtype=torch.bfloat16, device=cuda_device)
    full.copy_(bias)
    full[0, 0, 5, :] = -math.inf            # a row with no valid key
    full[0, 1, 10:40, 7::3] = -math.inf
    _run("bwd -inf", q, k, v, full, None)
