"""GPU parity of pair weighted averaging (pwa_forward, through the C ABI)
against the fp64 oracle, element by element.

Same tolerances as the attention: bf16 output within 1e-2 + 2^-8 |ref|
(bf16 weights P in the P V product, one bf16 rounding of the output), the
log-sum-exp within 1e-3, and the -inf pattern of the log-sum-exp exact.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import pair_biased_attention_b200 as pba
import workloads as W

pytestmark = pytest.mark.gpu

OUT_TOL = 1e-2
LSE_TOL = 1e-3
REL = 2.0 ** -8


def _cmp(name, out, lse, ref):
    o = out.double().cpu().numpy()
    excess = (np.abs(o - ref["o"]) - (OUT_TOL + REL * np.abs(ref["o"]))).max() if o.size else -1
    assert excess <= 0, f"{name}: output error exceeds its bound by {excess:.3e}"
    den = np.linalg.norm(ref["o"])
    if den > 0:
        assert np.linalg.norm(o - ref["o"]) / den <= 1e-2, name
    lg, lr = lse.double().cpu().numpy(), ref["lse"]
    fin = np.isfinite(lr)
    assert np.array_equal(fin, np.isfinite(lg)), f"{name}: -inf pattern of the log-sum-exp differs"
    if fin.any():
        assert np.abs(lg[fin] - lr[fin]).max() <= LSE_TOL, name


def _run(name, v, bias, mask, gate):
    out, lse = pba.pwa_forward(v, bias, mask, gate)
    torch.cuda.synchronize()
    assert pba.pba_last_device_error() == pba.PBA_OK
    _cmp(name, out, lse, oracle.pwa(v, bias, mask, gate))
    return out, lse


def _rand(S, N, H, D, seed, device, mask_frac=0.0, gate=True):
    g = torch.Generator(device.type).manual_seed(seed)
    v = torch.randn((S, N, H, D), generator=g, device=device).to(torch.bfloat16)
    bias = (torch.randn((H, N, N), generator=g, device=device) * 1.5).to(torch.bfloat16)
    gt = torch.randn((S, N, H, D), generator=g, device=device).to(torch.bfloat16) if gate else None
    mask = None
    if mask_frac:
        mask = (torch.rand((N,), generator=g, device=device) >= mask_frac).to(torch.uint8)
    return v, bias, mask, gt


def test_pwa512_full(cuda_device):
    v, bias, mask, gate = W.pwa_inputs(W.PWA512, cuda_device)
    _run("pwa512", v, bias, mask, gate)


@pytest.mark.parametrize("S,N,H,D,mask_frac,gate", [
    (8, 256, 2, 32, 0.0, False),    # one 256-feature tile exactly, whole key tiles, no mask
    (6, 256, 2, 32, 0.0, False),    # fewer sequences than a feature tile
    (7, 200, 3, 32, 0.1, True),     # ragged key tile, ragged row block
    (2, 128, 4, 32, 0.0, True),     # one key tile, one row block
    (5, 384, 2, 64, 0.2, True),     # D = 64 (4 sequences per feature tile): a ragged second tile
    (3, 1000, 1, 64, 0.5, False),   # long rows, half the keys masked
    (13, 520, 2, 32, 0.05, True),   # several units per CTA, ragged second feature tile
])
def test_shapes(cuda_device, S, N, H, D, mask_frac, gate):
    _run(f"pwa S={S} N={N} H={H} D={D}", *_rand(S, N, H, D, seed=S * 31 + N, device=cuda_device,
                                                mask_frac=mask_frac, gate=gate))


def test_minus_inf_logits_and_empty_rows(cuda_device):
    v, bias, _, gate = _rand(4, 264, 2, 32, seed=5, device=cuda_device)
    bias[0, 3, :] = -math.inf           # a row with no valid key
    bias[1, 10, ::2] = -math.inf        # scattered -inf logits
    bias[1, 100:200, :140] = -math.inf  # a tile region
    out, lse = _run("pwa -inf", v, bias, None, gate)
    assert torch.all(out[:, 3, 0] == 0) and lse[0, 3].item() == -math.inf
    mask = torch.zeros((264,), dtype=torch.uint8, device=cuda_device)  # no valid key at all
    out, lse = pba.pwa_forward(v, bias, mask, gate)
    assert torch.all(out == 0) and torch.all(lse == -math.inf)


def test_uniform_logits_give_mean_of_values(cuda_device):
    v, _, mask, _ = _rand(6, 256, 2, 32, seed=8, device=cuda_device, mask_frac=0.3, gate=False)
    bias = torch.zeros((2, 256, 256), dtype=torch.bfloat16, device=cuda_device)
    out, lse = pba.pwa_forward(v, bias, mask)
    mean = v.float()[:, mask.bool()].mean(dim=1, keepdim=True)
    assert (out.float() - mean).abs().max().item() <= 1e-2
    assert torch.allclose(lse, torch.full_like(lse, math.log(int(mask.sum()))), atol=1e-4)


def test_unaligned_key_mask(cuda_device):
    """A key mask at an odd address: both passes read it byte by byte."""
    v, bias, mask, gate = _rand(9, 264, 2, 32, seed=21, device=cuda_device, mask_frac=0.25)
    buf = torch.zeros((mask.numel() + 1,), dtype=torch.uint8, device=cuda_device)
    buf[1:] = mask
    odd = buf[1:]
    assert odd.data_ptr() % 8 != 0
    _run("pwa unaligned mask", v, bias, odd, gate)


def test_zero_sizes(cuda_device):
    v = torch.zeros((0, 64, 2, 32), dtype=torch.bfloat16, device=cuda_device)
    b = torch.zeros((2, 64, 64), dtype=torch.bfloat16, device=cuda_device)
    out, _ = pba.pwa_forward(v, b)
    assert out.numel() == 0
