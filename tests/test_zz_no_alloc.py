"""pba_backward_noalloc: the backward entry point that allocates nothing on
the device, for callers that hold only the tensors they were handed (no
device allocator of their own) or must keep cudaMalloc / cudaFree, which can
synchronise the device, off their path.  Its Delta rows live in a fixed array
inside the library instead of a caller buffer.

Called through the C ABI twice in a row, on two problems of different sizes
(the second finds the first one's Delta still in the shared array), each
result is compared with pba_backward's on the same inputs, within the
backward tests' per-element tolerance.  This file is collected last, so a
run that stops at the first failure has run every other test before it.
"""
import ctypes
import math

import pytest
import torch

import pair_biased_attention_b200 as pba
import workloads as W

pytestmark = pytest.mark.gpu

# the backward tests' element-wise bound, reduced to two runs of the same
# kernels: a bf16 rounding of dS (2^-8 relative) plus a floor for exact zeros
REL = 2.0 ** -8


def _close(name, got, ref):
    g, r = got.double(), ref.double()
    bound = REL * r.abs() + 1e-6 * max(1.0, r.abs().max().item())
    worst = ((g - r).abs() - bound).max().item() if g.numel() else -1.0
    assert worst <= 0, f"{name}: differs from pba_backward by more than its bound ({worst:.3e})"


def _problem(B, H, Nq, Nk, D, seed, mask_frac, device):
    q, k, v, bias, mask = W.random_attn(B, H, Nq, Nk, D, seed=seed, device=device, mask_frac=mask_frac)
    out, lse = pba.pba_forward(q, k, v, bias, mask)
    g = torch.Generator(device.type).manual_seed(seed + 1)
    dout = torch.randn(q.shape, generator=g, device=device).to(torch.bfloat16)
    return q, k, v, bias, mask, out, lse, dout


def test_noalloc_backward_matches_pba_backward_on_two_calls(cuda_device):
    pba.load_library()
    p1 = _problem(2, 3, 200, 264, 64, seed=31, mask_frac=0.1, device=cuda_device)
    p2 = _problem(1, 4, 136, 392, 32, seed=32, mask_frac=0.0, device=cuda_device)
    refs = [pba.pba_backward(*p)[:4] for p in (p1, p2)]
    # two calls in a row into the shared Delta array, the second smaller in rows
    # (2*3*200 then 1*4*136) and stream-ordered after the first
    got = [pba.pba_backward_noalloc(*p) for p in (p1, p2)]
    torch.cuda.synchronize()
    assert pba.pba_last_device_error() == pba.PBA_OK
    for n, (g, r) in enumerate(zip(got, refs)):
        for name, a, b in zip(("dq", "dk", "dv", "dbias"), g, r):
            _close(f"call {n + 1} {name}", a, b)
    # the same problem again after the other one has used the array
    again = pba.pba_backward_noalloc(*p1)
    torch.cuda.synchronize()
    for name, a, b in zip(("dq", "dk", "dv", "dbias"), again, refs[0]):
        _close(f"call 3 {name}", a, b)


def test_noalloc_backward_rejects_rows_beyond_its_array(cuda_device):
    lib = pba.load_library()
    d = pba.PbaAttnDesc()
    d.B, d.H, d.Nq, d.Nk, d.D, d.dtype = 1, 16, pba.PBA_BWD_NOALLOC_MAX_ROWS // 16 + 1, 128, 64, pba.PBA_BF16
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    st = lib.pba_backward_noalloc(ctypes.byref(d), *([fake] * 12), None)
    assert st == pba.PBA_ERR_INVALID_ARG
