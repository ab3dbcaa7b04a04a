"""GPU parity of the fp32 path (pba_forward / pba_partial with fp32 inputs)
against the fp64 oracle, element by element, at fp32-level tolerances.

fp32 inputs whose tiles the Tensor Memory Accelerator can address run on the
tensor cores as three tf32 products per product (high and low parts of each
operand); the others (rows not 16-byte aligned) run one warp per query row on
the CUDA cores.  Both are held to the same bound, derived from the split:
each product is off by at most about 3 * 2^-22 of |x y|, a score by that
times sum_d |q_d k_d| plus the fp32 sums, i.e. a few 1e-6 in these inputs'
scaled scores; the output, a convex combination of V rows, then moves by a
similar relative amount.  The checks use 2e-5 on O (|O| <= 3 here) and on
the log-sum-exp, against 1e-2 / 1e-3 for the bf16 path.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import pair_biased_attention_b200 as pba
import workloads as W

pytestmark = pytest.mark.gpu

F32_TOL = 2e-5


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_device):
    pba.load_library()
    torch.cuda.synchronize()
    assert pba.pba_last_device_error() == pba.PBA_OK
    yield
    assert pba.pba_last_device_error() == pba.PBA_OK, "a kernel recorded a device error"


def _np(x):
    return x.detach().double().cpu().numpy()


def _check(name, out, lse, ref, tol=F32_TOL):
    o = _np(out)
    err = np.abs(o - ref["o"]).max() if o.size else 0.0
    assert err <= tol, f"{name}: output max-abs error {err:.3e}"
    lg, lr = _np(lse), ref["lse"]
    fin = np.isfinite(lr)
    assert np.array_equal(fin, np.isfinite(lg)), f"{name}: -inf pattern of the log-sum-exp differs"
    assert np.all(lg[~fin] == -np.inf)
    if fin.any():
        lerr = np.abs(lg[fin] - lr[fin]).max()
        assert lerr <= tol, f"{name}: lse max-abs error {lerr:.3e}"


def _run(name, q, k, v, bias, mask, scale=None):
    out, lse = pba.pba_forward(q, k, v, bias, mask, softmax_scale=scale)
    B, H = q.shape[:2]
    ref = oracle.pba(q, k, v, bias.expand(B, H, -1, -1), mask, softmax_scale=scale)
    _check(f"{name} forward", out, lse, ref)
    o_p, m_p, l_p = pba.pba_partial(q, k, v, bias, mask, softmax_scale=scale)
    torch.cuda.synchronize()
    assert pba.pba_last_device_error() == pba.PBA_OK
    _check(f"{name} partial", o_p, m_p + torch.log(l_p), ref)
    fin = np.isfinite(ref["lse"])
    # m_p is the block's true maximum
    assert np.abs(_np(m_p)[fin] - ref["m"][fin]).max(initial=0) <= F32_TOL


@pytest.mark.parametrize("B,H,Nq,Nk,D,mask_frac", [
    (1, 4, 256, 256, 32, 0.0),     # the pr1 shape
    (1, 2, 128, 64, 64, 0.0),      # one query tile, one key tile
    (2, 3, 200, 264, 64, 0.1),     # ragged query and key tiles, mask
    (1, 2, 300, 100, 32, 0.2),     # key tail inside the second tile
    (1, 1, 129, 1000, 64, 0.05),   # a second query tile of one row
    (2, 2, 64, 2048, 32, 0.0),     # many key tiles (the rescale path)
    (1, 2, 17, 12, 64, 0.5),       # fewer keys than a tile, half masked
])
def test_f32_shapes(cuda_device, B, H, Nq, Nk, D, mask_frac):
    q, k, v, bias, mask = W.random_attn(B, H, Nq, Nk, D, dtype=torch.float32, seed=Nq * 3 + Nk + D,
                                        device=cuda_device, mask_frac=mask_frac)
    _run(f"f32 {B}x{H}x{Nq}x{Nk} D={D}", q, k, v, bias, mask)


def test_f32_pr1_config(cuda_device):
    """The pr1 config (fp32, N=256, H=4, D=32, no mask) with its own inputs."""
    q, k, v, bias, mask = W.attn_inputs(W.PR1, cuda_device)
    assert q.dtype == torch.float32
    _run("pr1", q, k, v, bias, mask)


@pytest.mark.parametrize("scale", [0.125, 0.3])
def test_f32_scale_bias_broadcast_and_large_scores(cuda_device, scale):
    """Other scales, a bias shared by every batch and head, and scores spread
    over tens of units (bias std 8), where the running maximum moves often."""
    q, k, v, bias, mask = W.random_attn(2, 3, 333, 420, 64, dtype=torch.float32, seed=21, device=cuda_device,
                                        mask_frac=0.1, bias_std=8.0)
    _run(f"f32 scale={scale}", q, k, v, bias, mask, scale=scale)
    _run(f"f32 broadcast scale={scale}", q, k, v, bias[:1, :1], mask, scale=scale)


def test_f32_minus_inf_bias_and_empty_rows(cuda_device):
    q, k, v, bias, mask = W.random_attn(1, 2, 300, 260, 32, dtype=torch.float32, seed=8, device=cuda_device,
                                        mask_frac=0.05)
    full = torch.zeros((1, 2, 300, 264), dtype=torch.float32, device=cuda_device)
    full[..., :260] = bias
    bias = full[..., :260]
    bias[0, 0, 5, :] = -math.inf              # a row with no valid key
    bias[0, 1, 7, ::3] = -math.inf            # scattered -inf entries
    bias[0, 1, 200:260, :130] = -math.inf     # whole key tiles of some rows
    _run("f32 -inf", q, k, v, bias, mask)
    out, lse = pba.pba_forward(q, k, v, bias, mask)
    assert torch.all(out[0, 0, 5] == 0) and lse[0, 0, 5].item() == -math.inf
    assert not torch.isnan(out).any()


def test_f32_unaligned_rows_take_the_cuda_core_kernel(cuda_device):
    """Bias rows of 17 fp32 (68 bytes) cannot be tile-loaded: the CUDA-core
    kernel answers, to the same bound."""
    q, k, v, bias, mask = W.random_attn(1, 2, 40, 17, 64, dtype=torch.float32, seed=2, device=cuda_device,
                                        mask_frac=0.2, bias_row_pad=0)
    assert bias.stride(2) == 17
    _run("f32 unaligned", q, k, v, bias, mask)


def test_f32_apb2k_shape_sampled_rows(cuda_device):
    """The apb2k workload's shape (N=2048, H=16, D=64, last 10 % of keys
    masked) in fp32, on sampled query rows of three heads."""
    cfg = W.APB2K
    q, k, v, bias, mask = (t if t is None or t.dtype == torch.uint8 else t.float()
                           for t in W.attn_inputs(cfg, cuda_device))
    out, lse = pba.pba_forward(q, k, v, bias, mask)
    rows = W.sample_rows(cfg.N, 48, seed=4)
    rows_t = torch.as_tensor(rows, device=cuda_device)
    for h in (0, 7, 15):
        sel = lambda x: x[:, h:h + 1].index_select(2, rows_t)
        ref = oracle.pba(sel(q), k[:, h:h + 1], v[:, h:h + 1], sel(bias), mask)
        _check(f"f32 apb2k h={h}", sel(out), sel(lse), ref)


def test_f32_strided_views_and_batch_broadcast_bias(cuda_device):
    """Every other head of larger q, k, v tensors (head strides doubled), a
    bias shared by the batch only (batch stride 0) and a partial over a key
    block given as column views, all on the tensor-core path."""
    qb, kb, vb, bias, mask = W.random_attn(2, 6, 140, 264, 64, dtype=torch.float32, seed=33, device=cuda_device,
                                           mask_frac=0.1)
    q, k, v = qb[:, ::2], kb[:, ::2], vb[:, ::2]
    assert q.stride(1) == 2 * 140 * 64
    b1 = bias[:1, ::2]  # [1, 3, 140, 264] -> batch stride 0 once expanded
    _run("f32 strided", q, k, v, b1, mask)
    # a key block of the same problem as column views (block start a multiple of 8 keys)
    sl = slice(64, 200)
    o_p, m_p, l_p = pba.pba_partial(q, k[:, :, sl], v[:, :, sl], b1[..., sl], mask[:, sl])
    ref = oracle.pba_partial(q, k, v, b1.expand(2, 3, -1, -1), mask, k0=64, L=136)
    assert np.abs(_np(o_p) - ref["o"]).max() <= F32_TOL
    fin = ref["l"] > 0
    lse_p = _np(m_p) + np.log(np.where(_np(l_p) > 0, _np(l_p), 1.0))
    assert np.abs(lse_p[fin] - (ref["m"] + np.log(np.where(fin, ref["l"], 1.0)))[fin]).max(initial=0) <= F32_TOL
