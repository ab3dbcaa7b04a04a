"""GPU parity of the backward (pba_backward, through the C ABI) against the
fp64 oracle, element by element.

Each gradient element must lie within the bound of the kernels' rounding model
(tests/bwd_bound.py): fp32 scores and exponents, bf16 dbias, bf16 P and dS in
fp32 tensor-core sums, and the forward's own measured errors in the lse and
the bf16 output the backward starts from.  The bound is about 0.6 % of |dS|
for dbias and a few percent of a typical dq, dk, dv element; the relative L2
error (<= 1e-2) stays as a second guard.  Small problems are checked in full;
the benchmark's shape (N=8192, H=16, D=64) on sampled query rows (dq, dbias,
every head) and sampled key rows (dk, dv, four heads).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import pair_biased_attention_b200 as pba
import workloads as W
from bwd_bound import dbias_bound, dk_bound, dq_bound, dv_bound, excess, head_terms

pytestmark = pytest.mark.gpu


def _np(x):
    return x.detach().double().cpu().numpy()


def _rel_l2(name, got, ref):
    den = np.linalg.norm(ref)
    if den > 0:
        rel = np.linalg.norm(got - ref) / den
        assert rel <= 1e-2, f"{name}: relative L2 error {rel:.3e}"


def _check_head(name, t, got, ref, k, q, dout, tau, full_rows=True, full_cols=True):
    """Element-wise bound checks of one (b, h); `t` from head_terms."""
    if "dbias" in got:
        e = excess(got["dbias"], ref["dbias"], dbias_bound(t))
        assert e <= 0, f"{name} dbias: error exceeds its bound by {e:.3e}"
    if "dq" in got and full_cols:
        e = excess(got["dq"], ref["dq"], dq_bound(t, k, tau))
        assert e <= 0, f"{name} dq: error exceeds its bound by {e:.3e}"
    if full_rows and "dk" in got:
        e = excess(got["dk"], ref["dk"], dk_bound(t, q, tau))
        assert e <= 0, f"{name} dk: error exceeds its bound by {e:.3e}"
        e = excess(got["dv"], ref["dv"], dv_bound(t, dout))
        assert e <= 0, f"{name} dv: error exceeds its bound by {e:.3e}"


def _run(name, q, k, v, bias, mask, seed=0, scale=None):
    out, lse = pba.pba_forward(q, k, v, bias, mask, softmax_scale=scale)
    g = torch.Generator(q.device.type).manual_seed(seed + 100)
    dout = torch.randn(q.shape, generator=g, device=q.device).to(torch.bfloat16)
    dq, dk, dv, dbias, delta = pba.pba_backward(q, k, v, bias, mask, out, lse, dout, softmax_scale=scale)
    torch.cuda.synchronize()
    assert pba.pba_last_device_error() == pba.PBA_OK
    B, H, Nq, D = q.shape
    bias_e = bias.expand(B, H, -1, -1)
    ref = oracle.pba_backward(q, k, v, bias_e, dout, mask, softmax_scale=scale)
    fwd = oracle.pba(q, k, v, bias_e, mask, softmax_scale=scale)
    tau = scale if scale else 1.0 / math.sqrt(D)
    got = {"dq": _np(dq), "dk": _np(dk), "dv": _np(dv), "dbias": _np(dbias)}
    qn, kn, vn, bn, don, on, ln = (_np(x) for x in (q, k, v, bias_e, dout, out, lse))
    for b in range(B):
        valid = np.ones(k.shape[2], dtype=bool) if mask is None else mask[b].cpu().numpy() != 0
        for h in range(H):
            t = head_terms(qn[b, h], kn[b, h], vn[b, h], bn[b, h], valid, don[b, h], on[b, h], ln[b, h],
                           fwd["o"][b, h], fwd["lse"][b, h], tau)
            _check_head(f"{name} b={b} h={h}", t, {n: x[b, h] for n, x in got.items()},
                        {n: ref[n][b, h] for n in got}, kn[b, h], qn[b, h], don[b, h], tau)
    for n in got:
        _rel_l2(f"{name} {n}", got[n], ref[n])
    d_ref = (dout.double() * out.double()).sum(-1).cpu().numpy()
    assert np.abs(_np(delta) - d_ref).max() <= 1e-3 * max(1.0, np.abs(d_ref).max())


@pytest.mark.parametrize("B,H,Nq,Nk,D,mask_frac", [
    (1, 2, 128, 128, 64, 0.0),     # one tile each way
    (2, 3, 200, 264, 64, 0.1),     # ragged query and key tiles, mask
    (1, 2, 384, 256, 32, 0.2),     # D = 32, several tiles
    (1, 1, 64, 512, 64, 0.5),      # half the keys masked
    (1, 2, 130, 1000, 32, 0.1),    # eight key steps with a ragged last one (the bias ring wraps twice)
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
    _run("bwd broadcast", q, k, v, bias[:1, :1], mask, seed=9, scale=0.2)


def test_backward_minus_inf_bias(cuda_device):
    q, k, v, bias, _ = W.random_attn(1, 2, 136, 264, 64, seed=4, device=cuda_device)
    full = torch.zeros((1, 2, 136, 264), dtype=torch.bfloat16, device=cuda_device)
    full.copy_(bias)
    full[0, 0, 5, :] = -math.inf            # a row with no valid key
    full[0, 1, 10:40, 7::3] = -math.inf
    _run("bwd -inf", q, k, v, full, None)


def _sampled(cfg, device, heads, n_rows=48, seed=11):
    """dq and dbias on sampled query rows of every head, dk and dv on sampled
    key rows of `heads`, each element within its bound."""
    q, k, v, bias, mask = W.attn_inputs(cfg, device)
    out, lse = pba.pba_forward(q, k, v, bias, mask)
    dout = torch.randn(q.shape, generator=torch.Generator(q.device.type).manual_seed(seed), device=q.device).to(
        torch.bfloat16)
    dq, dk, dv, dbias, _ = pba.pba_backward(q, k, v, bias, mask, out, lse, dout)
    torch.cuda.synchronize()
    assert pba.pba_last_device_error() == pba.PBA_OK
    N, D = cfg.N, cfg.D
    tau = 1.0 / math.sqrt(D)
    valid = np.ones(N, dtype=bool) if mask is None else mask[0].cpu().numpy() != 0
    rows = W.sample_rows(N, n_rows, seed=cfg.seed)
    rows_t = torch.as_tensor(rows, device=q.device)
    sel = lambda x, h: x[:, h:h + 1].index_select(2, rows_t)
    for h in range(cfg.H):
        # dq and dbias of a query row depend on that row alone
        ref = oracle.pba_backward(sel(q, h), k[:, h:h + 1], v[:, h:h + 1], sel(bias, h), sel(dout, h), mask)
        fwd = oracle.pba(sel(q, h), k[:, h:h + 1], v[:, h:h + 1], sel(bias, h), mask)
        t = head_terms(_np(sel(q, h))[0, 0], _np(k[0, h]), _np(v[0, h]), _np(sel(bias, h))[0, 0], valid,
                       _np(sel(dout, h))[0, 0], _np(sel(out, h))[0, 0], _np(lse[0, h])[rows], fwd["o"][0, 0],
                       fwd["lse"][0, 0], tau)
        got = {"dq": _np(sel(dq, h))[0, 0], "dbias": _np(sel(dbias, h))[0, 0]}
        _check_head(f"bwd {cfg.name} h={h} rows", t, got, {"dq": ref["dq"][0, 0], "dbias": ref["dbias"][0, 0]},
                    _np(k[0, h]), None, None, tau, full_rows=False)
        _rel_l2(f"bwd {cfg.name} h={h} dq rows", got["dq"], ref["dq"][0, 0])
    keys = W.sample_rows(N, n_rows, seed=cfg.seed + 1)
    hs = torch.as_tensor(heads, device=q.device)
    pick = lambda x: x.index_select(1, hs)
    # dk and dv of a key need every query row: the oracle's full backward on these heads
    ref = oracle.pba_backward(pick(q), pick(k), pick(v), pick(bias), pick(dout), mask)
    fwd = oracle.pba(pick(q), pick(k), pick(v), pick(bias), mask)
    for n, h in enumerate(heads):
        t = head_terms(_np(q[0, h]), _np(k[0, h]), _np(v[0, h]), _np(bias[0, h]), valid, _np(dout[0, h]),
                       _np(out[0, h]), _np(lse[0, h]), fwd["o"][0, n], fwd["lse"][0, n], tau, cols=keys)
        got = {"dk": _np(dk[0, h])[keys], "dv": _np(dv[0, h])[keys]}
        e = excess(got["dk"], ref["dk"][0, n][keys], dk_bound(t, _np(q[0, h]), tau))
        assert e <= 0, f"bwd {cfg.name} h={h} dk: error exceeds its bound by {e:.3e}"
        e = excess(got["dv"], ref["dv"][0, n][keys], dv_bound(t, _np(dout[0, h])))
        assert e <= 0, f"bwd {cfg.name} h={h} dv: error exceeds its bound by {e:.3e}"
        _rel_l2(f"bwd {cfg.name} h={h} dk keys", got["dk"], ref["dk"][0, n][keys])
        _rel_l2(f"bwd {cfg.name} h={h} dv keys", got["dv"], ref["dv"][0, n][keys])


def test_backward_benchmark_shape_sampled(cuda_device):
    """The benchmark's backward shapes (ring8k: N=8192, H=16, D=64, bf16, no
    mask) on sampled rows: dq and dbias of every head, dk and dv of four."""
    _sampled(W.RING8K, cuda_device, heads=[0, 5, 10, 15])
    torch.cuda.empty_cache()
