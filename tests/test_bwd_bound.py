"""CPU check of the backward's per-element error bound (tests/bwd_bound.py).

A float32 / bfloat16 replay of the kernels' arithmetic (the rounding model in
bwd_bound.py: fp32 scores and exponents, bf16 dbias and bf16 P / dS in the
fp32 products) must stay inside the bound against the fp64 oracle, and
plausible kernel mistakes must break it: small dbias entries off by 10 %, a
Delta off by 1 %, half of the small dS terms of dq dropped, P normalised by a
log-sum-exp off by 0.01.  The flat bound it replaced (1e-2 max|ref| + 2^-7
|ref|) lets the first of these through.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from bwd_bound import dbias_bound, dk_bound, dq_bound, dv_bound, excess, head_terms


def _replay(q, k, v, bias, valid, dout, out_bf16, lse32, tau, delta_scale=1.0, lse_shift=0.0):
    """The kernels' arithmetic for one (b, h) in fp32 with bf16 roundings."""
    f = torch.float32
    Q, K, V, Bm, dO, O = (x.to(f) for x in (q, k, v, bias, dout, out_bf16))
    l2e = torch.tensor(1.4426950408889634, dtype=f)
    cs = torch.tensor(tau, dtype=f) * l2e
    bm = torch.where(valid[None, :], Bm, torch.tensor(-math.inf, dtype=f))
    lse = lse32 + lse_shift
    lse2 = torch.where(lse == -math.inf, torch.zeros_like(lse), lse * l2e)
    a = (Q @ K.T) * cs + (bm * l2e - lse2[:, None])
    P = torch.exp2(a)
    dP = dO @ V.T
    delta = (dO * O).sum(-1) * delta_scale
    dS = P * (dP - delta[:, None])
    dS16 = dS.to(torch.bfloat16)
    t32 = torch.tensor(tau, dtype=f)
    return {"dbias": dS16, "dq": t32 * (dS16.to(f) @ K), "dk": t32 * (dS16.to(f).T @ Q),
            "dv": P.to(torch.bfloat16).to(f).T @ dO, "dS16": dS16}


@pytest.fixture(scope="module")
def problem():
    B, H, Nq, Nk, D = 1, 2, 200, 264, 64
    q, k, v, bias, mask = W.random_attn(B, H, Nq, Nk, D, seed=21, mask_frac=0.1)
    bias = bias.clone()
    bias[0, 1, 9, :] = -math.inf          # a row with no valid key
    bias[0, 0, 20:60, 5::4] = -math.inf   # scattered -inf entries
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(22)).to(torch.bfloat16)
    tau = 1.0 / math.sqrt(D)
    fwd = oracle.pba(q, k, v, bias, mask)
    bwd = oracle.pba_backward(q, k, v, bias, dout, mask)
    return dict(q=q, k=k, v=v, bias=bias, mask=mask, dout=dout, tau=tau, fwd=fwd, bwd=bwd)


def _terms(pr, h, out_bf16, lse32):
    f64 = lambda x: x[0, h].double().numpy()
    valid = pr["mask"][0].bool().numpy()
    return head_terms(f64(pr["q"]), f64(pr["k"]), f64(pr["v"]), f64(pr["bias"]), valid, f64(pr["dout"]),
                      out_bf16[0, h].double().numpy(), lse32[0, h].double().numpy(), pr["fwd"]["o"][0, h],
                      pr["fwd"]["lse"][0, h], pr["tau"])


def _forward_as_kernel(pr):
    """The forward's outputs as the backward receives them: bf16 out, fp32 lse."""
    out_bf16 = torch.from_numpy(pr["fwd"]["o"]).to(torch.bfloat16)
    lse32 = torch.from_numpy(pr["fwd"]["lse"]).to(torch.float32)
    return out_bf16, lse32


def _run(pr, h, **plant):
    out_bf16, lse32 = _forward_as_kernel(pr)
    valid = pr["mask"][0].bool()
    r = _replay(pr["q"][0, h], pr["k"][0, h], pr["v"][0, h], pr["bias"][0, h], valid, pr["dout"][0, h],
                out_bf16[0, h], lse32[0, h], pr["tau"], **plant)
    t = _terms(pr, h, out_bf16, lse32)
    return r, t


@pytest.mark.parametrize("h", [0, 1])
def test_kernel_arithmetic_replay_is_inside_the_bound(problem, h):
    pr = problem
    r, t = _run(pr, h)
    ref = {n: pr["bwd"][n][0, h] for n in ("dq", "dk", "dv", "dbias")}
    k64, q64, do64 = (pr[n][0, h].double().numpy() for n in ("k", "q", "dout"))
    assert excess(r["dbias"].double().numpy(), ref["dbias"], dbias_bound(t)) <= 0
    assert excess(r["dq"].double().numpy(), ref["dq"], dq_bound(t, k64, pr["tau"])) <= 0
    assert excess(r["dk"].double().numpy(), ref["dk"], dk_bound(t, q64, pr["tau"])) <= 0
    assert excess(r["dv"].double().numpy(), ref["dv"], dv_bound(t, do64)) <= 0
    # the bound is not vacuous: the replay's typical error is a few percent of it
    ratio = np.abs(r["dq"].double().numpy() - ref["dq"]) / dq_bound(t, k64, pr["tau"])
    assert np.median(ratio) < 0.2


def test_small_dbias_entries_off_by_ten_percent_break_the_bound(problem):
    pr = problem
    r, t = _run(pr, 0)
    ref = pr["bwd"]["dbias"][0, 0]
    db = r["dbias"].double().numpy()
    small = (np.abs(ref) < np.median(np.abs(ref[ref != 0]))) & (ref != 0)
    bad = np.where(small, db * 1.1, db)
    assert excess(bad, ref, dbias_bound(t)) > 0
    # the flat bound this replaces let it through
    flat = 1e-2 * np.abs(ref).max() + 2.0 ** -7 * np.abs(ref)
    assert (np.abs(bad - ref) - flat).max() <= 0


def test_delta_off_by_one_percent_breaks_the_bound(problem):
    pr = problem
    r, t = _run(pr, 0, delta_scale=1.01)
    ref = pr["bwd"]
    k64 = pr["k"][0, 0].double().numpy()
    assert excess(r["dbias"].double().numpy(), ref["dbias"][0, 0], dbias_bound(t)) > 0
    assert excess(r["dq"].double().numpy(), ref["dq"][0, 0], dq_bound(t, k64, pr["tau"])) > 0


def test_dq_missing_small_terms_breaks_the_bound(problem):
    pr = problem
    r, t = _run(pr, 0)
    dS = r["dS16"].to(torch.float32)
    med = dS.abs()[dS != 0].median()
    dropped = torch.where(dS.abs() < med, torch.zeros_like(dS), dS)
    dq_bad = torch.tensor(pr["tau"], dtype=torch.float32) * (dropped @ pr["k"][0, 0].to(torch.float32))
    k64 = pr["k"][0, 0].double().numpy()
    assert excess(dq_bad.double().numpy(), pr["bwd"]["dq"][0, 0], dq_bound(t, k64, pr["tau"])) > 0


def test_p_from_a_shifted_lse_breaks_the_dv_bound(problem):
    pr = problem
    r, t = _run(pr, 0, lse_shift=0.01)
    do64 = pr["dout"][0, 0].double().numpy()
    assert excess(r["dv"].double().numpy(), pr["bwd"]["dv"][0, 0], dv_bound(t, do64)) > 0
