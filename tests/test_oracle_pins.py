"""Pins of the fp64 oracle against things other than itself (CPU only).

Each check ties the oracle to something the pages or mathematics fix: a
library attention routine in fp64, brute force on tiny inputs, closed forms,
invariants, hand-derived worked examples (tests/golden/), and planted mistakes
that at least one pin must catch.  The definition checked is the one in the
header of oracle/pba_oracle.c (pair-biased attention, "Fold-CP: A Context
Parallelism Framework for Biomolecular Modeling", Table 1 and Figure 2).
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _num(x):
    if isinstance(x, str):
        return float(x)
    if isinstance(x, list):
        return [_num(y) for y in x]
    return x


def _rand_problem(B=2, H=3, Nq=37, Nk=53, D=16, seed=0, mask_frac=0.2, neg_inf_frac=0.0, bias_std=1.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, Nq, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, H, Nk, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, H, Nk, D, generator=g, dtype=torch.float64)
    bias = torch.randn(B, H, Nq, Nk, generator=g, dtype=torch.float64) * bias_std
    if neg_inf_frac > 0:
        bias[torch.rand(B, H, Nq, Nk, generator=g) < neg_inf_frac] = -math.inf
    mask = (torch.rand(B, Nk, generator=g) >= mask_frac).to(torch.uint8) if mask_frac > 0 else None
    return q, k, v, bias, mask


def _sdpa_reference(q, k, v, bias, mask):
    """torch's math-path scaled_dot_product_attention in fp64 with the bias
    and the key mask as an additive float mask."""
    add = bias.clone()
    if mask is not None:
        add = add + torch.where(mask.bool(), 0.0, -math.inf).to(torch.float64)[:, None, None, :]
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        o = F.scaled_dot_product_attention(q, k, v, attn_mask=add)
    scores = torch.einsum("bhid,bhjd->bhij", q, k) / math.sqrt(q.shape[-1]) + add
    lse = torch.logsumexp(scores, dim=-1)
    return o, lse, torch.isinf(lse)


# ---------------------------------------------------------------- library
@pytest.mark.parametrize("D", [4, 16, 32, 64])
@pytest.mark.parametrize("seed", [0, 1])
def test_matches_torch_sdpa_fp64(D, seed):
    q, k, v, bias, mask = _rand_problem(D=D, seed=seed, neg_inf_frac=0.05)
    r = oracle.pba(q, k, v, bias, mask)
    o_ref, lse_ref, empty = _sdpa_reference(q, k, v, bias, mask)
    keep = ~empty
    assert np.abs(r["o"][keep.numpy()] - o_ref[keep].numpy()).max() < 1e-12
    assert np.abs(r["lse"][keep.numpy()] - lse_ref[keep].numpy()).max() < 1e-12


def test_matches_torch_sdpa_fp64_n512():
    q, k, v, bias, mask = _rand_problem(B=1, H=2, Nq=512, Nk=512, D=32, seed=7, mask_frac=0.1)
    r = oracle.pba(q, k, v, bias, mask)
    o_ref, lse_ref, _ = _sdpa_reference(q, k, v, bias, mask)
    assert np.abs(r["o"] - o_ref.numpy()).max() < 1e-12
    assert np.abs(r["lse"] - lse_ref.numpy()).max() < 1e-12


# ---------------------------------------------------------------- brute force
def _brute_force(q, k, v, bias, mask):
    """Pure-Python loops, no max subtraction, math.fsum for the sums."""
    B, H, Nq, D = q.shape
    Nk = k.shape[2]
    tau = 1.0 / math.sqrt(D)
    o = np.zeros((B, H, Nq, D))
    lse = np.zeros((B, H, Nq))
    for b in range(B):
        for h in range(H):
            for i in range(Nq):
                w = []
                for j in range(Nk):
                    if mask is not None and mask[b, j] == 0:
                        continue
                    bij = float(bias[b, h, i, j])
                    if bij == -math.inf:
                        continue
                    s = tau * math.fsum(float(q[b, h, i, d]) * float(k[b, h, j, d]) for d in range(D)) + bij
                    w.append((math.exp(s), j))
                if not w:
                    lse[b, h, i] = -math.inf
                    continue
                Z = math.fsum(e for e, _ in w)
                lse[b, h, i] = math.log(Z)
                for d in range(D):
                    o[b, h, i, d] = math.fsum(e * float(v[b, h, j, d]) for e, j in w) / Z
    return o, lse


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_tiny(seed):
    q, k, v, bias, mask = _rand_problem(B=1, H=2, Nq=7, Nk=16, D=8, seed=seed, mask_frac=0.25, neg_inf_frac=0.1)
    r = oracle.pba(q, k, v, bias, mask)
    o_bf, lse_bf = _brute_force(q.numpy(), k.numpy(), v.numpy(), bias.numpy(), None if mask is None else mask.numpy())
    assert np.allclose(r["o"], o_bf, atol=1e-12, rtol=0)
    fin = np.isfinite(lse_bf)
    assert np.array_equal(fin, np.isfinite(r["lse"]))
    assert np.abs(r["lse"][fin] - lse_bf[fin]).max() < 1e-12


# ---------------------------------------------------------------- invariants and closed forms
def test_rows_sum_to_one():
    q, k, v, bias, mask = _rand_problem(seed=3, mask_frac=0.3)
    r = oracle.pba(q, k, torch.ones_like(v), bias, mask)
    assert np.abs(r["o"] - 1.0).max() < 1e-14


def test_shift_invariance_per_row():
    q, k, v, bias, mask = _rand_problem(seed=4, mask_frac=0.1)
    c = torch.randn(bias.shape[:-1], dtype=torch.float64, generator=torch.Generator().manual_seed(9)) * 5
    r0 = oracle.pba(q, k, v, bias, mask)
    r1 = oracle.pba(q, k, v, bias + c[..., None], mask)
    assert np.abs(r0["o"] - r1["o"]).max() < 1e-12
    assert np.abs((r0["lse"] + c.numpy()) - r1["lse"]).max() < 1e-12


def test_zero_q_zero_bias_gives_mean_of_valid_values():
    q, k, v, bias, mask = _rand_problem(seed=5, mask_frac=0.4)
    r = oracle.pba(torch.zeros_like(q), k, v, torch.zeros_like(bias), mask)
    mk = mask.numpy().astype(bool)
    for b in range(q.shape[0]):
        n_valid = mk[b].sum()
        mean = v[b][:, mk[b]].numpy().mean(axis=1)  # [H, D]
        assert np.abs(r["o"][b] - mean[:, None, :]).max() < 1e-13
        assert np.abs(r["lse"][b] - math.log(n_valid)).max() < 1e-13
        assert np.abs(r["l"][b] - n_valid).max() < 1e-12 and np.all(r["m"][b] == 0.0)


def test_one_hot_bias_closed_form():
    Nk, D = 20, 8
    q, k, v, bias, _ = _rand_problem(B=1, H=1, Nq=3, Nk=Nk, D=D, seed=6, mask_frac=0)
    bias = torch.zeros_like(bias)
    jstar = 11
    bias[..., jstar] = 30.0
    r = oracle.pba(torch.zeros_like(q), k, v, bias)
    e = math.exp(-30.0)
    vv = v[0, 0].numpy()
    expect = (vv[jstar] + e * (vv.sum(axis=0) - vv[jstar])) / (1.0 + (Nk - 1) * e)
    assert np.abs(r["o"][0, 0] - expect[None, :]).max() < 1e-14
    assert abs(r["lse"][0, 0, 0] - (30.0 + math.log1p((Nk - 1) * e))) < 1e-14


def test_single_key():
    q, k, v, bias, _ = _rand_problem(B=1, H=2, Nq=5, Nk=1, D=8, seed=7, mask_frac=0)
    r = oracle.pba(q, k, v, bias)
    assert np.abs(r["o"] - v.numpy()).max() == 0.0
    s0 = (q * k).sum(-1).numpy() / math.sqrt(8) + bias[..., 0].numpy()
    assert np.abs(r["lse"] - s0).max() < 1e-14


def test_fully_masked_rows():
    q, k, v, bias, _ = _rand_problem(B=1, H=2, Nq=4, Nk=9, D=8, seed=8, mask_frac=0)
    bias[0, 1, 2, :] = -math.inf
    mask = torch.ones(1, 9, dtype=torch.uint8)
    r = oracle.pba(q, k, v, bias, mask)
    assert np.all(r["o"][0, 1, 2] == 0.0) and r["lse"][0, 1, 2] == -math.inf
    assert r["m"][0, 1, 2] == -math.inf and r["l"][0, 1, 2] == 0.0
    r = oracle.pba(q, k, v, bias, torch.zeros(1, 9, dtype=torch.uint8))
    assert np.all(r["o"] == 0.0) and np.all(r["lse"] == -math.inf) and np.all(r["l"] == 0.0)


def test_permutations_and_head_independence():
    q, k, v, bias, mask = _rand_problem(seed=10, mask_frac=0.2)
    r0 = oracle.pba(q, k, v, bias, mask)
    g = torch.Generator().manual_seed(11)
    pk = torch.randperm(k.shape[2], generator=g)
    r1 = oracle.pba(q, k[:, :, pk], v[:, :, pk], bias[..., pk], mask[:, pk])
    assert np.abs(r0["o"] - r1["o"]).max() < 1e-13
    pq = torch.randperm(q.shape[2], generator=g)
    r2 = oracle.pba(q[:, :, pq], k, v, bias[:, :, pq], mask)
    assert np.abs(r0["o"][:, :, pq.numpy()] - r2["o"]).max() == 0.0
    q2 = q.clone()
    q2[:, 1] += 1.0
    r3 = oracle.pba(q2, k, v, bias, mask)
    assert np.array_equal(r0["o"][:, 0], r3["o"][:, 0]) and np.array_equal(r0["o"][:, 2], r3["o"][:, 2])
    assert np.abs(r0["o"][:, 1] - r3["o"][:, 1]).max() > 1e-3


# ---------------------------------------------------------------- partials and merge
@pytest.mark.parametrize("seed", range(5))
def test_merge_of_random_chunkings_equals_single_pass(seed):
    q, k, v, bias, mask = _rand_problem(B=1, H=2, Nq=9, Nk=61, D=8, seed=20 + seed, mask_frac=0.3,
                                        neg_inf_frac=0.05)
    full = oracle.pba(q, k, v, bias, mask)
    rng = np.random.default_rng(seed)
    Nk = k.shape[2]
    cuts = sorted(set(rng.integers(1, Nk, size=rng.integers(0, 8)).tolist()))
    edges = [0] + cuts + [Nk]
    blocks = list(zip(edges[:-1], edges[1:]))
    order = rng.permutation(len(blocks))
    parts = [oracle.pba_partial(q, k, v, bias, mask, k0=blocks[p][0], L=blocks[p][1] - blocks[p][0]) for p in order]
    o_parts = np.stack([p["o"] for p in parts])
    m_parts = np.stack([p["m"] for p in parts])
    l_parts = np.stack([p["l"] for p in parts])
    mrg = oracle.merge(o_parts, m_parts, l_parts)
    assert np.abs(mrg["o"] - full["o"]).max() < 1e-12
    fin = np.isfinite(full["lse"])
    assert np.array_equal(fin, np.isfinite(mrg["lse"]))
    assert np.abs(mrg["lse"][fin] - full["lse"][fin]).max() < 1e-12


def test_merge_identities():
    q, k, v, bias, mask = _rand_problem(B=1, H=2, Nq=6, Nk=30, D=8, seed=30, mask_frac=0.2)
    part = oracle.pba_partial(q, k, v, bias, mask, k0=0, L=30)
    full = oracle.pba(q, k, v, bias, mask)
    one = oracle.merge(part["o"][None], part["m"][None], part["l"][None])
    assert np.abs(one["o"] - full["o"]).max() < 1e-14 and np.abs(one["lse"] - full["lse"]).max() < 1e-14
    empty_o = np.zeros_like(part["o"])
    empty_m = np.full_like(part["m"], -np.inf)
    empty_l = np.zeros_like(part["l"])
    two = oracle.merge(np.stack([empty_o, part["o"]]), np.stack([empty_m, part["m"]]), np.stack([empty_l, part["l"]]))
    assert np.abs(two["o"] - full["o"]).max() < 1e-14 and np.abs(two["lse"] - full["lse"]).max() < 1e-14
    # a block with no valid key is exactly (0, -inf, 0)
    allmask = torch.zeros_like(mask)
    e = oracle.pba_partial(q, k, v, bias, allmask, k0=5, L=10)
    assert np.all(e["o"] == 0.0) and np.all(e["m"] == -np.inf) and np.all(e["l"] == 0.0)


def test_partial_block_sum_matches_brute_force():
    q, k, v, bias, mask = _rand_problem(B=1, H=1, Nq=5, Nk=16, D=8, seed=31, mask_frac=0.2)
    p = oracle.pba_partial(q, k, v, bias, mask, k0=4, L=7)
    sl = slice(4, 11)
    o_bf, lse_bf = _brute_force(q.numpy(), k[:, :, sl].numpy(), v[:, :, sl].numpy(), bias[..., sl].numpy(),
                                mask[:, sl].numpy())
    assert np.abs(p["o"] - o_bf).max() < 1e-12
    fin = np.isfinite(lse_bf)
    assert np.abs((p["m"] + np.log(p["l"]))[fin] - lse_bf[fin]).max() < 1e-12


# ---------------------------------------------------------------- triangle attention
def _tri_problem(N=12, H=2, D=8, seed=40, mask_frac=0.2):
    g = torch.Generator().manual_seed(seed)
    q, k, v, gt = (torch.randn(N, N, H, D, generator=g, dtype=torch.float64) for _ in range(4))
    bias = torch.randn(H, N, N, generator=g, dtype=torch.float64)
    pm = (torch.rand(N, N, generator=g) >= mask_frac).to(torch.uint8) if mask_frac > 0 else None
    return q, k, v, gt, bias, pm


def _tri_einsum(q, k, v, g, bias, pm, ending):
    """fp64 restatement with torch.einsum and torch.softmax (N <= 32)."""
    D = q.shape[-1]
    if not ending:
        s = torch.einsum("ijhd,ikhd->ijhk", q, k) / math.sqrt(D) + bias.permute(1, 0, 2)[None]  # b[h][j][k]
        if pm is not None:
            s = s + torch.where(pm.bool(), 0.0, -math.inf).double()[:, None, None, :]
        a = torch.softmax(s, dim=-1)
        o = torch.einsum("ijhk,ikhd->ijhd", a, v)
    else:
        s = torch.einsum("ijhd,kjhd->ijhk", q, k) / math.sqrt(D) + bias.permute(2, 0, 1)[:, None]  # b[h][k][i]
        if pm is not None:
            s = s + torch.where(pm.bool(), 0.0, -math.inf).double().t()[None, :, None, :]
        a = torch.softmax(s, dim=-1)
        o = torch.einsum("ijhk,kjhd->ijhd", a, v)
    lse = torch.logsumexp(s, dim=-1)
    return o * torch.sigmoid(g), lse


@pytest.mark.parametrize("ending", [False, True])
def test_tri_matches_einsum_restatement(ending):
    q, k, v, g, bias, pm = _tri_problem()
    r = oracle.tri_attn(q, k, v, bias, g, pm, ending=ending)
    o_ref, lse_ref = _tri_einsum(q, k, v, g, bias, pm, ending)
    if ending:  # line layout: line l = column j
        o_ref, lse_ref = o_ref.transpose(0, 1), lse_ref.transpose(0, 1)
    assert np.abs(r["o"] - o_ref.numpy()).max() < 1e-12
    assert np.abs(r["lse"] - lse_ref.numpy()).max() < 1e-12


def test_tri_starting_row_is_pair_biased_attention():
    q, k, v, g, bias, pm = _tri_problem(mask_frac=0.2)
    r = oracle.tri_attn(q, k, v, bias, None, pm, ending=False)
    for i in (0, 5, 11):
        # row i: queries j, keys k of head h -> [1, H, N, D]
        pr = oracle.pba(q[i].permute(1, 0, 2)[None], k[i].permute(1, 0, 2)[None], v[i].permute(1, 0, 2)[None],
                        bias[None], pm[i][None])
        assert np.abs(r["o"][i] - pr["o"][0].transpose(1, 0, 2)).max() < 1e-13
        assert np.abs(r["lse"][i] - pr["lse"][0].T).max() < 1e-13


def test_tri_ending_equals_starting_on_transpose():
    q, k, v, g, bias, pm = _tri_problem(mask_frac=0.2)
    end = oracle.tri_attn(q, k, v, bias, g, pm, ending=True)  # line l = column j
    T = lambda x: x.transpose(0, 1).contiguous()
    st = oracle.tri_attn(T(q), T(k), T(v), bias.transpose(1, 2).contiguous(), T(g), pm.t().contiguous(),
                         ending=False)  # line l = row l of the transpose = column l of the original
    assert np.abs(end["o"] - st["o"]).max() < 1e-13
    assert np.abs(end["lse"] - st["lse"]).max() < 1e-13


# ---------------------------------------------------------------- golden worked examples
def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("case", _golden()["attention"], ids=lambda c: c["name"])
def test_golden_attention(case):
    t = lambda x: torch.tensor(_num(x), dtype=torch.float64)[None, None]
    mask = None if case["key_mask"] is None else torch.tensor(case["key_mask"], dtype=torch.uint8)[None]
    r = oracle.pba(t(case["q"]), t(case["k"]), t(case["v"]), t(case["bias"]), mask)
    assert np.abs(r["o"][0, 0] - np.array(_num(case["o"]))).max() < 1e-14
    for key in ("lse", "m", "l"):
        exp = np.array(_num(case[key]))
        got = r[key][0, 0]
        assert np.array_equal(np.isfinite(exp), np.isfinite(got))
        fin = np.isfinite(exp)
        assert np.all(exp[~fin] == got[~fin])
        assert np.abs(got[fin] - exp[fin]).max(initial=0.0) < 1e-14


@pytest.mark.parametrize("case", _golden()["merge"], ids=lambda c: c["name"])
def test_golden_merge(case):
    r = oracle.merge(np.array(_num(case["o_parts"])), np.array(_num(case["m_parts"])), np.array(_num(case["l_parts"])))
    assert np.abs(r["o"] - np.array(_num(case["o"]))).max() < 1e-14
    assert np.abs(r["lse"] - np.array(_num(case["lse"]))).max() < 1e-14


@pytest.mark.parametrize("case", _golden()["triangle"], ids=lambda c: c["name"])
@pytest.mark.parametrize("gate", [False, True])
def test_golden_triangle(case, gate):
    bias = torch.tensor(_num(case["bias"]), dtype=torch.float64)
    v = torch.tensor(_num(case["v"]), dtype=torch.float64)
    z = torch.zeros_like(v)
    g = z if gate else None
    scale = 0.5 if gate else 1.0
    st = oracle.tri_attn(z, z, v, bias, g, None, ending=False)
    en = oracle.tri_attn(z, z, v, bias, g, None, ending=True)
    assert np.abs(st["o"] - scale * np.array(case["starting_o"])).max() < 1e-14
    assert np.abs(st["lse"] - np.array(case["starting_lse"])).max() < 1e-14
    # ending-node lines are columns: transpose back to [i][j]
    assert np.abs(en["o"].transpose(1, 0, 2, 3) - scale * np.array(case["ending_o"])).max() < 1e-14
    assert np.abs(en["lse"].transpose(1, 0, 2) - np.array(case["ending_lse"])).max() < 1e-14


# ---------------------------------------------------------------- triangle projections
# Fold-CP, Figure 2(a): q, k, v, g and the per-head bias of triangle attention
# are linear maps of the pair tensor z; the oracle writes them out as fp64 dot
# products.  Pinned against numpy's matmul (an independent implementation),
# closed forms and linearity.
def _proj_problem(N=6, c=16, F=24, H=3, seed=0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((N, N, c)), rng.standard_normal((c, F)), rng.standard_normal((c, H))


def test_proj_matches_numpy_matmul():
    z, w, wb = _proj_problem()
    r = oracle.tri_proj(z, w, wb)
    zf = z.reshape(-1, z.shape[-1])
    assert np.abs(r["out"] - zf @ w).max() < 1e-12
    assert np.abs(r["bias"] - (zf @ wb).T).max() < 1e-12
    assert r["bias"].shape == (3, 36)  # [H, N*N]: b[h, i, j] at h*N*N + i*N + j


def test_proj_one_hot_rows_select_weight_rows():
    _, w, wb = _proj_problem(c=16, F=24, H=3)
    z = np.eye(16)[[3, 0, 15, 7]]  # pair rows that pick weight rows 3, 0, 15, 7
    r = oracle.tri_proj(z, w, wb)
    assert np.array_equal(r["out"], w[[3, 0, 15, 7]])
    assert np.array_equal(r["bias"], wb[[3, 0, 15, 7]].T)


def test_proj_hand_worked_example():
    # z = [1, 2]; W = [[1, 0, 2], [3, 1, 0]]; W_b = [[1], [-1]]
    # out = [1*1 + 2*3, 1*0 + 2*1, 1*2 + 2*0] = [7, 2, 2]; bias = 1 - 2 = -1
    r = oracle.tri_proj(np.array([[1.0, 2.0]]), np.array([[1.0, 0, 2], [3, 1, 0]]), np.array([[1.0], [-1.0]]))
    assert np.array_equal(r["out"], [[7.0, 2.0, 2.0]]) and np.array_equal(r["bias"], [[-1.0]])


def test_proj_linearity_and_row_selection():
    z1, w, wb = _proj_problem(seed=1)
    z2, _, _ = _proj_problem(seed=2)
    a, b = 0.75, -2.5
    r = oracle.tri_proj(a * z1 + b * z2, w, wb)
    r1, r2 = oracle.tri_proj(z1, w, wb), oracle.tri_proj(z2, w, wb)
    assert np.abs(r["out"] - (a * r1["out"] + b * r2["out"])).max() < 1e-12
    rows = [35, 0, 17]
    rs = oracle.tri_proj(z1, w, wb, rows=rows)
    assert np.array_equal(rs["out"], r1["out"][rows]) and np.array_equal(rs["bias"], r1["bias"][:, rows])


# The output projection maps the concatenated heads of triangle attention back
# to the pair channels: out[r] = o[r, h*D + d] W_o.  Pinned on the flattening
# of (h, d), which is where a plausible mistake would sit.
def test_out_proj_one_hot_head_and_dim_select_weight_row():
    rng = np.random.default_rng(3)
    H, D, c = 4, 8, 16
    w_o = rng.standard_normal((H * D, c))
    o = np.zeros((2, 2, H, D))
    o[0, 1, 2, 5] = 1.0  # pair row 1 (i = 0, j = 1): head 2, dim 5 -> weight row 2*8 + 5
    o[1, 0, 0, 7] = -2.0  # pair row 2: head 0, dim 7 -> -2 x weight row 7
    out = oracle.tri_out_proj(o, w_o)
    assert out.shape == (4, c)
    assert np.array_equal(out[1], w_o[21]) and np.array_equal(out[2], -2.0 * w_o[7])
    assert not out[0].any() and not out[3].any()


def test_out_proj_identity_and_numpy():
    rng = np.random.default_rng(4)
    o = rng.standard_normal((3, 3, 2, 4))
    assert np.array_equal(oracle.tri_out_proj(o, np.eye(8)), o.reshape(9, 8))
    w = rng.standard_normal((8, 5))
    assert np.abs(oracle.tri_out_proj(o, w) - o.reshape(9, 8) @ w).max() < 1e-12


# ---------------------------------------------------------------- pair weighted averaging
# Fold-CP, Table 1 row "Pair Weighted Avg." (B*H*S*N^2*D; "2D ring + tiled
# softmax") and Figure 2 (grouped with the ring attention's merged softmax).  Reading: a
# softmax over the pair-bias logits alone, shared by the S sequences.  Pinned
# against pair-biased attention with zero queries (a different oracle path),
# torch's fp64 softmax and einsum, and closed forms.
def _pwa_problem(S=3, N=11, H=2, D=4, seed=0, mask_frac=0.3, neg_inf_frac=0.0):
    g = torch.Generator().manual_seed(seed)
    v = torch.randn((S, N, H, D), generator=g, dtype=torch.float64)
    bias = torch.randn((H, N, N), generator=g, dtype=torch.float64) * 2
    if neg_inf_frac:
        bias[torch.rand((H, N, N), generator=g) < neg_inf_frac] = -math.inf
    mask = (torch.rand((N,), generator=g) >= mask_frac).to(torch.uint8)
    gate = torch.randn((S, N, H, D), generator=g, dtype=torch.float64)
    return v, bias, mask, gate


def test_pwa_two_pass_reading_equals_one_pass():
    """The kernels take the softmax in two passes (the row log-sum-exp, then
    exp(b - lse) times the values); in exact arithmetic that is the one-pass
    softmax the oracle computes, masks and -inf logits included."""
    rng = np.random.default_rng(12)
    S, N, H, D = 3, 20, 2, 4
    v = rng.standard_normal((S, N, H, D))
    b = rng.standard_normal((H, N, N)) * 2.0
    b[1, 4, ::3] = -np.inf
    mask = (rng.random(N) > 0.25).astype(np.uint8)
    ref = oracle.pwa(v, b, mask)
    logits = np.where(mask[None, None, :] != 0, b, -np.inf)
    m = logits.max(axis=-1, keepdims=True)
    lse = (m + np.log(np.exp(logits - m).sum(axis=-1, keepdims=True)))[..., 0]
    w = np.exp(logits - lse[..., None])                     # second pass: normalised weights
    o = np.einsum("hij,sjhd->sihd", w, v)
    assert np.abs(lse - ref["lse"]).max() < 1e-12
    assert np.abs(o - ref["o"]).max() < 1e-12


def test_pwa_is_attention_with_zero_queries():
    v, bias, mask, _ = _pwa_problem(neg_inf_frac=0.1)
    r = oracle.pwa(v, bias, mask)
    S, N, H, D = v.shape
    q = torch.zeros((S, H, N, D), dtype=torch.float64)
    vt = v.permute(0, 2, 1, 3).contiguous()             # [S,H,N,D]
    bt = bias[None].expand(S, H, N, N).contiguous()      # the same logits for every sequence
    a = oracle.pba(q, q, vt, bt, mask[None].expand(S, N).contiguous())
    assert np.abs(r["o"] - a["o"].transpose(0, 2, 1, 3)).max() < 1e-13
    fin = np.isfinite(r["lse"])
    assert np.array_equal(fin, np.isfinite(a["lse"][0]))
    assert np.abs(r["lse"][fin] - a["lse"][0][fin]).max() < 1e-13


def test_pwa_matches_torch_softmax_einsum_with_gate():
    v, bias, mask, gate = _pwa_problem(S=4, N=17, H=3, D=5, seed=1)
    r = oracle.pwa(v, bias, mask, gate)
    logits = bias.masked_fill(mask[None, None, :] == 0, -math.inf)
    w = torch.softmax(logits, dim=-1)                    # [H,N,N]
    o = torch.einsum("hij,sjhd->sihd", w, v) * torch.sigmoid(gate)
    assert np.abs(r["o"] - o.numpy()).max() < 1e-13
    assert np.abs(r["lse"] - torch.logsumexp(logits, dim=-1).numpy()).max() < 1e-13


def test_pwa_closed_forms():
    v, _, mask, _ = _pwa_problem(S=2, N=9, H=2, D=3, seed=2, mask_frac=0.4)
    # equal logits: the mean of the valid values
    r = oracle.pwa(v, torch.zeros((2, 9, 9), dtype=torch.float64), mask)
    valid = mask.bool()
    assert np.abs(r["o"] - v[:, valid].mean(dim=1, keepdim=True).expand_as(v).numpy()).max() < 1e-14
    assert np.allclose(r["lse"], math.log(int(valid.sum())))
    # one finite logit per row: exactly that key's values
    pick = torch.tensor([4, 0, 8, 2, 2, 7, 1, 3, 5])
    bias = torch.full((2, 9, 9), -math.inf, dtype=torch.float64)
    bias[:, torch.arange(9), pick] = 1.5
    r = oracle.pwa(v, bias, None)
    assert np.array_equal(r["o"], v[:, pick].numpy()) and np.allclose(r["lse"], 1.5)
    # no valid key: zeros and -inf
    r = oracle.pwa(v, bias, torch.zeros(9, dtype=torch.uint8))
    assert np.all(r["o"] == 0) and np.all(r["lse"] == -np.inf)


# ---------------------------------------------------------------- backward
# Gradients of the same definition (training: Fold-CP, Figure 3 right).
# Pinned against torch autograd through its fp64 math-path attention (an
# independent implementation) and against central finite differences of the
# oracle's own forward on a tiny problem.
def _autograd_reference(q, k, v, bias, mask, dout):
    q, k, v, bias = (x.clone().requires_grad_(True) for x in (q, k, v, bias))
    add = bias
    if mask is not None:
        add = bias + torch.where(mask.bool(), 0.0, -math.inf).to(torch.float64)[:, None, None, :]
    with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
        o = F.scaled_dot_product_attention(q, k, v, attn_mask=add)
    o.backward(dout)
    return q.grad, k.grad, v.grad, bias.grad


@pytest.mark.parametrize("seed", [0, 1])
def test_backward_matches_torch_autograd(seed):
    q, k, v, bias, mask = _rand_problem(B=2, H=2, Nq=19, Nk=29, D=8, seed=seed, mask_frac=0.25)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(seed + 9), dtype=torch.float64)
    r = oracle.pba_backward(q, k, v, bias, dout, mask)
    dq, dk, dv, db = _autograd_reference(q, k, v, bias, mask, dout)
    for name, a, b in (("dq", r["dq"], dq), ("dk", r["dk"], dk), ("dv", r["dv"], dv), ("dbias", r["dbias"], db)):
        assert np.abs(a - b.numpy()).max() < 1e-12, name


def test_backward_finite_differences():
    q, k, v, bias, mask = _rand_problem(B=1, H=1, Nq=3, Nk=5, D=2, seed=4, mask_frac=0.0)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(5), dtype=torch.float64)
    r = oracle.pba_backward(q, k, v, bias, dout)
    loss = lambda qq, kk, vv, bb: float((oracle.pba(qq, kk, vv, bb)["o"] * dout.numpy()).sum())
    eps = 1e-6
    for name, t, pos in (("dq", q, 0), ("dk", k, 1), ("dv", v, 2), ("dbias", bias, 3)):
        flat = t.reshape(-1)
        for idx in range(0, flat.numel(), max(1, flat.numel() // 5)):
            args = [q, k, v, bias]
            plus, minus = [a.clone() for a in args], [a.clone() for a in args]
            plus[pos].reshape(-1)[idx] += eps
            minus[pos].reshape(-1)[idx] -= eps
            fd = (loss(*plus) - loss(*minus)) / (2 * eps)
            assert abs(fd - r[name].reshape(-1)[idx]) < 1e-7, (name, idx)


def test_backward_masked_keys_get_no_gradient():
    q, k, v, bias, mask = _rand_problem(B=1, H=2, Nq=7, Nk=13, D=4, seed=6, mask_frac=0.4)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(7), dtype=torch.float64)
    r = oracle.pba_backward(q, k, v, bias, dout, mask)
    dead = (mask[0] == 0).numpy()
    assert np.all(r["dbias"][..., dead] == 0) and np.all(r["dk"][:, :, dead] == 0) and np.all(r["dv"][:, :, dead] == 0)
    # dbias rows sum to zero (softmax Jacobian), dq is tau * dbias @ k
    assert np.abs(r["dbias"].sum(-1)).max() < 1e-12
    tau = 1.0 / math.sqrt(4)
    assert np.abs(r["dq"] - tau * np.einsum("bhij,bhjd->bhid", r["dbias"], k.numpy())).max() < 1e-12


# ---------------------------------------------------------------- planted mistakes
def _pin_suite(mutant):
    """Run a compact set of the pins against an oracle build; return the
    number that fail."""
    fails = 0
    gold = _golden()
    t = lambda x: torch.tensor(_num(x), dtype=torch.float64)[None, None]
    for case in gold["attention"]:
        mask = None if case["key_mask"] is None else torch.tensor(case["key_mask"], dtype=torch.uint8)[None]
        r = oracle.pba(t(case["q"]), t(case["k"]), t(case["v"]), t(case["bias"]), mask, mutant=mutant)
        exp_lse = np.array(_num(case["lse"]))
        fin = np.isfinite(exp_lse)
        if (np.abs(r["o"][0, 0] - np.array(_num(case["o"]))).max() > 1e-12
                or np.abs(r["lse"][0, 0][fin] - exp_lse[fin]).max(initial=0) > 1e-12):
            fails += 1
    for case in gold["merge"]:
        r = oracle.merge(np.array(_num(case["o_parts"])), np.array(_num(case["m_parts"])),
                         np.array(_num(case["l_parts"])), mutant=mutant)
        if np.abs(r["o"] - np.array(_num(case["o"]))).max() > 1e-12:
            fails += 1
    case = gold["triangle"][0]
    bias = torch.tensor(_num(case["bias"]), dtype=torch.float64)
    v = torch.tensor(_num(case["v"]), dtype=torch.float64)
    z = torch.zeros_like(v)
    en = oracle.tri_attn(z, z, v, bias, z, None, ending=True, mutant=mutant)
    if np.abs(en["o"].transpose(1, 0, 2, 3) - 0.5 * np.array(case["ending_o"])).max() > 1e-12:
        fails += 1
    q, k, v, bias, mask = _rand_problem(B=1, H=2, Nq=9, Nk=40, D=8, seed=21, mask_frac=0.2)
    full = oracle.pba(q, k, v, bias, mask, mutant=0)
    parts = [oracle.pba_partial(q, k, v, bias, mask, k0=a, L=b - a, mutant=mutant) for a, b in ((20, 40), (0, 7), (7, 20))]
    mrg = oracle.merge(np.stack([p["o"] for p in parts]), np.stack([p["m"] for p in parts]),
                       np.stack([p["l"] for p in parts]), mutant=mutant)
    if np.abs(mrg["o"] - full["o"]).max() > 1e-10:
        fails += 1
    q, k, v, bias, mask = _rand_problem(seed=0, neg_inf_frac=0.05)
    r = oracle.pba(q, k, v, bias, mask, mutant=mutant)
    o_ref, lse_ref, empty = _sdpa_reference(q, k, v, bias, mask)
    keep = (~empty).numpy()
    if np.abs(r["o"][keep] - o_ref.numpy()[keep]).max() > 1e-10:
        fails += 1
    z, w, wb = _proj_problem(seed=3)
    pr = oracle.tri_proj(z, w, wb, mutant=mutant)
    zf = z.reshape(-1, z.shape[-1])
    if np.abs(pr["out"] - zf @ w).max() > 1e-12 or np.abs(pr["bias"] - (zf @ wb).T).max() > 1e-12:
        fails += 1
    v, bias, mask, _ = _pwa_problem(seed=4)
    pw = oracle.pwa(v, bias, mask, mutant=mutant)
    logits = bias.masked_fill(mask[None, None, :] == 0, -math.inf)
    o = torch.einsum("hij,sjhd->sihd", torch.softmax(logits, dim=-1), v)
    if np.abs(pw["o"] - o.numpy()).max() > 1e-12:
        fails += 1
    q, k, v, bias, mask = _rand_problem(B=1, H=2, Nq=9, Nk=12, D=4, seed=8, mask_frac=0.2)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(3), dtype=torch.float64)
    bw = oracle.pba_backward(q, k, v, bias, dout, mask, mutant=mutant)
    ref = _autograd_reference(q, k, v, bias, mask, dout)
    if any(np.abs(bw[n] - t.numpy()).max() > 1e-12 for n, t in zip(("dq", "dk", "dv", "dbias"), ref)):
        fails += 1
    return fails


def test_default_build_passes_compact_pins():
    assert _pin_suite(0) == 0


@pytest.mark.parametrize("mutant", range(1, 16))
def test_planted_mistake_is_caught(mutant):
    assert _pin_suite(mutant) > 0, f"planted mistake {mutant} went unnoticed"
