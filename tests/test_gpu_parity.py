"""GPU parity: libpba (through its C ABI) against the fp64 oracle.

Every config of the workload list (workloads.py) plus edge cases.  Inputs are
the same seeded bf16/fp32 tensors on both sides (the oracle converts them to
fp64 exactly).  Tolerances: output max-abs <= 1e-2 and log-sum-exp max-abs
<= 1e-3 (bf16 inputs, fp32 accumulation, bf16 probabilities in P V); integer
mask and index handling bit-exact.  Large configs compare sampled rows the
oracle computes one by one.
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
# A bf16 output carries its own rounding, up to 2^-8 of |O| (half a unit in
# the last place of an 8-bit significand), which no kernel can avoid; bf16
# outputs are compared with OUT_TOL + BF16_OUT_REL * |O_ref| element by element.
BF16_OUT_REL = 2.0 ** -8
# internal guard on the relative L2 error of O (bf16 probabilities in P V)
REL_L2_TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_device):
    pba.load_library()
    torch.cuda.synchronize()
    assert pba.pba_last_device_error() == pba.PBA_OK
    yield
    assert pba.pba_last_device_error() == pba.PBA_OK, "a kernel recorded a device error"


def _cmp(name, o_gpu, lse_gpu, ref, rows_sel=None, out_tol=OUT_TOL, lse_tol=LSE_TOL):
    og = o_gpu.detach().double().cpu().numpy()
    o_ref = ref["o"]
    bound = out_tol + (BF16_OUT_REL * np.abs(o_ref) if o_gpu.dtype == torch.bfloat16 else 0.0)
    err = np.abs(og - o_ref).max() if og.size else 0.0
    excess = (np.abs(og - o_ref) - bound).max() if og.size else -1.0
    assert excess <= 0, f"{name}: output error {err:.3e} exceeds its bound by {excess:.3e}"
    den = np.linalg.norm(o_ref)
    if den > 0:
        rel = np.linalg.norm(og - o_ref) / den
        assert rel <= REL_L2_TOL, f"{name}: relative L2 error {rel:.3e}"
    if lse_gpu is not None:
        lg = lse_gpu.detach().double().cpu().numpy()
        lr = ref["lse"]
        fin = np.isfinite(lr)
        assert np.array_equal(fin, np.isfinite(lg)), f"{name}: -inf pattern of the log-sum-exp differs"
        assert np.all(lg[~fin] == -np.inf)
        if fin.any():
            lerr = np.abs(lg[fin] - lr[fin]).max()
            assert lerr <= lse_tol, f"{name}: lse max-abs error {lerr:.3e}"
    return err


def _oracle_rows(q, k, v, bias, mask, b, h, rows):
    """Oracle for query rows `rows` of (b, h)."""
    rows_t = torch.as_tensor(rows, device=q.device)
    qs = q[b:b + 1, h:h + 1].index_select(2, rows_t)
    bs = bias[b:b + 1, (h if bias.shape[1] > 1 else 0):(h if bias.shape[1] > 1 else 0) + 1].index_select(2, rows_t)
    m = None if mask is None else mask[b:b + 1]
    return oracle.pba(qs, k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1], bs, m)


# ------------------------------------------------------------------ configs
def test_pr1_fp32_forward_and_key_blocks(cuda_device):
    cfg = W.PR1
    q, k, v, bias, mask = W.attn_inputs(cfg, "cpu")
    ref = oracle.pba(q, k, v, bias, mask)
    qd, kd, vd, bd = (t.to(cuda_device) for t in (q, k, v, bias))
    out, lse = pba.pba_forward(qd, kd, vd, bd)
    _cmp("pr1 forward", out, lse, ref)
    # fp32 end to end: much tighter than the bf16 bound
    assert np.abs(out.double().cpu().numpy() - ref["o"]).max() < 1e-5
    # 4 key blocks of 64, merged in order and in a shuffled order
    L = cfg.N // cfg.blocks
    for order in (list(range(cfg.blocks)), [2, 0, 3, 1]):
        o_parts = torch.empty((cfg.blocks, cfg.B, cfg.H, cfg.N, cfg.D), device=cuda_device)
        m_parts = torch.empty((cfg.blocks, cfg.B, cfg.H, cfg.N), device=cuda_device)
        l_parts = torch.empty_like(m_parts)
        for slot, blk in enumerate(order):
            sl = slice(blk * L, (blk + 1) * L)
            pba.pba_partial(qd, kd[:, :, sl], vd[:, :, sl], bd[..., sl], None, o_parts[slot], m_parts[slot],
                            l_parts[slot])
        mo, ml = pba.softmax_merge(o_parts, m_parts, l_parts, out_dtype=torch.float32)
        _cmp(f"pr1 merge {order}", mo, ml, ref)
        assert np.abs(mo.double().cpu().numpy() - ref["o"]).max() < 1e-5


def test_apb2k_forward_full(cuda_device):
    cfg = W.APB2K
    q, k, v, bias, mask = W.attn_inputs(cfg, cuda_device)
    out, lse = pba.pba_forward(q, k, v, bias, mask)
    ref = oracle.pba(q, k, v, bias, mask)
    _cmp("apb2k", out, lse, ref)


def test_apb2k_partials_and_merge(cuda_device):
    cfg = W.APB2K
    q, k, v, bias, mask = W.attn_inputs(cfg, cuda_device)
    blocks = [(0, 1024), (1024, 1024)]  # the second block holds the masked tail
    o_parts = torch.empty((2, cfg.B, cfg.H, cfg.N, cfg.D), device=cuda_device)
    m_parts = torch.empty((2, cfg.B, cfg.H, cfg.N), device=cuda_device)
    l_parts = torch.empty_like(m_parts)
    for slot, (k0, L) in enumerate(blocks[::-1]):
        sl = slice(k0, k0 + L)
        pba.pba_partial(q, k[:, :, sl], v[:, :, sl], bias[..., sl], mask[:, sl], o_parts[slot], m_parts[slot],
                        l_parts[slot])
    mo, ml = pba.softmax_merge(o_parts, m_parts, l_parts, out_dtype=torch.bfloat16)
    rows = W.sample_rows(cfg.N, 64, seed=1)
    for h in (0, 7, 15):
        ref = _oracle_rows(q, k, v, bias, mask, 0, h, rows)
        _cmp(f"apb2k merge h={h}", mo[0:1, h:h + 1, rows], ml[0:1, h:h + 1, rows], ref)
        # partial of one block against the oracle's partial on that block
        pr = oracle.pba_partial(q[:, h:h + 1, rows], k[:, h:h + 1], v[:, h:h + 1], bias[:, h:h + 1, rows], mask,
                                k0=1024, L=1024)
        og = o_parts[0, :, h:h + 1, rows].double().cpu().numpy()
        assert np.abs(og - pr["o"]).max() <= OUT_TOL
        lse_p = (m_parts[0, :, h:h + 1, rows].double() + torch.log(l_parts[0, :, h:h + 1, rows].double())).cpu()
        assert np.abs(lse_p.numpy() - (pr["m"] + np.log(pr["l"]))).max() <= LSE_TOL


def _tri_lines_check(name, cfg, q, k, v, g, bias, ending, lines):
    out, lse = pba.tri_attn_forward(q, k, v, bias, g, None, "ending" if ending else "starting")
    ref = oracle.tri_attn(q, k, v, bias, g, None, ending=ending, lines=lines)
    if ending:
        o_sel = out[:, lines].transpose(0, 1)
        l_sel = lse[:, lines].transpose(0, 1)
    else:
        o_sel, l_sel = out[lines], lse[lines]
    _cmp(name, o_sel, l_sel, ref)
    return out, lse


@pytest.mark.parametrize("ending", [False, True])
def test_tri512_sampled_lines(cuda_device, ending):
    cfg = W.TRI512
    q, k, v, g, bias = W.tri_inputs(cfg, cuda_device)
    lines = W.sample_rows(cfg.N, 16, seed=cfg.seed)
    _tri_lines_check(f"tri512 ending={ending}", cfg, q, k, v, g, bias, ending, lines)


def test_ring8k_partials_merge_vs_forward_and_oracle(cuda_device):
    cfg = W.RING8K
    q, k, v, bias, mask = W.attn_inputs(cfg, cuda_device)
    L = cfg.N // cfg.blocks
    order = W.block_order(cfg)
    o_parts = torch.empty((cfg.blocks, cfg.B, cfg.H, cfg.N, cfg.D), device=cuda_device)
    m_parts = torch.empty((cfg.blocks, cfg.B, cfg.H, cfg.N), device=cuda_device)
    l_parts = torch.empty_like(m_parts)
    for slot, blk in enumerate(order):
        sl = slice(blk * L, (blk + 1) * L)
        pba.pba_partial(q, k[:, :, sl], v[:, :, sl], bias[..., sl], None, o_parts[slot], m_parts[slot], l_parts[slot])
    mo, ml = pba.softmax_merge(o_parts, m_parts, l_parts, out_dtype=torch.bfloat16)
    fo, fl = pba.pba_forward(q, k, v, bias)
    assert (mo.float() - fo.float()).abs().max().item() <= OUT_TOL
    assert (ml - fl).abs().max().item() <= LSE_TOL
    rows = W.sample_rows(cfg.N, 32, seed=cfg.seed)
    for h in range(cfg.H):
        ref = _oracle_rows(q, k, v, bias, mask, 0, h, rows)
        _cmp(f"ring8k merge h={h}", mo[:, h:h + 1, rows], ml[:, h:h + 1, rows], ref)
        _cmp(f"ring8k forward h={h}", fo[:, h:h + 1, rows], fl[:, h:h + 1, rows], ref)


def test_large16k_sampled_rows(cuda_device):
    cfg = W.LARGE16K
    q, k, v, bias, mask = W.attn_inputs(cfg, cuda_device)
    out, lse = pba.pba_forward(q, k, v, bias, mask)
    rows = W.sample_rows(cfg.N, 16, seed=cfg.seed)
    for h in range(cfg.H):
        ref = _oracle_rows(q, k, v, bias, mask, 0, h, rows)
        _cmp(f"large16k h={h}", out[:, h:h + 1, rows], lse[:, h:h + 1, rows], ref)
    del q, k, v, bias
    torch.cuda.empty_cache()


@pytest.mark.parametrize("ending", [False, True])
def test_tri1024_sampled_lines(cuda_device, ending):
    cfg = W.TRI1024
    q, k, v, g, bias = W.tri_inputs(cfg, cuda_device)
    lines = W.sample_rows(cfg.N, 8, seed=cfg.seed)
    _tri_lines_check(f"tri1024 ending={ending}", cfg, q, k, v, g, bias, ending, lines)


@pytest.mark.parametrize("N,H,D", [(136, 4, 32), (200, 2, 64)])
@pytest.mark.parametrize("ending", [False, True])
@pytest.mark.parametrize("masked", [False, True])
def test_tri_key_tail_and_pair_mask(cuda_device, N, H, D, ending, masked):
    """Triangle attention with N % 128 != 0: the last key tile runs past the
    end of every line and the last query tile is partly filled.  Both
    orientations, with and without a random pair mask, against the oracle's
    explicit index formulas.  With the mask, one line has every key masked
    and must give out = 0 and lse = -inf."""
    cfg = W.TriConfig(f"tail{N}", N=N, c=32, H=H, D=D, seed=N + (1 if ending else 0))
    q, k, v, g, bias = W.tri_inputs(cfg, cuda_device)
    dead = 3
    pm = None
    if masked:
        gen = torch.Generator("cuda").manual_seed(N * 3 + int(ending))
        pm = (torch.rand((N, N), generator=gen, device=cuda_device) > 0.25).to(torch.uint8)
        # the keys of line `dead`: row dead (starting node) or column dead (ending node)
        if ending:
            pm[:, dead] = 0
        else:
            pm[dead, :] = 0
    out, lse = pba.tri_attn_forward(q, k, v, bias, g, pm, "ending" if ending else "starting")
    lines = sorted({0, dead, 127, 128, N // 2, N - 1})
    ref = oracle.tri_attn(q, k, v, bias, g, pm, ending=ending, lines=lines)
    o_sel = out[:, lines].transpose(0, 1) if ending else out[lines]
    l_sel = lse[:, lines].transpose(0, 1) if ending else lse[lines]
    _cmp(f"tri tail N={N} D={D} ending={ending} masked={masked}", o_sel, l_sel, ref)
    if masked:
        o_dead = out[:, dead] if ending else out[dead]
        l_dead = lse[:, dead] if ending else lse[dead]
        assert torch.all(o_dead == 0) and torch.all(l_dead == -math.inf)


# ------------------------------------------------------------------ shapes and edge cases
@pytest.mark.parametrize("Nq,Nk,D,mask_frac", [
    (1, 1, 64, 0.0), (17, 17, 64, 0.0), (100, 100, 32, 0.2), (1000, 1000, 64, 0.05), (1025, 1025, 32, 0.0),
    (300, 129, 64, 0.1), (129, 700, 32, 0.0), (256, 256, 64, 0.5), (384, 1000, 64, 0.0), (77, 2048, 64, 0.02),
])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_shapes(cuda_device, Nq, Nk, D, mask_frac, dtype):
    q, k, v, bias, mask = W.random_attn(2, 3, Nq, Nk, D, dtype=dtype, seed=Nq * 7 + Nk, device=cuda_device,
                                        mask_frac=mask_frac)
    out, lse = pba.pba_forward(q, k, v, bias, mask)
    ref = oracle.pba(q, k, v, bias, mask)
    _cmp(f"shape {Nq}x{Nk} D={D} {dtype}", out, lse, ref)
    # a partial over the whole key range is the same problem in fp32
    o_p, m_p, l_p = pba.pba_partial(q, k, v, bias, mask)
    _cmp("partial over all keys", o_p, m_p + torch.log(l_p), ref)
    fin = np.isfinite(ref["lse"])
    mp = m_p.double().cpu().numpy()
    assert np.abs(mp[fin] - ref["m"][fin]).max(initial=0) <= LSE_TOL


@pytest.mark.parametrize("D", [32, 64])
@pytest.mark.parametrize("scale", [0.125, 0.25, 0.13, 0.3])
def test_bias_modes(cuda_device, D, scale):
    """The softmax warps add the bias to tau * (Q K^T) for every scale: powers
    of two (0.125, 0.25, where tau * s is exact) and others (0.13, 0.3).
    Against the oracle, masked and ragged, forward and partial, then unmasked
    whole tiles (no mask words)."""
    q, k, v, bias, mask = W.random_attn(2, 3, 333, 421, D, seed=int(scale * 1000) + D, device=cuda_device,
                                        mask_frac=0.1)
    out, lse = pba.pba_forward(q, k, v, bias, mask, softmax_scale=scale)
    ref = oracle.pba(q, k, v, bias, mask, softmax_scale=scale)
    _cmp(f"bias mode D={D} scale={scale}", out, lse, ref)
    o_p, m_p, l_p = pba.pba_partial(q, k, v, bias, mask, softmax_scale=scale)
    _cmp(f"bias mode partial D={D} scale={scale}", o_p, m_p + torch.log(l_p), ref)
    # unmasked whole tiles: the kernel instance without mask words
    q, k, v, bias, _ = W.random_attn(1, 2, 256, 512, D, seed=D + 1, device=cuda_device)
    out, lse = pba.pba_forward(q, k, v, bias, softmax_scale=scale)
    _cmp(f"bias mode unmasked D={D} scale={scale}", out, lse, oracle.pba(q, k, v, bias, softmax_scale=scale))


def test_bias_broadcast_over_heads_and_batch(cuda_device):
    q, k, v, bias, mask = W.random_attn(2, 4, 200, 300, 64, seed=5, device=cuda_device, mask_frac=0.1)
    b1 = bias[:1, :1]  # [1,1,Nq,Nk] -> strides 0 over b and h
    out, lse = pba.pba_forward(q, k, v, b1, mask)
    ref = oracle.pba(q, k, v, b1.expand(2, 4, -1, -1), mask)
    _cmp("broadcast bias", out, lse, ref)


def _padded_clone(b):
    """Copy of a bias view whose rows keep a 16-byte multiple stride."""
    nk = b.shape[-1]
    full = torch.zeros(b.shape[:-1] + (nk + (-nk) % 8,), dtype=b.dtype, device=b.device)
    full[..., :nk] = b
    return full[..., :nk]


@pytest.mark.parametrize("D,scale", [(64, None), (32, 0.25), (32, None), (64, 0.1)])
def test_minus_inf_bias_and_fully_masked_rows(cuda_device, D, scale):
    """-inf bias entries exclude their keys exactly like masked keys: a row
    with no valid key gives O = 0 and lse = -inf, scattered and tile-sized
    -inf regions drop out, and no NaN appears, with the default scale and a
    power-of-two scale alike."""
    q, k, v, bias, mask = W.random_attn(1, 2, 600, 260, D, seed=9, device=cuda_device, mask_frac=0.05)
    bias = _padded_clone(bias)
    bias[0, 0, 5, :] = -math.inf              # row with no valid key
    bias[0, 1, 7, ::3] = -math.inf            # scattered -inf entries
    bias[0, 1, 200:260, :130] = -math.inf     # a whole tile region
    out, lse = pba.pba_forward(q, k, v, bias, mask, softmax_scale=scale)
    ref = oracle.pba(q, k, v, bias, mask, softmax_scale=scale)
    _cmp("minus inf bias", out, lse, ref)
    assert torch.all(out[0, 0, 5] == 0) and lse[0, 0, 5].item() == -math.inf
    assert not torch.isnan(out.float()).any()
    o_p, m_p, l_p = pba.pba_partial(q, k, v, bias, mask, softmax_scale=scale)
    _cmp("minus inf bias, partial", o_p, m_p + torch.log(l_p), ref)
    assert not torch.isnan(o_p).any() and not torch.isnan(l_p).any()


def test_empty_inputs(cuda_device):
    q, k, v, bias, _ = W.random_attn(1, 2, 0, 64, 64, device=cuda_device)
    out, lse = pba.pba_forward(q, k, v, bias)
    assert out.numel() == 0
    # no keys: every row empty
    q, k, v, bias, _ = W.random_attn(1, 2, 40, 0, 64, device=cuda_device)
    out = torch.full((1, 2, 40, 64), 7.0, dtype=torch.bfloat16, device=cuda_device)
    lse = torch.zeros((1, 2, 40), device=cuda_device)
    pba.pba_forward(q, k, v, bias, None, out, lse)
    assert torch.all(out == 0) and torch.all(lse == -math.inf)
    o_p, m_p, l_p = pba.pba_partial(q, k, v, bias)
    assert torch.all(o_p == 0) and torch.all(m_p == -math.inf) and torch.all(l_p == 0)


def test_merge_edge_cases(cuda_device):
    g = torch.Generator("cuda").manual_seed(3)
    P, rows, D = 5, 1000, 64
    o_parts = torch.randn((P, rows, D), generator=g, device=cuda_device)
    m_parts = torch.randn((P, rows), generator=g, device=cuda_device) * 3
    l_parts = torch.rand((P, rows), generator=g, device=cuda_device) * 10 + 0.1
    # empty blocks in some rows, all-empty rows
    l_parts[1, ::7] = 0
    m_parts[1, ::7] = -math.inf
    l_parts[:, 13] = 0
    m_parts[:, 13] = -math.inf
    o_parts[:, 13] = 0
    ref = oracle.merge(o_parts, m_parts, l_parts)
    for dt in (torch.float32, torch.bfloat16):
        mo, ml = pba.softmax_merge(o_parts, m_parts, l_parts, out_dtype=dt)
        _cmp(f"merge {dt}", mo, ml, ref, out_tol=OUT_TOL if dt == torch.bfloat16 else 1e-5)
        assert torch.all(mo[13] == 0) and ml[13].item() == -math.inf
    # P = 1 is the identity on normalised O
    mo, ml = pba.softmax_merge(o_parts[:1].contiguous(), m_parts[:1].contiguous(), l_parts[:1].contiguous(),
                               out_dtype=torch.float32)
    assert (mo - o_parts[0]).abs().max().item() < 1e-6


@pytest.mark.parametrize("P,rows,D", [(11, 777, 32), (16, 300, 64), (3, 5, 32)])
def test_merge_many_blocks_and_ragged_rows(cuda_device, P, rows, D):
    """More partials than the unrolled kernels take (P > 8: the looping
    kernel), a row count that leaves the last block of threads part-filled,
    and very few rows; one block of every row empty."""
    g = torch.Generator("cuda").manual_seed(P * 100 + rows)
    o_parts = torch.randn((P, rows, D), generator=g, device=cuda_device)
    m_parts = torch.randn((P, rows), generator=g, device=cuda_device) * 4
    l_parts = torch.rand((P, rows), generator=g, device=cuda_device) * 10 + 0.1
    empty = torch.arange(rows, device=cuda_device) % P
    l_parts[empty, torch.arange(rows, device=cuda_device)] = 0
    m_parts[empty, torch.arange(rows, device=cuda_device)] = -math.inf
    ref = oracle.merge(o_parts, m_parts, l_parts)
    for dt in (torch.float32, torch.bfloat16):
        mo, ml = pba.softmax_merge(o_parts, m_parts, l_parts, out_dtype=dt)
        _cmp(f"merge P={P} rows={rows} D={D} {dt}", mo, ml, ref, out_tol=OUT_TOL if dt == torch.bfloat16 else 1e-5)


# ------------------------------------------------------------------ bit-exact integer / index handling
def test_bitexact_masked_entries_do_not_matter(cuda_device):
    q, k, v, bias, mask = W.random_attn(1, 4, 500, 777, 64, seed=11, device=cuda_device, mask_frac=0.3)
    o1, l1 = pba.pba_forward(q, k, v, bias, mask)
    k2, v2, b2 = k.clone(), v.clone(), _padded_clone(bias)
    dead = mask[0] == 0
    k2[:, :, dead] = 3.0
    v2[:, :, dead] = -5.0
    b2[..., dead] = 11.0
    o2, l2 = pba.pba_forward(q, k2, v2, b2, mask)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bitexact_block_in_place_vs_copy(cuda_device):
    q, k, v, bias, mask = W.random_attn(1, 2, 300, 1024, 64, seed=12, device=cuda_device, mask_frac=0.1)
    sl = slice(384, 384 + 256)
    a = pba.pba_partial(q, k[:, :, sl], v[:, :, sl], bias[..., sl], mask[:, sl])
    b = pba.pba_partial(q, k[:, :, sl].contiguous(), v[:, :, sl].contiguous(), bias[..., sl].contiguous(),
                        mask[:, sl].contiguous())
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("gate", [False, True])
def test_bitexact_ending_equals_starting_on_transposed_copy(cuda_device, gate):
    cfg = W.TriConfig("t", N=256, c=32, H=4, D=32, seed=13)
    q, k, v, g, bias = W.tri_inputs(cfg, cuda_device)
    g = g if gate else None
    e_out, e_lse = pba.tri_attn_forward(q, k, v, bias, g, None, "ending")
    T = lambda x: x.transpose(0, 1).contiguous()
    s_out, s_lse = pba.tri_attn_forward(T(q), T(k), T(v), bias.transpose(1, 2).contiguous(),
                                        None if g is None else T(g), None, "starting")
    assert torch.equal(e_out, T(s_out)) and torch.equal(e_lse, s_lse.transpose(0, 1))


def test_bitexact_tri_pair_mask_orientation(cuda_device):
    cfg = W.TriConfig("t", N=128, c=32, H=4, D=32, seed=14)
    q, k, v, g, bias = W.tri_inputs(cfg, cuda_device)
    pm = (torch.rand((128, 128), generator=torch.Generator("cuda").manual_seed(1), device=cuda_device) > 0.2)
    pm = pm.to(torch.uint8)
    for ending in (False, True):
        out, lse = pba.tri_attn_forward(q, k, v, bias, g, pm, "ending" if ending else "starting")
        lines = [0, 5, 64, 127]
        ref = oracle.tri_attn(q, k, v, bias, g, pm, ending=ending, lines=lines)
        o_sel = out[:, lines].transpose(0, 1) if ending else out[lines]
        l_sel = lse[:, lines].transpose(0, 1) if ending else lse[lines]
        _cmp(f"tri mask ending={ending}", o_sel, l_sel, ref)
    T = lambda x: x.transpose(0, 1).contiguous()
    e = pba.tri_attn_forward(q, k, v, bias, g, pm, "ending")
    s = pba.tri_attn_forward(T(q), T(k), T(v), bias.transpose(1, 2).contiguous(), T(g), T(pm), "starting")
    assert torch.equal(e[0], T(s[0])) and torch.equal(e[1], s[1].transpose(0, 1))


def test_bitexact_fully_masked_block_is_zero_minf_zero(cuda_device):
    q, k, v, bias, _ = W.random_attn(1, 2, 300, 512, 64, seed=15, device=cuda_device)
    mask = torch.ones((1, 512), dtype=torch.uint8, device=cuda_device)
    mask[:, 128:384] = 0
    sl = slice(128, 384)
    o_p, m_p, l_p = pba.pba_partial(q, k[:, :, sl], v[:, :, sl], bias[..., sl], mask[:, sl])
    assert torch.all(o_p == 0) and torch.all(m_p == -math.inf) and torch.all(l_p == 0)


def test_bitexact_valid_key_count(cuda_device):
    # q = 0 and bias = 0: every valid key has p = 1, so l is the count exactly
    q, k, v, bias, mask = W.random_attn(1, 3, 260, 1000, 64, seed=16, device=cuda_device, mask_frac=0.37)
    q.zero_()
    bias.zero_()
    o_p, m_p, l_p = pba.pba_partial(q, k, v, bias, mask)
    count = mask.sum().item()
    assert torch.all(l_p == float(count)) and torch.all(m_p == 0)
    ref = oracle.pba(q, k, v, bias, mask)
    _cmp("mean of valid values", o_p, m_p + torch.log(l_p), ref, out_tol=1e-4)


@pytest.mark.parametrize("D", [32, 64])
def test_bitexact_repeat_runs_are_identical(cuda_device, D):
    """Every output is a fixed function of the inputs: repeated calls give
    bitwise identical results.  Many short units per CTA (N=1024, 64 heads)
    make a race on a shared-memory ring or a Tensor Memory buffer show up as
    rows that differ from run to run."""
    q, k, v, bias, mask = W.random_attn(1, 64, 1024, 1024, D, seed=40 + D, device=cuda_device, mask_frac=0.05)
    runs = [pba.pba_partial(q, k, v, bias, mask) for _ in range(4)]
    fwd = [pba.pba_forward(q, k, v, bias, mask) for _ in range(4)]
    for r in runs[1:]:
        for x, y in zip(runs[0], r):
            assert torch.equal(x, y)
    for r in fwd[1:]:
        for x, y in zip(fwd[0], r):
            assert torch.equal(x, y)
    cfg = W.TriConfig("rep", N=256, c=32, H=4, D=32, seed=41)
    tq, tk, tv, tg, tb = W.tri_inputs(cfg, cuda_device)
    for orient in ("starting", "ending"):
        tri = [pba.tri_attn_forward(tq, tk, tv, tb, tg, None, orient) for _ in range(3)]
        for r in tri[1:]:
            assert torch.equal(tri[0][0], r[0]) and torch.equal(tri[0][1], r[1])


# ------------------------------------------------------------------ failure detection
def test_bounded_wait_reports_timeout_and_context_survives(cuda_device):
    assert pba.pba_last_device_error() == pba.PBA_OK
    pba.pba_selftest_wait_timeout(20_000_000)  # 20 ms
    assert pba.pba_last_device_error() == pba.PBA_ERR_TIMEOUT
    assert pba.pba_last_device_error() == pba.PBA_OK  # cleared by the read
    q, k, v, bias, _ = W.random_attn(1, 1, 128, 128, 64, seed=1, device=cuda_device)
    out, lse = pba.pba_forward(q, k, v, bias)
    torch.cuda.synchronize()
    assert pba.pba_last_device_error() == pba.PBA_OK
    assert torch.isfinite(out.float()).all()


def test_binding_refuses_cpu_tensors():
    q = torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        pba.pba_forward(q, q, q, torch.zeros((1, 1, 8, 8), dtype=torch.bfloat16))
