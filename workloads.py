"""Seeded synthetic inputs for pair-biased attention, shared by the tests, the
smoke check and the benchmark.

This module only draws random numbers and builds index sets; it holds none of
the attention arithmetic.  Neither the CUDA library nor the oracle imports it.

The workloads follow the shapes of the pages' runs ("Fold-CP: A Context
Parallelism Framework for Biomolecular Modeling", Table 2: 2,700 to 11,500
tokens; Table 1 symbols B, H, N, D) -- the pages publish no dataset or
benchmark inputs for this path, so every tensor here is synthetic:

  pr1       single pair-biased attention, B=1, N=256, H=4, D=32, fp32;
            q, k, v, bias ~ N(0,1) drawn in that order from one CPU seed (0);
            no mask; also split into 4 key blocks of 64.
  apb2k     B=1, N=2048, H=16, D=64, bf16; q,k,v ~ N(0,1), bias ~ N(0, var 2);
            key-padding mask with the last floor(N/10) keys masked (seed 1).
  tri512    triangle attention, pair tensor z [512,512,128] ~ N(0,1) bf16,
            weights ~ N(0, 1/c) bf16; q,k,v,g [N,N,H=4,D=32], bias [H,N,N]
            (seed 2).  Starting node; the ending node uses the same tensors.
  ring8k    N=8192, H=16, D=64, bf16, bias ~ N(0,1), no mask; P=8 key blocks
            of 1024 processed in the order randperm(8) (seed 3).
  large16k  N=16384, H=16, D=64, bf16, bias ~ N(0,1) (8.6 GB); a random key
            mask of round(0.05 N) = 819 keys (seed 4).
  tri1024   as tri512 with N=1024 (seed 5).
  pwa512    pair weighted averaging, S=16 sequences, N=512, H=8, D=32; v,
            gate, bias ~ N(0,1) bf16, last 5% of keys masked (seed 6).
  pwa4k     as pwa512 with S=64, N=4096 (seed 7).

"N(0, 2)" and "N(0, 1/c)" are read as (mean, variance).

The triangle projections q = z W_q (and k, v, g, bias) are part of how the
inputs are synthesised: the attention call takes q, k, v, g and the bias as
its inputs, and both the kernels and the oracle receive the same bf16 tensors.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class AttnConfig:
    name: str
    B: int
    N: int
    H: int
    D: int
    dtype: torch.dtype
    seed: int
    bias_std: float = 1.0
    mask: str | None = None  # None | "tail10" | "random5"
    blocks: int = 1  # key blocks (ring steps) for the partial/merge path


@dataclass(frozen=True)
class TriConfig:
    name: str
    N: int
    c: int
    H: int
    D: int
    seed: int


PR1 = AttnConfig("pr1", B=1, N=256, H=4, D=32, dtype=torch.float32, seed=0, blocks=4)
APB2K = AttnConfig("apb2k", B=1, N=2048, H=16, D=64, dtype=torch.bfloat16, seed=1, bias_std=math.sqrt(2.0),
                   mask="tail10")
RING8K = AttnConfig("ring8k", B=1, N=8192, H=16, D=64, dtype=torch.bfloat16, seed=3, blocks=8)
LARGE16K = AttnConfig("large16k", B=1, N=16384, H=16, D=64, dtype=torch.bfloat16, seed=4, mask="random5")
TRI512 = TriConfig("tri512", N=512, c=128, H=4, D=32, seed=2)
TRI1024 = TriConfig("tri1024", N=1024, c=128, H=4, D=32, seed=5)

ATTN_CONFIGS = {c.name: c for c in (PR1, APB2K, RING8K, LARGE16K)}
TRI_CONFIGS = {c.name: c for c in (TRI512, TRI1024)}


def key_mask(cfg: AttnConfig, device="cpu") -> torch.Tensor | None:
    """[B, N] uint8 key mask (1 = key takes part) or None."""
    if cfg.mask is None:
        return None
    m = torch.ones(cfg.B, cfg.N, dtype=torch.uint8)
    if cfg.mask == "tail10":
        m[:, cfg.N - cfg.N // 10:] = 0
    elif cfg.mask == "random5":
        g = torch.Generator("cpu").manual_seed(cfg.seed)
        n_masked = int(round(0.05 * cfg.N))
        for b in range(cfg.B):
            perm = torch.randperm(cfg.N, generator=g)
            m[b, perm[:n_masked]] = 0
    else:
        raise ValueError(cfg.mask)
    return m.to(device)


def attn_inputs(cfg: AttnConfig, device="cpu", bias_row_pad: int = 0):
    """q, k, v [B,H,N,D], bias [B,H,N,N], key_mask [B,N] or None.

    Drawn in the order q, k, v, bias from one generator on ``device``.  On a
    CUDA device the bias is drawn one head at a time so the fp32 temporary
    stays at one head.  ``bias_row_pad`` > 0 allocates bias rows of
    N + bias_row_pad elements and returns the [..., :N] view (for row strides
    that must be multiples of 16 bytes)."""
    dev = torch.device(device)
    g = torch.Generator(dev.type).manual_seed(cfg.seed)
    shape = (cfg.B, cfg.H, cfg.N, cfg.D)
    q = torch.randn(shape, generator=g, device=dev).to(cfg.dtype)
    k = torch.randn(shape, generator=g, device=dev).to(cfg.dtype)
    v = torch.randn(shape, generator=g, device=dev).to(cfg.dtype)
    ncol = cfg.N + bias_row_pad
    bias_full = torch.empty((cfg.B, cfg.H, cfg.N, ncol), dtype=cfg.dtype, device=dev)
    if bias_row_pad:
        bias_full.zero_()
    for b in range(cfg.B):
        for h in range(cfg.H):
            t = torch.randn((cfg.N, cfg.N), generator=g, device=dev)
            bias_full[b, h, :, :cfg.N] = (t * cfg.bias_std).to(cfg.dtype)
    bias = bias_full[..., :cfg.N]
    return q, k, v, bias, key_mask(cfg, dev)


def random_attn(B, H, Nq, Nk, D, dtype=torch.bfloat16, seed=0, device="cpu", bias_std=1.0, mask_frac=0.0,
                bias_row_pad=None):
    """Small random problems for edge-case tests (same drawing order).

    The bias row length is padded to a multiple of 8 elements by default so its
    row stride is a multiple of 16 bytes; the returned bias is the [..., :Nk]
    view."""
    dev = torch.device(device)
    g = torch.Generator(dev.type).manual_seed(seed)
    q = torch.randn((B, H, Nq, D), generator=g, device=dev).to(dtype)
    k = torch.randn((B, H, Nk, D), generator=g, device=dev).to(dtype)
    v = torch.randn((B, H, Nk, D), generator=g, device=dev).to(dtype)
    pad = ((-Nk) % 8) if bias_row_pad is None else bias_row_pad
    bias_full = torch.zeros((B, H, Nq, Nk + pad), dtype=dtype, device=dev)
    bias_full[..., :Nk] = (torch.randn((B, H, Nq, Nk), generator=g, device=dev) * bias_std).to(dtype)
    mask = None
    if mask_frac > 0:
        u = torch.rand((B, Nk), generator=g, device=dev)
        mask = (u >= mask_frac).to(torch.uint8)
    return q, k, v, bias_full[..., :Nk], mask


def block_order(cfg: AttnConfig) -> list[int]:
    """Order in which the ring-step emulation visits the key blocks."""
    if cfg.blocks <= 1:
        return [0]
    g = torch.Generator("cpu").manual_seed(cfg.seed)
    return torch.randperm(cfg.blocks, generator=g).tolist()


def tri_pair_inputs(cfg: TriConfig, device="cpu"):
    """The seeded draws of a triangle workload: z [N,N,c] ~ N(0,1) and the
    weights W_q | W_k | W_v | W_g as one [c, 4*H*D] matrix and W_b [c, H],
    ~ N(0, 1/c), all rounded to bf16."""
    dev = torch.device(device)
    gen = torch.Generator(dev.type).manual_seed(cfg.seed)
    N, c, H, D = cfg.N, cfg.c, cfg.H, cfg.D
    z = torch.randn((N, N, c), generator=gen, device=dev).to(torch.bfloat16)
    wstd = 1.0 / math.sqrt(c)
    ws = [(torch.randn((c, H * D), generator=gen, device=dev) * wstd).to(torch.bfloat16) for _ in range(4)]
    wb = (torch.randn((c, H), generator=gen, device=dev) * wstd).to(torch.bfloat16)
    return z, torch.cat(ws, dim=1).contiguous(), wb


def tri_inputs(cfg: TriConfig, device="cpu"):
    """q, k, v, g [N,N,H,D] bf16 and bias [H,N,N] bf16 from a seeded pair tensor.

    The draws of tri_pair_inputs; each projection is z W taken in fp32 and
    rounded to bf16 (input synthesis for the attention, which takes the bf16
    tensors as given).  The bias is laid out [H, N, N] with b[h, j, k] from
    pair (j, k)."""
    N, H, D = cfg.N, cfg.H, cfg.D
    z, w, wb = tri_pair_inputs(cfg, device)
    zf = z.float().reshape(N * N, cfg.c)
    outs = []
    for i in range(4):
        outs.append((zf @ w[:, i * H * D:(i + 1) * H * D].float()).to(torch.bfloat16).reshape(N, N, H, D).contiguous())
    bias = (zf @ wb.float()).to(torch.bfloat16).reshape(N, N, H).permute(2, 0, 1).contiguous()
    q, k, v, g = outs
    return q, k, v, g, bias


@dataclass(frozen=True)
class PwaConfig:
    """Pair weighted averaging: S sequences of N tokens, H heads of D values,
    one bias [H,N,N] shared by the sequences."""
    name: str
    S: int
    N: int
    H: int
    D: int
    seed: int
    pad_frac: float = 0.0  # last round(pad_frac*N) keys masked (padding)


PWA512 = PwaConfig("pwa512", S=16, N=512, H=8, D=32, seed=6, pad_frac=0.05)
PWA4K = PwaConfig("pwa4k", S=64, N=4096, H=8, D=32, seed=7, pad_frac=0.05)


def pwa_inputs(cfg: PwaConfig, device="cpu"):
    """v, gate [S,N,H,D] ~ N(0,1), bias [H,N,N] ~ N(0,1), all bf16, and a key
    padding mask [N] uint8 (or None), drawn in that order from one seed."""
    dev = torch.device(device)
    gen = torch.Generator(dev.type).manual_seed(cfg.seed)
    v = torch.randn((cfg.S, cfg.N, cfg.H, cfg.D), generator=gen, device=dev).to(torch.bfloat16)
    bias = torch.randn((cfg.H, cfg.N, cfg.N), generator=gen, device=dev).to(torch.bfloat16)
    gate = torch.randn((cfg.S, cfg.N, cfg.H, cfg.D), generator=gen, device=dev).to(torch.bfloat16)
    mask = None
    if cfg.pad_frac:
        mask = torch.ones((cfg.N,), dtype=torch.uint8, device=dev)
        mask[cfg.N - int(round(cfg.pad_frac * cfg.N)):] = 0
    return v, bias, mask, gate


def sample_rows(N: int, count: int, seed: int, tile: int = 128) -> list[int]:
    """Seeded sample of row indices that always contains the tile boundary rows
    0, tile-1, tile, N-1 (those that exist)."""
    fixed = sorted({r for r in (0, tile - 1, tile, 2 * tile - 1, N - 1) if 0 <= r < N})
    g = torch.Generator("cpu").manual_seed(seed + 1000)
    rest = torch.randperm(N, generator=g).tolist()
    out = list(fixed)
    for r in rest:
        if len(out) >= min(count, N):
            break
        if r not in fixed:
            out.append(r)
    return sorted(out)

