"""fp64 CPU oracle for pair-biased attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  The CUDA
library in ``pair_biased_attention_b200`` never imports it and shares no code
with it.

The arithmetic lives in ``pba_oracle.c`` (plain C, fp64, naive loops); this
module only builds that file with gcc, converts tensors to fp64 (exactly: every
bf16 and fp32 value is an fp64 value) and slices lines of the pair tensor for
triangle attention.  See the header of ``pba_oracle.c`` for the definition and
its sources ("Fold-CP: A Context Parallelism Framework for Biomolecular
Modeling", Table 1 and Figure 2; the "Builds on" list of "Design-CP: Context
Parallelism for Design of Protein Nanoparticles").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pba_oracle.c")
_LOCK = threading.Lock()
_LIBS: dict = {}

_i64 = ctypes.c_int64
_dbl = ctypes.c_double
_p = ctypes.c_void_p


def lib_path(mutant: int = 0) -> str:
    name = "liboracle.so" if mutant == 0 else f"liboracle_mutant{mutant}.so"
    return os.path.join(_HERE, name)


def build(mutant: int = 0, force: bool = False) -> str:
    """Compile pba_oracle.c with gcc (plain -O2, no fast-math) into a shared
    library beside it.  ``mutant`` > 0 compiles a planted mistake, used only
    by the tests that show the pins catch such mistakes."""
    out = lib_path(mutant)
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-shared", "-fPIC", "-o", out + ".tmp", _SRC, "-lpthread", "-lm"]
        if mutant:
            cmd.insert(1, f"-DORACLE_MUTANT={mutant}")
        subprocess.check_call(cmd)
        os.replace(out + ".tmp", out)
    return out


def _lib(mutant: int = 0):
    with _LOCK:
        if mutant not in _LIBS:
            lib = ctypes.CDLL(build(mutant))
            lib.oracle_pba_range.argtypes = [_i64] * 5 + [_dbl] + [_p] * 5 + [_i64, _i64] + [_p] * 4 + [ctypes.c_int]
            lib.oracle_pba_range.restype = ctypes.c_int
            lib.oracle_merge.argtypes = [_i64, _i64, _i64] + [_p] * 5
            lib.oracle_merge.restype = ctypes.c_int
            lib.oracle_tri_attn_lines.argtypes = [_i64, _i64, _i64, ctypes.c_int, _dbl, _i64] + [_p] * 8 + [ctypes.c_int]
            lib.oracle_tri_attn_lines.restype = ctypes.c_int
            lib.oracle_tri_proj.argtypes = [_i64] * 4 + [_p] * 5 + [ctypes.c_int]
            lib.oracle_tri_proj.restype = ctypes.c_int
            lib.oracle_pwa.argtypes = [_i64] * 4 + [_p] * 6 + [ctypes.c_int]
            lib.oracle_pwa.restype = ctypes.c_int
            lib.oracle_pba_backward.argtypes = [_i64] * 5 + [_dbl] + [_p] * 10 + [ctypes.c_int]
            lib.oracle_pba_backward.restype = ctypes.c_int
            lib.oracle_threads_used.argtypes = [ctypes.c_int]
            lib.oracle_threads_used.restype = ctypes.c_int
            _LIBS[mutant] = lib
        return _LIBS[mutant]


def threads_used(nthreads: int = 0) -> int:
    return _lib().oracle_threads_used(nthreads)


def _f64(x) -> np.ndarray:
    """Exact conversion of a torch tensor / array to a C-contiguous fp64 array."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (any device, bf16/fp32/fp64)
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _u8(x) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(x).astype(np.uint8))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _default_tau(D: int, softmax_scale) -> float:
    return float(softmax_scale) if softmax_scale else 1.0 / np.sqrt(D)


def pba(q, k, v, bias, key_mask=None, softmax_scale=None, k0: int = 0, k1: int | None = None,
        nthreads: int = 0, mutant: int = 0):
    """Pair-biased attention over keys [k0, k1) in fp64.

    q [B,H,Nq,D], k/v [B,H,Nk,D], bias [B,H,Nq,Nk], key_mask [B,Nk] (nonzero =
    key takes part) or None.  Returns dict with o [B,H,Nq,D] (normalised), m, l,
    lse [B,H,Nq] as fp64 numpy arrays."""
    q, k, v, bias = _f64(q), _f64(k), _f64(v), _f64(bias)
    mask = _u8(key_mask)
    B, H, Nq, D = q.shape
    Nk = k.shape[2]
    assert k.shape == (B, H, Nk, D) and v.shape == (B, H, Nk, D)
    assert bias.shape == (B, H, Nq, Nk)
    if mask is not None:
        assert mask.shape == (B, Nk)
    if k1 is None:
        k1 = Nk
    o = np.zeros((B, H, Nq, D))
    m = np.zeros((B, H, Nq))
    l = np.zeros((B, H, Nq))
    lse = np.zeros((B, H, Nq))
    rc = _lib(mutant).oracle_pba_range(B, H, Nq, Nk, D, _default_tau(D, softmax_scale), _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(bias), _ptr(mask), k0, k1, _ptr(o), _ptr(m), _ptr(l), _ptr(lse), nthreads)
    assert rc == 0, "oracle_pba_range rejected its arguments"
    return {"o": o, "m": m, "l": l, "lse": lse}


def pba_partial(q, k, v, bias, key_mask=None, softmax_scale=None, k0: int = 0, L: int | None = None,
                nthreads: int = 0, mutant: int = 0):
    """One ring-step partial over keys [k0, k0+L): (O_p normalised, m_p, l_p)."""
    Nk = k.shape[2]
    if L is None:
        L = Nk - k0
    r = pba(q, k, v, bias, key_mask, softmax_scale, k0, k0 + L, nthreads, mutant)
    return {"o": r["o"], "m": r["m"], "l": r["l"]}


def merge(o_parts, m_parts, l_parts, mutant: int = 0):
    """Tiled-softmax merge of P partials.  o_parts [P,...,D], m/l [P,...].
    Returns dict with o [...,D] and lse [...]."""
    o_parts, m_parts, l_parts = _f64(o_parts), _f64(m_parts), _f64(l_parts)
    P = o_parts.shape[0]
    D = o_parts.shape[-1]
    lead = o_parts.shape[1:-1]
    rows = int(np.prod(lead)) if len(lead) else 1
    assert m_parts.shape == (P,) + tuple(lead) and l_parts.shape == m_parts.shape
    out = np.zeros(tuple(lead) + (D,))
    lse = np.zeros(tuple(lead))
    rc = _lib(mutant).oracle_merge(P, rows, D, _ptr(o_parts), _ptr(m_parts), _ptr(l_parts), _ptr(out), _ptr(lse))
    assert rc == 0
    return {"o": out, "lse": lse}


STARTING = 0
ENDING = 1


def tri_attn_lines(q_lines, k_lines, v_lines, bias, g_lines=None, mask_lines=None, ending: bool = False,
                   softmax_scale=None, nthreads: int = 0, mutant: int = 0):
    """Triangle attention on LINES of the pair tensor (see pba_oracle.c).

    Starting node: line l is row i_l, x_lines[l] = x[i_l] ([N,H,D]),
    mask_lines[l] = pair_mask[i_l, :].
    Ending node:   line l is column j_l, x_lines[l] = x[:, j_l] ([N,H,D]),
    mask_lines[l] = pair_mask[:, j_l].
    bias [H,N,N].  Returns dict with out [nl,N,H,D] and lse [nl,N,H]."""
    q, k, v = _f64(q_lines), _f64(k_lines), _f64(v_lines)
    g = _f64(g_lines)
    b = _f64(bias)
    mask = _u8(mask_lines)
    nl, N, H, D = q.shape
    assert k.shape == q.shape and v.shape == q.shape and b.shape == (H, N, N)
    if g is not None:
        assert g.shape == q.shape
    if mask is not None:
        assert mask.shape == (nl, N)
    out = np.zeros((nl, N, H, D))
    lse = np.zeros((nl, N, H))
    rc = _lib(mutant).oracle_tri_attn_lines(N, H, D, 1 if ending else 0, _default_tau(D, softmax_scale), nl,
                                            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(mask), _ptr(out),
                                            _ptr(lse), nthreads)
    assert rc == 0
    return {"o": out, "lse": lse}


def tri_attn(q, k, v, bias, g=None, pair_mask=None, ending: bool = False, lines=None, softmax_scale=None,
             nthreads: int = 0, mutant: int = 0):
    """Triangle attention on full pair tensors q,k,v,g [N,N,H,D], bias [H,N,N],
    pair_mask [N,N].  ``lines`` selects rows i (starting node) or columns j
    (ending node); None = all.  Returns out [nl,N,H,D] and lse [nl,N,H] in line
    layout (for the starting node line l holds out[i_l, :]; for the ending node
    it holds out[:, j_l])."""
    N = q.shape[0]
    idx = list(range(N)) if lines is None else [int(x) for x in lines]

    def sl(x):
        if x is None:
            return None
        if ending:
            return _f64(x[:, idx]).transpose(1, 0, 2, 3)  # [nl, N(i), H, D]
        return _f64(x[idx])

    ml = None
    if pair_mask is not None:
        pm = _u8(pair_mask)
        ml = pm[:, idx].T if ending else pm[idx]
    return tri_attn_lines(sl(q), sl(k), sl(v), bias, sl(g), ml, ending, softmax_scale, nthreads, mutant)


def tri_proj(z, w, wb, rows=None, nthreads: int = 0, mutant: int = 0):
    """Triangle projections in fp64: z [N,N,c] (or [R,c]), w [c,F] (the
    q | k | v | g column blocks), wb [c,H].  ``rows`` selects flat pair rows
    r = i*N + j (None = all).  Returns out [R,F] and bias [H,R] for the
    selected rows."""
    c = z.shape[-1]
    zf = _f64(z).reshape(-1, c)
    if rows is not None:
        zf = np.ascontiguousarray(zf[np.asarray(rows, dtype=np.int64)])
    wf, wbf = _f64(w), _f64(wb)
    R, F, H = zf.shape[0], wf.shape[1], wbf.shape[1]
    out = np.zeros((R, F))
    bias = np.zeros((H, R))
    rc = _lib(mutant).oracle_tri_proj(R, c, F, H, _ptr(zf), _ptr(wf), _ptr(wbf), _ptr(out), _ptr(bias), nthreads)
    assert rc == 0
    return {"out": out, "bias": bias}


def tri_out_proj(o, w_o, rows=None, nthreads: int = 0, mutant: int = 0):
    """Output projection of triangle attention in fp64: o [N,N,H,D] (or
    [R, H*D]), w_o [H*D, c]; out[r] = o[r] (heads concatenated, h major) W_o.
    The same linear map as the input projections, so it runs through
    oracle_tri_proj with no bias columns.  Returns out [R, c] for the selected
    flat pair rows (None = all)."""
    of = _f64(o)
    of = of.reshape(-1, of.shape[-2] * of.shape[-1]) if of.ndim == 4 else of.reshape(-1, of.shape[-1])
    r = tri_proj(of, w_o, np.zeros((of.shape[1], 1)), rows=rows, nthreads=nthreads, mutant=mutant)
    return r["out"]


def pwa(v, bias, key_mask=None, g=None, nthreads: int = 0, mutant: int = 0):
    """Pair weighted averaging in fp64 (the reading stated in pba_oracle.c):
    v [S,N,H,D], bias [H,N,N], key_mask [N] or None, g [S,N,H,D] or None.
    Returns out [S,N,H,D] and lse [H,N]."""
    vf, bf, gf, mk = _f64(v), _f64(bias), _f64(g), _u8(key_mask)
    S, N, H, D = vf.shape
    out = np.zeros((S, N, H, D))
    lse = np.zeros((H, N))
    rc = _lib(mutant).oracle_pwa(S, N, H, D, _ptr(vf), _ptr(bf), _ptr(gf), _ptr(mk), _ptr(out), _ptr(lse), nthreads)
    assert rc == 0
    return {"o": out, "lse": lse}


def pba_backward(q, k, v, bias, dout, key_mask=None, softmax_scale=None, nthreads: int = 0, mutant: int = 0):
    """Gradients of pair-biased attention in fp64 (see pba_oracle.c): q, dout
    [B,H,Nq,D], k, v [B,H,Nk,D], bias [B,H,Nq,Nk] (broadcast views are
    expanded), key_mask [B,Nk] or None.  Returns dq, dk, dv, dbias."""
    qf, kf, vf, of = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, Nq, D = qf.shape
    Nk = kf.shape[2]
    bf = np.ascontiguousarray(np.broadcast_to(_f64(bias), (B, H, Nq, Nk)))
    mk = _u8(key_mask)
    dq, dk, dv = np.zeros_like(qf), np.zeros_like(kf), np.zeros_like(vf)
    dbias = np.zeros((B, H, Nq, Nk))
    rc = _lib(mutant).oracle_pba_backward(B, H, Nq, Nk, D, _default_tau(D, softmax_scale), _ptr(qf), _ptr(kf),
                                          _ptr(vf), _ptr(bf), _ptr(mk), _ptr(of), _ptr(dq), _ptr(dk), _ptr(dv),
                                          _ptr(dbias), nthreads)
    assert rc == 0
    return {"dq": dq, "dk": dk, "dv": dv, "dbias": dbias}
