"""Python binding of libpba (include/pba.h): pair-biased attention on B200.

Argument marshalling only.  Every function here checks and converts torch
tensors into pointers, strides and sizes, calls the C entry point of the same
name on the current CUDA stream and raises PbaError on a non-OK status.  All
arithmetic runs in the CUDA kernels of libpba.so; there is no CPU path, and an
import without the built library fails loudly.

The operation ("Fold-CP: A Context Parallelism Framework for Biomolecular
Modeling", Table 1 "Attn Pair Bias" / "Triangle Attention", Figure 2):
    O = softmax_keys(tau Q K^T + bias + mask) V,  tau = 1/sqrt(D),
computed in one pass (pba_forward) or as per-key-block partials (pba_partial)
combined by the tiled-softmax merge (softmax_merge); triangle attention runs it
along one axis of a pair tensor (tri_attn_forward).
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "PbaError", "PBA_OK", "PBA_ERR_INVALID_ARG", "PBA_ERR_UNSUPPORTED", "PBA_ERR_CUDA", "PBA_ERR_TIMEOUT",
    "library_path", "load_library", "pba_forward", "pba_partial", "softmax_merge", "tri_attn_forward", "tri_proj_forward", "tri_out_proj_forward", "pwa_forward", "pba_backward",
    "pba_backward_noalloc", "PBA_BWD_NOALLOC_MAX_ROWS",
    "pba_last_device_error", "pba_set_wait_timeout_ns", "pba_selftest_wait_timeout", "pba_selftest_exp2",
    "pba_status_string",
]

PBA_OK, PBA_ERR_INVALID_ARG, PBA_ERR_UNSUPPORTED, PBA_ERR_CUDA, PBA_ERR_TIMEOUT = 0, 1, 2, 3, 4
PBA_BF16, PBA_F32 = 0, 1
PBA_TRI_STARTING, PBA_TRI_ENDING = 0, 1
# rows (B * H * Nq) of the fixed Delta array of pba_backward_noalloc (include/pba.h)
PBA_BWD_NOALLOC_MAX_ROWS = 1048576

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(_HERE, "libpba.so")


class PbaAttnDesc(ctypes.Structure):
    """Mirror of pba_attn_desc."""
    _fields_ = [
        ("B", ctypes.c_int64), ("H", ctypes.c_int64), ("Nq", ctypes.c_int64), ("Nk", ctypes.c_int64),
        ("D", ctypes.c_int64), ("dtype", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
        ("q_stride", ctypes.c_int64 * 3), ("k_stride", ctypes.c_int64 * 3), ("v_stride", ctypes.c_int64 * 3),
        ("bias_stride", ctypes.c_int64 * 3), ("mask_stride_b", ctypes.c_int64),
        ("out_stride", ctypes.c_int64 * 3), ("lse_stride", ctypes.c_int64 * 3),
    ]


class PbaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {pba_status_string(status)} ({status})")
        self.status = status


_LIB = None
_p = ctypes.c_void_p


def load_library() -> ctypes.CDLL:
    """Load libpba.so from this package directory (built by
    ``python -m pair_biased_attention_b200.build``)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(f"libpba.so is not built ({path}); run: python -m pair_biased_attention_b200.build")
    lib = ctypes.CDLL(path)
    st = ctypes.c_int
    desc_p = ctypes.POINTER(PbaAttnDesc)
    lib.pba_forward.argtypes = [desc_p, _p, _p, _p, _p, _p, _p, _p, _p]
    lib.pba_forward.restype = st
    lib.pba_partial.argtypes = [desc_p, _p, _p, _p, _p, _p, _p, _p, _p, _p]
    lib.pba_partial.restype = st
    lib.softmax_merge.argtypes = [ctypes.c_int32, ctypes.c_int64, ctypes.c_int64, _p, _p, _p, ctypes.c_int32, _p,
                                  _p, _p]
    lib.softmax_merge.restype = st
    lib.tri_attn_forward.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_float,
                                     _p, _p, _p, _p, _p, _p, _p, _p, _p]
    lib.tri_attn_forward.restype = st
    lib.tri_proj_forward.argtypes = [ctypes.c_int64] * 4 + [_p] * 9
    lib.tri_proj_forward.restype = st
    lib.tri_out_proj_forward.argtypes = [ctypes.c_int64] * 4 + [_p] * 4
    lib.tri_out_proj_forward.restype = st
    lib.pwa_forward.argtypes = [ctypes.c_int64] * 4 + [_p] * 7
    lib.pwa_forward.restype = st
    lib.pba_backward.argtypes = [desc_p] + [_p] * 14
    lib.pba_backward.restype = st
    lib.pba_backward_noalloc.argtypes = [desc_p] + [_p] * 13
    lib.pba_backward_noalloc.restype = st
    lib.pba_status_string.argtypes = [st]
    lib.pba_status_string.restype = ctypes.c_char_p
    lib.pba_last_device_error.argtypes = [_p]
    lib.pba_last_device_error.restype = st
    lib.pba_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.pba_set_wait_timeout_ns.restype = ctypes.c_uint64
    lib.pba_selftest_wait_timeout.argtypes = [ctypes.c_uint64, _p]
    lib.pba_selftest_wait_timeout.restype = st
    lib.pba_selftest_exp2.argtypes = [_p, _p, ctypes.c_int64, _p]
    lib.pba_selftest_exp2.restype = st
    _LIB = lib
    return lib


def pba_status_string(status: int) -> str:
    return load_library().pba_status_string(status).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn: str, status: int):
    if status != PBA_OK:
        raise PbaError(fn, status)


def _cuda(name, t, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _dtype_code(dt) -> int:
    if dt == torch.bfloat16:
        return PBA_BF16
    if dt == torch.float32:
        return PBA_F32
    raise ValueError(f"unsupported dtype {dt}")


def _bhn(name, t, shape_len=4):
    if t.dim() != shape_len:
        raise ValueError(f"{name} must have {shape_len} dims")
    if shape_len == 4 and t.stride(3) != 1 and t.shape[3] > 1:
        raise ValueError(f"{name} must be contiguous along its last axis")
    return t.stride(0), t.stride(1), t.stride(2)


def _desc(q, k, v, bias, key_mask, out_strides, lse_strides, softmax_scale) -> PbaAttnDesc:
    B, H, Nq, D = q.shape
    Nk = k.shape[2]
    if k.shape != (B, H, Nk, D) or v.shape != (B, H, Nk, D):
        raise ValueError("k and v must be [B,H,Nk,D] matching q")
    if bias.dim() != 4 or bias.shape[2] != Nq or bias.shape[3] != Nk or bias.shape[0] not in (1, B) or \
            bias.shape[1] not in (1, H):
        raise ValueError("bias must be [B|1, H|1, Nq, Nk]")
    if bias.stride(3) != 1 and Nk > 1:
        raise ValueError("bias must be contiguous along keys")
    d = PbaAttnDesc()
    d.B, d.H, d.Nq, d.Nk, d.D = B, H, Nq, Nk, D
    d.dtype = _dtype_code(q.dtype)
    d.softmax_scale = float(softmax_scale or 0.0)
    d.q_stride[:] = _bhn("q", q)
    d.k_stride[:] = _bhn("k", k)
    d.v_stride[:] = _bhn("v", v)
    bsb = 0 if (bias.shape[0] == 1 and B > 1) else bias.stride(0)
    bsh = 0 if (bias.shape[1] == 1 and H > 1) else bias.stride(1)
    d.bias_stride[:] = (bsb, bsh, bias.stride(2))
    if key_mask is not None:
        if key_mask.shape != (B, Nk) or (key_mask.stride(1) != 1 and Nk > 1):
            raise ValueError("key_mask must be [B, Nk] uint8, contiguous along keys")
        d.mask_stride_b = key_mask.stride(0)
    d.out_stride[:] = out_strides
    d.lse_stride[:] = lse_strides
    return d


def pba_forward(q, k, v, bias, key_mask=None, out=None, lse=None, softmax_scale=None, return_lse=True,
                stream=None):
    """O (and the natural-log log-sum-exp) of pair-biased attention over all
    keys.  q [B,H,Nq,D], k/v [B,H,Nk,D], bias [B|1,H|1,Nq,Nk] (bf16 or fp32, all
    the same dtype), key_mask [B,Nk] uint8 (1 = key takes part) or None.
    bf16 runs on the tensor cores; fp32 keeps fp32-level accuracy, on the
    tensor cores as three tf32 products per product (high and low parts of
    each operand) when the rows are 16-byte aligned, else on the CUDA cores."""
    for n, t in (("q", q), ("k", k), ("v", v), ("bias", bias)):
        _cuda(n, t, q.dtype)
    _cuda("key_mask", key_mask, torch.uint8)
    B, H, Nq, D = q.shape
    if out is None:
        out = torch.empty((B, H, Nq, D), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _cuda("out", out, q.dtype)
    _cuda("lse", lse, torch.float32)
    lse_strides = lse.stride() if lse is not None else (0, 0, 0)
    d = _desc(q, k, v, bias, key_mask, _bhn("out", out), lse_strides, softmax_scale)
    _check("pba_forward", load_library().pba_forward(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(bias),
                                                     _ptr(key_mask), _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def pba_partial(q, k, v, bias, key_mask=None, o_part=None, m_part=None, l_part=None, softmax_scale=None,
                stream=None):
    """One ring step: the online-softmax partial (O_p, m_p, l_p) of the queries
    against the keys that k, v, bias and key_mask hold (pass column views of
    the full tensors for a block of keys).  Outputs are fp32."""
    for n, t in (("q", q), ("k", k), ("v", v), ("bias", bias)):
        _cuda(n, t, q.dtype)
    _cuda("key_mask", key_mask, torch.uint8)
    B, H, Nq, D = q.shape
    if o_part is None:
        o_part = torch.empty((B, H, Nq, D), dtype=torch.float32, device=q.device)
    if m_part is None:
        m_part = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    if l_part is None:
        l_part = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    for n, t in (("o_part", o_part), ("m_part", m_part), ("l_part", l_part)):
        _cuda(n, t, torch.float32)
    if m_part.stride() != l_part.stride():
        raise ValueError("m_part and l_part must share strides")
    d = _desc(q, k, v, bias, key_mask, _bhn("o_part", o_part), m_part.stride(), softmax_scale)
    _check("pba_partial", load_library().pba_partial(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(bias),
                                                     _ptr(key_mask), _ptr(o_part), _ptr(m_part), _ptr(l_part),
                                                     _stream(stream)))
    return o_part, m_part, l_part


def softmax_merge(o_parts, m_parts, l_parts, out_dtype=torch.bfloat16, out=None, lse=None, return_lse=True,
                  stream=None):
    """Tiled-softmax merge of P stacked partials: o_parts [P,...,D], m_parts and
    l_parts [P,...] (fp32, contiguous).  Returns out [...,D] (out_dtype) and
    lse [...]."""
    for n, t in (("o_parts", o_parts), ("m_parts", m_parts), ("l_parts", l_parts)):
        _cuda(n, t, torch.float32)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    P, D = o_parts.shape[0], o_parts.shape[-1]
    lead = tuple(o_parts.shape[1:-1])
    if tuple(m_parts.shape) != (P,) + lead or tuple(l_parts.shape) != (P,) + lead:
        raise ValueError("m_parts and l_parts must be [P, ...] matching o_parts")
    rows = 1
    for x in lead:
        rows *= x
    if out is None:
        out = torch.empty(lead + (D,), dtype=out_dtype, device=o_parts.device)
    if lse is None and return_lse:
        lse = torch.empty(lead, dtype=torch.float32, device=o_parts.device)
    _cuda("out", out, out_dtype)
    if not out.is_contiguous() or (lse is not None and not lse.is_contiguous()):
        raise ValueError("out and lse must be contiguous")
    _check("softmax_merge", load_library().softmax_merge(P, rows, D, _ptr(o_parts), _ptr(m_parts), _ptr(l_parts),
                                                         _dtype_code(out_dtype), _ptr(out), _ptr(lse),
                                                         _stream(stream)))
    return out, lse


def tri_attn_forward(q, k, v, bias, gate=None, pair_mask=None, orientation="starting", out=None, lse=None,
                     softmax_scale=None, return_lse=True, stream=None):
    """Triangle attention on a pair tensor, bf16.  q, k, v, gate [N,N,H,D]
    (contiguous), bias [H,N,N], pair_mask [N,N] uint8 or None; orientation
    "starting" (attend along j of row i, bias b[h][j][k]) or "ending" (attend
    along i of column j, bias b[h][k][i]).  Returns out [N,N,H,D] and lse
    [N,N,H]."""
    for n, t in (("q", q), ("k", k), ("v", v), ("bias", bias), ("gate", gate)):
        _cuda(n, t, torch.bfloat16)
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    _cuda("pair_mask", pair_mask, torch.uint8)
    N, N2, H, D = q.shape
    if N2 != N or k.shape != q.shape or v.shape != q.shape or (gate is not None and gate.shape != q.shape):
        raise ValueError("q, k, v, gate must be [N,N,H,D]")
    if tuple(bias.shape) != (H, N, N):
        raise ValueError("bias must be [H,N,N]")
    if pair_mask is not None and (tuple(pair_mask.shape) != (N, N) or not pair_mask.is_contiguous()):
        raise ValueError("pair_mask must be a contiguous [N,N] uint8 tensor")
    orient = {"starting": PBA_TRI_STARTING, "ending": PBA_TRI_ENDING}[orientation]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((N, N, H), dtype=torch.float32, device=q.device)
    _cuda("out", out, torch.bfloat16)
    _cuda("lse", lse, torch.float32)
    _check("tri_attn_forward", load_library().tri_attn_forward(N, H, D, orient, float(softmax_scale or 0.0), _ptr(q),
                                                               _ptr(k), _ptr(v), _ptr(bias), _ptr(gate),
                                                               _ptr(pair_mask), _ptr(out), _ptr(lse),
                                                               _stream(stream)))
    return out, lse


def tri_proj_forward(z, w_qkvg, w_b, H, out=None, bias=None, stream=None):
    """Triangle projections of a pair tensor, bf16.  z [N,N,c] (contiguous),
    w_qkvg [c, 4*H*D] (column blocks W_q | W_k | W_v | W_g), w_b [c, H].
    Returns q, k, v, g [N,N,H,D] and bias [H,N,N]; ``out`` may pass the four
    output tensors."""
    for n, t in (("z", z), ("w_qkvg", w_qkvg), ("w_b", w_b)):
        _cuda(n, t, torch.bfloat16)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    N, N2, c = z.shape
    if N2 != N or w_qkvg.shape[0] != c or w_b.shape != (c, H) or w_qkvg.shape[1] % (4 * H) != 0:
        raise ValueError("z must be [N,N,c], w_qkvg [c, 4*H*D], w_b [c,H]")
    D = w_qkvg.shape[1] // (4 * H)
    if out is None:
        out = tuple(torch.empty((N, N, H, D), dtype=torch.bfloat16, device=z.device) for _ in range(4))
    if bias is None:
        bias = torch.empty((H, N, N), dtype=torch.bfloat16, device=z.device)
    for n, t in zip(("q", "k", "v", "g", "bias"), tuple(out) + (bias,)):
        _cuda(n, t, torch.bfloat16)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    q, k, v, g = out
    _check("tri_proj_forward", load_library().tri_proj_forward(N, c, H, D, _ptr(z), _ptr(w_qkvg), _ptr(w_b), _ptr(q),
                                                               _ptr(k), _ptr(v), _ptr(g), _ptr(bias),
                                                               _stream(stream)))
    return q, k, v, g, bias


def tri_out_proj_forward(o, w_o, out=None, stream=None):
    """Output projection of triangle attention, bf16: o [N,N,H,D]
    (contiguous, H*D = 128), w_o [H*D, c].  Returns out [N,N,c] = o W_o."""
    for n, t in (("o", o), ("w_o", w_o)):
        _cuda(n, t, torch.bfloat16)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    N, N2, H, D = o.shape
    if N2 != N or w_o.dim() != 2 or w_o.shape[0] != H * D:
        raise ValueError("o must be [N,N,H,D] and w_o [H*D, c]")
    c = w_o.shape[1]
    if out is None:
        out = torch.empty((N, N, c), dtype=torch.bfloat16, device=o.device)
    _cuda("out", out, torch.bfloat16)
    if not out.is_contiguous() or tuple(out.shape) != (N, N, c):
        raise ValueError("out must be a contiguous [N,N,c] tensor")
    _check("tri_out_proj_forward", load_library().tri_out_proj_forward(N, c, H, D, _ptr(o), _ptr(w_o), _ptr(out),
                                                                       _stream(stream)))
    return out


def pwa_forward(v, bias, key_mask=None, gate=None, out=None, lse=None, return_lse=True, stream=None):
    """Pair weighted averaging, bf16: v, gate [S,N,H,D] (contiguous), bias
    [H,N,N], key_mask [N] uint8 or None.  Returns out [S,N,H,D] and lse [H,N]
    (the kernels always write lse; return_lse=False only drops it from the
    result)."""
    for n, t in (("v", v), ("bias", bias), ("gate", gate)):
        _cuda(n, t, torch.bfloat16)
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    _cuda("key_mask", key_mask, torch.uint8)
    S, N, H, D = v.shape
    if tuple(bias.shape) != (H, N, N) or (gate is not None and gate.shape != v.shape):
        raise ValueError("bias must be [H,N,N] and gate [S,N,H,D]")
    if key_mask is not None and (tuple(key_mask.shape) != (N,) or not key_mask.is_contiguous()):
        raise ValueError("key_mask must be a contiguous [N] uint8 tensor")
    if out is None:
        out = torch.empty_like(v)
    lse_out = lse if lse is not None else torch.empty((H, N), dtype=torch.float32, device=v.device)
    _cuda("out", out, torch.bfloat16)
    _cuda("lse", lse_out, torch.float32)
    _check("pwa_forward", load_library().pwa_forward(S, N, H, D, _ptr(v), _ptr(bias), _ptr(key_mask), _ptr(gate),
                                                     _ptr(out), _ptr(lse_out), _stream(stream)))
    return out, (lse_out if (lse is not None or return_lse) else None)


def pba_backward(q, k, v, bias, key_mask, out, lse, dout, softmax_scale=None, stream=None):
    """Gradients of pba_forward, bf16 inputs (contiguous [B,H,n,D]; bias as
    for pba_forward).  Returns dq, dk, dv (fp32), dbias [B,H,Nq,Nk] (bf16) and
    delta = rowsum(dout * out) [B,H,Nq] (fp32)."""
    for n, t in (("out", out), ("dout", dout)):
        _cuda(n, t, torch.bfloat16)
    _cuda("lse", lse, torch.float32)
    for n, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout), ("lse", lse)):
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    B, H, Nq, D = q.shape
    Nk = k.shape[2]
    if out.shape != q.shape or dout.shape != q.shape or tuple(lse.shape) != (B, H, Nq):
        raise ValueError("out and dout must be [B,H,Nq,D], lse [B,H,Nq]")
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    dbias = torch.empty((B, H, Nq, Nk), dtype=torch.bfloat16, device=q.device)
    delta = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    d = _desc(q, k, v, bias, key_mask, out.stride()[:3] if out.dim() == 4 else None, lse.stride(), softmax_scale)
    _check("pba_backward", load_library().pba_backward(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(bias),
                                                       _ptr(key_mask), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                                                       _ptr(dk), _ptr(dv), _ptr(dbias), _ptr(delta),
                                                       _stream(stream)))
    return dq, dk, dv, dbias, delta


def pba_backward_noalloc(q, k, v, bias, key_mask, out, lse, dout, softmax_scale=None, stream=None, grads=None):
    """pba_backward through the entry point that allocates nothing on the
    device: Delta goes to the library's fixed array (B*H*Nq rows at most,
    PBA_BWD_NOALLOC_MAX_ROWS), so no delta buffer is passed.  For callers
    that cannot allocate device memory; ``grads`` = (dq, dk, dv, dbias)
    preallocated by the caller (allocated here when None).  Calls that
    overlap on the GPU race on the shared array.  Returns dq, dk, dv, dbias."""
    for n, t in (("out", out), ("dout", dout)):
        _cuda(n, t, torch.bfloat16)
    _cuda("lse", lse, torch.float32)
    for n, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout), ("lse", lse)):
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    B, H, Nq, D = q.shape
    Nk = k.shape[2]
    if out.shape != q.shape or dout.shape != q.shape or tuple(lse.shape) != (B, H, Nq):
        raise ValueError("out and dout must be [B,H,Nq,D], lse [B,H,Nq]")
    if grads is None:
        grads = (torch.empty(q.shape, dtype=torch.float32, device=q.device),
                 torch.empty(k.shape, dtype=torch.float32, device=q.device),
                 torch.empty(v.shape, dtype=torch.float32, device=q.device),
                 torch.empty((B, H, Nq, Nk), dtype=torch.bfloat16, device=q.device))
    dq, dk, dv, dbias = grads
    for n, t, dt, shape in (("dq", dq, torch.float32, q.shape), ("dk", dk, torch.float32, k.shape),
                            ("dv", dv, torch.float32, v.shape), ("dbias", dbias, torch.bfloat16, (B, H, Nq, Nk))):
        _cuda(n, t, dt)
        if tuple(t.shape) != tuple(shape) or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous {tuple(shape)} tensor")
    d = _desc(q, k, v, bias, key_mask, out.stride()[:3] if out.dim() == 4 else None, lse.stride(), softmax_scale)
    _check("pba_backward_noalloc",
           load_library().pba_backward_noalloc(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(bias),
                                               _ptr(key_mask), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                                               _ptr(dv), _ptr(dbias), _stream(stream)))
    return dq, dk, dv, dbias


def pba_last_device_error(stream=None) -> int:
    """Synchronise the stream; return and clear the device error word."""
    return load_library().pba_last_device_error(_stream(stream))


def pba_set_wait_timeout_ns(ns: int) -> int:
    return load_library().pba_set_wait_timeout_ns(int(ns))


def pba_selftest_exp2(x, out=None, stream=None):
    """The kernels' software 2^x applied to a CUDA fp32 tensor (test hook)."""
    _cuda("x", x, torch.float32)
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    if out is None:
        out = torch.empty_like(x)
    _check("pba_selftest_exp2", load_library().pba_selftest_exp2(_ptr(x), _ptr(out), x.numel(), _stream(stream)))
    return out


def pba_selftest_wait_timeout(ns: int, stream=None) -> None:
    _check("pba_selftest_wait_timeout", load_library().pba_selftest_wait_timeout(int(ns), _stream(stream)))
