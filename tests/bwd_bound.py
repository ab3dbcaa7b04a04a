"""Per-element error bounds of the backward kernels (pba_backward), derived
from their rounding model, for the GPU parity tests and for the CPU test that
checks the bound itself.

What the kernels do (bf16 inputs q, k, v, bias, dout; the forward's bf16 out
and fp32 lse):
  s_ij    = q_i . k_j                    fp32 sum of exact bf16 products
  a_ij    = (tau s_ij + b_ij - lse_i) log2(e)   three fp32 roundings
  P_ij    = ex2.approx(a_ij)             fp32, relative error below 2^-21
  dP_ij   = dout_i . v_j                 fp32 sum of exact products
  Delta_i = sum_d dout_id out_id         fp32, from the forward's bf16 out
  dS_ij   = P_ij (dP_ij - Delta_i)       two fp32 roundings
  dbias   = bf16(dS)                     one bf16 rounding (unit roundoff 2^-8)
  dq_i = tau sum_j bf16(dS_ij) k_j,  dk_j = tau sum_i bf16(dS_ij) q_i,
  dv_j = sum_i bf16(P_ij) dout_i          fp32 tensor-core sums
Against the exact values (fp64 oracle, from the exact forward), with the
forward's own errors |lse_gpu - lse| and |out_gpu - out| taken as measured:
  eps_P = |dlse_i| + tau gamma_D (|q||k|^T)_ij + 2^-20 (|tau s| + |b| + |lse| + 1)
  E_dS  = P (eps_P |dP - Delta| + gamma_D (|dout||v|^T) + e_Delta_i) + 2^-22 P |dP - Delta|
  e_Delta_i = sum_d |dout_id| |out_gpu - out|_id + gamma_D sum_d |dout_id out_id|
  |dbias - dS|  <= 2^-8 |dS| + (1 + 2^-8) E_dS
  |dq - dq_ref| <= tau (M @ |K|),  M = 2^-8 |dS| + (1 + 2^-8) E_dS + gamma_Nk |dS|
  |dk - dk_ref| <= tau (M^T @ |Q|)   (gamma_Nq in M)
  |dv - dv_ref| <= (P (2^-8 + (1 + 2^-8) eps_P + gamma_Nq))^T @ |dout|
with gamma_n = n 2^-23 (a generous fp32 sum bound).  Every term is a worst
case: rounding errors of one sign all along a sum.  Typical errors are a
small fraction of it, but a kernel that drops, rescales or misplaces terms
breaks it element by element (see test_bwd_bound.py).
"""
from __future__ import annotations

import numpy as np

U_BF16 = 2.0 ** -8


def _gamma(n: int) -> float:
    return n * 2.0 ** -23


def head_terms(q, k, v, bias, valid, dout, out_gpu, lse_gpu, out_ref, lse_ref, tau, rows=None, cols=None):
    """Exact P, dS and the fp32-path error E_dS, eps_P of one (b, h) on the
    query rows `rows` and key columns `cols` (None = all), in fp64.

    q, dout, out_gpu, out_ref [Nq, D]; k, v [Nk, D]; bias [Nq, Nk]; valid [Nk]
    bool; lse_gpu, lse_ref [Nq]."""
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    cols = np.arange(k.shape[0]) if cols is None else np.asarray(cols)
    D = q.shape[1]
    gD = _gamma(D)
    qr, dor = q[rows], dout[rows]
    kc, vc = k[cols], v[cols]
    b = bias[np.ix_(rows, cols)]
    qk = qr @ kc.T
    s = tau * qk + b
    ok = valid[cols][None, :] & np.isfinite(b)
    lse = lse_ref[rows][:, None]
    with np.errstate(invalid="ignore", over="ignore"):
        P = np.where(ok & np.isfinite(lse), np.exp(np.where(ok, s, 0.0) - np.where(np.isfinite(lse), lse, 0.0)), 0.0)
    dP = dor @ vc.T
    delta = np.sum(dor * out_ref[rows], axis=1)[:, None]
    dS = P * (dP - delta)
    fin = np.isfinite(lse_ref[rows])
    dlse = np.abs(np.where(fin, lse_gpu[rows] - np.where(fin, lse_ref[rows], 0.0), 0.0))[:, None]
    eps_P = (dlse + tau * gD * (np.abs(qr) @ np.abs(kc).T) +
             2.0 ** -20 * (np.abs(tau * qk) + np.abs(np.where(ok, b, 0.0)) + np.abs(np.where(np.isfinite(lse), lse, 0.0)) + 1.0))
    e_delta = (np.sum(np.abs(dor) * np.abs(out_gpu[rows] - out_ref[rows]), axis=1) +
               gD * np.sum(np.abs(dor * out_gpu[rows]), axis=1))[:, None]
    E_dS = P * (eps_P * np.abs(dP - delta) + gD * (np.abs(dor) @ np.abs(vc).T) + e_delta) + \
        2.0 ** -22 * P * np.abs(dP - delta)
    return {"P": P, "dS": dS, "E_dS": E_dS, "eps_P": eps_P}


def dbias_bound(t) -> np.ndarray:
    return U_BF16 * np.abs(t["dS"]) + (1 + U_BF16) * t["E_dS"] + 1e-30


def dq_bound(t, k_cols, tau) -> np.ndarray:
    """Bound of dq on the rows of `t`; t must span every key (cols = all)."""
    n = t["dS"].shape[1]
    M = U_BF16 * np.abs(t["dS"]) + (1 + U_BF16) * t["E_dS"] + _gamma(n) * np.abs(t["dS"])
    return tau * (M @ np.abs(k_cols)) + 1e-30


def dk_bound(t, q_rows, tau) -> np.ndarray:
    """Bound of dk on the columns of `t`; t must span every query (rows = all)."""
    n = t["dS"].shape[0]
    M = U_BF16 * np.abs(t["dS"]) + (1 + U_BF16) * t["E_dS"] + _gamma(n) * np.abs(t["dS"])
    return tau * (M.T @ np.abs(q_rows)) + 1e-30


def dv_bound(t, dout_rows) -> np.ndarray:
    """Bound of dv on the columns of `t`; t must span every query (rows = all)."""
    n = t["P"].shape[0]
    M = t["P"] * (U_BF16 + (1 + U_BF16) * t["eps_P"] + _gamma(n))
    return M.T @ np.abs(dout_rows) + 1e-30


def excess(got, ref, bound) -> float:
    """Largest amount by which |got - ref| exceeds its bound (<= 0: within)."""
    got = np.asarray(got, dtype=np.float64)
    if got.size == 0:
        return -1.0
    return float((np.abs(got - ref) - bound).max())
