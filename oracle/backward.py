"""Gradient of causal softmax attention, from the definition, in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages give no backward formulas; they say only that activations are recomputed rather
than stored ("スケーラビリティとメモリ管理" in "長いシーケンスのLLMトレーニングの進展") and that
gradients travel back to their ranks by the inverse exchanges (§3 of "05. 長系列の分散学習
（Context Parallelism）").  The reading taken is the textbook gradient of
O = softmax(S) V with S = scale * Q K^T (masked), recomputing P from the stored LSE:

    P_ij  = exp(s_ij - LSE_i)               (0 where masked)
    dV    = P^T dO
    dP    = dO V^T
    D_i   = sum_j P_ij dP_ij = <dO_i, O_i>
    dS    = P o (dP - D)
    dQ    = scale * dS K
    dK    = scale * dS^T Q
GQA: dK, dV of a KV head are summed over the G query heads that share it.
"""
from __future__ import annotations

import numpy as np


def _probs(q, k, lse_row, rows, causal, scale):
    s = scale * (q @ k.T)
    if causal:
        s = np.where(np.arange(k.shape[0])[None, :] <= rows[:, None], s, -np.inf)
    return np.exp(s - lse_row[:, None])


def attention_backward(q, k, v, do, causal: bool = True, scale: float | None = None, o=None):
    """q [B,Hq,L,d], k/v [B,Hkv,L,d], do [B,Hq,L,d] (float64) -> dq, dk, dv (same shapes).

    P is recomputed here from q, k (the plain definition).  ``o`` is the forward output the
    backward is given, used only in D = rowsum(dO * O): the backward works from the stored
    forward state (recompute, do not store), and what the forward stores is its output as
    written (bf16).  Default: the exact O."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    rows = np.arange(L)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            s = scale * (q[b, h] @ k[b, g].T)
            if causal:
                s = np.where(rows[None, :] <= rows[:, None], s, -np.inf)
            m = s.max(axis=1)
            lse = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
            p = np.exp(s - lse[:, None])
            o_bh = p @ v[b, g] if o is None else np.asarray(o[b, h], np.float64)
            dv[b, g] += p.T @ do[b, h]
            dp = do[b, h] @ v[b, g].T
            D = (do[b, h] * o_bh).sum(axis=1)
            ds = p * (dp - D[:, None])
            dq[b, h] = scale * (ds @ k[b, g])
            dk[b, g] += scale * (ds.T @ q[b, h])
    return dq, dk, dv


def backward_rows_dq(q_rows, k, v, do_rows, o_rows, lse_rows, rows, causal: bool = True,
                     scale: float | None = None):
    """dQ for selected query rows of one head.  Needs only that row's LSE and O (both
    computable exactly per row with ``attention_rows``), so any sampled row is exact."""
    q_rows = np.asarray(q_rows, np.float64)
    rows = np.asarray(rows, np.int64)
    d = q_rows.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    p = _probs(q_rows, k, np.asarray(lse_rows, np.float64), rows, causal, scale)
    dp = np.asarray(do_rows, np.float64) @ v.T
    D = (np.asarray(do_rows, np.float64) * np.asarray(o_rows, np.float64)).sum(axis=1)
    ds = p * (dp - D[:, None])
    return scale * (ds @ k)


def backward_rows_dkdv(q, k, v, do, o, lse, key_rows, causal: bool = True,
                       scale: float | None = None, q_lo: int = 0):
    """dK, dV for selected key rows of one KV head, summed over its query heads.

    q, do, o [Gh, Lq', d] and lse [Gh, Lq'] hold the query rows q_lo .. q_lo+Lq'-1 of the G
    query heads of this KV head; under a causal mask the rows below min(key_rows) see none of
    the selected keys, so only the tail from q_lo = min(key_rows) is needed.  k, v [Lk, d].
    Returns dk [R, d], dv [R, d] for the R selected keys."""
    q = np.asarray(q, np.float64)
    do = np.asarray(do, np.float64)
    o = np.asarray(o, np.float64)
    lse = np.asarray(lse, np.float64)
    key_rows = np.asarray(key_rows, np.int64)
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    kk = np.asarray(k, np.float64)
    vv = np.asarray(v, np.float64)
    rows = q_lo + np.arange(q.shape[1])
    dk = np.zeros((len(key_rows), d))
    dv = np.zeros((len(key_rows), d))
    for g in range(q.shape[0]):
        s = scale * (q[g] @ kk[key_rows].T)                  # [Lq', R]
        if causal:
            s = np.where(key_rows[None, :] <= rows[:, None], s, -np.inf)
        p = np.exp(s - lse[g][:, None])
        dp = do[g] @ vv[key_rows].T
        D = (do[g] * o[g]).sum(axis=1)
        ds = p * (dp - D[:, None])
        dv += p.T @ do[g]
        dk += scale * (ds.T @ q[g])
    return dk, dv
