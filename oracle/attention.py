"""Causal softmax attention with log-sum-exp, written as its definition, in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

What ring attention, Ulysses and the 2D grid all compute is plain full attention: after
N_cp ring steps every query has seen every key/value ("ring attention: key/value をリングで
回す", step 4, in "05. 長系列の分散学習（Context Parallelism）"), and Ulysses computes full
attention per head after its all-to-all ("Ulyssesシーケンス並列化の核心", step 3).  So the
oracle for the fused path is the definition itself, per batch b, query head h, query i:

    s_ij  = scale * <q_i, k_j>          for keys j visible to i (causal: j <= i)
    LSE_i = ln sum_j exp(s_ij)          (natural log, scale included)
    O_i   = sum_j exp(s_ij - LSE_i) v_j

GQA: a group of G = Hq/Hkv consecutive query heads shares one K/V head, kv = h // G
("LLMのアーキテクチャを理解する" in "長いシーケンスのLLMトレーニングの進展").
"""
from __future__ import annotations

import numpy as np


def _kv_head(h: int, hq: int, hkv: int) -> int:
    return h // (hq // hkv)


def attention_full(q, k, v, causal: bool = True, scale: float | None = None):
    """Full attention.  q [B,Hq,L,d], k/v [B,Hkv,L,d] (float64) -> O [B,Hq,L,d], LSE [B,Hq,L].

    Rows with no visible key (only possible with an empty key set) get O = 0, LSE = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    Lk = k.shape[2]
    assert Hq % Hkv == 0 and v.shape == k.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((B, Hq, L, d))
    lse = np.full((B, Hq, L), -np.inf)
    visible = np.ones((L, Lk), dtype=bool)
    if causal:
        visible = np.arange(Lk)[None, :] <= np.arange(L)[:, None]
    for b in range(B):
        for h in range(Hq):
            g = _kv_head(h, Hq, Hkv)
            s = scale * (q[b, h] @ k[b, g].T)
            s = np.where(visible, s, -np.inf)
            m = s.max(axis=1)
            has = np.isfinite(m)
            m_safe = np.where(has, m, 0.0)
            e = np.exp(s - m_safe[:, None])
            l = e.sum(axis=1)
            lse[b, h] = np.where(has, m_safe + np.log(np.where(has, l, 1.0)), -np.inf)
            p = e / np.where(has, l, 1.0)[:, None]
            o[b, h] = p @ v[b, g]
    return o, lse


def attention_rows(q_rows, k, v, rows, causal: bool = True, scale: float | None = None):
    """Attention for selected query rows of ONE head (sampled checks of large shapes).

    q_rows [R,d] are the query vectors at global positions ``rows`` [R]; k/v [Lk,d] are the
    head's full key/value sequence.  Returns O [R,d], LSE [R].  Each row follows the same
    definition as ``attention_full``, so any sampled row is exact.
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.int64)
    d = q_rows.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    hi = int(rows.max()) + 1 if causal else k.shape[0]
    s = scale * (q_rows @ k[:hi].T)
    if causal:
        s = np.where(np.arange(hi)[None, :] <= rows[:, None], s, -np.inf)
    m = s.max(axis=1)
    e = np.exp(s - m[:, None])
    l = e.sum(axis=1)
    return (e / l[:, None]) @ v[:hi], m + np.log(l)


def forward_flops(B: int, Hq: int, L: int, d: int, causal: bool = True) -> float:
    """Algorithmic forward FLOPs: 2 GEMMs of 2*d flops per visible (query, key) pair."""
    pairs = L * (L + 1) / 2 if causal else float(L) * L
    return 4.0 * B * Hq * d * pairs
