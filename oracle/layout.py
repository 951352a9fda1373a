"""Ulysses sequence<->head re-layout by its index formula.

TEST INFRASTRUCTURE ONLY (see the package docstring).

All-to-all re-layout ("05. 長系列の分散学習（Context Parallelism）" §2, and step 2 of
"Ulyssesシーケンス並列化の核心：All-to-All通信"): each of N ranks holds a sequence shard
[L/N, H] (here [B, c, H, d], c = L/N); after the exchange rank r' holds the channel
(head) group [H/N, L] for the full sequence (here [B, H/N, L, d], d innermost — the reading
taken where the pages give only [H/N, L]).  Index formula, for source rank s, position t,
destination rank r', local head h':

    out[r'][b, h', s*c + t, :] = in[s][b, t, r'*H/N + h', :]

head2seq is its exact inverse (step 4 of the same 4-step algorithm).
"""
from __future__ import annotations

import numpy as np


def seq2head(x_ranks):
    """list of N arrays [B, c, H, d] (rank s holds positions [s*c,(s+1)*c)) ->
    list of N arrays [B, H/N, L, d] (rank r' holds heads [r'*H/N, (r'+1)*H/N))."""
    n = len(x_ranks)
    B, c, H, d = x_ranks[0].shape
    assert H % n == 0, "Ulysses degree must divide the head count"
    hn = H // n
    out = [np.empty((B, hn, n * c, d), dtype=x_ranks[0].dtype) for _ in range(n)]
    for r2 in range(n):
        for h2 in range(hn):
            for s in range(n):
                out[r2][:, h2, s * c:(s + 1) * c, :] = x_ranks[s][:, :, r2 * hn + h2, :]
    return out


def head2seq(y_ranks):
    """Inverse of seq2head: list of N arrays [B, H/N, L, d] -> list of N arrays [B, c, H, d]."""
    n = len(y_ranks)
    B, hn, L, d = y_ranks[0].shape
    assert L % n == 0
    c = L // n
    out = [np.empty((B, c, hn * n, d), dtype=y_ranks[0].dtype) for _ in range(n)]
    for s in range(n):
        for r2 in range(n):
            for h2 in range(hn):
                out[s][:, :, r2 * hn + h2, :] = y_ranks[r2][:, h2, s * c:(s + 1) * c, :]
    return out
