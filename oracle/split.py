"""Rank-to-sequence maps for causal load balance, and the ring and Ulysses flows under them.

TEST INFRASTRUCTURE ONLY (see the package docstring).

"05. 長系列の分散学習（Context Parallelism）" §5 (因果モデルの負荷分散): under a causal mask a
contiguous split gives later ranks more work, so the sequence is cut into 2 N_cp shards of
L / (2 N_cp) positions and each rank holds two of them.  Zig-zag splitting pairs the front
and back halves: with 8 shards and N_cp = 4 the ranks hold [x0, x7], [x1, x6], [x2, x5],
[x3, x4], i.e. rank r holds shards r and 2 N_cp - 1 - r.

Readings taken where the page is terse:
  * a rank's local rows are its first shard followed by its second (in the order listed);
  * striped ordering ("CP ランク数の2倍のシャードに分け、各ランクに2枚を縞状に配置") is read
    as rank r holding shards r and r + N_cp;
  * contiguous is the same machinery with rank r holding shards 2r and 2r + 1;
  * every other reading of ring.py holds: at step s rank r holds the KV of rank
    (r - s) mod N_cp, partials are merged by the LSE merge, causal means key <= query in
    global positions;
  * the LSE output stays in global position order [B, H, L] whatever the split.
"""
from __future__ import annotations

import numpy as np

from .attention import attention_full
from .ring import lse_merge

SPLITS = ("contiguous", "zigzag", "striped")


def shards_of_rank(split: str, n_cp: int, r: int):
    """The two shard indices (of 2 n_cp, each L / (2 n_cp) long) held by rank r."""
    if split == "contiguous":
        return (2 * r, 2 * r + 1)
    if split == "zigzag":
        return (r, 2 * n_cp - 1 - r)
    if split == "striped":
        return (r, r + n_cp)
    raise ValueError(split)


def rank_positions(split: str, n_cp: int, L: int, r: int) -> np.ndarray:
    """Global positions of rank r's local rows, in local order."""
    assert L % (2 * n_cp) == 0, "two shards per rank need 2 N_cp | L"
    w = L // (2 * n_cp)
    return np.concatenate([np.arange(a * w, (a + 1) * w) for a in shards_of_rank(split, n_cp, r)])


def rank_order(split: str, n_cp: int, L: int) -> np.ndarray:
    """Global position of every row of the rank-major layout (rank 0's rows, rank 1's, ...)."""
    return np.concatenate([rank_positions(split, n_cp, L, r) for r in range(n_cp)])


def causal_pairs(positions) -> int:
    """Visible (query, key) pairs of a set of query positions under the causal mask."""
    return int(np.sum(np.asarray(positions, dtype=np.int64) + 1))


def step_pairs(split: str, n_cp: int, L: int, r: int, s: int) -> int:
    """Visible pairs of rank r at ring step s (its queries against the KV of rank (r-s) mod N)."""
    qp = rank_positions(split, n_cp, L, r)
    kp = rank_positions(split, n_cp, L, (r - s) % n_cp)
    return int(np.sum(kp[None, :] <= qp[:, None]))


def partial(q_rows, k_rows, v_rows, q_pos, k_pos, causal: bool = True, scale: float | None = None):
    """Normalised partial attention of queries at global positions q_pos against keys/values at
    k_pos (one head): O [cq, d], LSE [cq]; a row with no visible key gives (0, -inf)."""
    q_rows = np.asarray(q_rows, dtype=np.float64)
    k_rows = np.asarray(k_rows, dtype=np.float64)
    v_rows = np.asarray(v_rows, dtype=np.float64)
    cq, d = q_rows.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((cq, d))
    lse = np.full(cq, -np.inf)
    k_pos = np.asarray(k_pos)
    for t in range(cq):
        vis = k_pos <= q_pos[t] if causal else np.ones(len(k_pos), dtype=bool)
        if not vis.any():
            continue
        sc = scale * (k_rows[vis] @ q_rows[t])
        m = sc.max()
        e = np.exp(sc - m)
        l = e.sum()
        o[t] = (e @ v_rows[vis]) / l
        lse[t] = m + np.log(l)
    return o, lse


def ring_step_split(q, k, v, n_cp: int, split: str, rank: int, step: int, causal: bool = True,
                    scale: float | None = None):
    """The partial of rank `rank` at ring step `step` under the split: its local rows (in local
    order) against the KV rows of rank (rank - step) mod N.  q [B,Hq,L,d], k/v [B,Hkv,L,d].
    Returns O [B,Hq,c,d], LSE [B,Hq,c] (c = L / N)."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, L, d = q.shape
    G = Hq // k.shape[1]
    qp = rank_positions(split, n_cp, L, rank)
    kp = rank_positions(split, n_cp, L, (rank - step) % n_cp)
    o = np.zeros((B, Hq, len(qp), d))
    lse = np.full((B, Hq, len(qp)), -np.inf)
    for b in range(B):
        for h in range(Hq):
            o[b, h], lse[b, h] = partial(q[b, h, qp], k[b, h // G, kp], v[b, h // G, kp], qp, kp, causal, scale)
    return o, lse


def ring_attention_split(q, k, v, n_cp: int, split: str, causal: bool = True, scale: float | None = None,
                         order=None):
    """Ring attention with each rank holding its split's rows: every rank merges its partials
    over all N steps (``order[r]``: rank r's visit order of steps, default 0..N-1).  Returns O
    [B,Hq,L,d] and LSE [B,Hq,L] in global position order."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, L, d = q.shape
    o = np.zeros((B, Hq, L, d))
    lse = np.full((B, Hq, L), -np.inf)
    for r in range(n_cp):
        qp = rank_positions(split, n_cp, L, r)
        acc_o = np.zeros((B, Hq, len(qp), d))
        acc_l = np.full((B, Hq, len(qp)), -np.inf)
        steps = range(n_cp) if order is None else order[r]
        for s in steps:
            po, pl = ring_step_split(q, k, v, n_cp, split, r, s, causal, scale)
            acc_o, acc_l = lse_merge(acc_o, acc_l, po, pl)
        o[:, :, qp] = acc_o
        lse[:, :, qp] = acc_l
    return o, lse


def seq2head_split(x, n: int, split: str):
    """Ulysses all-to-all from the rank-major sequence layout: x [B, L, H, d] holds rank s's
    local rows at [s*c, (s+1)*c) (global positions rank_positions(split, n, L, s)); the result
    [B, H, L, d] is in global position order (all ranks' head groups side by side):
        out[b, h, rank_positions(s)[t], :] = x[b, s*c + t, h, :]"""
    x = np.asarray(x)
    B, L, H, d = x.shape
    c = L // n
    out = np.empty((B, H, L, d), dtype=x.dtype)
    for s in range(n):
        pos = rank_positions(split, n, L, s)
        for t in range(c):
            out[:, :, pos[t], :] = x[:, s * c + t, :, :]
    return out


def head2seq_split(y, n: int, split: str):
    """Inverse of seq2head_split: [B, H, L, d] in position order -> rank-major [B, L, H, d]."""
    y = np.asarray(y)
    B, H, L, d = y.shape
    c = L // n
    out = np.empty((B, L, H, d), dtype=y.dtype)
    for s in range(n):
        pos = rank_positions(split, n, L, s)
        for t in range(c):
            out[:, s * c + t, :, :] = y[:, :, pos[t], :]
    return out


def ulysses_attention_split(q_seq, k_seq, v_seq, n: int, split: str, causal: bool = True,
                            scale: float | None = None):
    """The 4-step Ulysses flow with rank-major inputs under the split: all-to-all to heads in
    position order, full attention per head group, all-to-all back.  Returns O in the input's
    rank-major layout [B, L, Hq, d] and LSE [B, Hq, L] in position order."""
    qh = seq2head_split(q_seq, n, split)
    kh = seq2head_split(k_seq, n, split)
    vh = seq2head_split(v_seq, n, split)
    oh, lse = attention_full(qh, kh, vh, causal=causal, scale=scale)
    return head2seq_split(oh, n, split), lse
