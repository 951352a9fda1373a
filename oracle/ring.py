"""Chunked (ring) attention, the LSE merge, and the Ulysses / 2D flows, in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Ring attention ("ring attention: key/value をリングで回す" in "05. 長系列の分散学習（Context
Parallelism）"): N_cp ranks in a ring; rank r keeps its query chunk, key/value chunks pass to
the neighbour one step at a time (step 1); each step computes a partial attention of the
local queries against the chunk just received (step 2); the softmax statistics are updated
online (step 3); after N_cp steps every query has seen every key/value (step 4).

Readings taken where the page is silent:
  * contiguous split: rank r owns global positions [r*c, (r+1)*c), c = L / N_cp;
  * at step s rank r holds KV chunk j = (r - s) mod N_cp (chunks move to the next rank);
  * a partial is normalised, O_rj = P V / l, and carries LSE_rj = m + ln l; a partial with
    no visible key is (O=0, LSE=-inf), which the merge treats as the identity;
  * causal: key j visible to query i iff j <= i in global positions.
"""
from __future__ import annotations

import numpy as np

from .layout import seq2head, head2seq


def chunk_partial(q_r, k_j, v_j, q_pos0: int, k_pos0: int, causal: bool = True,
                  scale: float | None = None):
    """One ring step for one head: queries q_r [cq,d] at global positions q_pos0 + t against
    keys/values k_j, v_j [ck,d] at positions k_pos0 + u.  Returns the normalised partial
    O [cq,d] and its LSE [cq] (natural log, scale included)."""
    q_r = np.asarray(q_r, dtype=np.float64)
    k_j = np.asarray(k_j, dtype=np.float64)
    v_j = np.asarray(v_j, dtype=np.float64)
    cq, d = q_r.shape
    ck = k_j.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((cq, d))
    lse = np.full(cq, -np.inf)
    qpos = q_pos0 + np.arange(cq)
    kpos = k_pos0 + np.arange(ck)
    for t in range(cq):
        vis = kpos <= qpos[t] if causal else np.ones(ck, dtype=bool)
        if not vis.any():
            continue
        s = scale * (k_j[vis] @ q_r[t])
        m = s.max()
        e = np.exp(s - m)
        l = e.sum()
        o[t] = (e @ v_j[vis]) / l
        lse[t] = m + np.log(l)
    return o, lse


def lse_merge(o_a, lse_a, o_b, lse_b):
    """Online-softmax merge of two normalised partials (rows along axis 0 of lse, O [...,d]).

    m = max(la, lb); wa = e^(la-m); wb = e^(lb-m); LSE = m + ln(wa+wb);
    O = (wa*Oa + wb*Ob) / (wa+wb).  A partial with LSE = -inf is the identity.
    """
    o_a = np.asarray(o_a, dtype=np.float64)
    o_b = np.asarray(o_b, dtype=np.float64)
    lse_a = np.asarray(lse_a, dtype=np.float64)
    lse_b = np.asarray(lse_b, dtype=np.float64)
    m = np.maximum(lse_a, lse_b)
    empty = np.isneginf(m)
    m_safe = np.where(empty, 0.0, m)
    wa = np.where(np.isneginf(lse_a), 0.0, np.exp(lse_a - m_safe))
    wb = np.where(np.isneginf(lse_b), 0.0, np.exp(lse_b - m_safe))
    w = wa + wb
    w_safe = np.where(empty, 1.0, w)
    lse = np.where(empty, -np.inf, m_safe + np.log(w_safe))
    o = (wa[..., None] * o_a + wb[..., None] * o_b) / w_safe[..., None]
    o = np.where(empty[..., None], 0.0, o)
    return o, lse


def ring_attention(q, k, v, n_cp: int, causal: bool = True, scale: float | None = None,
                   order=None):
    """Ring attention over N_cp virtual ranks.  q [B,Hq,L,d], k/v [B,Hkv,L,d] float64.

    ``order[r]`` optionally gives rank r's visit order of KV chunks (a permutation of
    range(N_cp)); the default is the ring order j = (r - s) mod N_cp.  Every chunk is
    visited, including chunks wholly above the causal diagonal, whose empty partial the
    merge absorbs.  Returns O [B,Hq,L,d], LSE [B,Hq,L].
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    assert L % n_cp == 0, "contiguous split needs N_cp | L"
    c = L // n_cp
    G = Hq // Hkv
    o = np.zeros((B, Hq, L, d))
    lse = np.full((B, Hq, L), -np.inf)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for r in range(n_cp):
                acc_o = np.zeros((c, d))
                acc_l = np.full(c, -np.inf)
                visit = [(r - s) % n_cp for s in range(n_cp)] if order is None else list(order[r])
                assert sorted(visit) == list(range(n_cp))
                for j in visit:
                    po, pl = chunk_partial(q[b, h, r * c:(r + 1) * c], k[b, g, j * c:(j + 1) * c],
                                           v[b, g, j * c:(j + 1) * c], r * c, j * c, causal, scale)
                    acc_o, acc_l = lse_merge(acc_o, acc_l, po, pl)
                o[b, h, r * c:(r + 1) * c] = acc_o
                lse[b, h, r * c:(r + 1) * c] = acc_l
    return o, lse


def _attention_heads(q, k, v, causal, scale):
    """Full attention over [B,h,L,d] blocks (used per Ulysses rank); GQA kv = h // G."""
    from .attention import attention_full
    return attention_full(q, k, v, causal=causal, scale=scale)


def ulysses_attention(q_seq, k_seq, v_seq, n: int, causal: bool = True, scale: float | None = None):
    """The 4-step Ulysses flow on N virtual ranks ("Ulyssesシーケンス並列化の核心：All-to-All
    通信", steps 1-4).  Inputs are sequence-major [B,L,H,d]; rank s holds rows [s*c,(s+1)*c).

    step 2: all-to-all seq->head: rank r receives heads [r*H/N, (r+1)*H/N) for all of L;
    step 3: full attention on its own heads;
    step 4: all-to-all head->seq of the output.
    Returns O [B,L,Hq,d] (sequence-major) and LSE [B,Hq,L].
    """
    q_seq = np.asarray(q_seq, dtype=np.float64)
    B, L, Hq, d = q_seq.shape
    Hkv = k_seq.shape[2]
    assert L % n == 0 and Hq % n == 0 and Hkv % n == 0
    c = L // n
    split = lambda x: [x[:, s * c:(s + 1) * c] for s in range(n)]  # noqa: E731
    qh, kh, vh = seq2head(split(q_seq)), seq2head(split(np.asarray(k_seq, np.float64))), \
        seq2head(split(np.asarray(v_seq, np.float64)))
    o_heads, lse_heads = [], []
    for r in range(n):
        o_r, l_r = _attention_heads(qh[r], kh[r], vh[r], causal, scale)
        o_heads.append(o_r)
        lse_heads.append(l_r)
    o_ranks = head2seq(o_heads)
    return np.concatenate(o_ranks, axis=1), np.concatenate(lse_heads, axis=1)


def attention_2d(q_seq, k_seq, v_seq, n_hp: int, n_cp: int, causal: bool = True,
                 scale: float | None = None):
    """2D head x context attention on an n_hp x n_cp virtual grid ("2Dアテンションの導入" in
    "長いシーケンスのLLMトレーニングの進展": tensors distributed over heads and chunked
    along the context at the same time).

    Reading taken (the page gives no rank map): the input [B,L,H,d] is sequence-sharded over
    all n_hp*n_cp ranks; rank (h, k) starts with shard k*n_hp + h, so the n_hp ranks of
    context group k together hold context chunk k.  An all-to-all inside each context group
    turns that into head group h over chunk k; a ring over k then computes attention for each
    head group; a second all-to-all inside the group restores the sequence sharding.
    Returns O [B,L,Hq,d] and LSE [B,Hq,L].
    """
    q_seq = np.asarray(q_seq, dtype=np.float64)
    k_seq = np.asarray(k_seq, dtype=np.float64)
    v_seq = np.asarray(v_seq, dtype=np.float64)
    B, L, Hq, d = q_seq.shape
    Hkv = k_seq.shape[2]
    assert L % (n_hp * n_cp) == 0 and Hq % n_hp == 0 and Hkv % n_hp == 0
    cs = L // (n_hp * n_cp)          # initial shard length
    cc = L // n_cp                   # context chunk length
    shard = lambda x, i: x[:, i * cs:(i + 1) * cs]  # noqa: E731
    # head-group all-to-all inside each context group k -> per (h,k): [B, H/n_hp, cc, d]
    grid_q, grid_k, grid_v = {}, {}, {}
    for kk in range(n_cp):
        for src, dst in ((q_seq, grid_q), (k_seq, grid_k), (v_seq, grid_v)):
            parts = seq2head([shard(src, kk * n_hp + h) for h in range(n_hp)])
            for h in range(n_hp):
                dst[(h, kk)] = parts[h]
    # ring over the context axis for each head group, then the inverse all-to-all
    o_seq = np.zeros((B, L, Hq, d))
    lse = np.full((B, Hq, L), -np.inf)
    hq_g = Hq // n_hp
    grid_o = {}
    for h in range(n_hp):
        qg = np.concatenate([grid_q[(h, kk)] for kk in range(n_cp)], axis=2)
        kg = np.concatenate([grid_k[(h, kk)] for kk in range(n_cp)], axis=2)
        vg = np.concatenate([grid_v[(h, kk)] for kk in range(n_cp)], axis=2)
        og, lg = ring_attention(qg, kg, vg, n_cp, causal=causal, scale=scale)
        lse[:, h * hq_g:(h + 1) * hq_g] = lg
        for kk in range(n_cp):
            grid_o[(h, kk)] = og[:, :, kk * cc:(kk + 1) * cc]
    for kk in range(n_cp):
        back = head2seq([grid_o[(h, kk)] for h in range(n_hp)])
        for h in range(n_hp):
            i = kk * n_hp + h
            o_seq[:, i * cs:(i + 1) * cs] = back[h]
    return o_seq, lse
