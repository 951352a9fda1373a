"""Ring attention across GPUs, one rank per GPU ("05. 長系列の分散学習（Context Parallelism）",
"ring attention: key/value をリングで回す", steps 1-4: each rank keeps its queries, passes its
key/value shard to the next rank, computes a partial attention against the shard it holds at
each step, and merges the partials with the online-softmax statistics).

Rank r holds the query shard Q_r and the key/value shard (K_r, V_r) of a sequence split into
N = world contiguous shards.  At step s = 0 .. N-1 it holds the shard of rank j = (r - s) mod N:
while the partial of Q_r against it runs on the GPU (the library's ring-step kernel with a
one-chunk plan: causal at j = r, full for j < r, skipped for j > r under the causal mask), the
shard is sent on to rank r + 1 and the next one received from rank r - 1 into a second buffer
(one message of [2, B, Hkv, c, d] per step, point-to-point over the process group: NCCL over
NVLink on GPUs).  The partials merge into an fp32 accumulator with the library's LSE merge.

Two-shard splits (§5 因果モデルの負荷分散): with split = "zigzag" (rank r holds shards r and
2N-1-r of 2N) or "striped" (shards r and r+N), every rank's local rows are its two shards in
that order, each w = c/2 rows, and so are the key/value rows it passes on.  The partial of a
step is then the merge of up to four shard-pair partials: shard a's queries against shard b's
keys are full when b < a, masked (key <= query) when b == a, and skipped when b > a.  Every
step carries the same causal work under zig-zag, which is why the split is used.

The exchange lands every remote shard in this rank's own memory before a kernel reads it;
no kernel reads a peer's memory.  It is injectable: the default passes the device buffers
point to point over the group (NCCL); `host_staged_exchange` passes them through host memory,
for process groups that move only host tensors (gloo), e.g. several ranks sharing one GPU.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist

from .binding import Plan, lse_merge


class _PlanCache:
    """One-chunk plans by (shape, diagonal, scale): plans are host objects, cheap to keep."""

    def __init__(self):
        self._plans = {}

    def get(self, B, Hq, Hkv, c, d, diagonal, scale):
        key = (B, Hq, Hkv, c, d, bool(diagonal), float(scale))
        p = self._plans.get(key)
        if p is None:
            p = Plan(B, Hq, Hkv, c, d, n_cp=1, causal=bool(diagonal), scale=float(scale))
            self._plans[key] = p
        return p


_plans = _PlanCache()


def cuda_partial(q, k, v, diagonal: bool, scale: float):
    """The partial (fp32 O normalised, LSE) of q [B, Hq, c, d] against one key/value shard
    k, v [B, Hkv, c, d]: the ring-step kernel on a one-chunk plan (causal mask at the
    diagonal shard, none below it)."""
    B, Hq, c, d = q.shape
    return _plans.get(B, Hq, k.shape[1], c, d, diagonal, scale).ring_step(0, 0, q, k, v)


def p2p_exchange(send, recv, nxt: int, prv: int, group=None):
    """Start sending `send` to rank `nxt` and receiving `recv` from rank `prv`; returns the
    requests to wait on (after which `recv` holds the message)."""
    return dist.batch_isend_irecv([dist.P2POp(dist.isend, send, nxt, group),
                                   dist.P2POp(dist.irecv, recv, prv, group)])


class _HostRecv:
    """Completes a host-staged exchange: waits for the messages, then copies the received
    host buffer into the device buffer (stream-ordered before any later kernel)."""

    def __init__(self, reqs, host_recv, recv):
        self.reqs, self.host_recv, self.recv = reqs, host_recv, recv

    def wait(self):
        for r in self.reqs:
            r.wait()
        self.recv.copy_(self.host_recv, non_blocking=False)


def host_staged_exchange(send, recv, nxt: int, prv: int, group=None):
    """The same exchange as p2p_exchange with the message staged through host memory: `send`
    is copied to the host, sent over the group, and the received host message copied into
    `recv` on wait().  For process groups whose backend moves only host tensors (gloo)."""
    host_send = send.to("cpu")
    host_recv = torch.empty_like(host_send)
    reqs = dist.batch_isend_irecv([dist.P2POp(dist.isend, host_send, nxt, group),
                                   dist.P2POp(dist.irecv, host_recv, prv, group)])
    return [_HostRecv(reqs, host_recv, recv)]


def shards_of_rank(split: str, n: int, r: int):
    """The two shard indices (of 2n) held by rank r under a two-shard split."""
    if split == "zigzag":
        return (r, 2 * n - 1 - r)
    if split == "striped":
        return (r, r + n)
    raise ValueError(f"unknown split {split!r}")


def ring_attention(q, k, v, group=None, *, causal: bool = True, scale: float = 0.0, split: str = "contiguous",
                   partial_fn: Optional[Callable] = None, merge_fn: Optional[Callable] = None,
                   exchange_fn: Optional[Callable] = None):
    """This rank's share of ring attention over the process group.

    q [B, Hq, c, d], k, v [B, Hkv, c, d]: this rank's rows (contiguous: sequence positions
    [r c, (r+1) c); zigzag / striped: its two shards of c/2 positions, in order).  Returns
    (O [B, Hq, c, d] normalised, LSE [B, Hq, c]) of this rank's queries over the whole
    sequence, in fp32 on the GPU.  partial_fn(q, k, v, diagonal, scale) -> (O, LSE) and
    merge_fn(acc_o, acc_lse, o, lse) (in place) default to the library's kernels;
    exchange_fn(send, recv, next_rank, prev_rank, group) -> waitables defaults to
    p2p_exchange."""
    partial_fn = partial_fn or cuda_partial
    merge_fn = merge_fn or lse_merge
    exchange_fn = exchange_fn or p2p_exchange
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    if group is not None:
        nxt, prv = dist.get_global_rank(group, nxt), dist.get_global_rank(group, prv)
    kv_cur = torch.stack([k, v]).contiguous()       # one message: [2, B, Hkv, c, d]
    kv_nxt = torch.empty_like(kv_cur)
    B, Hq, c, d = q.shape
    if split != "contiguous" and c % 2:
        raise ValueError("a two-shard split needs an even number of local rows")
    acc_o = torch.zeros((B, Hq, c, d), dtype=torch.float32 if q.is_cuda else torch.float64, device=q.device)
    acc_l = torch.full((B, Hq, c), -float("inf"), dtype=acc_o.dtype, device=q.device)
    for s in range(world):
        j = (rank - s) % world
        reqs = []
        if s < world - 1:
            # pass the shard held now to the next rank, receive the next one from the previous
            reqs = exchange_fn(kv_cur, kv_nxt, nxt, prv, group)
        if split == "contiguous":
            if not (causal and j > rank):
                po, pl = partial_fn(q, kv_cur[0], kv_cur[1], causal and j == rank, scale)
                merge_fn(acc_o, acc_l, po, pl)
        else:
            w = c // 2
            for qa, a in enumerate(shards_of_rank(split, world, rank)):
                for kb, b in enumerate(shards_of_rank(split, world, j)):
                    if causal and b > a:
                        continue
                    qs, ks = slice(qa * w, (qa + 1) * w), slice(kb * w, (kb + 1) * w)
                    po, pl = partial_fn(q[:, :, qs], kv_cur[0][:, :, ks], kv_cur[1][:, :, ks],
                                        causal and b == a, scale)
                    merge_fn(acc_o[:, :, qs], acc_l[:, :, qs], po, pl)
        for r in reqs:
            r.wait()
        kv_cur, kv_nxt = kv_nxt, kv_cur
    return acc_o, acc_l
