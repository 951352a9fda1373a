"""The ring across processes ("05. 長系列の分散学習（Context Parallelism）", ring attention steps
1-4, and the two-shard splits of §5) on CPU: gloo ranks, one per shard, run
ring_dist.ring_attention's exchange schedule (send the held key/value rows to the next rank,
receive the next from the previous, N - 1 exchanges, causal skip above the diagonal, shard
pairs under zig-zag / striped) with the oracle's chunk partial and merge standing in for the
GPU kernels.  Every rank's result must equal full attention on its rows.

On GPUs the same schedule runs the library's ring-step and merge kernels over NCCL; that form
needs several GPUs in one job and is not run here."""
import os
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _inputs(world, B=1, Hq=4, Hkv=2, c=6, d=8):
    # c = 6 local rows: shards of 3 under a two-shard split
    rng = np.random.default_rng(100 + world)
    L = c * world
    return (rng.standard_normal((B, Hq, L, d)), rng.standard_normal((B, Hkv, L, d)),
            rng.standard_normal((B, Hkv, L, d)))


def _positions(split, world, L, r):
    from oracle import split as osp
    if split == "contiguous":
        c = L // world
        return np.arange(r * c, (r + 1) * c)
    return osp.rank_positions(split, world, L, r)


def _rank(rank, world, port, causal, split, out, staged=False):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from sequence_long_context_ring_b200 import ring_dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = _inputs(world)
        B, Hq, L, d = q.shape
        G = Hq // k.shape[1]
        pos = _positions(split, world, L, rank)
        qr, kr, vr = (torch.from_numpy(np.ascontiguousarray(x[:, :, pos])) for x in (q, k, v))
        calls = []

        def partial(qq, kk, vv, diagonal, scale):
            # the oracle's one-step partial of a shard pair: masked (key <= query inside the
            # pair) at the diagonal shard, full below it
            calls.append(bool(diagonal))
            qq, kk, vv = qq.numpy(), kk.numpy(), vv.numpy()
            o = np.zeros(qq.shape)
            lse = np.zeros(qq.shape[:3])
            for b in range(B):
                for h in range(Hq):
                    o[b, h], lse[b, h] = oracle.chunk_partial(qq[b, h], kk[b, h // G], vv[b, h // G], 0, 0,
                                                              causal=bool(diagonal), scale=scale or None)
            return torch.from_numpy(o), torch.from_numpy(lse)

        def merge(acc_o, acc_l, po, pl):
            o2, l2 = oracle.lse_merge(acc_o.numpy(), acc_l.numpy(), po.numpy(), pl.numpy())
            acc_o.copy_(torch.from_numpy(o2))
            acc_l.copy_(torch.from_numpy(l2))

        exchange = ring_dist.host_staged_exchange if staged else None
        o, lse = ring_dist.ring_attention(qr, kr, vr, causal=causal, split=split, partial_fn=partial, merge_fn=merge,
                                          exchange_fn=exchange)
        out[rank] = (o.numpy(), lse.numpy(), calls)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal,split", [
    (1, True, "contiguous"), (2, True, "contiguous"), (3, True, "contiguous"), (4, True, "contiguous"),
    (1, False, "contiguous"), (3, False, "contiguous"),
    (2, True, "zigzag"), (3, True, "zigzag"), (4, True, "zigzag"), (3, True, "striped"), (2, False, "zigzag"),
    (8, True, "zigzag"), (6, False, "striped"), (5, True, "contiguous"),
])
def test_ring_across_processes_equals_full_attention(world, causal, split):
    import oracle
    port = 29600 + (os.getpid() * 7 + world * 13 + int(causal) + 3 * len(split)) % 2000
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.spawn(_rank, args=(world, port, causal, split, out), nprocs=world, join=True)
        res = dict(out)
    q, k, v = _inputs(world)
    L = q.shape[2]
    o_ref, l_ref = oracle.attention_full(q, k, v, causal=causal)
    for r in range(world):
        o, lse, calls = res[r]
        pos = _positions(split, world, L, r)
        np.testing.assert_allclose(o, o_ref[:, :, pos], atol=1e-12)
        np.testing.assert_allclose(lse, l_ref[:, :, pos], atol=1e-12)
        if split == "contiguous":
            # causal: rank r computes its r + 1 shards at or below the diagonal (the diagonal
            # one masked, first) and skips the rest; otherwise all N shards, none masked
            assert calls == ([True] + [False] * r if causal else [False] * world)
        elif causal:
            # two shards per rank: the shard pairs at or below the diagonal, one masked pair per
            # own shard; under zig-zag every step but the first carries 2 full pairs
            n_pairs = sum(1 for s in range(world)
                          for a in ring_dist_shards(split, world, r)
                          for b in ring_dist_shards(split, world, (r - s) % world) if b <= a)
            assert len(calls) == n_pairs and sum(calls) == 2
            if split == "zigzag":
                assert n_pairs == 3 + 2 * (world - 1)


@pytest.mark.parametrize("world,split", [(3, "zigzag"), (4, "contiguous")])
def test_host_staged_exchange_gives_the_same_ring(world, split):
    # the exchange through host buffers (for groups that move only host tensors) runs the same
    # schedule: every rank's rows equal full attention
    import oracle
    port = 29550 + (os.getpid() * 5 + world * 17 + len(split)) % 2000
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.spawn(_rank, args=(world, port, True, split, out, True), nprocs=world, join=True)
        res = dict(out)
    q, k, v = _inputs(world)
    o_ref, l_ref = oracle.attention_full(q, k, v)
    for r in range(world):
        pos = _positions(split, world, q.shape[2], r)
        np.testing.assert_allclose(res[r][0], o_ref[:, :, pos], atol=1e-12)
        np.testing.assert_allclose(res[r][1], l_ref[:, :, pos], atol=1e-12)


def ring_dist_shards(split, world, r):
    from oracle import split as osp
    return osp.shards_of_rank(split, world, r)


def _rank_groups(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from sequence_long_context_ring_b200 import ring_dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # two independent rings of two ranks each: global ranks {0, 2} and {1, 3}, so the
        # neighbours inside a group are not the neighbours in the world
        groups = [dist.new_group([0, 2]), dist.new_group([1, 3])]
        g = rank % 2
        gr = rank // 2
        q, k, v = _inputs(10 + g)                 # each group attends over its own problem
        B, Hq, L, d = q.shape
        G = Hq // k.shape[1]
        c = L // 2
        sl = slice(gr * c, (gr + 1) * c)
        qr, kr, vr = (torch.from_numpy(np.ascontiguousarray(x[:, :, sl])) for x in (q, k, v))

        def partial(qq, kk, vv, diagonal, scale):
            qq, kk, vv = qq.numpy(), kk.numpy(), vv.numpy()
            o = np.zeros(qq.shape)
            lse = np.zeros(qq.shape[:3])
            for b in range(B):
                for h in range(Hq):
                    o[b, h], lse[b, h] = oracle.chunk_partial(qq[b, h], kk[b, h // G], vv[b, h // G], 0, 0,
                                                              causal=bool(diagonal))
            return torch.from_numpy(o), torch.from_numpy(lse)

        def merge(acc_o, acc_l, po, pl):
            o2, l2 = oracle.lse_merge(acc_o.numpy(), acc_l.numpy(), po.numpy(), pl.numpy())
            acc_o.copy_(torch.from_numpy(o2))
            acc_l.copy_(torch.from_numpy(l2))

        o, lse = ring_dist.ring_attention(qr, kr, vr, groups[g], partial_fn=partial, merge_fn=merge)
        out[rank] = (o.numpy(), lse.numpy())
    finally:
        dist.destroy_process_group()


def test_rings_in_process_subgroups():
    import oracle
    port = 29650 + (os.getpid() * 11) % 2000
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.spawn(_rank_groups, args=(4, port, out), nprocs=4, join=True)
        res = dict(out)
    for rank in range(4):
        g, gr = rank % 2, rank // 2
        q, k, v = _inputs(10 + g)
        o_ref, l_ref = oracle.attention_full(q, k, v)
        c = q.shape[2] // 2
        np.testing.assert_allclose(res[rank][0], o_ref[:, :, gr * c:(gr + 1) * c], atol=1e-12)
        np.testing.assert_allclose(res[rank][1], l_ref[:, :, gr * c:(gr + 1) * c], atol=1e-12)


def _rank_failure(rank, world, port, mode, out):
    import datetime
    import time

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from sequence_long_context_ring_b200 import ring_dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=2))
    if rank == 1:
        # the failing peer: it leaves before its first exchange, or stalls past the timeout
        out[rank] = mode
        if mode == "stalls":
            time.sleep(5)
        dist.destroy_process_group()
        return
    q = torch.zeros((1, 2, 4, 8), dtype=torch.float64)
    zeros = lambda qq, kk, vv, diag, scale: (torch.zeros_like(qq), torch.zeros(qq.shape[:3], dtype=qq.dtype))
    t0 = time.time()
    try:
        ring_dist.ring_attention(q, q[:, :1], q[:, :1], partial_fn=zeros, merge_fn=lambda *a: None)
        out[rank] = ("returned", time.time() - t0)
    except RuntimeError:
        out[rank] = ("raised", time.time() - t0)
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


@pytest.mark.parametrize("mode", ["leaves", "stalls"])
def test_a_failing_peer_ends_the_ring_with_an_error(mode):
    # failure detection on the host: the surviving rank's exchange raises (connection closed,
    # or the process group's 2 s timeout) instead of waiting for ever
    port = 29750 + (os.getpid() * 13 + len(mode)) % 2000
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.spawn(_rank_failure, args=(2, port, mode, out), nprocs=2, join=True)
        res = dict(out)
    assert res[1] == mode
    outcome, seconds = res[0]
    assert outcome == "raised"
    assert seconds < 4.5
