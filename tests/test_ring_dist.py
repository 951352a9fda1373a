"""The ring across processes ("05. 長系列の分散学習（Context Parallelism）", ring attention steps
1-4) on CPU: gloo ranks, one per shard, run ring_dist.ring_attention's exchange schedule
(send the held key/value shard to the next rank, receive the next from the previous, N - 1
exchanges, causal skip above the diagonal) with the oracle's chunk partial and merge standing
in for the GPU kernels.  Every rank's result must equal full attention on its rows.

On GPUs the same schedule runs the library's ring-step and merge kernels over NCCL; that form
needs several GPUs in one job and is not run here."""
import os
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _inputs(world, B=1, Hq=4, Hkv=2, c=6, d=8):
    rng = np.random.default_rng(100 + world)
    L = c * world
    return (rng.standard_normal((B, Hq, L, d)), rng.standard_normal((B, Hkv, L, d)),
            rng.standard_normal((B, Hkv, L, d)))


def _rank(rank, world, port, causal, out):
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
        c = L // world
        sl = slice(rank * c, (rank + 1) * c)
        qr, kr, vr = (torch.from_numpy(np.ascontiguousarray(x[:, :, sl])) for x in (q, k, v))
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

        o, lse = ring_dist.ring_attention(qr, kr, vr, causal=causal, partial_fn=partial, merge_fn=merge)
        out[rank] = (o.numpy(), lse.numpy(), calls)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_across_processes_equals_full_attention(world, causal):
    import oracle
    port = 29600 + (os.getpid() * 7 + world * 13 + int(causal)) % 2000
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.spawn(_rank, args=(world, port, causal, out), nprocs=world, join=True)
        res = dict(out)
    q, k, v = _inputs(world)
    o_ref, l_ref = oracle.attention_full(q, k, v, causal=causal)
    c = q.shape[2] // world
    for r in range(world):
        o, lse, calls = res[r]
        np.testing.assert_allclose(o, o_ref[:, :, r * c:(r + 1) * c], atol=1e-12)
        np.testing.assert_allclose(lse, l_ref[:, :, r * c:(r + 1) * c], atol=1e-12)
        # causal: rank r computes its r + 1 shards at or below the diagonal (the diagonal one
        # masked, first) and skips the rest; otherwise all N shards, none masked
        if causal:
            assert calls == [True] + [False] * r
        else:
            assert calls == [False] * world
