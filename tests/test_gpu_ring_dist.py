"""GPU checks of ring_dist's compute path (the library's ring-step kernel on one-chunk plans and
its LSE merge):
  * one rank: the ring reduces to the diagonal shard;
  * 2-4 ranks as processes sharing the one GPU, the key/value message passed through host
    memory over gloo (NCCL does not run two ranks on one device): the whole schedule -- the
    exchange, the buffer swap, the causal skips and the shard pairs of the two-shard splits --
    with the real kernels on every rank.  No kernel waits on another rank's; ranks meet only
    on the host.
Every rank's rows must match the fp64 oracle."""
import datetime
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sequence_long_context_ring_b200 import ring_dist, synth

from _helpers import to_dev, to_f64, inputs, assert_attn_close

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def test_one_rank_ring_matches_the_oracle(cuda_lib):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(29700 + os.getpid() % 1000))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        B, Hq, Hkv, c, d = 1, 8, 2, 1000, 128
        q, k, v = inputs(950, (B, Hq, c, d), (B, Hkv, c, d))
        o, lse = ring_dist.ring_attention(to_dev(q), to_dev(k), to_dev(v))
        torch.cuda.synchronize()
        o_ref, l_ref = oracle.attention_full(*(to_f64(to_dev(x)) for x in (q, k, v)))
        assert_attn_close(to_f64(o), o_ref, to_f64(lse), l_ref, "one-rank ring")
        # non-causal: the full shard
        o2, l2 = ring_dist.ring_attention(to_dev(q), to_dev(k), to_dev(v), causal=False)
        torch.cuda.synchronize()
        o2_ref, l2_ref = oracle.attention_full(*(to_f64(to_dev(x)) for x in (q, k, v)), causal=False)
        assert_attn_close(to_f64(o2), o2_ref, to_f64(l2), l2_ref, "one-rank ring, non-causal")
        # zig-zag with one rank: its two shards (first and second half) as shard pairs on
        # strided views -- (0,0) masked, (1,0) full, (1,1) masked -- equal full causal attention
        o3, l3 = ring_dist.ring_attention(to_dev(q), to_dev(k), to_dev(v), split="zigzag")
        torch.cuda.synchronize()
        assert_attn_close(to_f64(o3), o_ref, to_f64(l3), l_ref, "one-rank zig-zag ring")
    finally:
        dist.destroy_process_group()


def _positions(split, world, L, r):
    from oracle import split as osp
    if split == "contiguous":
        c = L // world
        return np.arange(r * c, (r + 1) * c)
    return osp.rank_positions(split, world, L, r)


def _shape(world):
    return 1, 4, 2, 256 * world, 128   # B, Hq, Hkv, L, d: 256 rows per rank


def _gpu_rank(rank, world, port, causal, split, out):
    sys.path.insert(0, ROOT)
    from sequence_long_context_ring_b200 import ring_dist as rd
    torch.cuda.set_device(0)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        B, Hq, Hkv, L, d = _shape(world)
        q, k, v = inputs(960 + world, (B, Hq, L, d), (B, Hkv, L, d))
        pos = _positions(split, world, L, rank)
        qr, kr, vr = (to_dev(np.ascontiguousarray(x[:, :, pos])) for x in (q, k, v))
        o, lse = rd.ring_attention(qr, kr, vr, causal=causal, split=split, exchange_fn=rd.host_staged_exchange)
        torch.cuda.synchronize()
        out[rank] = (o.cpu().numpy(), lse.cpu().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal,split", [
    (2, True, "contiguous"), (4, True, "contiguous"), (3, False, "contiguous"),
    (3, True, "zigzag"), (4, True, "zigzag"), (2, True, "striped"),
])
def test_ring_across_processes_on_one_gpu(cuda_lib, world, causal, split):
    port = 29800 + (os.getpid() * 7 + world * 13 + int(causal) + 3 * len(split)) % 2000
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.spawn(_gpu_rank, args=(world, port, causal, split, out), nprocs=world, join=True)
        res = dict(out)
    B, Hq, Hkv, L, d = _shape(world)
    q, k, v = inputs(960 + world, (B, Hq, L, d), (B, Hkv, L, d))
    o_ref, l_ref = oracle.attention_full(*(synth.bf16_bits_to_f64(x) for x in (q, k, v)), causal=causal)
    for r in range(world):
        pos = _positions(split, world, L, r)
        o, lse = res[r]
        assert_attn_close(o, o_ref[:, :, pos], lse, l_ref[:, :, pos], f"{split} world {world} rank {r}")
