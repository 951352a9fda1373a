"""GPU check of ring_dist's default compute path (the library's ring-step kernel on one-chunk
plans and its LSE merge) in a one-rank process group: the ring reduces to the diagonal shard,
whose result must match the fp64 oracle.  Several ranks need one GPU each (NCCL does not run
two ranks on one device); their exchange schedule is covered on CPU by test_ring_dist.py."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from sequence_long_context_ring_b200 import ring_dist

from _helpers import to_dev, to_f64, inputs, assert_attn_close

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
