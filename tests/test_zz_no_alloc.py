"""cp_attn_fwd_noalloc: the forward for callers that cannot allocate device memory (code inside
a framework that owns the whole device-memory budget, or a process that reserved all device
memory up front).  The library uses its static 64 MiB scratch instead of a caller workspace.
This file is collected last, so a run that stops at the first failure has run every other
test already; it also passes on its own in a fresh process."""
import numpy as np
import pytest
import torch

import oracle
from oracle import split as osp
from sequence_long_context_ring_b200 import synth
from sequence_long_context_ring_b200.binding import Plan, CpError, CP_ERR_WORKSPACE, CP_ERR_INVALID_ARG

from _helpers import to_dev, to_f64, inputs, assert_attn_close


@pytest.mark.gpu
@pytest.mark.parametrize("mode,n_cp,n_hp,split", [("ulysses", 4, 1, "contiguous"), ("2d", 2, 2, "contiguous"),
                                                  ("ulysses", 4, 1, "zigzag")])
def test_noalloc_matches_workspace_entry_point_twice(cuda_lib, mode, n_cp, n_hp, split):
    # Both entry points run the same kernels on the same inputs, so their results must agree
    # bit for bit; the first is also checked against the fp64 oracle.  Two calls in a row with
    # different inputs: nothing left in the shared scratch by the first may leak into the second.
    B, L, Hq, Hkv, d = 1, 1024, 8, 4, 128
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n_cp, n_hp=n_hp, mode=mode, split=split)
    assert plan.workspace_size() <= 64 << 20
    for call, seed in enumerate((71, 72)):
        qb, kb, vb = inputs(seed, (B, L, Hq, d), (B, L, Hkv, d))
        q, k, v = to_dev(qb), to_dev(kb), to_dev(vb)
        o_ws, lse_ws = plan.fwd(q, k, v)
        o = torch.full_like(o_ws, float("nan"))
        lse = torch.full_like(lse_ws, float("nan"))
        plan.fwd_noalloc(q, k, v, o, lse)
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int16), o_ws.view(torch.int16)), f"{mode}/{split} call {call}: O differs"
        assert torch.equal(lse, lse_ws), f"{mode}/{split} call {call}: LSE differs"
        q64, k64, v64 = (synth.bf16_bits_to_f64(x) for x in (qb, kb, vb))
        if mode == "2d":
            o_ref, l_ref = oracle.attention_2d(q64, k64, v64, n_hp, n_cp)
        elif split == "contiguous":
            o_ref, l_ref = oracle.ulysses_attention(q64, k64, v64, n_cp)
        else:
            o_ref, l_ref = osp.ulysses_attention_split(q64, k64, v64, n_cp, split)
        assert_attn_close(to_f64(o), o_ref, to_f64(lse), l_ref, f"{mode}/{split} call {call} vs oracle")


@pytest.mark.gpu
def test_noalloc_rejects_problems_beyond_the_scratch(cuda_lib):
    B, L, H, d = 1, 16384, 16, 128     # forward workspace 128 MiB > 64 MiB
    plan = Plan(B, H, H, L, d, n_cp=4, mode="ulysses")
    assert plan.workspace_size() > 64 << 20
    x = torch.zeros((B, L, H, d), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(x)
    lse = torch.empty((B, H, L), dtype=torch.float32, device="cuda")
    with pytest.raises(CpError) as e:
        plan.fwd_noalloc(x, x, x, o, lse)
    assert e.value.status == CP_ERR_WORKSPACE
    ring = Plan(1, 4, 4, 1024, 64, n_cp=4)
    y = torch.zeros((1, 4, 1024, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(CpError) as e:
        ring.fwd_noalloc(y, y, y, torch.empty_like(y), torch.empty((1, 4, 1024), dtype=torch.float32, device="cuda"))
    assert e.value.status == CP_ERR_INVALID_ARG
