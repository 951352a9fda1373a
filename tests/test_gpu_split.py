"""GPU parity of the two-shard splits (zig-zag and striped, "05. 長系列の分散学習（Context
Parallelism）" §5 因果モデルの負荷分散) through the C ABI: the rank-major layouts (bit-exact),
every ring step's partial, the step-wise ring merged in random order, and the Ulysses forward
and backward with rank-major tensors, each against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from oracle import split as osp
from sequence_long_context_ring_b200 import synth
from sequence_long_context_ring_b200.binding import Plan, seq2head, head2seq, lse_merge

from _helpers import to_dev, to_f64, to_bits, inputs, assert_attn_close

pytestmark = pytest.mark.gpu

SPLITS = ["zigzag", "striped"]


@pytest.mark.parametrize("split", SPLITS)
@pytest.mark.parametrize("B,L,H,d,n", [(2, 64, 8, 128, 4), (1, 96, 6, 64, 3), (1, 16, 2, 128, 2)])
def test_split_layouts_bit_exact(cuda_lib, split, B, L, H, d, n):
    x = synth.tagged_u16((B, L, H, d)) ^ synth.normal_bf16(9, 0, (B, L, H, d))
    y = to_bits(seq2head(n, to_dev(x), split=split))
    np.testing.assert_array_equal(y, osp.seq2head_split(x, n, split))
    back = to_bits(head2seq(n, to_dev(y), split=split))
    np.testing.assert_array_equal(back, x)
    np.testing.assert_array_equal(back, osp.head2seq_split(y, n, split))


@pytest.mark.parametrize("split", SPLITS)
@pytest.mark.parametrize("B,Hq,Hkv,L,d,n,causal", [
    (1, 4, 2, 1024, 128, 4, True),    # shards of 128: one tile each
    (1, 2, 2, 1200, 64, 3, True),     # shards of 200: a ragged tile per shard
    (1, 4, 4, 512, 128, 2, False),
])
def test_ring_step_partials_under_a_split(cuda_lib, split, B, Hq, Hkv, L, d, n, causal):
    q, k, v = inputs(700 + L, (B, Hq, L, d), (B, Hkv, L, d))
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n, causal=causal, split=split)
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    q64, k64, v64 = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    for r in range(n):
        for s in range(n):
            po, pl = plan.ring_step(r, s, tq, tk, tv)
            torch.cuda.synchronize()
            ro, rl = osp.ring_step_split(q64, k64, v64, n, split, r, s, causal=causal)
            got_o, got_l = to_f64(po), to_f64(pl)
            empty = np.isneginf(rl)
            assert np.array_equal(np.isneginf(got_l), empty), f"{split} r{r} s{s}: empty rows differ"
            assert not np.any(got_o[empty]), f"{split} r{r} s{s}: identity rows not zero"
            keep = ~empty
            assert_attn_close(got_o[keep], ro[keep], got_l[keep], rl[keep], f"{split} r{r} s{s}")
    assert plan.device_status()[0] == 0


@pytest.mark.parametrize("split", SPLITS)
def test_stepwise_split_ring_any_order_equals_full_attention(cuda_lib, split):
    B, Hq, Hkv, L, d, n = 1, 4, 2, 1024, 128, 4
    q, k, v = inputs(731, (B, Hq, L, d), (B, Hkv, L, d))
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n, split=split)
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    c = L // n
    rng = np.random.default_rng(5)
    o_all = np.zeros((B, Hq, L, d))
    l_all = np.zeros((B, Hq, L))
    for r in range(n):
        acc_o = torch.zeros((B, Hq, c, d), dtype=torch.float32, device="cuda")
        acc_l = torch.full((B, Hq, c), -float("inf"), dtype=torch.float32, device="cuda")
        for s in rng.permutation(n):
            po, pl = plan.ring_step(r, int(s), tq, tk, tv)
            lse_merge(acc_o, acc_l, po, pl)
        torch.cuda.synchronize()
        pos = osp.rank_positions(split, n, L, r)
        o_all[:, :, pos] = to_f64(acc_o)
        l_all[:, :, pos] = to_f64(acc_l)
    o_ref, l_ref = oracle.attention_full(*(synth.bf16_bits_to_f64(x) for x in (q, k, v)))
    assert_attn_close(o_all, o_ref, l_all, l_ref, f"{split} step-wise")
    # the fused forward of a split plan computes the same global result as a contiguous plan
    o_s, l_s = plan.fwd(tq, tk, tv)
    o_c, l_c = Plan(B, Hq, Hkv, L, d, n_cp=n).fwd(tq, tk, tv)
    torch.cuda.synchronize()
    assert torch.equal(o_s.view(torch.int16), o_c.view(torch.int16)) and torch.equal(l_s, l_c)


@pytest.mark.parametrize("split", SPLITS)
def test_ulysses_forward_and_backward_under_a_split(cuda_lib, split):
    B, L, Hq, Hkv, d, n = 1, 512, 8, 4, 64, 4
    q, k, v, do = inputs(741, (B, L, Hq, d), (B, L, Hkv, d), with_do=True)
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n, mode="ulysses", split=split)
    tq, tk, tv, tdo = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    o, lse = plan.fwd(tq, tk, tv)
    gq, gk, gv = plan.bwd(tq, tk, tv, o, lse, tdo)
    torch.cuda.synchronize()
    assert plan.device_status()[0] == 0
    q64, k64, v64, do64 = (synth.bf16_bits_to_f64(x) for x in (q, k, v, do))
    o_ref, l_ref = osp.ulysses_attention_split(q64, k64, v64, n, split)
    assert_attn_close(to_f64(o), o_ref, to_f64(lse), l_ref, f"{split} ulysses")
    # gradients in position order, head-major, against the plain backward
    order = osp.rank_order(split, n, L)
    inv = np.argsort(order)                       # rank-major row of each position
    head = lambda x: np.transpose(np.asarray(x)[:, inv], (0, 2, 1, 3))
    oh_ref, _ = oracle.attention_full(head(q64), head(k64), head(v64))
    stored = synth.bf16_bits_to_f64(synth.f32_to_bf16_bits(np.asarray(oh_ref, np.float32)))
    rq, rk, rv = oracle.attention_backward(head(q64), head(k64), head(v64), head(do64), o=stored)
    for g, ref, name in ((gq, rq, "dq"), (gk, rk, "dk"), (gv, rv, "dv")):
        got = head(to_f64(g))
        err = np.abs(got - ref)
        assert err.max() <= 2.0 ** -7 * np.abs(ref).max(), f"{split} {name} max-abs {err.max():.3e}"
        assert err.mean() <= 2.0 ** -7 * np.abs(ref).mean(), f"{split} {name} mean-abs {err.mean():.3e}"


@pytest.mark.parametrize("split", SPLITS)
def test_two_shard_step_is_ordered_on_the_callers_stream(cuda_lib, split):
    """Under a two-shard split the step's second query shard runs on the plan's own stream,
    forked from the caller's stream and joined back into it.  So work queued on the caller's
    stream before the call (here: outputs filled with NaN) is seen by both shards, and work
    queued after it (a copy) sees both shards' final values: bit for bit those of the same
    step run alone on the default stream."""
    B, Hq, Hkv, L, d, n = 1, 8, 2, 8192, 128, 4   # shards of 1024 rows, both with work at r = n-1
    q, k, v = inputs(771, (B, Hq, L, d), (B, Hkv, L, d))
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n, split=split)
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    r, st = n - 1, 1
    ref_o, ref_l = plan.ring_step(r, st, tq, tk, tv)
    torch.cuda.synchronize()
    ref_o, ref_l = ref_o.clone(), ref_l.clone()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o = torch.full_like(ref_o, float("nan"))
        lse = torch.full_like(ref_l, float("nan"))
        plan.ring_step(r, st, tq, tk, tv, o, lse, stream=s)
        o2, l2 = o.clone(), lse.clone()
    torch.cuda.synchronize()
    assert torch.equal(o2, ref_o) and torch.equal(l2, ref_l), f"{split}: the copy after the call saw unfinished rows"
    assert plan.device_status()[0] == 0
