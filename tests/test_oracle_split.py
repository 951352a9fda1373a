"""Pins of the oracle's rank-to-sequence maps (zig-zag, striped, contiguous) and of the ring and
Ulysses flows under them ("05. 長系列の分散学習（Context Parallelism）" §5 因果モデルの負荷分散)."""
import json
import os
from itertools import permutations

import numpy as np
import pytest

import oracle
from oracle import split as sp

HERE = os.path.dirname(os.path.abspath(__file__))


def test_zigzag_matches_the_pages_worked_example():
    g = json.load(open(os.path.join(HERE, "golden", "zigzag_shards_n4.json")))
    got = [list(sp.shards_of_rank("zigzag", g["n_cp"], r)) for r in range(g["n_cp"])]
    assert got == g["shards_per_rank"]


def test_striped_matches_the_fixture_of_its_reading():
    g = json.load(open(os.path.join(HERE, "golden", "striped_shards_n4.json")))
    n = g["n_cp"]
    assert [list(sp.shards_of_rank("striped", n, r)) for r in range(n)] == g["shards_per_rank"]
    assert [sp.rank_positions("striped", n, g["L"], r).tolist() for r in range(n)] == g["positions_per_rank"]


@pytest.mark.parametrize("n", [1, 2, 3, 4, 8])
def test_striped_deals_shards_round_robin(n):
    # stripes: walking the shards in sequence order, the ranks take turns, so shard s belongs
    # to rank s mod N (any other permutation of shards would break this for some n)
    owner = {}
    for r in range(n):
        for s in sp.shards_of_rank("striped", n, r):
            owner[s] = r
    assert [owner[s] for s in range(2 * n)] == [s % n for s in range(2 * n)]


@pytest.mark.parametrize("split", sp.SPLITS)
@pytest.mark.parametrize("n,L", [(1, 8), (2, 8), (3, 12), (4, 32), (5, 40)])
def test_every_position_belongs_to_exactly_one_rank(split, n, L):
    order = sp.rank_order(split, n, L)
    assert sorted(order.tolist()) == list(range(L))


@pytest.mark.parametrize("n,L", [(2, 16), (4, 64), (8, 160)])
def test_zigzag_balances_the_causal_work_exactly(n, L):
    # the page's reason for zig-zag: every rank gets the same causal work.  With shards of w,
    # rank r's queries are shards r and 2N-1-r: sum of (pos+1) is (2N-1)*w*w + w*(w+1) for all r
    work = [oracle.split.causal_pairs(sp.rank_positions("zigzag", n, L, r)) for r in range(n)]
    w = L // (2 * n)
    assert work == [(2 * n - 1) * w * w + w * (w + 1)] * n
    contiguous = [oracle.split.causal_pairs(sp.rank_positions("contiguous", n, L, r)) for r in range(n)]
    assert all(a < b for a, b in zip(contiguous, contiguous[1:]))


@pytest.mark.parametrize("n", [2, 3, 4])
def test_zigzag_steps_carry_equal_work(n):
    # under zig-zag every off-diagonal ring step of every rank sees two full w x w shard blocks
    # (one of its shards is above the other rank's pair, one below); the diagonal step sees one
    # full block and two triangular ones: w^2 + 2 * w(w+1)/2
    L = 8 * n
    w = L // (2 * n)
    for r in range(n):
        for s in range(n):
            expect = 2 * w * w + (w if s == 0 else 0)
            assert sp.step_pairs("zigzag", n, L, r, s) == expect


def _inputs(seed, B, Hq, Hkv, L, d):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, Hq, L, d)), rng.standard_normal((B, Hkv, L, d)),
            rng.standard_normal((B, Hkv, L, d)))


@pytest.mark.parametrize("split", sp.SPLITS)
@pytest.mark.parametrize("n,L,causal", [(1, 8, True), (2, 16, True), (3, 24, True), (4, 32, False)])
def test_ring_under_a_split_equals_full_attention(split, n, L, causal):
    q, k, v = _inputs(L + n, 1, 4, 2, L, 8)
    o, lse = sp.ring_attention_split(q, k, v, n, split, causal=causal)
    o_ref, l_ref = oracle.attention_full(q, k, v, causal=causal)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, l_ref, rtol=0, atol=1e-12)


def test_ring_under_zigzag_is_step_order_invariant():
    q, k, v = _inputs(7, 1, 2, 1, 24, 8)
    o_ref, l_ref = oracle.attention_full(q, k, v)
    for perm in permutations(range(3)):
        o, lse = sp.ring_attention_split(q, k, v, 3, "zigzag", order=[perm] * 3)
        np.testing.assert_allclose(o, o_ref, atol=1e-12)
        np.testing.assert_allclose(lse, l_ref, atol=1e-12)


def test_contiguous_split_reduces_to_the_plain_ring_step():
    q, k, v = _inputs(11, 1, 2, 2, 16, 8)
    for r in range(4):
        for s in range(4):
            o, lse = sp.ring_step_split(q, k, v, 4, "contiguous", r, s)
            j = (r - s) % 4
            for h in range(2):
                po, pl = oracle.chunk_partial(q[0, h, 4 * r:4 * r + 4], k[0, h, 4 * j:4 * j + 4],
                                              v[0, h, 4 * j:4 * j + 4], 4 * r, 4 * j)
                np.testing.assert_allclose(o[0, h], po, atol=1e-12)
                np.testing.assert_allclose(lse[0, h], pl, atol=1e-12)


@pytest.mark.parametrize("split", sp.SPLITS)
def test_split_layouts_invert_and_follow_the_index_formula(split):
    n, L, H, d = 4, 16, 8, 4
    x = np.arange(L * H * d, dtype=np.int64).reshape(1, L, H, d)
    y = sp.seq2head_split(x, n, split)
    np.testing.assert_array_equal(sp.head2seq_split(y, n, split), x)
    order = sp.rank_order(split, n, L)
    for u in range(L):  # rank-major row u holds global position order[u]
        np.testing.assert_array_equal(y[0, :, order[u], :], x[0, u, :, :])
    if split == "contiguous":
        np.testing.assert_array_equal(y, np.concatenate(oracle.seq2head([x[:, s * 4:(s + 1) * 4] for s in range(n)]), 1))


@pytest.mark.parametrize("split", ["zigzag", "striped"])
def test_ulysses_under_a_split_equals_full_attention(split):
    n, L, H, d = 2, 16, 4, 8
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((1, L, H, d)) for _ in range(3))
    o, lse = sp.ulysses_attention_split(q, k, v, n, split)
    order = sp.rank_order(split, n, L)
    to_head = lambda x: np.transpose(x[:, np.argsort(order)], (0, 2, 1, 3))  # rank-major -> [B,H,L,d]
    o_ref, l_ref = oracle.attention_full(to_head(q), to_head(k), to_head(v))
    np.testing.assert_allclose(to_head(o), o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, l_ref, atol=1e-12)
