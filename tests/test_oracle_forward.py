"""Pins of the fp64 oracle's forward path against facts fixed outside the oracle itself.

Each test states what pins it: a property the pages state (chunked = full, order does not
matter, all-to-all then its inverse restores the layout), a closed form, or a library
routine on a special case.  No expected value comes from the CUDA path.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
from sequence_long_context_ring_b200 import synth


def _qkv(seed, B, Hq, Hkv, L, d, scale=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, L, d)) * scale
    k = rng.standard_normal((B, Hkv, L, d)) * scale
    v = rng.standard_normal((B, Hkv, L, d))
    return q, k, v


def _sdpa64(q, k, v, causal, scale):
    """torch's SDPA in float64 on CPU, with GQA handled by repeating each KV head G times."""
    G = q.shape[1] // k.shape[1]
    tq = torch.from_numpy(q)
    tk = torch.from_numpy(k).repeat_interleave(G, dim=1)
    tv = torch.from_numpy(v).repeat_interleave(G, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
    return o.numpy()


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2), (4, 1)])
def test_full_matches_library_sdpa(causal, hq, hkv):
    # Library routine on the N_cp = 1 special case (GQA by explicit head repetition).
    q, k, v = _qkv(1, 2, hq, hkv, 19, 8)
    o, _ = oracle.attention_full(q, k, v, causal=causal)
    ref = _sdpa64(q, k, v, causal, 1.0 / np.sqrt(8))
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


def test_lse_closed_form_and_row0():
    # Causal row 0 sees only key 0: O_0 = V_0 exactly and LSE_0 = scale * <q_0, k_0>.
    q, k, v = _qkv(2, 1, 2, 2, 12, 16)
    o, lse = oracle.attention_full(q, k, v, causal=True)
    scale = 1.0 / 4.0
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], scale * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]),
                               rtol=0, atol=1e-14)
    # LSE_i = ln sum_j exp(s_ij) by brute force on every row
    for i in range(12):
        s = scale * (k[0, 1, :i + 1] @ q[0, 1, i])
        assert abs(lse[0, 1, i] - np.log(np.sum(np.exp(s)))) < 1e-12


def test_zero_queries_give_prefix_mean():
    # Q = 0 makes every visible score 0: O_i = mean(V_0..V_i), LSE_i = ln(i+1).
    _, k, v = _qkv(3, 1, 2, 1, 10, 4)
    q = np.zeros((1, 2, 10, 4))
    o, lse = oracle.attention_full(q, k, v, causal=True)
    for i in range(10):
        np.testing.assert_allclose(o[0, 1, i], v[0, 0, :i + 1].mean(axis=0), atol=1e-14)
        assert abs(lse[0, 0, i] - np.log(i + 1)) < 1e-14


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2)])
def test_chunked_equals_full_for_every_divisor(causal, hq, hkv):
    # After N_cp ring steps every query has seen every key: chunked == full, for all N | L.
    L = 24
    q, k, v = _qkv(4, 1, hq, hkv, L, 8)
    o_ref, l_ref = oracle.attention_full(q, k, v, causal=causal)
    for n in [n for n in range(1, L + 1) if L % n == 0]:
        o, l = oracle.ring_attention(q, k, v, n, causal=causal)
        np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l, l_ref, rtol=0, atol=1e-12)


def test_visit_order_invariance_all_permutations():
    # The result does not depend on the order in which KV chunks arrive (N = 4: all 24 orders).
    q, k, v = _qkv(5, 1, 2, 1, 16, 8)
    o_ref, l_ref = oracle.ring_attention(q, k, v, 4)
    for perm in itertools.permutations(range(4)):
        o, l = oracle.ring_attention(q, k, v, 4, order=[perm] * 4)
        np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l, l_ref, rtol=0, atol=1e-12)


def test_visit_order_invariance_random_per_rank():
    rng = np.random.default_rng(6)
    q, k, v = _qkv(6, 1, 2, 2, 32, 4)
    o_ref, l_ref = oracle.attention_full(q, k, v)
    for _ in range(5):
        order = [rng.permutation(8) for _ in range(8)]
        o, l = oracle.ring_attention(q, k, v, 8, order=order)
        np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l, l_ref, rtol=0, atol=1e-12)


def test_chunk_partial_of_whole_sequence_is_full():
    q, k, v = _qkv(7, 1, 1, 1, 9, 4)
    o, l = oracle.chunk_partial(q[0, 0], k[0, 0], v[0, 0], 0, 0, causal=True)
    o_ref, l_ref = oracle.attention_full(q, k, v)
    np.testing.assert_allclose(o, o_ref[0, 0], atol=1e-13)
    np.testing.assert_allclose(l, l_ref[0, 0], atol=1e-13)


def test_chunk_above_diagonal_is_empty():
    q, k, v = _qkv(8, 1, 1, 1, 8, 4)
    o, l = oracle.chunk_partial(q[0, 0, :4], k[0, 0, 4:], v[0, 0, 4:], 0, 4, causal=True)
    assert np.all(o == 0) and np.all(np.isneginf(l))


def test_merge_identity_commutative_associative():
    rng = np.random.default_rng(9)
    parts = [(rng.standard_normal((5, 3)), rng.standard_normal(5) * 3) for _ in range(3)]
    ident = (np.zeros((5, 3)), np.full(5, -np.inf))
    a, b, c = parts
    o, l = oracle.lse_merge(*a, *ident)
    np.testing.assert_array_equal(o, a[0]) ; np.testing.assert_array_equal(l, a[1])
    o1, l1 = oracle.lse_merge(*a, *b)
    o2, l2 = oracle.lse_merge(*b, *a)
    np.testing.assert_allclose(o1, o2, atol=1e-14) ; np.testing.assert_allclose(l1, l2, atol=1e-14)
    x = oracle.lse_merge(*oracle.lse_merge(*a, *b), *c)
    y = oracle.lse_merge(*a, *oracle.lse_merge(*b, *c))
    np.testing.assert_allclose(x[0], y[0], atol=1e-13) ; np.testing.assert_allclose(x[1], y[1], atol=1e-13)
    # both empty stays empty, without NaN
    o, l = oracle.lse_merge(*ident, *ident)
    assert np.all(o == 0) and np.all(np.isneginf(l))


def test_merge_of_two_halves_is_attention_over_the_union():
    # Closed form: merging the partials over disjoint key sets equals attention over their union.
    q, k, v = _qkv(10, 1, 1, 1, 12, 4)
    pa = oracle.chunk_partial(q[0, 0], k[0, 0, :5], v[0, 0, :5], 0, 0, causal=False)
    pb = oracle.chunk_partial(q[0, 0], k[0, 0, 5:], v[0, 0, 5:], 0, 5, causal=False)
    o, l = oracle.lse_merge(*pa, *pb)
    ref = _sdpa64(q, k, v, False, 0.5)
    np.testing.assert_allclose(o, ref[0, 0], atol=1e-13)


def test_seq2head_head2seq_inverse_and_index_map():
    # a2a then reverse a2a restores the layout; after seq2head rank r' holds heads
    # [r'H/N, (r'+1)H/N) over the FULL sequence (channels split, sequence whole).
    B, L, H, d, n = 2, 12, 6, 4, 3
    c = L // n
    # each element encodes (global position, head, channel) uniquely
    full = (np.arange(L)[None, :, None, None] * 1000 + np.arange(H)[None, None, :, None] * 10
            + np.arange(d)[None, None, None, :] + np.arange(B)[:, None, None, None] * 10 ** 6)
    ranks = [full[:, s * c:(s + 1) * c] for s in range(n)]
    out = oracle.seq2head(ranks)
    for r2 in range(n):
        assert out[r2].shape == (B, H // n, L, d)
        for b in range(B):
            for h2 in range(H // n):
                for pos in range(L):
                    for e in range(d):
                        assert out[r2][b, h2, pos, e] == b * 10 ** 6 + pos * 1000 + (r2 * (H // n) + h2) * 10 + e
    back = oracle.head2seq(out)
    for s in range(n):
        np.testing.assert_array_equal(back[s], ranks[s])


def test_ulysses_flow_equals_full_attention():
    # Ulysses computes full attention per head after the all-to-all (step 3).
    B, L, Hq, Hkv, d, n = 1, 16, 4, 2, 8, 2
    q, k, v = _qkv(11, B, Hq, Hkv, L, d)
    o_ref, l_ref = oracle.attention_full(q, k, v)
    o_seq, lse = oracle.ulysses_attention(q.transpose(0, 2, 1, 3), k.transpose(0, 2, 1, 3),
                                          v.transpose(0, 2, 1, 3), n)
    np.testing.assert_allclose(o_seq.transpose(0, 2, 1, 3), o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, l_ref, atol=1e-12)


def test_2d_flow_equals_full_attention():
    B, L, H, d = 1, 32, 4, 4
    q, k, v = _qkv(12, B, H, H, L, d)
    o_ref, l_ref = oracle.attention_full(q, k, v)
    o_seq, lse = oracle.attention_2d(q.transpose(0, 2, 1, 3), k.transpose(0, 2, 1, 3),
                                     v.transpose(0, 2, 1, 3), 2, 4)
    np.testing.assert_allclose(o_seq.transpose(0, 2, 1, 3), o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, l_ref, atol=1e-12)


def test_rows_match_full():
    q, k, v = _qkv(13, 1, 2, 1, 40, 8)
    o_ref, l_ref = oracle.attention_full(q, k, v)
    rows = np.array([0, 1, 7, 8, 20, 39])
    o, l = oracle.attention_rows(q[0, 1, rows], k[0, 0], v[0, 0], rows)
    np.testing.assert_allclose(o, o_ref[0, 1, rows], atol=1e-13)
    np.testing.assert_allclose(l, l_ref[0, 1, rows], atol=1e-13)


def test_forward_flops_counts_visible_pairs():
    for L in (1, 5, 64):
        pairs = sum(1 for i in range(L) for j in range(L) if j <= i)
        assert oracle.forward_flops(2, 3, L, 8) == 4.0 * 2 * 3 * 8 * pairs


def test_bf16_rounding_is_nearest_even():
    # Input generator: RNE on the bit pattern (ties to even), exact upcast.
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -9], dtype=np.float32)
    got = synth.bf16_bits_to_f64(synth.f32_to_bf16_bits(x))
    np.testing.assert_array_equal(got, [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 1.0])
    t = torch.from_numpy(np.random.default_rng(0).standard_normal(4096).astype(np.float32))
    ref = t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(synth.f32_to_bf16_bits(t.numpy()), ref)


def test_generator_is_deterministic_and_blocked():
    a = synth.normal_bf16(3, 1, (2, 5, 7))
    b = synth.normal_bf16(3, 1, (2, 5, 7))
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, synth.normal_bf16(3, 2, (2, 5, 7)))
