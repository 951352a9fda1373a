"""Pins of the oracle's causal FIR convolution and its point-to-point form with an l_h - 1 halo
("05. 長系列の分散学習（Context Parallelism）" §3 Hyena 演算子をどう分散するか, p2p 畳み込み).

Each pin rests on something other than the oracle's own formula: numpy's convolution routine,
closed forms (delta filters, impulse inputs, the sum of a full convolution), and the locality
property the page states (only the first l_h - 1 outputs of a shard depend on another rank)."""
import numpy as np
import pytest

from oracle import conv


def _xh(seed, B, D, L, lh):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((B, D, L)), rng.standard_normal((D, lh))


@pytest.mark.parametrize("B,D,L,lh", [(1, 1, 1, 1), (1, 3, 17, 5), (2, 4, 40, 9), (1, 2, 6, 11)])
def test_definition_equals_numpys_convolution_truncated(B, D, L, lh):
    # np.convolve(a, v)[t] = sum_k v[k] a[t-k]: its first L samples are the causal convolution
    x, h = _xh(1, B, D, L, lh)
    y = conv.fir_conv(x, h)
    for b in range(B):
        for c in range(D):
            np.testing.assert_allclose(y[b, c], np.convolve(x[b, c], h[c])[:L], rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("k", [0, 1, 4, 7])
def test_delta_filter_delays_the_input(k):
    x, _ = _xh(2, 2, 3, 20, 8)
    h = np.zeros((3, 8))
    h[:, k] = [1.0, -2.0, 0.5]
    y = conv.fir_conv(x, h)
    expect = np.zeros_like(x)
    expect[:, :, k:] = x[:, :, :20 - k] * np.array([1.0, -2.0, 0.5])[None, :, None]
    np.testing.assert_array_equal(y, expect)


@pytest.mark.parametrize("t0", [0, 3, 15])
def test_impulse_input_reads_out_the_filter_in_order(t0):
    # an asymmetric filter catches a correlation written in place of a convolution
    L, lh = 20, 6
    h = np.arange(1.0, 1.0 + 2 * lh).reshape(2, lh) ** 2
    x = np.zeros((1, 2, L))
    x[0, :, t0] = 1.0
    y = conv.fir_conv(x, h)
    expect = np.zeros((1, 2, L))
    n = min(lh, L - t0)
    expect[0, :, t0:t0 + n] = h[:, :n]
    np.testing.assert_array_equal(y, expect)


def test_full_length_convolution_sums_to_the_product_of_sums():
    # with l_h - 1 zeros appended nothing is truncated: sum_t y = (sum x)(sum h) per channel
    B, D, L, lh = 2, 3, 25, 7
    x, h = _xh(3, B, D, L, lh)
    xp = np.concatenate([x, np.zeros((B, D, lh - 1))], axis=2)
    y = conv.fir_conv(xp, h)
    np.testing.assert_allclose(y.sum(axis=2), x.sum(axis=2) * h.sum(axis=1)[None], rtol=1e-12)


@pytest.mark.parametrize("L,n", [(12, 1), (12, 2), (12, 3), (12, 4), (24, 6), (30, 5)])
@pytest.mark.parametrize("lh", [1, 2, 3])
def test_point_to_point_equals_the_whole_sequence(L, n, lh):
    x, h = _xh(4, 2, 3, L, lh)
    np.testing.assert_allclose(conv.fir_conv_cp(x, h, n), conv.fir_conv(x, h), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("c,n", [(5, 3), (8, 4), (16, 2)])
def test_point_to_point_with_the_longest_halo(c, n):
    # l_h - 1 == c: a rank's halo is the whole previous shard, the largest the page allows
    x, h = _xh(5, 1, 2, c * n, c + 1)
    np.testing.assert_allclose(conv.fir_conv_cp(x, h, n), conv.fir_conv(x, h), rtol=1e-12, atol=1e-12)
    with pytest.raises(AssertionError):
        conv.fir_conv_cp(x, np.ones((2, c + 2)), n)


def test_only_the_first_lh_minus_1_outputs_depend_on_the_previous_rank():
    # the page's locality statement, checked on the definition: perturb rank r-1's inputs and
    # exactly rank r's first l_h - 1 outputs move; perturb anything before its last l_h - 1
    # inputs and rank r does not move at all
    B, D, c, n, lh = 1, 2, 10, 3, 4
    x, h = _xh(6, B, D, c * n, lh)
    h[:, -1] = 1.0 + np.abs(h[:, -1])          # the longest tap is non-zero
    y = conv.fir_conv(x, h)
    r = 2
    far = x.copy()
    far[:, :, (r - 1) * c:r * c - (lh - 1)] += 1.0
    np.testing.assert_array_equal(conv.fir_conv(far, h)[:, :, r * c:], y[:, :, r * c:])
    near = x.copy()
    near[:, :, r * c - (lh - 1):r * c] += 1.0
    moved = conv.fir_conv(near, h)[:, :, r * c:] != y[:, :, r * c:]
    assert moved[:, :, :lh - 1].all() and not moved[:, :, lh - 1:].any()


def test_shard_without_a_halo_is_the_zero_padded_first_stage():
    # rank 0 (no predecessor) and the overlap variant's first stage are the same computation
    x, h = _xh(7, 2, 3, 16, 5)
    np.testing.assert_array_equal(conv.fir_conv_shard(x, None, h), conv.fir_conv(x, h))
    zero_halo = conv.fir_conv_shard(x, np.zeros((2, 3, 4)), h)
    np.testing.assert_array_equal(zero_halo, conv.fir_conv(x, h))


def test_shard_boundary_terms_come_from_the_halo_in_order():
    # a halo that is an impulse at its m-th entry (input position m - (l_h - 1) relative to the
    # shard) adds h[t - m + l_h - 1] to output t, for the taps that reach back that far
    lh, c = 6, 9
    h = (np.arange(1.0, 1.0 + lh) ** 2)[None, :]
    for m in range(lh - 1):
        halo = np.zeros((1, 1, lh - 1))
        halo[0, 0, m] = 1.0
        y = conv.fir_conv_shard(np.zeros((1, 1, c)), halo, h)
        expect = np.zeros(c)
        for t in range(c):
            k = t - (m - (lh - 1))
            if k < lh:
                expect[t] = h[0, k]
        np.testing.assert_array_equal(y[0, 0], expect)
