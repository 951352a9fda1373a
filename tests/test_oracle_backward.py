"""Pins of the fp64 oracle's backward: finite differences, float64 autograd, identities."""
import numpy as np
import pytest
import torch

import oracle


def _inputs(seed, B, Hq, Hkv, L, d):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, Hq, L, d)), rng.standard_normal((B, Hkv, L, d)),
            rng.standard_normal((B, Hkv, L, d)), rng.standard_normal((B, Hq, L, d)))


def _loss(q, k, v, do, causal):
    o, _ = oracle.attention_full(q, k, v, causal=causal)
    return float(np.sum(o * do))


@pytest.mark.parametrize("causal", [True, False])
def test_backward_central_differences(causal):
    # <dO, O(x)> has gradient (dq, dk, dv); check every coordinate by central differences.
    q, k, v, do = _inputs(1, 1, 4, 2, 6, 3)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, causal=causal)
    h = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        for idx in np.ndindex(*x.shape):
            old = x[idx]
            x[idx] = old + h
            fp = _loss(q, k, v, do, causal)
            x[idx] = old - h
            fm = _loss(q, k, v, do, causal)
            x[idx] = old
            fd = (fp - fm) / (2 * h)
            assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(fd)), (idx, fd, g[idx])


def test_backward_matches_float64_autograd():
    q, k, v, do = _inputs(2, 2, 4, 1, 11, 8)
    dq, dk, dv = oracle.attention_backward(q, k, v, do)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(4, dim=1), tv.repeat_interleave(4, dim=1), is_causal=True)
    o.backward(torch.from_numpy(do))
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-12)


def test_backward_identities():
    # Rows of P sum to 1: sum over keys of dV = sum over queries (of the group) of dO.
    # Rows of dS sum to 0: sum over keys of dK = 0.
    q, k, v, do = _inputs(3, 1, 4, 2, 13, 4)
    dq, dk, dv = oracle.attention_backward(q, k, v, do)
    for g in range(2):
        np.testing.assert_allclose(dv[0, g].sum(axis=0), do[0, 2 * g:2 * g + 2].sum(axis=(0, 1)), atol=1e-12)
        np.testing.assert_allclose(dk[0, g].sum(axis=0), 0.0, atol=1e-12)
    z = oracle.attention_backward(q, k, v, np.zeros_like(do))
    assert all(np.all(t == 0) for t in z)


def test_sampled_rows_match_full_backward():
    q, k, v, do = _inputs(4, 1, 2, 1, 30, 8)
    dq, dk, dv = oracle.attention_backward(q, k, v, do)
    o, lse = oracle.attention_full(q, k, v)
    rows = np.array([0, 3, 17, 29])
    dq_r = oracle.backward_rows_dq(q[0, 1, rows], k[0, 0], v[0, 0], do[0, 1, rows], o[0, 1, rows],
                                   lse[0, 1, rows], rows)
    np.testing.assert_allclose(dq_r, dq[0, 1, rows], atol=1e-12)
    keys = np.array([20, 25, 29])
    lo = 20
    dk_r, dv_r = oracle.backward_rows_dkdv(q[0, :, lo:], k[0, 0], v[0, 0], do[0, :, lo:], o[0, :, lo:],
                                           lse[0, :, lo:], keys, q_lo=lo)
    np.testing.assert_allclose(dk_r, dk[0, 0, keys], atol=1e-12)
    np.testing.assert_allclose(dv_r, dv[0, 0, keys], atol=1e-12)


def test_stored_output_enters_only_through_D():
    # Closed form: replacing O by O' in D = rowsum(dO * O) changes dS by -P * dD (dD = D' - D),
    # so dV is unchanged, dQ changes by -scale * dD_i * sum_j P_ij k_j and dK by
    # -scale * sum_i dD_i P_ij q_i; giving the exact O reproduces the default (to rounding).
    q, k, v, do = _inputs(5, 1, 2, 2, 9, 4)
    o, _ = oracle.attention_full(q, k, v)
    base = oracle.attention_backward(q, k, v, do)
    same = oracle.attention_backward(q, k, v, do, o=o)
    for a, b in zip(base, same):
        np.testing.assert_allclose(a, b, atol=1e-13)
    o2 = o + 0.01 * np.random.default_rng(1).standard_normal(o.shape)
    dq2, dk2, dv2 = oracle.attention_backward(q, k, v, do, o=o2)
    np.testing.assert_allclose(dv2, base[2], atol=1e-13)
    scale = 0.5
    rows = np.arange(9)
    for h in range(2):
        s = scale * (q[0, h] @ k[0, h].T)
        s = np.where(rows[None, :] <= rows[:, None], s, -np.inf)
        p = np.exp(s - np.log(np.exp(s).sum(axis=1))[:, None])
        dD = (do[0, h] * (o2[0, h] - o[0, h])).sum(axis=1)
        np.testing.assert_allclose(dq2[0, h] - base[0][0, h], -scale * dD[:, None] * (p @ k[0, h]), atol=1e-12)
        np.testing.assert_allclose(dk2[0, h] - base[1][0, h], -scale * (p * dD[:, None]).T @ q[0, h], atol=1e-12)
