"""Causal FIR (finite impulse response) convolution under context parallelism, in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

"05. 長系列の分散学習（Context Parallelism）" §3 (Hyena 演算子をどう分散するか), the point-to-point
convolution: each rank holds every channel of its sequence shard x[D, L/N_cp] and a copy of
the filters; a causal FIR filter of length l_h needs, for the first l_h - 1 outputs of a
shard, the last l_h - 1 inputs of the previous rank (its halo), and nothing else from other
ranks.  The overlap variant computes the shard with a zero halo first and adds the boundary
terms once the halo has arrived.

Readings taken where the page is terse:
  * the filter is depthwise (one filter per channel, as in Hyena): h [D, l_h];
  * causal: y[c, t] = sum_{k=0}^{l_h-1} h[c, k] x[c, t-k], with x[c, t] = 0 for t < 0;
  * the halo of rank r comes from rank r-1 alone, so l_h - 1 <= L / N_cp;
  * rank 0 has no predecessor: its halo is zero (the same zero as x[c, t<0]).
"""
from __future__ import annotations

import numpy as np


def fir_conv(x, h):
    """The definition: x [B, D, L], h [D, l_h] -> y [B, D, L] (float64)."""
    x = np.asarray(x, dtype=np.float64)
    h = np.asarray(h, dtype=np.float64)
    B, D, L = x.shape
    lh = h.shape[1]
    y = np.zeros((B, D, L))
    for k in range(min(lh, L)):
        y[:, :, k:] += h[None, :, k, None] * x[:, :, :L - k]
    return y


def fir_conv_shard(x_shard, halo, h):
    """One rank of the point-to-point convolution: its shard x_shard [B, D, c] and the halo
    [B, D, l_h - 1] received from the previous rank (None: no predecessor, zeros) ->
    y_shard [B, D, c].  Taken in the overlap variant's two stages: the shard convolved with a
    zero halo, then the boundary terms, in which a tap reaches back past the shard's start,
    added to the first l_h - 1 outputs."""
    x_shard = np.asarray(x_shard, dtype=np.float64)
    h = np.asarray(h, dtype=np.float64)
    B, D, c = x_shard.shape
    lh = h.shape[1]
    assert lh - 1 <= c, "the halo must come from the previous rank alone"
    y = fir_conv(x_shard, h)                                   # stage 1: zero halo
    if halo is None or lh == 1:
        return y
    halo = np.asarray(halo, dtype=np.float64)
    assert halo.shape == (B, D, lh - 1)
    # halo[..., m] is the input at shard-relative position m - (l_h - 1)
    for t in range(lh - 1):                                    # stage 2: boundary terms
        for k in range(t + 1, lh):                             # taps with t - k < 0
            y[:, :, t] += h[None, :, k] * halo[:, :, lh - 1 + t - k]
    return y


def fir_conv_cp(x, h, n_cp: int):
    """The point-to-point convolution on n_cp ranks of contiguous shards: rank r convolves
    x[..., r c:(r+1) c] with the last l_h - 1 inputs of rank r - 1 as its halo."""
    x = np.asarray(x, dtype=np.float64)
    B, D, L = x.shape
    lh = np.asarray(h).shape[1]
    assert L % n_cp == 0
    c = L // n_cp
    y = np.zeros((B, D, L))
    for r in range(n_cp):
        halo = x[:, :, r * c - (lh - 1):r * c] if r > 0 and lh > 1 else None
        y[:, :, r * c:(r + 1) * c] = fir_conv_shard(x[:, :, r * c:(r + 1) * c], halo, h)
    return y
