"""Distributed FFT convolution (radix-N_cp decimation in frequency), in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

"05. 長系列の分散学習（Context Parallelism）" §4 (FFT 畳み込み：周波数領域の魔法):
  * convolution theorem: x * h = F^-1(F(x) . F(h));
  * DFT: y(k) = sum_j x(j) w_l^(jk), w_l = exp(-2 pi i / l);
  * decimation-in-frequency (DiF) butterfly: X = x + y, Y = (x - y) w^j;
  * the DiF split matches point-to-point CP: each shard stays on its device; a DiF forward
    transform followed by the mirrored inverse puts the result back in the input's shard
    layout, with no all-to-all (the spectrum is used in its decimated order, never reordered);
  * N_cp > 2: radix-N (an l-point DFT as N sub-DFTs of l/N points) with N = N_cp.

Readings taken where the page is terse:
  * the operator is the causal linear convolution of a long filter (Hyena-LI): h [D, L],
    y[c, t] = sum_{k<=t} h[c, k] x[c, t-k] for t < L; it needs a transform of l = 2L points
    (zero padding), so the first DiF stage is radix-2N over the N data shards and N zero
    shards: z_q(n) = w_2L^(n q) sum_r x(n + c r) w_2N^(r q), q in [0, 2N);
  * the l/N = c point transforms run per virtual rank q ("local"); the spectral product and the
    local inverse transform too; the last stage is the mirrored cross-rank sum
    y(n + c r) = (1/2L) sum_q w_2N^(-r q) w_q(n);
  * the local DFT is a library step (numpy's FFT), as the page allows any FFT there.
"""
from __future__ import annotations

import numpy as np


def dft(a, inverse: bool = False):
    """The definition, O(l^2): y(k) = sum_j a(j) w^(jk), w = exp(-+2 pi i / l); the inverse is
    unnormalised (w^-1)."""
    a = np.asarray(a, dtype=np.complex128)
    l = a.shape[-1]
    s = 1.0 if inverse else -1.0
    jk = np.outer(np.arange(l), np.arange(l))
    return a @ np.exp(s * 2j * np.pi * jk / l)


def dif_butterfly(x, y, w):
    """The page's DiF butterfly: X = x + y, Y = (x - y) w."""
    return x + y, (x - y) * w


def causal_conv(x, h):
    """The definition: x [..., L], h [..., L] -> y[t] = sum_{k<=t} h[k] x[t-k] (float64)."""
    x = np.asarray(x, dtype=np.float64)
    h = np.asarray(h, dtype=np.float64)
    L = x.shape[-1]
    y = np.zeros(np.broadcast_shapes(x.shape, h.shape))
    for k in range(L):
        y[..., k:] += h[..., k:k + 1] * x[..., :L - k]
    return y


def dft_distributed(a, n: int):
    """An l-point DFT of a sequence held in n contiguous shards (rank r: a(m0 + c r), c = l/n),
    by one radix-n DiF stage across the ranks and a local c-point DFT on each: rank k2 ends
    with the frequencies n k1 + k2.  Returns spec [n, c] with spec[k2, k1] = A(n k1 + k2)."""
    a = np.asarray(a, dtype=np.complex128)
    l = a.shape[-1]
    c = l // n
    shards = a.reshape(n, c)                                   # shards[r, m] = a(m + c r)
    m = np.arange(c)
    spec = np.empty((n, c), dtype=np.complex128)
    for k2 in range(n):
        # cross-rank stage: N-point DFT across the shards at each local position, then the
        # twiddle w_l^(m k2)
        z = np.exp(-2j * np.pi * m * k2 / l) * sum(shards[r] * np.exp(-2j * np.pi * r * k2 / n) for r in range(n))
        spec[k2] = np.fft.fft(z)                                # local c-point DFT
    return spec


def spectra(x, n_cp: int):
    """Forward half of the convolution: the 2L-point spectrum of x zero-padded, as 2N local
    spectra: out[..., q, k1] = X~(2N k1 + q).  x [..., L], L = n_cp * c."""
    x = np.asarray(x, dtype=np.float64)
    L = x.shape[-1]
    N = n_cp
    c = L // N
    shards = x.reshape(x.shape[:-1] + (N, c))                  # [..., r, n]
    nn = np.arange(c)
    out = np.empty(x.shape[:-1] + (2 * N, c), dtype=np.complex128)
    for q in range(2 * N):
        # radix-2N DiF stage over the N data shards (the N zero shards add nothing)
        acc = sum(shards[..., r, :] * np.exp(-2j * np.pi * r * q / (2 * N)) for r in range(N))
        z = np.exp(-2j * np.pi * nn * q / (2 * L)) * acc
        out[..., q, :] = np.fft.fft(z, axis=-1)
    return out


def fft_conv_distributed(x, h, n_cp: int):
    """Causal convolution of x [..., L] with the long filter h [..., L] by the distributed
    radix-2N DiF FFT: spectra of x and h in the decimated layout, their product, the local
    inverse DFT with the mirrored twiddle, and the cross-rank inverse sum back into the
    contiguous shards.  Returns y [..., L] (float64)."""
    x = np.asarray(x, dtype=np.float64)
    L = x.shape[-1]
    N = n_cp
    c = L // N
    P = spectra(x, N) * spectra(h, N)                          # [..., 2N, c]
    nn = np.arange(c)
    w = np.empty_like(P)
    for q in range(2 * N):
        # local inverse DFT (unnormalised), then the conjugate twiddle w_2L^(-n q)
        w[..., q, :] = np.exp(2j * np.pi * nn * q / (2 * L)) * np.fft.ifft(P[..., q, :], axis=-1) * c
    y = np.empty(x.shape[:-1] + (N, c))
    for r in range(N):
        # cross-rank inverse: y(n + c r) = (1/2L) sum_q w_2N^(-r q) w_q(n)
        s = sum(w[..., q, :] * np.exp(2j * np.pi * r * q / (2 * N)) for q in range(2 * N))
        y[..., r, :] = (s / (2 * L)).real
    return y.reshape(x.shape)
