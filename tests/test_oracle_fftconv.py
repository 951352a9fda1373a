"""Pins of the oracle's distributed FFT convolution ("05. 長系列の分散学習（Context Parallelism）"
§4 FFT 畳み込み): the DFT definition against numpy's FFT, the page's DiF butterfly as the
two-rank stage, the decimated-frequency layout of every rank's spectrum, and the whole
convolution against the causal-convolution definition and a library FFT convolution."""
import numpy as np
import pytest

from oracle import conv, fftconv


def test_dft_definition_matches_the_library_fft():
    rng = np.random.default_rng(1)
    a = rng.standard_normal(12) + 1j * rng.standard_normal(12)
    np.testing.assert_allclose(fftconv.dft(a), np.fft.fft(a), atol=1e-12)
    np.testing.assert_allclose(fftconv.dft(a, inverse=True), np.fft.ifft(a) * 12, atol=1e-12)


def test_two_rank_stage_is_the_pages_butterfly():
    # with N = 2 the cross-rank stage at local position m is X = x + y, Y = (x - y) w_l^m
    rng = np.random.default_rng(2)
    l = 16
    a = rng.standard_normal(l)
    spec = fftconv.dft_distributed(a, 2)
    m = np.arange(l // 2)
    X, Y = fftconv.dif_butterfly(a[:l // 2], a[l // 2:], np.exp(-2j * np.pi * m / l))
    np.testing.assert_allclose(spec[0], np.fft.fft(X), atol=1e-12)
    np.testing.assert_allclose(spec[1], np.fft.fft(Y), atol=1e-12)
    # and rank k2 holds the frequencies 2 k1 + k2 of the whole sequence (decimation in frequency)
    full = fftconv.dft(a)
    np.testing.assert_allclose(spec[0], full[0::2], atol=1e-11)
    np.testing.assert_allclose(spec[1], full[1::2], atol=1e-11)


@pytest.mark.parametrize("l,n", [(8, 1), (12, 3), (16, 4), (24, 8), (30, 5)])
def test_every_rank_holds_its_decimated_frequencies(l, n):
    rng = np.random.default_rng(l + n)
    a = rng.standard_normal(l) + 1j * rng.standard_normal(l)
    spec = fftconv.dft_distributed(a, n)
    full = fftconv.dft(a)
    for k2 in range(n):
        np.testing.assert_allclose(spec[k2], full[k2::n], atol=1e-10)


@pytest.mark.parametrize("L,n", [(8, 2), (12, 3), (16, 4)])
def test_padded_spectra_are_the_2L_point_dft_in_decimated_order(L, n):
    rng = np.random.default_rng(7)
    x = rng.standard_normal(L)
    s = fftconv.spectra(x, n)
    full = fftconv.dft(np.concatenate([x, np.zeros(L)]))
    for q in range(2 * n):
        np.testing.assert_allclose(s[q], full[q::2 * n], atol=1e-10)


@pytest.mark.parametrize("L,n", [(1, 1), (8, 1), (8, 2), (12, 3), (32, 4), (48, 8), (40, 5)])
def test_distributed_fft_convolution_equals_the_definition(L, n):
    rng = np.random.default_rng(L * 10 + n)
    x = rng.standard_normal((2, 3, L))
    h = rng.standard_normal((3, L))
    y = fftconv.fft_conv_distributed(x, h, n)
    np.testing.assert_allclose(y, fftconv.causal_conv(x, h), atol=1e-10)
    # the same definition as the FIR oracle with l_h = L
    np.testing.assert_allclose(y, conv.fir_conv(x, h), atol=1e-10)


def test_distributed_fft_convolution_matches_a_library_fft_convolution():
    rng = np.random.default_rng(3)
    L, n = 256, 8
    x = rng.standard_normal(L)
    h = rng.standard_normal(L)
    lib = np.fft.irfft(np.fft.rfft(x, 2 * L) * np.fft.rfft(h, 2 * L), 2 * L)[:L]
    np.testing.assert_allclose(fftconv.fft_conv_distributed(x, h, n), lib, atol=1e-10)


def test_impulses_give_exact_shifts():
    # x = delta(t0) reads out h from t0 on; h = delta(k) delays x by k (to rounding)
    L, n = 64, 4
    rng = np.random.default_rng(5)
    h = rng.standard_normal(L)
    x = np.zeros(L)
    x[9] = 1.0
    y = fftconv.fft_conv_distributed(x, h, n)
    np.testing.assert_allclose(y, np.concatenate([np.zeros(9), h[:L - 9]]), atol=1e-12)
    d = np.zeros(L)
    d[5] = 1.0
    xs = rng.standard_normal(L)
    np.testing.assert_allclose(fftconv.fft_conv_distributed(xs, d, n),
                               np.concatenate([np.zeros(5), xs[:L - 5]]), atol=1e-12)
