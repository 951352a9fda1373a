"""GPU parity of the distributed FFT convolution ("05. 長系列の分散学習（Context Parallelism）" §4
FFT 畳み込み) through the C ABI, against the fp64 oracle.

Tolerance, from the arithmetic: the transforms run in fp32 with exact-argument twiddles, and the
error of an FFT convolution is bounded in norm, not per element, by a few log2(2L) u ||y|| (u =
2^-24): below 2^-9 RMS(y) per row for every size here even if one element took all of it; the
output's bf16 rounding adds at most 2^-8 |y|.  Each element must satisfy
|y - y_ref| <= 2^-8 |y_ref| + 2^-9 RMS_row(y_ref); impulse cases, where one bf16 value is
reproduced up to fp32 noise, are compared bit-exactly."""
import numpy as np
import pytest
import torch

from oracle import fftconv as ofc
from sequence_long_context_ring_b200 import synth
from sequence_long_context_ring_b200.binding import FftConvPlan, CpError
from sequence_long_context_ring_b200.configs import FFT_WORKLOADS

from _helpers import to_dev, to_f64, to_bits

pytestmark = pytest.mark.gpu


def _xh(seed, B, D, L):
    return (synth.normal_bf16(seed, synth.TENSOR_ID["x"], (B, D, L)),
            synth.normal_bf16(seed, synth.TENSOR_ID["h"], (D, L), L ** -0.5))


def _assert_close(got, ref, what):
    rms = np.sqrt(np.mean(ref ** 2, axis=-1, keepdims=True))
    tol = 2.0 ** -8 * np.abs(ref) + 2.0 ** -9 * rms
    err = np.abs(got - ref)
    bad = err > tol
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside the bound, worst "
                           f"{np.max(err - tol):.3e} at {np.unravel_index(np.argmax(err - tol), err.shape)}")
    assert np.linalg.norm(got - ref) <= 2.0 ** -7 * np.linalg.norm(ref), what


@pytest.mark.parametrize("B,D,L,n", [
    (1, 3, 4 * 16, 16),         # the smallest shard: c = 4
    (2, 3, 256, 8),
    (1, 2, 1024, 1),            # one rank: a plain 2L-point FFT convolution
    (1, 2, 2048, 2),            # two ranks: the page's butterfly across the shards
    (1, 2, 512 * 32, 32),       # the most ranks
    (1, 2, 8192 * 4, 4),        # the longest shard a CTA transforms: c = 8192
])
def test_fftconv_matches_the_oracle(cuda_lib, B, D, L, n):
    x, h = _xh(20 + n, B, D, L)
    plan = FftConvPlan(B, D, L, n)
    y = plan.fwd(to_dev(x), to_dev(h))
    torch.cuda.synchronize()
    x64, h64 = synth.bf16_bits_to_f64(x), synth.bf16_bits_to_f64(h)
    ref = ofc.causal_conv(x64, h64) if L <= 4096 else ofc.fft_conv_distributed(x64, h64, n)
    _assert_close(to_f64(y), ref, f"B{B} D{D} L{L} N{n}")


@pytest.mark.parametrize("t0", [0, 1, 511, 512, 3000])
def test_impulse_input_reproduces_the_filter_exactly(cuda_lib, t0):
    B, D, L, n = 1, 2, 4096, 8
    x = np.zeros((B, D, L), np.uint16)
    x[:, :, t0] = synth.f32_to_bf16_bits(np.float32([1.0]))[0]
    h = synth.normal_bf16(6, synth.TENSOR_ID["h"], (D, L), 0.05)
    y = to_bits(FftConvPlan(B, D, L, n).fwd(to_dev(x), to_dev(h)))
    expect = np.zeros_like(y)
    expect[:, :, t0:] = h[None, :, :L - t0]
    hv = np.abs(synth.bf16_bits_to_f64(expect))
    sure = hv > 1e-3                  # fp32 noise (~1e-7 here) cannot move these across an ulp boundary
    np.testing.assert_array_equal(y[sure], expect[sure])
    assert np.all(np.abs(synth.bf16_bits_to_f64(y[~sure])) <= 1.1e-3)


@pytest.mark.parametrize("k0", [0, 1, 255, 256, 4095])
def test_delta_filter_delays_the_input_exactly(cuda_lib, k0):
    B, D, L, n = 2, 2, 4096, 16
    x = synth.normal_bf16(7, synth.TENSOR_ID["x"], (B, D, L))
    h = np.zeros((D, L), np.uint16)
    h[:, k0] = synth.f32_to_bf16_bits(np.float32([1.0]))[0]
    y = to_bits(FftConvPlan(B, D, L, n).fwd(to_dev(x), to_dev(h)))
    expect = np.zeros_like(y)
    expect[:, :, k0:] = x[:, :, :L - k0]
    xv = np.abs(synth.bf16_bits_to_f64(expect))
    sure = xv > 1e-3
    np.testing.assert_array_equal(y[sure], expect[sure])
    assert np.all(np.abs(synth.bf16_bits_to_f64(y[~sure])) <= 1.1e-3)


def test_strided_views_and_argument_errors(cuda_lib):
    B, D, L, n = 2, 3, 1024, 4
    x, h = _xh(9, B, D, L)
    big = torch.zeros((B, D + 1, L + 6), dtype=torch.bfloat16, device="cuda")
    big[:, 1:, 3:3 + L] = to_dev(x)
    xv = big[:, 1:, 3:3 + L]
    y = torch.full((B, D, L + 2), 5.0, dtype=torch.bfloat16, device="cuda")
    plan = FftConvPlan(B, D, L, n)
    plan.fwd(xv, to_dev(h), y=y[:, :, :L])
    torch.cuda.synchronize()
    ref = ofc.causal_conv(synth.bf16_bits_to_f64(x), synth.bf16_bits_to_f64(h))
    _assert_close(to_f64(y[:, :, :L]), ref, "strided")
    assert torch.all(y[:, :, L:] == 5.0)
    small = torch.empty(plan.workspace_size() - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(CpError):
        plan.fwd(xv, to_dev(h), y=y[:, :, :L], ws=small)
    with pytest.raises(CpError):
        plan.fwd(xv, to_dev(h)[:, :L - 1], y=y[:, :, :L])


def test_full_size_workload_sampled_rows(cuda_lib):
    # the bench's launch at full size; 16 whole rows compared against the oracle
    w = FFT_WORKLOADS["fft_long"]
    x = synth.normal_bf16(w.cfg_id, synth.TENSOR_ID["x"], w.x_shape())
    h = synth.normal_bf16(w.cfg_id, synth.TENSOR_ID["h"], w.h_shape(), w.h_scale)
    plan = FftConvPlan(w.B, w.D, w.L, w.n_cp)
    ty = plan.fwd(to_dev(x), to_dev(h))
    torch.cuda.synchronize()
    rows = np.random.default_rng(42).choice(w.D, 16, replace=False)
    got = to_f64(ty[0][torch.as_tensor(rows, device="cuda")])
    ref = ofc.fft_conv_distributed(synth.bf16_bits_to_f64(x[0, rows]), synth.bf16_bits_to_f64(h[rows]), w.n_cp)
    _assert_close(got, ref, "full size")
