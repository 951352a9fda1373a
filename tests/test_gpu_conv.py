"""GPU parity of the point-to-point FIR convolution ("05. 長系列の分散学習（Context Parallelism）"
§3 Hyena 演算子をどう分散するか, p2p 畳み込み) through the C ABI, against the fp64 oracle.

Tolerance, from the arithmetic: products of two bf16 values are exact in fp32; the fp32
accumulation of at most 2 x 128 terms errs by at most 256 * 2^-24 = 2^-16 of sum |h||x|; the
bf16 rounding of the output by at most half an ulp, 2^-8 of |y|.  The test allows
2^-8 |y| + 2^-14 sum_k |h_k| |x_{t-k}| per element (4x margin on the accumulation term)."""
import numpy as np
import pytest
import torch

from oracle import conv as oconv
from sequence_long_context_ring_b200 import synth
from sequence_long_context_ring_b200.binding import ConvPlan, CpError
from sequence_long_context_ring_b200.configs import CONV_WORKLOADS

from _helpers import to_dev, to_f64, to_bits

pytestmark = pytest.mark.gpu


def _xh(seed, B, D, L, lh):
    x = synth.normal_bf16(seed, synth.TENSOR_ID["x"], (B, D, L))
    h = synth.normal_bf16(seed, synth.TENSOR_ID["h"], (D, lh), lh ** -0.5)
    return x, h


def _assert_conv_close(got, ref, abs_ref, what):
    tol = 2.0 ** -8 * np.abs(ref) + 2.0 ** -14 * abs_ref
    err = np.abs(got - ref)
    bad = err > tol
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside the bound, worst "
                           f"{np.max(err - tol):.3e} at {np.unravel_index(np.argmax(err - tol), err.shape)}")


def _ref(x, h):
    x64, h64 = synth.bf16_bits_to_f64(x), synth.bf16_bits_to_f64(h)
    return oconv.fir_conv(x64, h64), oconv.fir_conv(np.abs(x64), np.abs(h64))


@pytest.mark.parametrize("B,D,L,lh,n", [
    (1, 3, 128 * 133 + 56, 7, 4),      # 2 tiles per row (the second ragged) + a 56-sample tail
    (2, 5, 128 * 133 + 56, 128, 2),    # medium filter, two previous-block boxes
    (1, 4, 128 * 130, 65, 8),          # the longest filter served by one previous-block box
    (1, 4, 128 * 130, 66, 8),          # the shortest that needs both
    (1, 2, 128 * 40, 129, 40),         # the longest filter: halo = a whole shard of 128
    (2, 80, 128 * 129, 33, 3),         # 320 tiles on 148 CTAs: channel changes inside a CTA
    (1, 70, 128 * 300, 128, 4),        # 210 tiles: CTA ranges that start inside a row
    (1, 3, 104, 9, 2),                 # shorter than one block: the direct kernel alone
    (3, 2, 1024, 1, 4),                # one tap: no halo
])
def test_fir_fwd_matches_the_oracle(cuda_lib, B, D, L, lh, n):
    x, h = _xh(11 + lh, B, D, L, lh)
    plan = ConvPlan(B, D, L, lh, n)
    y = plan.fwd(to_dev(x), to_dev(h))
    torch.cuda.synchronize()
    assert plan.device_status()[0] == 0
    ref, abs_ref = _ref(x, h)
    _assert_conv_close(to_f64(y), ref, abs_ref, f"fwd B{B} D{D} L{L} lh{lh}")


def test_one_tap_is_a_bit_exact_scaling(cuda_lib):
    # h0 * x is exact in fp32; both sides round the same real number to bf16 (nearest even)
    B, D, L = 2, 6, 128 * 9 + 8
    x, h = _xh(3, B, D, L, 1)
    y = ConvPlan(B, D, L, 1, 1).fwd(to_dev(x), to_dev(h))
    ref = oconv.fir_conv(synth.bf16_bits_to_f64(x), synth.bf16_bits_to_f64(h))
    expect = synth.f32_to_bf16_bits(ref.astype(np.float32))    # exact in fp32, so one rounding
    np.testing.assert_array_equal(to_bits(y), expect)


def test_impulse_reads_out_every_tap_at_every_offset(cuda_lib):
    # x = impulses at offsets that straddle block and tile boundaries: y = h shifted, exactly
    B, D, L, lh = 1, 3, 128 * 260, 129
    x = np.zeros((B, D, L), np.uint16)
    starts = [0, 1, 127, 128, 255, 128 * 128 - 1, 128 * 128, 128 * 200 + 77]
    for s in starts:
        x[:, :, s] = synth.f32_to_bf16_bits(np.float32([1.0]))[0]
    h = synth.normal_bf16(4, synth.TENSOR_ID["h"], (D, lh), 0.1)
    y = to_bits(ConvPlan(B, D, L, lh, 1).fwd(to_dev(x), to_dev(h)))
    ref = oconv.fir_conv(synth.bf16_bits_to_f64(x), synth.bf16_bits_to_f64(h))
    # impulses sit >= lh apart except the first few: compare against the oracle, bit-exact where
    # a single tap lands on the output (sums of several taps round once, like the oracle)
    expect = synth.f32_to_bf16_bits(ref.astype(np.float32))
    single = np.ones(L, bool)
    for a in starts:
        for b in starts:
            if a < b < a + lh:
                single[b:a + lh] = False
    np.testing.assert_array_equal(y[:, :, single], expect[:, :, single])


@pytest.mark.parametrize("B,D,c,lh,n", [
    (1, 3, 128 * 3 + 40, 7, 3),
    (2, 4, 128 * 2, 128, 4),
    (1, 2, 128, 129, 3),        # halo = the whole previous shard; all outputs take the halo path
    (1, 2, 96, 20, 3),          # shard shorter than a block
])
def test_fir_shard_with_a_received_halo(cuda_lib, B, D, c, lh, n):
    L = c * n
    x, h = _xh(40 + lh, B, D, L, lh)
    plan = ConvPlan(B, D, L, lh, n)
    tx, th = to_dev(x), to_dev(h)
    x64, h64 = synth.bf16_bits_to_f64(x), synth.bf16_bits_to_f64(h)
    for r in range(n):
        shard = tx[:, :, r * c:(r + 1) * c]                       # a strided view of x
        halo = tx[:, :, r * c - (lh - 1):r * c].clone() if r > 0 and lh > 1 else None
        y = plan.shard(r, shard, halo, th)
        torch.cuda.synchronize()
        h_ref = x64[:, :, r * c - (lh - 1):r * c] if r > 0 and lh > 1 else None
        ref = oconv.fir_conv_shard(x64[:, :, r * c:(r + 1) * c], h_ref, h64)
        habs = np.abs(h_ref) if h_ref is not None else None
        abs_ref = oconv.fir_conv_shard(np.abs(x64[:, :, r * c:(r + 1) * c]), habs, np.abs(h64))
        _assert_conv_close(to_f64(y), ref, abs_ref, f"shard r{r} lh{lh}")
    assert plan.device_status()[0] == 0


def test_shards_together_equal_the_whole_sequence(cuda_lib):
    B, D, L, lh, n = 1, 4, 128 * 64, 100, 8
    x, h = _xh(77, B, D, L, lh)
    plan = ConvPlan(B, D, L, lh, n)
    tx, th = to_dev(x), to_dev(h)
    c = L // n
    parts = [plan.shard(r, tx[:, :, r * c:(r + 1) * c], tx[:, :, r * c - lh + 1:r * c] if r else None, th)
             for r in range(n)]
    whole = plan.fwd(tx, th)
    torch.cuda.synchronize()
    ref, abs_ref = _ref(x, h)
    _assert_conv_close(to_f64(torch.cat(parts, dim=2)), ref, abs_ref, "shards")
    _assert_conv_close(to_f64(whole), ref, abs_ref, "whole")
    # outside each shard's first l_h - 1 samples the two paths run the same tensor-core tiles
    got_p, got_w = to_bits(torch.cat(parts, dim=2)), to_bits(whole)
    for r in range(n):
        lo = r * c + (lh - 1 if r else 0)
        np.testing.assert_array_equal(got_p[:, :, lo:(r + 1) * c], got_w[:, :, lo:(r + 1) * c])


def test_strided_views_and_argument_errors(cuda_lib):
    B, D, L, lh = 2, 3, 128 * 5, 17
    x, h = _xh(8, B, D, L, lh)
    big = torch.zeros((B, D + 2, L + 64), dtype=torch.bfloat16, device="cuda")
    big[:, 1:D + 1, 32:32 + L] = to_dev(x)
    xv = big[:, 1:D + 1, 32:32 + L]                    # strides (D+2)(L+64), L+64, 1
    hbig = torch.zeros((D, 40), dtype=torch.bfloat16, device="cuda")
    hbig[:, :lh] = to_dev(h)
    ybig = torch.full((B, D, L + 8), 7.0, dtype=torch.bfloat16, device="cuda")
    plan = ConvPlan(B, D, L, lh, 5)
    plan.fwd(xv, hbig[:, :lh], y=ybig[:, :, :L])
    torch.cuda.synchronize()
    ref, abs_ref = _ref(x, h)
    _assert_conv_close(to_f64(ybig[:, :, :L]), ref, abs_ref, "strided")
    assert torch.all(ybig[:, :, L:] == 7.0)            # nothing written past the view
    with pytest.raises(CpError):
        plan.fwd(xv, hbig[:, :lh - 1], y=ybig[:, :, :L])        # wrong filter length
    with pytest.raises(CpError):
        plan.fwd(big[:, 1:D + 1, 33:33 + L], hbig[:, :lh], y=ybig[:, :, :L])   # unaligned base
    with pytest.raises(CpError):
        plan.shard(0, xv[:, :, :128], xv[:, :, :lh - 1], hbig[:, :lh])          # rank 0 takes no halo
    with pytest.raises(CpError):
        plan.shard(1, xv[:, :, 128:256], None, hbig[:, :lh])                    # rank 1 needs one


@pytest.mark.parametrize("key", ["fir_short", "fir_medium"])
def test_full_size_workload_sampled(cuda_lib, key):
    # the bench's launch at full size; outputs sampled at every shard boundary (the halo
    # region), tile boundaries and seeded-random positions, each computed from the definition
    w = CONV_WORKLOADS[key]
    x = synth.normal_bf16(w.cfg_id, synth.TENSOR_ID["x"], w.x_shape())
    h = synth.normal_bf16(w.cfg_id, synth.TENSOR_ID["h"], w.h_shape(), w.h_scale)
    plan = ConvPlan(w.B, w.D, w.L, w.lh, w.n_cp)
    ty = plan.fwd(to_dev(x), to_dev(h))
    torch.cuda.synchronize()
    assert plan.device_status()[0] == 0
    c = w.L // w.n_cp
    rng = np.random.default_rng(99)
    ts = set()
    for r in range(w.n_cp):
        ts.update(range(max(r * c - 1, 0), r * c + w.lh + 1))
    ts.update(t for t in (16383, 16384, 16385, w.L - 1) if t < w.L)
    ts.update(rng.integers(0, w.L, 200).tolist())
    ts = np.array(sorted(ts))
    rows = rng.choice(w.D, 24, replace=False)
    got = to_f64(ty[0][torch.as_tensor(rows, device="cuda")][:, torch.as_tensor(ts, device="cuda")])
    h64 = synth.bf16_bits_to_f64(h)
    for a, ch in enumerate(rows):
        xr = synth.bf16_bits_to_f64(x[0, ch])
        for b, t in enumerate(ts):
            k = np.arange(min(w.lh, t + 1))
            terms = h64[ch, k] * xr[t - k]
            ref, abs_ref = terms.sum(), np.abs(terms).sum()
            assert abs(got[a, b] - ref) <= 2.0 ** -8 * abs(ref) + 2.0 ** -14 * abs_ref, (ch, t, got[a, b], ref)
