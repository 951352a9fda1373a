"""GPU parity of the Ulysses re-layout (bit-exact) and of the Ulysses and 2D forward flows."""
import numpy as np
import pytest
import torch

import oracle
from sequence_long_context_ring_b200 import synth
from sequence_long_context_ring_b200.binding import Plan, seq2head, head2seq
from sequence_long_context_ring_b200.configs import WORKLOADS

from _helpers import to_dev, to_f64, to_bits, inputs, assert_attn_close, sample_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,L,H,d,n", [(2, 64, 8, 128, 4), (1, 96, 6, 64, 3), (1, 8, 2, 128, 2)])
def test_seq2head_head2seq_bit_exact(cuda_lib, B, L, H, d, n):
    x = synth.tagged_u16((B, L, H, d)) ^ synth.normal_bf16(7, 0, (B, L, H, d))
    y = to_bits(seq2head(n, to_dev(x)))
    c = L // n
    ref = np.concatenate(oracle.seq2head([x[:, s * c:(s + 1) * c] for s in range(n)]), axis=1)
    np.testing.assert_array_equal(y, ref)
    back = to_bits(head2seq(n, to_dev(y)))
    np.testing.assert_array_equal(back, x)
    ref_back = np.concatenate(oracle.head2seq([y[:, r * (H // n):(r + 1) * (H // n)] for r in range(n)]), axis=1)
    np.testing.assert_array_equal(back, ref_back)


def test_seq2head_strided_views(cuda_lib):
    # a view with padded strides: in [B, L, H, d] taken from a larger buffer
    big = torch.from_numpy(synth.normal_bf16(8, 0, (1, 64, 10, 128)).view(np.int16)).cuda().view(torch.bfloat16)
    x = big[:, :, 1:9, :]
    y = seq2head(4, x)
    np.testing.assert_array_equal(to_bits(y), to_bits(x).transpose(0, 2, 1, 3))


def test_full_size_permute_c4(cuda_lib):
    w = WORKLOADS["c4"]
    x = synth.normal_bf16(w.cfg_id, 0, w.q_shape())
    dx = to_dev(x)
    y = seq2head(w.n_cp, dx)
    back = head2seq(w.n_cp, y)
    torch.cuda.synchronize()
    assert torch.equal(back.view(torch.int16), dx.view(torch.int16))
    # sampled rows against the index formula out[b, h, l, :] = in[b, l, h, :]
    rng = np.random.default_rng(4)
    for h, l in zip(rng.integers(0, w.Hq, 64), rng.integers(0, w.L, 64)):
        np.testing.assert_array_equal(to_bits(y[0, h, l]), x[0, l, h])


def test_ulysses_small_matches_oracle(cuda_lib):
    B, L, Hq, Hkv, d, n = 1, 512, 8, 4, 128, 4
    q, k, v = inputs(41, (B, L, Hq, d), (B, L, Hkv, d))
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n, mode="ulysses")
    o, lse = plan.fwd(to_dev(q), to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    assert plan.device_status()[0] == 0
    o_ref, l_ref = oracle.ulysses_attention(*(synth.bf16_bits_to_f64(x) for x in (q, k, v)), n)
    assert_attn_close(to_f64(o), o_ref, to_f64(lse), l_ref, "ulysses")


def test_2d_small_matches_oracle(cuda_lib):
    B, L, H, d = 1, 1024, 8, 64
    q, k, v = inputs(42, (B, L, H, d), (B, L, H, d))
    plan = Plan(B, H, H, L, d, n_cp=4, n_hp=2, mode="2d")
    o, lse = plan.fwd(to_dev(q), to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    assert plan.device_status()[0] == 0
    o_ref, l_ref = oracle.attention_2d(*(synth.bf16_bits_to_f64(x) for x in (q, k, v)), 2, 4)
    assert_attn_close(to_f64(o), o_ref, to_f64(lse), l_ref, "2d")


@pytest.mark.parametrize("name", ["c4", "c5"])
def test_full_size_seq_major_forward_sampled(cuda_lib, name):
    w = WORKLOADS[name]
    q, k, v = inputs(w.cfg_id, w.q_shape(), w.kv_shape(), w.input_scale)
    plan = Plan(w.B, w.Hq, w.Hkv, w.L, w.d, n_cp=w.n_cp, n_hp=w.n_hp, mode=w.mode)
    o, lse = plan.fwd(to_dev(q), to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    assert plan.device_status()[0] == 0
    assert bool(torch.isfinite(o.float()).all())
    np.testing.assert_array_equal(to_bits(o[:, 0]), v[:, 0])
    rows = sample_rows(w.L, w.n_cp * w.n_hp, 8, w.cfg_id)
    o_rows = to_f64(o[:, rows])      # [B, R, H, d]
    l_rows = to_f64(lse[:, :, rows])
    for h in range(0, w.Hq, 3):
        k64 = synth.bf16_bits_to_f64(k[0, :, h])
        v64 = synth.bf16_bits_to_f64(v[0, :, h])
        ro, rl = oracle.attention_rows(synth.bf16_bits_to_f64(q[0, rows, h]), k64, v64, rows, scale=plan.scale)
        assert_attn_close(o_rows[0, :, h], ro, l_rows[0, h], rl, f"{name} head {h}")
