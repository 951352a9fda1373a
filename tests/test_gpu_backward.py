"""GPU parity of the backward (cp_attn_bwd) against the fp64 oracle, through the C ABI.

Reference: the oracle's gradient given the forward's stored output (its own O rounded to bf16,
which is what cp_attn_bwd receives), so D = rowsum(dO * O_stored) on both sides.
Tolerance (the pages fix none for gradients; derived from the arithmetic): the kernel rounds
P and dS to bf16 (relative error <= 2^-9 each) before the tensor-core products, accumulates in
fp32, and rounds each gradient to bf16 once (<= 2^-9).  Three such roundings stay below
2^-7 of the tensor's own scale, so: max-abs <= 2^-7 * max|ref| and mean-abs <= 2^-7 *
mean|ref| for each gradient tensor (or sampled block of it).
"""
import numpy as np
import pytest
import torch

import oracle
from sequence_long_context_ring_b200 import synth
from sequence_long_context_ring_b200.binding import Plan
from sequence_long_context_ring_b200.configs import WORKLOADS

from _helpers import to_dev, to_f64, inputs, sample_rows

pytestmark = pytest.mark.gpu

BWD_REL = 2.0 ** -7


def stored(o64):
    """The oracle's own forward output as the forward stores it: rounded to bf16 (nearest even)."""
    return synth.bf16_bits_to_f64(synth.f32_to_bf16_bits(np.asarray(o64, np.float32)))


def assert_grad_close(g, ref, what):
    g = np.asarray(g, np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite"
    err = np.abs(g - ref)
    scale_max, scale_mean = np.abs(ref).max(), np.abs(ref).mean()
    assert err.max() <= BWD_REL * scale_max, f"{what}: max-abs {err.max():.3e} vs max|ref| {scale_max:.3e}"
    assert err.mean() <= BWD_REL * scale_mean, f"{what}: mean-abs {err.mean():.3e} vs mean|ref| {scale_mean:.3e}"
    return err.max() / scale_max, err.mean() / scale_mean


@pytest.mark.parametrize("B,Hq,Hkv,L,d,n,causal", [
    (1, 4, 4, 512, 64, 4, True),      # MHA, d = 64
    (1, 4, 2, 640, 128, 2, True),     # GQA G=2, ragged chunk of 320
    (2, 8, 2, 1024, 128, 4, True),    # GQA G=4, B=2
    (1, 2, 1, 390, 128, 3, True),     # ragged chunks of 130
    (1, 4, 4, 768, 128, 3, False),    # non-causal
])
def test_ring_backward_matches_oracle(cuda_lib, B, Hq, Hkv, L, d, n, causal):
    q, k, v, do = inputs(500 + L, (B, Hq, L, d), (B, Hkv, L, d), with_do=True)
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n, causal=causal)
    dq_, dk_, dv_, ddo = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    o, lse = plan.fwd(dq_, dk_, dv_)
    gq, gk, gv = plan.bwd(dq_, dk_, dv_, o, lse, ddo)
    torch.cuda.synchronize()
    assert plan.device_status()[0] == 0
    q64, k64, v64, do64 = (synth.bf16_bits_to_f64(x) for x in (q, k, v, do))
    o_ref, _ = oracle.attention_full(q64, k64, v64, causal=causal)
    # the backward is given the forward's stored output, i.e. O rounded to bf16
    rq, rk, rv = oracle.attention_backward(q64, k64, v64, do64, causal=causal, o=stored(o_ref))
    assert_grad_close(to_f64(gq), rq, "dq")
    assert_grad_close(to_f64(gk), rk, "dk")
    assert_grad_close(to_f64(gv), rv, "dv")


def test_backward_identities_and_zero_grad(cuda_lib):
    # sum over keys of dV = sum over the group's queries of dO; sum over keys of dK = 0
    B, Hq, Hkv, L, d, n = 1, 4, 2, 1024, 128, 4
    q, k, v, do = inputs(601, (B, Hq, L, d), (B, Hkv, L, d), with_do=True)
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n)
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    o, lse = plan.fwd(tq, tk, tv)
    gq, gk, gv = plan.bwd(tq, tk, tv, o, lse, to_dev(do))
    zq, zk, zv = plan.bwd(tq, tk, tv, o, lse, torch.zeros_like(o))
    torch.cuda.synchronize()
    do64 = synth.bf16_bits_to_f64(do)
    gv64, gk64 = to_f64(gv), to_f64(gk)
    for g in range(Hkv):
        lhs = gv64[0, g].sum(axis=0)
        rhs = do64[0, 2 * g:2 * g + 2].sum(axis=(0, 1))
        assert np.abs(lhs - rhs).max() <= 0.02 * np.abs(rhs).max() + 0.5
        assert np.abs(gk64[0, g].sum(axis=0)).max() <= 0.02 * np.abs(gk64[0, g]).sum(axis=0).max() + 0.05
    for z in (zq, zk, zv):
        assert not bool(z.float().abs().max() > 0)


def test_ulysses_and_2d_backward_small(cuda_lib):
    B, L, H, d = 1, 512, 8, 64
    q, k, v, do = inputs(602, (B, L, H, d), (B, L, H, d), with_do=True)
    q64, k64, v64, do64 = (synth.bf16_bits_to_f64(x).transpose(0, 2, 1, 3) for x in (q, k, v, do))
    o_ref, _ = oracle.attention_full(q64, k64, v64)
    rq, rk, rv = oracle.attention_backward(q64, k64, v64, do64, o=stored(o_ref))
    for mode, n_cp, n_hp in (("ulysses", 4, 1), ("2d", 2, 2)):
        plan = Plan(B, H, H, L, d, n_cp=n_cp, n_hp=n_hp, mode=mode)
        tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
        o, lse = plan.fwd(tq, tk, tv)
        gq, gk, gv = plan.bwd(tq, tk, tv, o, lse, to_dev(do))
        torch.cuda.synchronize()
        assert plan.device_status()[0] == 0
        assert_grad_close(to_f64(gq).transpose(0, 2, 1, 3), rq, f"{mode} dq")
        assert_grad_close(to_f64(gk).transpose(0, 2, 1, 3), rk, f"{mode} dk")
        assert_grad_close(to_f64(gv).transpose(0, 2, 1, 3), rv, f"{mode} dv")


def test_c5_full_size_backward_sampled(cuda_lib):
    # 2D 4x4 grid, 7B-MHA, L = 65536: dQ on sampled rows (exact per row), dK/dV on the last
    # 128 keys (only the last queries see them), plus the sum identities over all keys.
    w = WORKLOADS["c5"]
    q, k, v, do = inputs(w.cfg_id, w.q_shape(), w.kv_shape(), with_do=True)
    plan = Plan(w.B, w.Hq, w.Hkv, w.L, w.d, n_cp=w.n_cp, n_hp=w.n_hp, mode=w.mode)
    tq, tk, tv, tdo = to_dev(q), to_dev(k), to_dev(v), to_dev(do)
    o, lse = plan.fwd(tq, tk, tv)
    gq, gk, gv = plan.bwd(tq, tk, tv, o, lse, tdo)
    torch.cuda.synchronize()
    assert plan.device_status()[0] == 0
    for t in (gq, gk, gv):
        assert bool(torch.isfinite(t.float()).all())
    rows = sample_rows(w.L, w.n_cp * w.n_hp, 4, 5)
    tail = np.arange(w.L - 128, w.L)
    for h in range(0, w.Hq, 8):
        k64 = synth.bf16_bits_to_f64(k[0, :, h])
        v64 = synth.bf16_bits_to_f64(v[0, :, h])
        q_r = synth.bf16_bits_to_f64(q[0, rows, h])
        do_r = synth.bf16_bits_to_f64(do[0, rows, h])
        o_r, l_r = oracle.attention_rows(q_r, k64, v64, rows)
        ref_dq = oracle.backward_rows_dq(q_r, k64, v64, do_r, stored(o_r), l_r, rows)
        assert_grad_close(to_f64(gq[0, rows, h]), ref_dq, f"c5 dq head {h}")
        q_t = synth.bf16_bits_to_f64(q[0, tail, h])
        do_t = synth.bf16_bits_to_f64(do[0, tail, h])
        o_t, l_t = oracle.attention_rows(q_t, k64, v64, tail)
        ref_dk, ref_dv = oracle.backward_rows_dkdv(q_t[None], k64, v64, do_t[None], stored(o_t)[None], l_t[None], tail,
                                                   q_lo=int(tail[0]))
        assert_grad_close(to_f64(gk[0, tail, h]), ref_dk, f"c5 dk head {h}")
        assert_grad_close(to_f64(gv[0, tail, h]), ref_dv, f"c5 dv head {h}")
    # identities over the whole sequence (per head, MHA)
    sdv = gv.float().sum(dim=1)
    sdo = tdo.float().sum(dim=1)
    assert float((sdv - sdo).abs().max()) <= 0.02 * float(sdo.abs().max()) + 1.0
    sdk = gk.float().sum(dim=1)
    assert float(sdk.abs().max()) <= 0.02 * float(gk.float().abs().sum(dim=1).max()) + 0.1
