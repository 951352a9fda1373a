"""GPU parity of the fused forward (cp_attn_fwd, ring mode) and the step-wise path
(cp_ring_step + cp_lse_merge) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from sequence_long_context_ring_b200 import synth
from sequence_long_context_ring_b200.binding import Plan, lse_merge, CP_ERR_TIMEOUT
from sequence_long_context_ring_b200.configs import WORKLOADS

from _helpers import to_dev, to_f64, to_bits, inputs, assert_attn_close, sample_rows

pytestmark = pytest.mark.gpu


def _run_ring(B, Hq, Hkv, L, d, n, causal=True, cfg_id=100, scale=0.0, in_scale=1.0):
    q, k, v = inputs(cfg_id, (B, Hq, L, d), (B, Hkv, L, d), in_scale)
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n, causal=causal, scale=scale)
    o, lse = plan.fwd(to_dev(q), to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    assert plan.device_status()[0] == 0
    return plan, (q, k, v), o, lse


def test_c1_tiny_ring_matches_oracle(cuda_lib):
    w = WORKLOADS["c1"]
    plan, (q, k, v), o, lse = _run_ring(w.B, w.Hq, w.Hkv, w.L, w.d, w.n_cp, cfg_id=w.cfg_id)
    o_ref, l_ref = oracle.attention_full(*(synth.bf16_bits_to_f64(x) for x in (q, k, v)), causal=True)
    assert_attn_close(to_f64(o), o_ref, to_f64(lse), l_ref, "c1")
    # causal row 0 sees only key 0: O_0 = V_0 bit for bit
    np.testing.assert_array_equal(to_bits(o)[:, :, 0], v[:, :, 0])


@pytest.mark.parametrize("B,Hq,Hkv,L,d,n,causal", [
    (2, 4, 2, 640, 128, 2, True),     # GQA G=2, chunk 320 = 2.5 tiles (ragged tail)
    (1, 3, 1, 384, 64, 3, True),      # odd G=3 -> consecutive-tile pairing
    (1, 2, 2, 200, 128, 1, True),     # single ragged chunk shorter than two tiles
    (1, 8, 2, 1536, 128, 4, False),   # non-causal, G=4
    (1, 4, 4, 1000, 64, 5, True),     # MHA, chunk 200 (ragged), 5 ranks
    (1, 2, 1, 130, 64, 2, True),      # chunks of 65: one KV tile spans two chunks
    (1, 2, 2, 1, 64, 1, True),        # L = 1
    (1, 8, 8, 2048, 128, 8, True),    # MHA, many tiles per rank
])
def test_ring_forward_shapes(cuda_lib, B, Hq, Hkv, L, d, n, causal):
    plan, (q, k, v), o, lse = _run_ring(B, Hq, Hkv, L, d, n, causal, cfg_id=1000 + L + n)
    o_ref, l_ref = oracle.attention_full(*(synth.bf16_bits_to_f64(x) for x in (q, k, v)), causal=causal)
    assert_attn_close(to_f64(o), o_ref, to_f64(lse), l_ref, f"{(B, Hq, Hkv, L, d, n, causal)}")


def test_custom_scale(cuda_lib):
    plan, (q, k, v), o, lse = _run_ring(1, 4, 2, 512, 128, 2, scale=0.05, cfg_id=77)
    o_ref, l_ref = oracle.attention_full(*(synth.bf16_bits_to_f64(x) for x in (q, k, v)), causal=True, scale=0.05)
    assert_attn_close(to_f64(o), o_ref, to_f64(lse), l_ref, "scale")


@pytest.mark.parametrize("B,Hq,Hkv,L,d,n", [(1, 4, 4, 1024, 64, 4), (1, 4, 2, 1000, 128, 4), (1, 2, 1, 390, 64, 3)])
def test_stepwise_ring_any_order_matches_fused_and_oracle(cuda_lib, B, Hq, Hkv, L, d, n):
    # Each rank visits its KV chunks in a random order; the merged partials equal the fused
    # result and full attention (order invariance, on the GPU).
    q, k, v = inputs(300 + L, (B, Hq, L, d), (B, Hkv, L, d))
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    o_fused, lse_fused = plan.fwd(dq, dk, dv)
    c = L // n
    rng = np.random.default_rng(L)
    o_all = torch.empty((B, Hq, L, d), dtype=torch.float32, device="cuda")
    l_all = torch.empty((B, Hq, L), dtype=torch.float32, device="cuda")
    for r in range(n):
        acc_o = o_all[:, :, r * c:(r + 1) * c]
        acc_l = l_all[:, :, r * c:(r + 1) * c]
        acc_o.zero_()
        acc_l.fill_(-float("inf"))
        for s in rng.permutation(n):
            po, pl = plan.ring_step(r, int(s), dq, dk, dv)
            lse_merge(acc_o, acc_l, po, pl)
    torch.cuda.synchronize()
    assert plan.device_status()[0] == 0
    o_ref, l_ref = oracle.attention_full(*(synth.bf16_bits_to_f64(x) for x in (q, k, v)))
    assert_attn_close(to_f64(o_all), o_ref, to_f64(l_all), l_ref, "stepwise vs oracle")
    assert_attn_close(to_f64(o_all), to_f64(o_fused), to_f64(l_all), to_f64(lse_fused), "stepwise vs fused")


def test_ring_step_partial_matches_oracle_chunk_partial(cuda_lib):
    B, Hq, Hkv, L, d, n = 1, 2, 1, 768, 128, 3
    q, k, v = inputs(55, (B, Hq, L, d), (B, Hkv, L, d))
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n)
    c = L // n
    q64, k64, v64 = (synth.bf16_bits_to_f64(x) for x in (q, k, v))
    for r in range(n):
        for s in range(n):
            j = (r - s) % n
            po, pl = plan.ring_step(r, s, to_dev(q), to_dev(k), to_dev(v))
            torch.cuda.synchronize()
            for h in range(Hq):
                ro, rl = oracle.chunk_partial(q64[0, h, r * c:(r + 1) * c], k64[0, h // 2, j * c:(j + 1) * c],
                                              v64[0, h // 2, j * c:(j + 1) * c], r * c, j * c)
                go, gl = to_f64(po)[0, h], to_f64(pl)[0, h]
                if j > r:
                    assert np.all(go == 0) and np.all(np.isneginf(gl))
                else:
                    assert_attn_close(go, ro, gl, rl, f"partial r={r} j={j}")


def _sampled_check(plan, w, q, k, v, o, lse, n_random=16):
    rows = sample_rows(w.L, w.n_cp, n_random, w.cfg_id)
    o_rows = to_f64(o[:, :, rows])
    l_rows = to_f64(lse[:, :, rows])
    G = w.Hq // w.Hkv
    errs = []
    for g in range(w.Hkv):
        k64 = synth.bf16_bits_to_f64(k[0, g])
        v64 = synth.bf16_bits_to_f64(v[0, g])
        for h in range(g * G, (g + 1) * G):
            ro, rl = oracle.attention_rows(synth.bf16_bits_to_f64(q[0, h, rows]), k64, v64, rows, causal=True,
                                           scale=plan.scale)
            errs.append(assert_attn_close(o_rows[0, h], ro, l_rows[0, h], rl, f"{w.name} head {h}"))
    return errs


@pytest.mark.parametrize("name", ["c2", "c3"])
def test_full_size_gqa_sampled_rows(cuda_lib, name):
    w = WORKLOADS[name]
    q, k, v = inputs(w.cfg_id, w.q_shape(), w.kv_shape(), w.input_scale)
    plan = Plan(w.B, w.Hq, w.Hkv, w.L, w.d, n_cp=w.n_cp)
    o, lse = plan.fwd(to_dev(q), to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    assert plan.device_status()[0] == 0
    assert bool(torch.isfinite(o.float()).all()) and bool(torch.isfinite(lse).all())
    np.testing.assert_array_equal(to_bits(o[:, :, 0]), v[:, np.arange(w.Hq) // (w.Hq // w.Hkv), 0])
    _sampled_check(plan, w, q, k, v, o, lse)


def test_timeout_path_reports_error_and_context_survives(cuda_lib):
    # The load warp skips the query-tile load (host flag), so every consumer's bounded wait
    # expires; the kernel must end with CP_ERR_TIMEOUT in the status word, without a fault.
    B, Hq, Hkv, L, d, n = 1, 2, 2, 512, 128, 2
    q, k, v = inputs(9, (B, Hq, L, d), (B, Hkv, L, d))
    bad = Plan(B, Hq, Hkv, L, d, n_cp=n, wait_limit_ns=20_000_000, debug_fault=1)
    bad.fwd(to_dev(q), to_dev(k), to_dev(v))
    st, word = bad.device_status()
    assert st == CP_ERR_TIMEOUT and (word & 0xFF) == 6 and (word >> 8) > 0
    # the context is still usable and a correct plan still gives the right answer
    good = Plan(B, Hq, Hkv, L, d, n_cp=n)
    o, lse = good.fwd(to_dev(q), to_dev(k), to_dev(v))
    torch.cuda.synchronize()
    assert good.device_status()[0] == 0
    o_ref, l_ref = oracle.attention_full(*(synth.bf16_bits_to_f64(x) for x in (q, k, v)))
    assert_attn_close(to_f64(o), o_ref, to_f64(lse), l_ref, "after timeout")
