"""Stand-ins for the memory and race checkers, which are closed on this pool.

Poisoned buffers: every workspace and output is filled with 0xFF bytes (NaN in bf16 and fp32)
before a call, and the result must equal, bit for bit, the same call on zero-filled buffers.  A
kernel that read a byte it had not written first -- a workspace word left from nothing, an
output element assumed zero -- would carry the NaN or the difference into the result.

Bounded waits: a host flag makes one producer leave out a load (or, in the dQ kernel, the
report that Q and dO are in TMEM), so every wait that depends on it expires.  The kernel must then end with CP_ERR_TIMEOUT and the wait site in the plan's status
word, without a fault, and a correct call on the same context must still match the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import conv as oconv
from sequence_long_context_ring_b200 import synth
from sequence_long_context_ring_b200.binding import (Plan, ConvPlan, FftConvPlan, seq2head, head2seq,
                                                     CP_ERR_TIMEOUT)

from _helpers import to_dev, to_f64, inputs, assert_attn_close

pytestmark = pytest.mark.gpu


def poisoned(t):
    if t is not None:
        t.view(torch.uint8).fill_(0xFF)
    return t


def zeroed(t):
    if t is not None:
        t.view(torch.uint8).zero_()
    return t


def same_bits(a, b):
    return torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


def finite(*ts):
    return all(bool(torch.isfinite(t.float()).all()) for t in ts)


@pytest.mark.parametrize("mode,n_cp,n_hp,split", [
    ("ring", 4, 1, "contiguous"), ("ulysses", 4, 1, "contiguous"), ("ulysses", 4, 1, "zigzag"),
    ("ulysses", 4, 1, "striped"), ("2d", 2, 2, "contiguous"),
])
def test_forward_and_backward_on_poisoned_buffers(cuda_lib, mode, n_cp, n_hp, split):
    B, L, Hq, Hkv, d = 1, 1024, 8, 4, 128
    qs, kvs = ((B, Hq, L, d), (B, Hkv, L, d)) if mode == "ring" else ((B, L, Hq, d), (B, L, Hkv, d))
    q, k, v, do = (to_dev(x) for x in inputs(811, qs, kvs, with_do=True))
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n_cp, n_hp=n_hp, mode=mode, split=split)
    runs = []
    for fill in (zeroed, poisoned):
        o, lse = fill(torch.empty_like(q)), fill(torch.empty((B, Hq, L), dtype=torch.float32, device="cuda"))
        plan.fwd(q, k, v, o, lse, ws=fill(plan.workspace(False)))
        dq, dk, dv = fill(torch.empty_like(q)), fill(torch.empty_like(k)), fill(torch.empty_like(v))
        plan.bwd(q, k, v, o, lse, do, dq, dk, dv, ws=fill(plan.workspace(True)))
        torch.cuda.synchronize()
        assert plan.device_status()[0] == 0
        runs.append((o, lse, dq, dk, dv))
    for a, b, name in zip(runs[0], runs[1], ("o", "lse", "dq", "dk", "dv")):
        assert finite(b), f"{mode}/{split} {name}: NaN from a poisoned buffer"
        assert same_bits(a, b), f"{mode}/{split} {name}: differs between zeroed and poisoned buffers"


def test_ring_step_partials_and_layouts_on_poisoned_outputs(cuda_lib):
    B, L, Hq, Hkv, d, n = 1, 1024, 4, 2, 128, 4
    q, k, v = (to_dev(x) for x in inputs(812, (B, Hq, L, d), (B, Hkv, L, d)))
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n)
    c = L // n
    for r in range(n):
        for s in range(n):
            parts = []
            for fill in (zeroed, poisoned):
                po = fill(torch.empty((B, Hq, c, d), dtype=torch.float32, device="cuda"))
                pl = fill(torch.empty((B, Hq, c), dtype=torch.float32, device="cuda"))
                plan.ring_step(r, s, q, k, v, po, pl)
                parts.append((po, pl))
            torch.cuda.synchronize()
            assert same_bits(parts[0][0], parts[1][0]) and same_bits(parts[0][1], parts[1][1]), f"r{r} s{s}"
    assert plan.device_status()[0] == 0
    x = to_dev(synth.normal_bf16(813, 0, (2, 512, 8, 64)))
    for split in ("contiguous", "zigzag"):
        y0 = seq2head(4, x, out=zeroed(torch.empty((2, 8, 512, 64), dtype=torch.bfloat16, device="cuda")), split=split)
        y1 = seq2head(4, x, out=poisoned(torch.empty_like(y0)), split=split)
        z1 = head2seq(4, y1, out=poisoned(torch.empty_like(x)), split=split)
        torch.cuda.synchronize()
        assert same_bits(y0, y1) and same_bits(z1, x), split


def test_host_forward_on_poisoned_staging_and_outputs(cuda_lib):
    B, Hq, Hkv, L, d, n = 1, 8, 2, 1024, 128, 4
    q, k, v = inputs(814, (B, Hq, L, d), (B, Hkv, L, d))
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n)
    o_dev, l_dev = plan.fwd(to_dev(q), to_dev(k), to_dev(v))
    pin = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).pin_memory()
    oh = poisoned(torch.empty((B, Hq, L, d), dtype=torch.bfloat16).pin_memory())
    lh = poisoned(torch.empty((B, Hq, L), dtype=torch.float32).pin_memory())
    ws = poisoned(torch.empty(plan.host_workspace_size(), dtype=torch.uint8, device="cuda"))
    plan.fwd_host(pin(q), pin(k), pin(v), oh, lh, ws=ws)
    torch.cuda.synchronize()
    assert plan.device_status()[0] == 0
    assert same_bits(oh, o_dev.cpu()) and same_bits(lh, l_dev.cpu())


def test_convolutions_on_poisoned_workspace_and_outputs(cuda_lib):
    B, D, L, n = 1, 6, 128 * 64, 8
    x = to_dev(synth.normal_bf16(815, synth.TENSOR_ID["x"], (B, D, L)))
    h_long = to_dev(synth.normal_bf16(815, synth.TENSOR_ID["h"], (D, L), L ** -0.5))
    h_fir = to_dev(synth.normal_bf16(815, synth.TENSOR_ID["h"], (D, 33), 33 ** -0.5))
    fft = FftConvPlan(B, D, L, n)
    fir = ConvPlan(B, D, L, 33, n)
    c = L // n
    halo = x[:, :, 2 * c - 32:2 * c].contiguous()
    outs = []
    for fill in (zeroed, poisoned):
        y_fft = fft.fwd(x, h_long, y=fill(torch.empty_like(x)), ws=fill(fft.workspace(x.device)))
        y_fir = fir.fwd(x, h_fir, y=fill(torch.empty_like(x)))
        y_shard = fir.shard(2, x[:, :, 2 * c:3 * c].contiguous(), halo, h_fir,
                            y=fill(torch.empty((B, D, c), dtype=torch.bfloat16, device="cuda")))
        outs.append((y_fft, y_fir, y_shard))
    torch.cuda.synchronize()
    assert fir.device_status()[0] == 0
    for a, b, name in zip(outs[0], outs[1], ("fft", "fir", "fir shard")):
        assert finite(b), name
        assert same_bits(a, b), name


@pytest.mark.parametrize("fault,sites", [(2, range(17, 27)), (3, range(33, 44))])
def test_backward_wait_expiry_reports_timeout_and_context_survives(cuda_lib, fault, sites):
    # fault 2: the dK/dV kernel's load warp leaves out the K/V tile; 3: the dQ kernel's leaves
    # out the Q/dO tile.  The forward of the same plan is untouched.
    B, Hq, Hkv, L, d, n = 1, 4, 2, 512, 128, 2
    qb, kb, vb, dob = inputs(816, (B, Hq, L, d), (B, Hkv, L, d), with_do=True)
    q, k, v, do = (to_dev(x) for x in (qb, kb, vb, dob))
    bad = Plan(B, Hq, Hkv, L, d, n_cp=n, wait_limit_ns=20_000_000, debug_fault=fault)
    o, lse = bad.fwd(q, k, v)
    torch.cuda.synchronize()
    assert bad.device_status()[0] == 0
    bad.bwd(q, k, v, o, lse, do)
    st, word = bad.device_status()
    assert st == CP_ERR_TIMEOUT and (word & 0xFF) == 6 and (word >> 8) in sites, (st, hex(word))
    good = Plan(B, Hq, Hkv, L, d, n_cp=n)
    o, lse = good.fwd(q, k, v)
    gq, gk, gv = good.bwd(q, k, v, o, lse, do)
    torch.cuda.synchronize()
    assert good.device_status()[0] == 0
    q64, k64, v64, do64 = (synth.bf16_bits_to_f64(x) for x in (qb, kb, vb, dob))
    o_ref, _ = oracle.attention_full(q64, k64, v64)
    stored = synth.bf16_bits_to_f64(synth.f32_to_bf16_bits(np.asarray(o_ref, np.float32)))
    for g, ref, name in zip((gq, gk, gv), oracle.attention_backward(q64, k64, v64, do64, o=stored),
                            ("dq", "dk", "dv")):
        err = np.abs(to_f64(g) - ref)
        assert err.max() <= 2.0 ** -7 * np.abs(ref).max(), name
        assert err.mean() <= 2.0 ** -7 * np.abs(ref).mean(), name


def test_fir_wait_expiry_reports_timeout_and_context_survives(cuda_lib):
    B, D, L, lh, n = 1, 4, 128 * 64, 7, 4
    x = synth.normal_bf16(817, synth.TENSOR_ID["x"], (B, D, L))
    h = synth.normal_bf16(817, synth.TENSOR_ID["h"], (D, lh), lh ** -0.5)
    bad = ConvPlan(B, D, L, lh, n, wait_limit_ns=20_000_000, debug_fault=1)
    bad.fwd(to_dev(x), to_dev(h))
    st, word = bad.device_status()
    assert st == CP_ERR_TIMEOUT and (word & 0xFF) == 6 and 1 <= (word >> 8) <= 7, (st, hex(word))
    good = ConvPlan(B, D, L, lh, n)
    y = good.fwd(to_dev(x), to_dev(h))
    torch.cuda.synchronize()
    assert good.device_status()[0] == 0
    x64, h64 = synth.bf16_bits_to_f64(x), synth.bf16_bits_to_f64(h)
    ref, abs_ref = oconv.fir_conv(x64, h64), oconv.fir_conv(np.abs(x64), np.abs(h64))
    err = np.abs(to_f64(y) - ref)
    assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 2.0 ** -14 * abs_ref)
