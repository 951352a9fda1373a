"""Host-side tests of the C ABI (no GPU): the library loads, exports every declared symbol,
and plan validation / ring map / FLOP counts behave as the header states."""
import ctypes
import os
import re

import pytest

from sequence_long_context_ring_b200 import binding, build
from sequence_long_context_ring_b200.binding import Plan, CpError

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(cp_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    lib = binding.lib()
    declared = _declared_functions()
    assert "cp_attn_fwd" in declared and "cp_layout_seq2head" in declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(binding.EXPORTS) <= set(declared)


def test_version_and_status_strings():
    lib = binding.lib()
    assert b"sm_100a" in lib.cp_version()
    for st in range(-6, 1):
        assert lib.cp_status_string(st)


@pytest.mark.parametrize("kw,err", [
    (dict(Hq=6, Hkv=4), binding.CP_ERR_INVALID_ARG),            # Hq % Hkv != 0
    (dict(L=1000, n_cp=3), binding.CP_ERR_INVALID_ARG),         # L % N != 0
    (dict(d=96), binding.CP_ERR_UNSUPPORTED),                    # d not in {64, 128}
    (dict(n_hp=2), binding.CP_ERR_INVALID_ARG),                  # ring needs n_hp == 1
    (dict(mode="ulysses", n_cp=3, L=999), binding.CP_ERR_INVALID_ARG),   # H % N != 0
    (dict(mode="ulysses", Hq=32, Hkv=4, n_cp=8), binding.CP_ERR_INVALID_ARG),  # degree > KV groups
    (dict(mode="2d", n_hp=3, n_cp=2), binding.CP_ERR_INVALID_ARG),       # Hq % n_hp != 0
    (dict(mode="2d", n_hp=2, n_cp=2, split="zigzag"), binding.CP_ERR_UNSUPPORTED),  # 2D: contiguous only
    (dict(split="zigzag", L=1028, n_cp=4), binding.CP_ERR_INVALID_ARG),   # two shards per rank: 2N | L
    (dict(split="striped", mode="ulysses", L=1020, n_cp=4), binding.CP_ERR_INVALID_ARG),
    (dict(B=0), binding.CP_ERR_INVALID_ARG),
    (dict(debug_fault=4), binding.CP_ERR_INVALID_ARG),          # the fault seams are 1..3
    (dict(debug_fault=-1), binding.CP_ERR_INVALID_ARG),
])
def test_plan_validation_errors(kw, err):
    args = dict(B=1, Hq=8, Hkv=8, L=1024, d=128, n_cp=4)
    args.update(kw)
    with pytest.raises(CpError) as e:
        Plan(**args)
    assert e.value.status == err


def test_ring_map_and_skip_set():
    # step s: rank r holds chunk (r - s) mod N; j > r skipped, j == r diagonal.
    p = Plan(B=1, Hq=4, Hkv=4, L=1024, d=64, n_cp=4)
    for r in range(4):
        seen = []
        for s in range(4):
            j, kind = p.step_chunk(r, s)
            assert j == (r - s) % 4
            assert kind == (0 if j > r else 2 if j == r else 1)
            seen.append(j)
        assert sorted(seen) == [0, 1, 2, 3]
    with pytest.raises(CpError):
        p.step_chunk(4, 0)
    nc = Plan(B=1, Hq=4, Hkv=4, L=1024, d=64, n_cp=4, causal=False)
    assert all(nc.step_chunk(r, s)[1] == 1 for r in range(4) for s in range(4))


@pytest.mark.parametrize("split", ["zigzag", "striped"])
def test_two_shard_splits_plan_and_ring_map(split):
    # ring and Ulysses plans accept the two-shard splits; at every ring step some shard of the
    # KV rank is visible to some shard of the query rank, the diagonal step holds masked blocks
    Plan(B=1, Hq=8, Hkv=8, L=1024, d=128, n_cp=4, mode="ulysses", split=split)
    p = Plan(B=1, Hq=8, Hkv=8, L=1024, d=128, n_cp=4, split=split)
    for r in range(4):
        for s in range(4):
            j, kind = p.step_chunk(r, s)
            assert j == (r - s) % 4
            assert kind == (2 if j == r else 1)


def test_flops_and_work_items():
    p = Plan(B=1, Hq=32, Hkv=8, L=212992, d=128, n_cp=16)
    assert abs(p.flops() - 4 * 32 * 128 * 212992 * 212993 / 2) < 1.0
    assert abs(p.flops(True) - 2.5 * p.flops()) < 1.0
    # GQA pairs two heads of a group at the same 128 query rows: 8 KV heads x 2 pairs x 1664 tiles
    assert p.num_work_items() == 8 * 2 * 16 * 104
    m = Plan(B=1, Hq=4, Hkv=4, L=1024, d=64, n_cp=4)
    assert m.num_work_items() == 4 * 4 * 1  # MHA: two consecutive tiles of a 256-row chunk


def test_workspace_sizes():
    p = Plan(B=1, Hq=32, Hkv=32, L=131072, d=128, n_cp=8, mode="ulysses")
    assert p.workspace_size(False) >= 4 * 32 * 131072 * 128 * 2
    r = Plan(B=1, Hq=4, Hkv=4, L=1024, d=64, n_cp=4)
    assert r.workspace_size(False) == 0
    # ring backward: only D = rowsum(dO * O), fp32 [B, Hq, L] (dQ has no accumulator)
    assert r.workspace_size(True) == 4 * 1024 * 4
    # sequence-major backward: D plus head-major copies of q, dO (Hq) and k, v, dk, dv (Hkv)
    n = 32 * 131072 * 128 * 2
    assert p.workspace_size(True) == 32 * 131072 * 4 + 2 * n + 4 * n


# ---- the point-to-point FIR convolution (include/cp_conv.h) --------------------------------
@pytest.mark.parametrize("kw", [
    dict(lh=0), dict(lh=130),                  # taps outside 1..129
    dict(L=1000, n_cp=3),                      # L % n_cp != 0
    dict(L=64, n_cp=4, lh=18),                 # halo of 17 > shard of 16
    dict(B=0), dict(D=0), dict(n_cp=0),
    dict(debug_fault=2),                       # the one fault seam is 1
])
def test_conv_plan_validation_errors(kw):
    args = dict(B=1, D=4, L=1024, lh=7, n_cp=4)
    args.update(kw)
    with pytest.raises(CpError) as e:
        binding.ConvPlan(**args)
    assert e.value.status == binding.CP_ERR_INVALID_ARG


def test_conv_plan_accepts_the_longest_halo_and_reports_its_cost():
    p = binding.ConvPlan(1, 4, 512, 129, 4)    # l_h - 1 = 128 = the shard length
    nbytes, fmas = p.cost()
    assert nbytes == 2 * 2 * 4 * 512 + 2 * 4 * 129
    # sum over t < 512 of min(t + 1, 129), per channel
    assert fmas == 4 * sum(min(t + 1, 129) for t in range(512))
    p7 = binding.ConvPlan(2, 3, 40, 7, 2)
    assert p7.cost()[1] == 2 * 3 * sum(min(t + 1, 7) for t in range(40))


def test_conv_calls_reject_bad_arguments_before_any_launch():
    # argument checks run on the host: null tensors and a missing plan fail without a GPU
    lib = binding.lib()
    assert lib.cp_conv_fir_fwd(None, None, None, None, None) == binding.CP_ERR_INVALID_ARG
    p = binding.ConvPlan(1, 2, 256, 5, 2)
    assert lib.cp_conv_fir_fwd(p._h, None, None, None, None) == binding.CP_ERR_INVALID_ARG
    assert lib.cp_conv_fir_shard(p._h, 2, None, None, None, None, None) == binding.CP_ERR_INVALID_ARG
    assert lib.cp_conv_device_status(None, None, None) == binding.CP_ERR_INVALID_ARG


# ---- the distributed FFT convolution (include/cp_fftconv.h) --------------------------------
@pytest.mark.parametrize("kw,err", [
    (dict(L=1000, n_cp=3), binding.CP_ERR_INVALID_ARG),        # L % n_cp != 0
    (dict(L=3 * 512, n_cp=3), binding.CP_ERR_UNSUPPORTED),     # n_cp not a power of two
    (dict(L=64 * 1000, n_cp=64), binding.CP_ERR_UNSUPPORTED),  # more than 32 ranks
    (dict(L=4 * 1000, n_cp=4), binding.CP_ERR_UNSUPPORTED),    # shard not a power of two
    (dict(L=4 * 16384, n_cp=4), binding.CP_ERR_UNSUPPORTED),   # shard above 8192
    (dict(L=4 * 2, n_cp=4), binding.CP_ERR_UNSUPPORTED),       # shard below 4
    (dict(B=0), binding.CP_ERR_INVALID_ARG),
])
def test_fftconv_plan_validation(kw, err):
    args = dict(B=1, D=2, L=1024, n_cp=4)
    args.update(kw)
    with pytest.raises(CpError) as e:
        binding.FftConvPlan(**args)
    assert e.value.status == err


def test_fftconv_workspace_and_cost():
    p = binding.FftConvPlan(2, 3, 1024, 4)
    tw = 16 * 1024 + ((8 * 256 // 2 + 8 + 255) // 256) * 256      # w_2L^m, then w_c^m (c = 256)
    assert p.workspace_size() == 16 * 3 * 1024 + 16 * 2 * 3 * 1024 + tw
    nbytes, flops = p.cost()
    D, L, B = 3, 1024, 2
    assert nbytes == 18 * D * L + B * (34 * D * L) + B * 18 * D * L
    assert flops > 0
    lib = binding.lib()
    assert lib.cp_fftconv_fwd(p._h, None, None, None, None, 0, None) == binding.CP_ERR_INVALID_ARG


# ---- the host-buffer forward (cp_attn_fwd_host): argument checks run before any CUDA call ----
def _host_desc(shape, dtype_code, strides=None):
    d = binding.CpTensor()
    d.data = 4096            # never dereferenced: the checks reject the call first
    d.dtype = dtype_code
    d.ndim = len(shape)
    st = strides
    if st is None:
        st, acc = [], 1
        for n in reversed(shape):
            st.insert(0, acc)
            acc *= n
    for i, n in enumerate(shape):
        d.shape[i] = n
        d.stride[i] = st[i]
    return d


def test_host_forward_workspace_size_and_argument_checks():
    B, Hq, Hkv, L, d = 1, 8, 2, 512, 64
    plan = Plan(B, Hq, Hkv, L, d, n_cp=4)
    a256 = lambda n: (n + 255) // 256 * 256
    nq, nkv = B * Hq * L * d, B * Hkv * L * d
    assert plan.host_workspace_size() == 2 * a256(nq * 2) + 2 * a256(nkv * 2) + a256(B * Hq * L * 4)
    lib = binding.lib()
    q = _host_desc((B, Hq, L, d), binding.CP_BF16)
    k = _host_desc((B, Hkv, L, d), binding.CP_BF16)
    o = _host_desc((B, Hq, L, d), binding.CP_BF16)
    lse = _host_desc((B, Hq, L), binding.CP_FP32)
    r = ctypes.byref
    # workspace missing
    assert lib.cp_attn_fwd_host(plan._h, r(q), r(k), r(k), r(o), r(lse), None, 0, None) == binding.CP_ERR_WORKSPACE
    # wrong shape, wrong dtype, non-canonical strides
    bad = _host_desc((B, Hq, L, d + 8), binding.CP_BF16)
    assert lib.cp_attn_fwd_host(plan._h, r(bad), r(k), r(k), r(o), r(lse), None, 0, None) == binding.CP_ERR_INVALID_ARG
    badt = _host_desc((B, Hq, L), binding.CP_BF16)
    assert lib.cp_attn_fwd_host(plan._h, r(q), r(k), r(k), r(o), r(badt), None, 0, None) == binding.CP_ERR_INVALID_ARG
    strided = _host_desc((B, Hq, L, d), binding.CP_BF16, [Hq * L * d * 2, L * d * 2, d * 2, 1])
    assert lib.cp_attn_fwd_host(plan._h, r(strided), r(k), r(k), r(o), r(lse), None, 0, None) == binding.CP_ERR_ALIGNMENT
    # ring plans only
    uly = Plan(B, Hq, Hkv, L, d, n_cp=2, mode="ulysses")
    assert lib.cp_attn_fwd_host(uly._h, r(q), r(k), r(k), r(o), r(lse), None, 0, None) == binding.CP_ERR_UNSUPPORTED


def test_binding_refuses_tensors_in_the_wrong_memory():
    # a host tensor handed to a kernel would be a GPU memory fault: refused before any call
    import torch
    q = torch.zeros((1, 2, 64, 64), dtype=torch.bfloat16)
    plan = Plan(1, 2, 2, 64, 64, n_cp=2)
    with pytest.raises(ValueError):
        plan.fwd(q, q, q)
    with pytest.raises(ValueError):
        plan.ring_step(0, 0, q, q, q)
    with pytest.raises(ValueError):
        binding.lse_merge(q.float(), q[:, :, :, 0].float(), q.float(), q[:, :, :, 0].float())
    with pytest.raises(ValueError):
        binding.seq2head(2, q)
    x = torch.zeros((1, 2, 256), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.ConvPlan(1, 2, 256, 5, 2).fwd(x, torch.zeros((2, 5), dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        binding.FftConvPlan(1, 2, 256, 2).fwd(x, torch.zeros((2, 256), dtype=torch.bfloat16))


def test_binding_refuses_a_tensor_on_another_gpu(monkeypatch):
    # the kernels launch on the current device: a tensor on another GPU is refused before any
    # call (stand-in tensors, so no GPU is needed)
    import types

    import torch
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    on0 = types.SimpleNamespace(is_cuda=True, device=torch.device("cuda", 0))
    on1 = types.SimpleNamespace(is_cuda=True, device=torch.device("cuda", 1))
    binding._on_device(on0, None, on0)
    with pytest.raises(ValueError, match="cuda:1"):
        binding._on_device(on0, on1)


def test_workspace_size_is_counted_in_bytes():
    import torch
    assert binding._ws_args(None) == (None, 0)
    ws = torch.empty(10, dtype=torch.float32)
    assert binding._ws_args(ws) == (ws.data_ptr(), 40)
    with pytest.raises(ValueError):
        binding._ws_args(torch.empty((4, 4), dtype=torch.uint8)[:, ::2])


def test_noalloc_forward_refuses_fault_injection_before_any_launch():
    # the allocation-free forward has no status word to report an injected wait expiry, so a
    # plan with debug_fault set is refused before the tensors are even looked at
    lib = binding.lib()
    plan = Plan(1, 8, 8, 512, 64, n_cp=4, mode="ulysses", debug_fault=1)
    assert lib.cp_attn_fwd_noalloc(plan._h, None, None, None, None, None, None) == binding.CP_ERR_UNSUPPORTED
    ring = Plan(1, 8, 8, 512, 64, n_cp=4, debug_fault=1)
    assert lib.cp_attn_fwd_noalloc(ring._h, None, None, None, None, None, None) == binding.CP_ERR_INVALID_ARG
