"""GPU test of the host-buffer forward (cp_attn_fwd_host): host Q/K/V in, host O/LSE out, the
copies pipelined by KV-head block against the kernels.  The blocks are independent GQA
problems run by the same kernel, so the result must equal cp_attn_fwd's bit for bit."""
import numpy as np
import pytest
import torch

from sequence_long_context_ring_b200.binding import Plan, CpError

from _helpers import to_dev, inputs

pytestmark = pytest.mark.gpu


def _pinned(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()


@pytest.mark.parametrize("B,Hq,Hkv,L,d,n", [
    (1, 32, 8, 4096, 128, 8),    # 8 blocks of one KV head (4 query heads each)
    (2, 12, 6, 1024, 64, 4),     # B = 2: blocks run over (batch, KV block) pairs
    (1, 4, 4, 1000, 128, 4),     # MHA, ragged chunks
    (1, 6, 3, 512, 128, 2),      # 3 KV heads: blocks of one head
])
def test_host_forward_equals_the_device_forward(cuda_lib, B, Hq, Hkv, L, d, n):
    q, k, v = inputs(900 + L, (B, Hq, L, d), (B, Hkv, L, d))
    plan = Plan(B, Hq, Hkv, L, d, n_cp=n)
    o_dev, l_dev = plan.fwd(to_dev(q), to_dev(k), to_dev(v))
    qh, kh, vh = _pinned(q), _pinned(k), _pinned(v)
    oh = torch.empty((B, Hq, L, d), dtype=torch.bfloat16).pin_memory()
    lh = torch.empty((B, Hq, L), dtype=torch.float32).pin_memory()
    oh.fill_(3.0)
    plan.fwd_host(qh, kh, vh, oh, lh)
    torch.cuda.synchronize()
    assert plan.device_status()[0] == 0
    assert torch.equal(oh.view(torch.int16), o_dev.cpu().view(torch.int16))
    assert torch.equal(lh, l_dev.cpu())


def test_host_forward_rejects_bad_arguments(cuda_lib):
    B, Hq, Hkv, L, d = 1, 4, 2, 512, 64
    plan = Plan(B, Hq, Hkv, L, d, n_cp=2)
    q = torch.zeros((B, Hq, L, d), dtype=torch.bfloat16).pin_memory()
    k = torch.zeros((B, Hkv, L, d), dtype=torch.bfloat16).pin_memory()
    o = torch.zeros_like(q).pin_memory()
    lse = torch.zeros((B, Hq, L), dtype=torch.float32).pin_memory()
    small = torch.empty(plan.host_workspace_size() - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(CpError):
        plan.fwd_host(q, k, k, o, lse, ws=small)                        # workspace too small
    with pytest.raises(CpError):
        plan.fwd_host(q.transpose(2, 3), k, k, o, lse)                  # not the canonical layout
    uly = Plan(B, Hq, Hkv, L, d, n_cp=2, mode="ulysses")
    with pytest.raises(CpError):
        uly.fwd_host(q, k, k, o, lse)                                   # ring plans only
