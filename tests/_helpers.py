"""Shared helpers for the GPU parity tests: seeded inputs, uploads, tolerances, sampled rows."""
from __future__ import annotations

import numpy as np
import torch

from sequence_long_context_ring_b200 import synth

# Tolerances against the fp64 oracle on identical bf16 inputs (forward).
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def to_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> bf16 device tensor (same shape)."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return synth.bf16_bits_to_f64(to_bits(t))
    return t.detach().double().cpu().numpy()


def inputs(cfg_id: int, q_shape, kv_shape, scale: float = 1.0, with_do: bool = False):
    q = synth.normal_bf16(cfg_id, synth.TENSOR_ID["q"], q_shape, scale)
    k = synth.normal_bf16(cfg_id, synth.TENSOR_ID["k"], kv_shape, scale)
    v = synth.normal_bf16(cfg_id, synth.TENSOR_ID["v"], kv_shape, scale)
    if with_do:
        return q, k, v, synth.normal_bf16(cfg_id, synth.TENSOR_ID["do"], q_shape, 1.0)
    return q, k, v


def assert_attn_close(o, o_ref, lse=None, lse_ref=None, what=""):
    err = np.abs(np.asarray(o, np.float64) - o_ref)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    assert err.max() <= O_MAX_ABS, f"{what}: O max-abs {err.max():.3e}"
    assert err.mean() <= O_MEAN_ABS, f"{what}: O mean-abs {err.mean():.3e}"
    if lse is not None:
        le = np.abs(np.asarray(lse, np.float64) - lse_ref)
        assert le.max() <= LSE_ABS, f"{what}: LSE max-abs {le.max():.3e}"
    return err.max(), err.mean()


def sample_rows(L: int, n_chunks: int, n_random: int, seed: int) -> np.ndarray:
    """Rows 0, 1, last; every chunk boundary +-1; plus seeded random rows."""
    c = L // n_chunks
    rows = {0, 1, L - 1, L - 2}
    for j in range(1, n_chunks):
        rows |= {j * c - 1, j * c, j * c + 1}
    rng = np.random.default_rng(seed)
    rows |= set(rng.integers(0, L, n_random).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < L), dtype=np.int64)
