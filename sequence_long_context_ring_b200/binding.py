"""ctypes binding of libcpattn.so (argument marshalling only: every step runs in the CUDA kernels).

Names follow the C ABI in include/cp_attn.h, include/cp_conv.h and include/cp_fftconv.h.  torch tensors are passed as strided views
(data pointer, shape, strides in elements); streams default to torch's current stream.
There is no fallback: if the library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcpattn.so")
_lib = None

CP_OK, CP_ERR_INVALID_ARG, CP_ERR_UNSUPPORTED, CP_ERR_ALIGNMENT = 0, -1, -2, -3
CP_ERR_WORKSPACE, CP_ERR_CUDA, CP_ERR_TIMEOUT = -4, -5, -6
CP_BF16, CP_FP32 = 0, 1
MODES = {"ring": 0, "ulysses": 1, "2d": 2}
SPLITS = {"contiguous": 0, "zigzag": 1, "striped": 2}


class CpError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().cp_status_string(status).decode()} ({status})")


class CpTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int), ("ndim", ctypes.c_int),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class CpConfig(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("L", ctypes.c_int),
                ("d", ctypes.c_int), ("n_cp", ctypes.c_int), ("n_hp", ctypes.c_int), ("causal", ctypes.c_int),
                ("mode", ctypes.c_int), ("split", ctypes.c_int), ("softmax_scale", ctypes.c_float),
                ("wait_limit_ns", ctypes.c_uint64), ("debug_fault", ctypes.c_int)]


class ConvConfig(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("D", ctypes.c_int), ("L", ctypes.c_int), ("lh", ctypes.c_int),
                ("n_cp", ctypes.c_int), ("wait_limit_ns", ctypes.c_uint64), ("debug_fault", ctypes.c_int)]


class FftConvConfig(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("D", ctypes.c_int), ("L", ctypes.c_int), ("n_cp", ctypes.c_int)]


EXPORTS = [
    "cp_attn_plan", "cp_attn_plan_destroy", "cp_attn_workspace_size", "cp_attn_fwd", "cp_attn_bwd",
    "cp_layout_seq2head", "cp_layout_head2seq", "cp_ring_step", "cp_lse_merge", "cp_device_status",
    "cp_status_string", "cp_plan_step_chunk", "cp_plan_flops", "cp_plan_num_work_items", "cp_version",
    "cp_attn_fwd_noalloc", "cp_layout_seq2head_split", "cp_layout_head2seq_split",
    "cp_conv_plan", "cp_conv_plan_destroy", "cp_conv_fir_fwd", "cp_conv_fir_shard", "cp_conv_device_status",
    "cp_conv_cost", "cp_attn_fwd_host", "cp_attn_host_workspace_size", "cp_fftconv_plan", "cp_fftconv_plan_destroy", "cp_fftconv_workspace_size", "cp_fftconv_fwd",
    "cp_fftconv_cost",
]


def lib() -> ctypes.CDLL:
    """Load libcpattn.so (built in-tree by ``sequence_long_context_ring_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"libcpattn.so not found at {_LIB_PATH}; run sequence_long_context_ring_b200/build.py")
        L = ctypes.CDLL(_LIB_PATH)
        P, T = ctypes.c_void_p, ctypes.POINTER(CpTensor)
        sig = {
            "cp_attn_plan": ([ctypes.POINTER(CpConfig), ctypes.POINTER(ctypes.c_void_p)], ctypes.c_int),
            "cp_attn_plan_destroy": ([P], None),
            "cp_attn_workspace_size": ([P, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
            "cp_attn_fwd": ([P, T, T, T, T, T, P, ctypes.c_size_t, P], ctypes.c_int),
            "cp_attn_bwd": ([P, T, T, T, T, T, T, T, T, T, P, ctypes.c_size_t, P], ctypes.c_int),
            "cp_layout_seq2head": ([ctypes.c_int, T, T, P], ctypes.c_int),
            "cp_layout_head2seq": ([ctypes.c_int, T, T, P], ctypes.c_int),
            "cp_ring_step": ([P, ctypes.c_int, ctypes.c_int, T, T, T, T, T, P], ctypes.c_int),
            "cp_lse_merge": ([T, T, T, T, P], ctypes.c_int),
            "cp_device_status": ([P, P, ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
            "cp_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "cp_plan_step_chunk": ([P, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                    ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
            "cp_plan_flops": ([P, ctypes.c_int, ctypes.POINTER(ctypes.c_double)], ctypes.c_int),
            "cp_plan_num_work_items": ([P, ctypes.POINTER(ctypes.c_int64)], ctypes.c_int),
            "cp_version": ([], ctypes.c_char_p),
            "cp_attn_fwd_noalloc": ([P, T, T, T, T, T, P], ctypes.c_int),
            "cp_layout_seq2head_split": ([ctypes.c_int, ctypes.c_int, T, T, P], ctypes.c_int),
            "cp_layout_head2seq_split": ([ctypes.c_int, ctypes.c_int, T, T, P], ctypes.c_int),
            "cp_attn_fwd_host": ([P, T, T, T, T, T, P, ctypes.c_size_t, P], ctypes.c_int),
            "cp_attn_host_workspace_size": ([P, ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
            "cp_conv_plan": ([ctypes.POINTER(ConvConfig), ctypes.POINTER(ctypes.c_void_p)], ctypes.c_int),
            "cp_conv_plan_destroy": ([P], None),
            "cp_conv_fir_fwd": ([P, T, T, T, P], ctypes.c_int),
            "cp_conv_fir_shard": ([P, ctypes.c_int, T, T, T, T, P], ctypes.c_int),
            "cp_conv_device_status": ([P, P, ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
            "cp_conv_cost": ([P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)], ctypes.c_int),
            "cp_fftconv_plan": ([ctypes.POINTER(FftConvConfig), ctypes.POINTER(ctypes.c_void_p)], ctypes.c_int),
            "cp_fftconv_plan_destroy": ([P], None),
            "cp_fftconv_workspace_size": ([P, ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
            "cp_fftconv_fwd": ([P, T, T, T, P, ctypes.c_size_t, P], ctypes.c_int),
            "cp_fftconv_cost": ([P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != CP_OK:
        raise CpError(status, what)


def tensor_desc(t: torch.Tensor) -> CpTensor:
    """Strided-view descriptor of a device tensor (bf16 or fp32, 2-D to 4-D)."""
    if t.dtype == torch.bfloat16:
        dt = CP_BF16
    elif t.dtype == torch.float32:
        dt = CP_FP32
    else:
        raise TypeError(f"unsupported dtype {t.dtype}")
    if t.dim() not in (2, 3, 4):
        raise ValueError("expected a 2-D, 3-D or 4-D tensor")
    d = CpTensor()
    d.data = t.data_ptr()
    d.dtype = dt
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _on_device(*tensors) -> None:
    """The device entry points dereference their pointers in kernels launched on the current
    device: a host tensor, or one on another GPU, would be a memory fault there, so it is
    refused before the call."""
    cur = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("expected a CUDA tensor (this call's kernels read and write device memory)")
        if cur is None:
            cur = torch.cuda.current_device()
        if t.device.index != cur:
            raise ValueError(f"tensor on {t.device}, but the kernels launch on cuda:{cur} "
                             "(select the tensor's device first)")


def _ws_args(ws):
    """(pointer, size in bytes) of a workspace tensor, or (None, 0) without one."""
    if ws is None:
        return None, 0
    if not ws.is_contiguous():
        raise ValueError("the workspace must be contiguous")
    return ws.data_ptr(), ws.numel() * ws.element_size()


def _on_host(*tensors) -> None:
    for t in tensors:
        if t is not None and t.is_cuda:
            raise ValueError("expected a host tensor (this call copies host memory in and out itself)")


class Plan:
    """A cp_attn plan: validated problem geometry (host only until the first launch)."""

    def __init__(self, B: int, Hq: int, Hkv: int, L: int, d: int, n_cp: int = 1, n_hp: int = 1,
                 causal: bool = True, mode: str = "ring", split: str = "contiguous", scale: float = 0.0,
                 wait_limit_ns: int = 0, debug_fault: int = 0):
        self.cfg = CpConfig(B, Hq, Hkv, L, d, n_cp, n_hp, int(bool(causal)), MODES[mode], SPLITS[split],
                            float(scale), int(wait_limit_ns), int(debug_fault))
        self.mode = mode
        h = ctypes.c_void_p()
        _check(lib().cp_attn_plan(ctypes.byref(self.cfg), ctypes.byref(h)), "cp_attn_plan")
        self._h = h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.cp_attn_plan_destroy(h)
            self._h = None

    @property
    def scale(self) -> float:
        return self.cfg.softmax_scale if self.cfg.softmax_scale > 0 else 1.0 / math.sqrt(self.cfg.d)

    def workspace_size(self, backward: bool = False) -> int:
        n = ctypes.c_size_t()
        _check(lib().cp_attn_workspace_size(self._h, int(backward), ctypes.byref(n)), "cp_attn_workspace_size")
        return n.value

    def workspace(self, backward: bool = False, device=None) -> Optional[torch.Tensor]:
        n = self.workspace_size(backward)
        return torch.empty(max(n, 1), dtype=torch.uint8, device=device or "cuda") if n else None

    def step_chunk(self, rank: int, step: int):
        c, k = ctypes.c_int(), ctypes.c_int()
        _check(lib().cp_plan_step_chunk(self._h, rank, step, ctypes.byref(c), ctypes.byref(k)), "cp_plan_step_chunk")
        return c.value, k.value

    def flops(self, backward: bool = False) -> float:
        f = ctypes.c_double()
        _check(lib().cp_plan_flops(self._h, int(backward), ctypes.byref(f)), "cp_plan_flops")
        return f.value

    def num_work_items(self) -> int:
        n = ctypes.c_int64()
        _check(lib().cp_plan_num_work_items(self._h, ctypes.byref(n)), "cp_plan_num_work_items")
        return n.value

    def fwd(self, q, k, v, o=None, lse=None, ws=None, stream=None):
        """Forward; returns (o, lse).  Layouts per mode (see cp_attn.h)."""
        _on_device(q, k, v, o, lse, ws)
        c = self.cfg
        if o is None:
            o = torch.empty_like(q)
        if lse is None:
            lse = torch.empty((c.B, c.Hq, c.L), dtype=torch.float32, device=q.device)
        if ws is None:
            ws = self.workspace(False, q.device)
        wptr, wlen = _ws_args(ws)
        td = [tensor_desc(t) for t in (q, k, v, o, lse)]
        _check(lib().cp_attn_fwd(self._h, *[ctypes.byref(t) for t in td], wptr, wlen, _stream(stream)),
               "cp_attn_fwd")
        return o, lse

    def host_workspace_size(self) -> int:
        n = ctypes.c_size_t()
        _check(lib().cp_attn_host_workspace_size(self._h, ctypes.byref(n)), "cp_attn_host_workspace_size")
        return n.value

    def fwd_host(self, q, k, v, o, lse, ws=None, stream=None):
        """Forward of a ring plan on HOST tensors (contiguous, preferably pinned): the library
        copies in, computes and copies out, overlapping the transfers with the kernels.  ws:
        device staging of host_workspace_size() bytes."""
        _on_host(q, k, v, o, lse)
        _on_device(ws)
        if ws is None:
            ws = torch.empty(self.host_workspace_size(), dtype=torch.uint8, device="cuda")
        td = [tensor_desc(t) for t in (q, k, v, o, lse)]
        _check(lib().cp_attn_fwd_host(self._h, *[ctypes.byref(t) for t in td], *_ws_args(ws), _stream(stream)),
               "cp_attn_fwd_host")
        return o, lse

    def fwd_noalloc(self, q, k, v, o, lse, stream=None):
        """Forward of a Ulysses / 2D plan through cp_attn_fwd_noalloc: the library uses its
        static 64 MiB scratch instead of a workspace and allocates nothing.  o and lse must
        be given (preallocated by the caller)."""
        _on_device(q, k, v, o, lse)
        td = [tensor_desc(t) for t in (q, k, v, o, lse)]
        _check(lib().cp_attn_fwd_noalloc(self._h, *[ctypes.byref(t) for t in td], _stream(stream)),
               "cp_attn_fwd_noalloc")
        return o, lse

    def bwd(self, q, k, v, o, lse, dout, dq=None, dk=None, dv=None, ws=None, stream=None):
        """Backward; returns (dq, dk, dv)."""
        _on_device(q, k, v, o, lse, dout, dq, dk, dv, ws)
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(k) if dk is None else dk
        dv = torch.empty_like(v) if dv is None else dv
        if ws is None:
            ws = self.workspace(True, q.device)
        wptr, wlen = _ws_args(ws)
        td = [tensor_desc(t) for t in (q, k, v, o, lse, dout, dq, dk, dv)]
        _check(lib().cp_attn_bwd(self._h, *[ctypes.byref(t) for t in td], wptr, wlen, _stream(stream)),
               "cp_attn_bwd")
        return dq, dk, dv

    def ring_step(self, rank: int, step: int, q, k, v, o_part=None, lse_part=None, stream=None):
        """One ring step's fp32 partial (O normalised, LSE) of query chunk `rank`."""
        _on_device(q, k, v, o_part, lse_part)
        c = self.cfg
        ch = c.L // c.n_cp
        if o_part is None:
            o_part = torch.empty((c.B, c.Hq, ch, c.d), dtype=torch.float32, device=q.device)
        if lse_part is None:
            lse_part = torch.empty((c.B, c.Hq, ch), dtype=torch.float32, device=q.device)
        td = [tensor_desc(t) for t in (q, k, v, o_part, lse_part)]
        _check(lib().cp_ring_step(self._h, rank, step, *[ctypes.byref(t) for t in td], _stream(stream)),
               "cp_ring_step")
        return o_part, lse_part

    def device_status(self, stream=None):
        """Synchronise and read/clear the device status word -> (status, raw word)."""
        w = ctypes.c_int()
        st = lib().cp_device_status(self._h, _stream(stream), ctypes.byref(w))
        return st, w.value


def lse_merge(o_acc, lse_acc, o_part, lse_part, stream=None) -> None:
    _on_device(o_acc, lse_acc, o_part, lse_part)
    td = [tensor_desc(t) for t in (o_acc, lse_acc, o_part, lse_part)]
    _check(lib().cp_lse_merge(*[ctypes.byref(t) for t in td], _stream(stream)), "cp_lse_merge")


def seq2head(n_ranks: int, x, out=None, stream=None, split: str = "contiguous"):
    """[B, L, H, d] (rank-major under a two-shard split) -> [B, H, L, d] in position order
    (Ulysses all-to-all, bit-exact)."""
    _on_device(x, out)
    if out is None:
        B, L, H, d = x.shape
        out = torch.empty((B, H, L, d), dtype=x.dtype, device=x.device)
    a, b = tensor_desc(x), tensor_desc(out)
    if split == "contiguous":
        _check(lib().cp_layout_seq2head(n_ranks, ctypes.byref(a), ctypes.byref(b), _stream(stream)), "cp_layout_seq2head")
    else:
        _check(lib().cp_layout_seq2head_split(n_ranks, SPLITS[split], ctypes.byref(a), ctypes.byref(b), _stream(stream)),
               "cp_layout_seq2head_split")
    return out


def head2seq(n_ranks: int, x, out=None, stream=None, split: str = "contiguous"):
    """[B, H, L, d] in position order -> [B, L, H, d] (rank-major under a two-shard split),
    the inverse all-to-all, bit-exact."""
    _on_device(x, out)
    if out is None:
        B, H, L, d = x.shape
        out = torch.empty((B, L, H, d), dtype=x.dtype, device=x.device)
    a, b = tensor_desc(x), tensor_desc(out)
    if split == "contiguous":
        _check(lib().cp_layout_head2seq(n_ranks, ctypes.byref(a), ctypes.byref(b), _stream(stream)), "cp_layout_head2seq")
    else:
        _check(lib().cp_layout_head2seq_split(n_ranks, SPLITS[split], ctypes.byref(a), ctypes.byref(b), _stream(stream)),
               "cp_layout_head2seq_split")
    return out


class ConvPlan:
    """A cp_conv plan: the causal depthwise FIR convolution of a sequence sharded over n_cp
    contiguous virtual ranks (include/cp_conv.h)."""

    def __init__(self, B: int, D: int, L: int, lh: int, n_cp: int = 1, wait_limit_ns: int = 0,
                 debug_fault: int = 0):
        self.cfg = ConvConfig(B, D, L, lh, n_cp, int(wait_limit_ns), int(debug_fault))
        h = ctypes.c_void_p()
        _check(lib().cp_conv_plan(ctypes.byref(self.cfg), ctypes.byref(h)), "cp_conv_plan")
        self._h = h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.cp_conv_plan_destroy(h)
            self._h = None

    def cost(self):
        """(HBM bytes, multiply-adds) of one whole-sequence convolution."""
        b, f = ctypes.c_double(), ctypes.c_double()
        _check(lib().cp_conv_cost(self._h, ctypes.byref(b), ctypes.byref(f)), "cp_conv_cost")
        return b.value, f.value

    def fwd(self, x, h, y=None, stream=None):
        """y = x * h over the whole sequence [B, D, L] (every virtual rank, halos in place)."""
        _on_device(x, h, y)
        y = torch.empty_like(x) if y is None else y
        td = [tensor_desc(t) for t in (x, h, y)]
        _check(lib().cp_conv_fir_fwd(self._h, *[ctypes.byref(t) for t in td], _stream(stream)), "cp_conv_fir_fwd")
        return y

    def shard(self, rank: int, x, halo, h, y=None, stream=None):
        """One rank's shard [B, D, L/n_cp] with the halo [B, D, lh-1] from rank-1 (None at rank 0)."""
        _on_device(x, halo, h, y)
        y = torch.empty_like(x) if y is None else y
        dx, dh, dy = tensor_desc(x), tensor_desc(h), tensor_desc(y)
        dg = ctypes.byref(tensor_desc(halo)) if halo is not None else None
        _check(lib().cp_conv_fir_shard(self._h, int(rank), ctypes.byref(dx), dg, ctypes.byref(dh),
                                       ctypes.byref(dy), _stream(stream)), "cp_conv_fir_shard")
        return y

    def device_status(self, stream=None):
        detail = ctypes.c_int()
        st = lib().cp_conv_device_status(self._h, _stream(stream), ctypes.byref(detail))
        return st, detail.value


class FftConvPlan:
    """A cp_fftconv plan: the causal convolution with a filter as long as the sequence by the
    distributed radix-2N DiF FFT over n_cp contiguous virtual ranks (include/cp_fftconv.h)."""

    def __init__(self, B: int, D: int, L: int, n_cp: int = 1):
        self.cfg = FftConvConfig(B, D, L, n_cp)
        h = ctypes.c_void_p()
        _check(lib().cp_fftconv_plan(ctypes.byref(self.cfg), ctypes.byref(h)), "cp_fftconv_plan")
        self._h = h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.cp_fftconv_plan_destroy(h)
            self._h = None

    def workspace_size(self) -> int:
        n = ctypes.c_size_t()
        _check(lib().cp_fftconv_workspace_size(self._h, ctypes.byref(n)), "cp_fftconv_workspace_size")
        return n.value

    def workspace(self, device=None) -> torch.Tensor:
        return torch.empty(self.workspace_size(), dtype=torch.uint8, device=device or "cuda")

    def cost(self):
        """(HBM bytes, flops) of one convolution."""
        b, f = ctypes.c_double(), ctypes.c_double()
        _check(lib().cp_fftconv_cost(self._h, ctypes.byref(b), ctypes.byref(f)), "cp_fftconv_cost")
        return b.value, f.value

    def fwd(self, x, h, y=None, ws=None, stream=None):
        """y = x * h, x [B, D, L], h [D, L] (bf16)."""
        _on_device(x, h, y, ws)
        y = torch.empty_like(x) if y is None else y
        ws = self.workspace(x.device) if ws is None else ws
        td = [tensor_desc(t) for t in (x, h, y)]
        _check(lib().cp_fftconv_fwd(self._h, *[ctypes.byref(t) for t in td], *_ws_args(ws), _stream(stream)),
               "cp_fftconv_fwd")
        return y
