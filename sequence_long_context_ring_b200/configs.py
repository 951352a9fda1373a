"""Named workloads: shapes of the pages' models on one GPU (synthetic, seeded inputs).

  c1  tiny ring attention, MHA, d=64, L=1024, N_cp=4 (chunks of 256)
  c2  Llama-3-8B-shaped GQA ring attention: 32 q heads / 8 KV heads, d=128, L=32768, N_cp=8,
      inputs N(0,1)/sqrt(2)
  c3  long-context Llama-3-8B-shaped GQA ring attention: L=212992 (208K), N_cp=16 (13312)
  c4  Ulysses, 7B-MHA: H=32, d=128, L=131072, degree 8; sequence-major per-rank input
  c5  2D head x context grid 4 x 4, 7B-MHA: H=32, d=128, L=65536, forward + backward

Point-to-point FIR convolution ("05. 長系列の分散学習（Context Parallelism）" §3), on c3's
sequence and chunking at the Llama-3-8B width (D = 4096 channels):
  fir_short   l_h = 7 taps    (a short explicit filter: halo of 6 samples per rank)
  fir_medium  l_h = 128 taps  (a medium filter: halo of 127 samples per rank)
Inputs: x ~ N(0, 1), h ~ N(0, 1/l_h), both rounded to bf16.

Distributed FFT convolution ("05. 長系列の分散学習（Context Parallelism）" §4), a long filter
(Hyena-LI: as long as the sequence) on c4's 128K sequence at the Llama-3-8B width:
  fft_long    D = 4096, L = 131072, N_cp = 16 (shards of 8192); h ~ N(0, 1/L)
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Workload:
    name: str
    cfg_id: int
    B: int
    Hq: int
    Hkv: int
    L: int
    d: int
    n_cp: int
    n_hp: int
    mode: str            # ring | ulysses | 2d
    causal: bool = True
    input_scale: float = 1.0
    backward: bool = False

    @property
    def seq_major(self) -> bool:
        return self.mode != "ring"

    def q_shape(self):
        return (self.B, self.L, self.Hq, self.d) if self.seq_major else (self.B, self.Hq, self.L, self.d)

    def kv_shape(self):
        return (self.B, self.L, self.Hkv, self.d) if self.seq_major else (self.B, self.Hkv, self.L, self.d)

    def fwd_flops(self) -> float:
        pairs = self.L * (self.L + 1) / 2 if self.causal else float(self.L) ** 2
        return 4.0 * self.B * self.Hq * self.d * pairs


WORKLOADS = {
    "c1": Workload("c1_tiny_ring_mha_L1024_N4", 1, 1, 4, 4, 1024, 64, 4, 1, "ring"),
    "c2": Workload("c2_llama3_8b_gqa_L32768_N8", 2, 1, 32, 8, 32768, 128, 8, 1, "ring", input_scale=2 ** -0.5),
    "c3": Workload("c3_llama3_8b_gqa_L212992_N16", 3, 1, 32, 8, 212992, 128, 16, 1, "ring"),
    "c4": Workload("c4_ulysses_7b_mha_L131072_N8", 4, 1, 32, 32, 131072, 128, 8, 1, "ulysses"),
    "c5": Workload("c5_2d_4x4_7b_mha_L65536_fwd_bwd", 5, 1, 32, 32, 65536, 128, 4, 4, "2d", backward=True),
}


@dataclass(frozen=True)
class ConvWorkload:
    name: str
    cfg_id: int
    B: int
    D: int
    L: int
    lh: int
    n_cp: int

    def x_shape(self):
        return (self.B, self.D, self.L)

    def h_shape(self):
        return (self.D, self.lh)

    @property
    def h_scale(self) -> float:
        return self.lh ** -0.5


CONV_WORKLOADS = {
    "fir_short": ConvWorkload("fir_short_D4096_L212992_N16_lh7", 6, 1, 4096, 212992, 7, 16),
    "fir_medium": ConvWorkload("fir_medium_D4096_L212992_N16_lh128", 7, 1, 4096, 212992, 128, 16),
}


@dataclass(frozen=True)
class FftConvWorkload:
    name: str
    cfg_id: int
    B: int
    D: int
    L: int
    n_cp: int

    def x_shape(self):
        return (self.B, self.D, self.L)

    def h_shape(self):
        return (self.D, self.L)

    @property
    def h_scale(self) -> float:
        return self.L ** -0.5


FFT_WORKLOADS = {
    "fft_long": FftConvWorkload("fft_long_D4096_L131072_N16", 8, 1, 4096, 131072, 16),
}
