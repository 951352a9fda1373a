"""fp64 CPU oracle for context-parallel causal attention.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously correct statement of
what the CUDA path computes.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import it; the library under
``sequence_long_context_ring_b200`` never does, and the oracle imports nothing from it.

Sources (web pages on long-context sequence parallelism):
  * "05. 長系列の分散学習（Context Parallelism）", homemade-llm, StripedHyena 2 series —
    §1 (CP sharding [D, L] -> [D, L/N_cp]), §2 (all-to-all vs point-to-point),
    "ring attention: key/value をリングで回す" (steps 1-4), §5 (causal load balance).
  * "百万トークンのコンテキストでLLMを訓練する：Ulyssesシーケンス並列化の仕組みと可能性" —
    "Ulyssesシーケンス並列化の核心：All-to-All通信" (the 4-step algorithm).
  * "長いシーケンスのLLMトレーニングの進展" (2D-Attention summary) — "2Dアテンションの導入"
    (head x context grid), "LLMのアーキテクチャを理解する" (GQA), "スケーラビリティとメモリ管理"
    (recompute instead of store).
  * "05. 長系列の分散学習（Context Parallelism）" §3 (Hyena 演算子をどう分散するか): the
    point-to-point FIR convolution whose shards need only the previous rank's last l_h - 1 inputs;
    §4 (FFT 畳み込み): the DiF butterfly and the radix-N_cp distributed FFT convolution.

Modules:
  attention  full causal softmax attention with LSE (the plain definition), row-sampled form
  ring       per-(rank, step) chunk partials, the LSE merge, ring / Ulysses / 2D flows
  layout     Ulysses sequence<->head re-layout by index formula
  split      zig-zag / striped / contiguous rank-to-sequence maps, ring and Ulysses under them
  backward   gradient of softmax attention from its definition
  conv       causal depthwise FIR convolution and its point-to-point form with an l_h - 1 halo
  fftconv    causal long convolution by the distributed radix-N DiF FFT (decimated spectra)

Every pin of this oracle is listed in tests/test_oracle_*.py; there is no function here
marked "parity unpinned".
"""
from .attention import attention_full, attention_rows, forward_flops
from .ring import chunk_partial, lse_merge, ring_attention, ulysses_attention, attention_2d
from .layout import seq2head, head2seq
from .backward import attention_backward, backward_rows_dq, backward_rows_dkdv
from .split import (rank_positions, rank_order, shards_of_rank, step_pairs, ring_step_split,
                    ring_attention_split, seq2head_split, head2seq_split, ulysses_attention_split)
from .conv import fir_conv, fir_conv_shard, fir_conv_cp
from .fftconv import causal_conv, fft_conv_distributed

__all__ = [
    "attention_full", "attention_rows", "forward_flops",
    "chunk_partial", "lse_merge", "ring_attention", "ulysses_attention", "attention_2d",
    "seq2head", "head2seq",
    "attention_backward", "backward_rows_dq", "backward_rows_dkdv",
    "rank_positions", "rank_order", "shards_of_rank", "step_pairs", "ring_step_split",
    "ring_attention_split", "seq2head_split", "head2seq_split", "ulysses_attention_split",
    "fir_conv", "fir_conv_shard", "fir_conv_cp", "causal_conv", "fft_conv_distributed",
]
