/*
 * cp_conv.h — C ABI of libcpattn.so, second sequence-mixing operator: the causal depthwise
 * FIR convolution of a context-parallel sequence, all virtual ranks on one B200.
 *
 * Source: "05. 長系列の分散学習（Context Parallelism）", homemade-llm StripedHyena 2 series,
 * §3 (Hyena 演算子をどう分散するか), the point-to-point convolution: each rank holds every
 * channel of its shard x[D, L/N_cp] and a copy of the filters; a causal FIR filter of length
 * l_h makes all but the first l_h - 1 outputs of a shard local, and those need only the last
 * l_h - 1 inputs of the previous rank (the halo).  The overlap variant computes the shard
 * with a zero halo first and adds the boundary terms once the halo has arrived.
 *
 *   y[b, c, t] = sum_{k=0}^{l_h-1} h[c, k] * x[b, c, t - k],   x[b, c, t < 0] = 0
 *
 * Readings of the page taken here: depthwise filters h[D, l_h] (one per channel); a rank's
 * halo comes from the previous rank alone (l_h - 1 <= L / N_cp); x, h and y are bf16 (the
 * tensor cores' operand type, both operands alike), products accumulate in fp32 and y is
 * rounded to bf16 (nearest, ties to even).
 *
 * Conventions are those of cp_attn.h (ownership, asynchronous calls on `stream`, argument
 * errors before any launch, device errors through the plan's status word, strides in
 * elements).  Layout: x, y [B, D, L] with the sequence innermost (stride 1), the page's
 * [D, L/N_cp] per rank being the view [:, :, r*c:(r+1)*c]; the other strides of x and y
 * multiples of 8 elements and their base addresses 16-byte aligned (the TMA rules).
 */
#ifndef CP_CONV_H
#define CP_CONV_H

#include "cp_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int B, D, L;            /* batch, channels, sequence length                                  */
  int lh;                 /* filter taps l_h, 1..129 (the halo l_h - 1 fits one 128-sample block) */
  int n_cp;               /* virtual ranks holding contiguous shards of c = L / n_cp samples;
                             L % n_cp == 0 and l_h - 1 <= c                                    */
  uint64_t wait_limit_ns; /* bound of every device-side wait; 0 => 2 s                          */
  int debug_fault;        /* 0 in production.  1 => the tensor-core kernel's load warp leaves out
                             its first tile's load, so the bounded waits expire and the call's
                             status word reads CP_ERR_TIMEOUT (a test of the timeout path;
                             nothing faults or hangs).  Other values: CP_ERR_INVALID_ARG.       */
} cp_conv_config_t;

typedef struct cp_conv_plan cp_conv_plan_t;

/* Validate the configuration and create a plan (host only; CP_ERR_INVALID_ARG on a bad
 * shape, l_h outside 1..129, L % n_cp != 0 or l_h - 1 > L / n_cp).  Free with
 * cp_conv_plan_destroy. */
cp_status_t cp_conv_plan(const cp_conv_config_t* cfg, cp_conv_plan_t** out);
void cp_conv_plan_destroy(cp_conv_plan_t* plan);

/* The whole sequence, every virtual rank at once: y = x * h.  Each rank's halo is the
 * previous rank's tail, read where it lies in x (the one-GPU form of the point-to-point
 * exchange); rank 0's halo is zero.  x, y [B, D, L] bf16 (distinct, non-overlapping);
 * h [D, l_h] bf16, innermost stride 1, 2-byte aligned. */
cp_status_t cp_conv_fir_fwd(const cp_conv_plan_t* plan, const cp_tensor_t* x, const cp_tensor_t* h,
                            cp_tensor_t* y, void* stream);

/* One rank of the point-to-point convolution: its shard x [B, D, c] and the halo
 * [B, D, l_h - 1] bf16 received from rank - 1 (any strides; halo[..., m] is the input at
 * shard position m - (l_h - 1)) -> y [B, D, c].  Rank 0 has no predecessor: halo must be
 * NULL (zeros); every other rank must pass one when l_h > 1.  Runs as the overlap variant's
 * two stages: the shard with a zero halo, then the first l_h - 1 outputs recomputed with
 * the halo. */
cp_status_t cp_conv_fir_shard(const cp_conv_plan_t* plan, int rank, const cp_tensor_t* x,
                              const cp_tensor_t* halo, const cp_tensor_t* h, cp_tensor_t* y, void* stream);

/* Synchronise `stream`, read and clear the plan's device status word (as cp_device_status). */
cp_status_t cp_conv_device_status(const cp_conv_plan_t* plan, void* stream, int* detail);

/* Algorithmic cost of one cp_conv_fir_fwd: bytes that must cross HBM (x read once, y written
 * once, the filters) and multiply-adds (B*D*sum over t of the taps that fall inside the
 * sequence). */
cp_status_t cp_conv_cost(const cp_conv_plan_t* plan, double* hbm_bytes, double* fmas);

#ifdef __cplusplus
}
#endif

#endif /* CP_CONV_H */
