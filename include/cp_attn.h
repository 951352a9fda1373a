/*
 * cp_attn.h — C ABI of libcpattn.so: the per-rank compute of context-parallel causal
 * attention (ring, Ulysses, 2D head x context) with all virtual ranks on one B200.
 *
 * Sources (web pages on long-context sequence parallelism):
 *  [CP]  "05. 長系列の分散学習（Context Parallelism）", homemade-llm StripedHyena 2 series:
 *        §1 (input [D, L] split along the sequence into N_cp shards [D, L/N_cp]),
 *        §2 (all-to-all re-layout [D, L/N_cp] -> [H/N_cp, L]; point-to-point exchange),
 *        "ring attention: key/value をリングで回す" (steps 1-4: queries stay, KV chunks pass
 *        to the neighbour, a partial attention per step, online softmax statistics),
 *        §3 (backward returns gradients by the inverse exchanges),
 *        §5 (causal attention is a triangular workload).
 *  [UL]  "百万トークンのコンテキストでLLMを訓練する：Ulyssesシーケンス並列化の仕組みと可能性",
 *        "Ulyssesシーケンス並列化の核心：All-to-All通信" (4 steps), and "Ring Attentionと
 *        Ulyssesの設計上の違い" (the head-parallel degree is capped by the KV-group count).
 *  [2D]  "長いシーケンスのLLMトレーニングの進展": "2Dアテンションの導入" (heads distributed and
 *        context chunked at the same time), "LLMのアーキテクチャを理解する" (GQA: query heads
 *        in a group share one K/V head), "スケーラビリティとメモリ管理" (recompute, not store).
 *  [USP] "USP: A Unified Sequence Parallelism Approach for Long Context Generative AI"
 *        summary, "2. 先行研究との差別化ポイント" (Ulysses degree <= head count).
 *
 * Conventions (all entry points):
 *  - Ownership: the caller owns every tensor and the workspace (device memory).  A plan owns
 *    host metadata and one small device status word (allocated on the first launch on a
 *    device).  A plan is immutable after creation and may be shared across host threads and
 *    streams; calls that share a status word report the first device error of any of them.
 *  - Execution: every compute call is asynchronous on `stream` (a cudaStream_t passed as
 *    void*; NULL = legacy default stream).  No exception crosses the ABI.
 *  - Errors: argument errors return before any launch (nothing is written).  CP_ERR_CUDA
 *    reports a launch error.  Device-side problems (a bounded wait that expired) are read
 *    with cp_device_status().
 *  - Tensors: cp_tensor_t describes a strided device view; strides are in ELEMENTS.  The
 *    innermost stride must be 1; every other stride a multiple of 8 elements (16 bytes, the
 *    TMA rule); the base address 16-byte aligned.  bf16 tensors carry CP_BF16; fp32 CP_FP32.
 *  - Canonical head-major layout [B, H, L, d].  A virtual rank r of a ring of N owns the
 *    sequence view [:, :, r*c:(r+1)*c, :], c = L/N — the [D, L/N_cp] shard of [CP] §1.
 *    The sequence-major layout [B, L, H, d] is the per-rank Ulysses input [L/N, H, d] of
 *    [UL] step 1, concatenated over ranks.
 */
#ifndef CP_ATTN_H
#define CP_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CP_OK = 0,
  CP_ERR_INVALID_ARG = -1, /* bad shape, dtype, null pointer, rank/step out of range       */
  CP_ERR_UNSUPPORTED = -2, /* valid request outside what the kernels implement (d, G, ...) */
  CP_ERR_ALIGNMENT = -3,   /* base address not 16 B aligned or stride not a multiple of 8  */
  CP_ERR_WORKSPACE = -4,   /* workspace missing or smaller than cp_attn_workspace_size()   */
  CP_ERR_CUDA = -5,        /* a CUDA runtime/driver call or a launch failed                */
  CP_ERR_TIMEOUT = -6      /* a bounded device-side wait expired (see cp_device_status)    */
} cp_status_t;

typedef enum { CP_BF16 = 0, CP_FP32 = 1 } cp_dtype_t;

/* RING: ring attention over N = n_cp virtual ranks on head-major [B,H,L,d] ([CP] ring steps).
 * ULYSSES: the 4-step all-to-all flow with degree N = n_cp on sequence-major [B,L,H,d]:
 *   seq->head re-layout, full attention per head group, head->seq ([UL] steps 1-4).
 * TWO_D: n_hp x n_cp grid on sequence-major [B,L,H,d]: head-group re-layout over n_hp,
 *   ring over n_cp context chunks per head group, inverse re-layout ([2D]). */
typedef enum { CP_MODE_RING = 0, CP_MODE_ULYSSES = 1, CP_MODE_2D = 2 } cp_mode_t;

/* Chunk-to-rank map ([CP] §5, "因果モデルの負荷分散": a contiguous split gives later ranks more
 * causal work).  CONTIGUOUS: rank r owns positions [r*c, (r+1)*c).  The two-shard splits cut
 * the sequence into 2N shards of w = c/2 positions and give each rank two, its local rows
 * being its first shard followed by its second:
 *   ZIGZAG   rank r holds shards r and 2N-1-r (the page's example: 8 shards, N = 4 ->
 *            [x0,x7],[x1,x6],[x2,x5],[x3,x4]); every rank has the same causal work;
 *   STRIPED  rank r holds shards r and r+N (the page's "striped ordering", read as two
 *            shards per rank placed in stripes).
 * Two-shard splits need L % (2 n_cp) == 0 and apply to RING and ULYSSES plans (TWO_D:
 * CP_ERR_UNSUPPORTED).  In RING mode they define the virtual ranks of cp_ring_step;
 * cp_attn_fwd/bwd on the head-major tensors compute the same global result for every split.
 * In ULYSSES mode the sequence-major tensors are rank-major: rank s's local rows at
 * [s*c, (s+1)*c).  LSE is in position order [B, Hq, L] in every case. */
typedef enum { CP_SPLIT_CONTIGUOUS = 0, CP_SPLIT_ZIGZAG = 1, CP_SPLIT_STRIPED = 2 } cp_split_t;

typedef struct {
  void* data;         /* device pointer                                    */
  cp_dtype_t dtype;
  int ndim;           /* 3 or 4                                            */
  int64_t shape[4];
  int64_t stride[4];  /* in elements                                       */
} cp_tensor_t;

typedef struct {
  int B, Hq, Hkv, L, d; /* batch, query heads, KV heads (GQA: Hq % Hkv == 0), length, head dim */
  int n_cp;             /* ring size (RING, TWO_D) or Ulysses degree (ULYSSES)                 */
  int n_hp;             /* head-group degree (TWO_D); must be 1 otherwise                       */
  int causal;           /* 1: key j visible to query i iff j <= i (global positions); 0: all    */
  cp_mode_t mode;
  cp_split_t split;
  float softmax_scale;  /* 0 => 1/sqrt(d)                                                       */
  uint64_t wait_limit_ns; /* bound of every device-side wait; 0 => 2 s                          */
  int debug_fault;      /* 0 in production.  A test of the timeout path, where one load warp
                           leaves out a load so that every consumer's bounded wait expires and
                           the kernel ends with CP_ERR_TIMEOUT in the status word (nothing
                           faults or hangs): 1 => the forward kernel skips the query-tile load;
                           2 => the backward's dK/dV kernel skips the K/V tile load; 3 => the
                           backward's dQ kernel never reports its Q/dO rows as stored in TMEM
                           (its MMA thread's wait for them expires).  Other values:
                           CP_ERR_INVALID_ARG.                                                  */
} cp_attn_config_t;

typedef struct cp_plan cp_plan_t;

/* Validate `cfg` and build a plan (host only; touches no GPU).
 * Rules: B,Hq,Hkv,L,d,n_cp >= 1; Hq % Hkv == 0; d in {64, 128}; a two-shard split needs
 * L % (2 n_cp) == 0 and is not supported for TWO_D; RING: n_hp == 1,
 * L % n_cp == 0.  ULYSSES: n_hp == 1, L % n_cp == 0, Hq % n_cp == 0 and Hkv % n_cp == 0 (the
 * head-parallel degree cannot exceed the KV-group count: [UL] "Ring AttentionとUlyssesの設計上の
 * 違い", [USP] §2).  TWO_D: L % (n_hp*n_cp) == 0, Hq % n_hp == 0, Hkv % n_hp == 0.
 * Returns CP_ERR_INVALID_ARG / CP_ERR_UNSUPPORTED on violation and leaves *out untouched. */
cp_status_t cp_attn_plan(const cp_attn_config_t* cfg, cp_plan_t** out);
void cp_attn_plan_destroy(cp_plan_t* plan);

/* Device workspace (bytes) that cp_attn_fwd (backward=0) or cp_attn_bwd (backward=1) need.
 * RING forward: 0.  ULYSSES/TWO_D forward: head-major copies of q, k, v, o.  Backward:
 * D = rowsum(dO*O) [B,Hq,L] fp32 (+ head-major copies of q, dO, k, v, dk, dv for
 * ULYSSES/TWO_D, and of dq under a two-shard split).  Sizes include 256 B alignment padding. */
cp_status_t cp_attn_workspace_size(const cp_plan_t* plan, int backward, size_t* bytes);

/* Forward.  Each query of each virtual rank accumulates causal softmax attention over every
 * visible KV chunk, one ring step at a time ([CP] ring steps 1-4), merged by the online-softmax
 * (LSE) merge; chunks wholly above the diagonal are skipped, the diagonal chunk is masked.
 * RING:        q [B,Hq,L,d], k/v [B,Hkv,L,d], o [B,Hq,L,d] (all bf16).
 * ULYSSES/2D:  q [B,L,Hq,d], k/v [B,L,Hkv,d], o [B,L,Hq,d] (all bf16).
 * lse [B,Hq,L] fp32 in every mode: natural-log log-sum-exp of the scaled scores.
 * o is rounded to bf16 (nearest even) once, after the last merge. */
cp_status_t cp_attn_fwd(const cp_plan_t* plan, const cp_tensor_t* q, const cp_tensor_t* k,
                        const cp_tensor_t* v, cp_tensor_t* o, cp_tensor_t* lse, void* ws,
                        size_t ws_bytes, void* stream);

/* Backward, recomputing P = exp(S - LSE) from the forward's stored LSE ([2D] "スケーラビリティと
 * メモリ管理"): D = rowsum(dO*O); dV += P^T dO; dP = dO V^T; dS = P*(dP - D); dQ += scale dS K;
 * dK += scale dS^T Q; dK/dV summed over the query heads of a KV group.  Layouts as for the
 * forward (dq like q, dk/dv like k/v, dout like o); o and lse are the forward's outputs. */
cp_status_t cp_attn_bwd(const cp_plan_t* plan, const cp_tensor_t* q, const cp_tensor_t* k,
                        const cp_tensor_t* v, const cp_tensor_t* o, const cp_tensor_t* lse,
                        const cp_tensor_t* dout, cp_tensor_t* dq, cp_tensor_t* dk,
                        cp_tensor_t* dv, void* ws, size_t ws_bytes, void* stream);

/* Forward for callers that cannot allocate device memory — for example code running inside
 * another framework that owns the whole device-memory budget and forbids allocations of its
 * own, or a host process that reserved all device memory up front.  The pages have no
 * counterpart to this entry point: it is a deployment variant of cp_attn_fwd.
 * Same computation and tensors as cp_attn_fwd for ULYSSES and TWO_D plans (RING plans need no
 * workspace: use cp_attn_fwd; they get CP_ERR_INVALID_ARG here).  Instead of a caller
 * workspace it uses a scratch array of 64 MiB that the library declares statically: every GPU
 * that loads the library holds those 64 MiB until the process exits.  Problems whose forward
 * workspace (cp_attn_workspace_size) exceeds 64 MiB are rejected with CP_ERR_WORKSPACE before
 * any launch.  The library calls no allocating routine here.  The first call on a device looks
 * up the scratch's device address (cudaGetSymbolAddress) and caches it for the rest of the
 * process, per device ordinal, so a cudaDeviceReset afterwards leaves a stale address; make
 * that first call before any stream capture.  All calls share the one scratch array: calls whose GPU
 * work overlaps (on different streams, or from different threads) race on it and must be
 * serialised by the caller.  The scratch keeps the last call's contents; every byte a call
 * reads is written earlier in the same call.  Device-side wait expiries are not recorded
 * (there is no status word without an allocation); the waits stay bounded.  For the same
 * reason a plan with debug_fault set gets CP_ERR_UNSUPPORTED before any launch. */
cp_status_t cp_attn_fwd_noalloc(const cp_plan_t* plan, const cp_tensor_t* q, const cp_tensor_t* k,
                                const cp_tensor_t* v, cp_tensor_t* o, cp_tensor_t* lse, void* stream);

/* Forward of a RING plan with the tensors in HOST memory: q, k, v, o [B, H, L, d] bf16 and lse
 * [B, Hq, L] fp32, each contiguous (canonical strides), preferably page-locked (pageable memory
 * works but its copies do not overlap the kernels).  The library copies the inputs in, runs
 * the same forward kernel, and copies O and LSE out, pipelined over blocks of KV heads: while
 * one block computes on `stream`, the next block's Q/K/V arrive and the previous block's O/LSE
 * leave on two copy streams (created with their events at the plan's first such call on a
 * device and kept until cp_attn_plan_destroy; calls on one plan enqueue one at a time, so the
 * plan stays shareable between threads) (GQA blocks are independent problems, so the result is
 * bit-identical to cp_attn_fwd).  Device staging for all five tensors comes from `ws`, a
 * device buffer of at least cp_attn_host_workspace_size bytes, 256-byte aligned.  Everything
 * is enqueued behind the work already on `stream`; the host buffers are complete, and `ws`
 * free, when `stream` reaches the point of this call's return.  Other modes: CP_ERR_UNSUPPORTED. */
cp_status_t cp_attn_fwd_host(const cp_plan_t* plan, const cp_tensor_t* q, const cp_tensor_t* k,
                             const cp_tensor_t* v, cp_tensor_t* o, cp_tensor_t* lse, void* ws,
                             size_t ws_bytes, void* stream);
/* Device bytes cp_attn_fwd_host stages through (Q, K, V, O, LSE, each 256-byte aligned). */
cp_status_t cp_attn_host_workspace_size(const cp_plan_t* plan, size_t* bytes);

/* Ulysses all-to-all on one GPU ([CP] §2, [UL] step 2): in [B, L, H, d] (rank s holds rows
 * [s*c, (s+1)*c)) -> out [B, H, L, d] (rank r' holds heads [r'*H/N, (r'+1)*H/N) for all L):
 *     out[b, r'*H/N + h', s*c + t, :] = in[b, s*c + t, r'*H/N + h', :].
 * n_ranks = N must divide H and L.  Bit-exact copy; both tensors the same dtype. */
cp_status_t cp_layout_seq2head(int n_ranks, const cp_tensor_t* in, cp_tensor_t* out, void* stream);
/* Exact inverse ([UL] step 4): in [B, H, L, d] -> out [B, L, H, d]. */
cp_status_t cp_layout_head2seq(int n_ranks, const cp_tensor_t* in, cp_tensor_t* out, void* stream);

/* The same all-to-all under a chunk-to-rank map ([CP] §5): in [B, L, H, d] is rank-major
 * (rank s's local rows at [s*c, (s+1)*c), in its shards' order), out [B, H, L, d] is in
 * position order:  out[b, h, pos_s(t), :] = in[b, s*c + t, h, :], pos_s(t) the global
 * position of rank s's local row t.  CONTIGUOUS equals cp_layout_seq2head.  Two-shard splits
 * need L % (2 n_ranks) == 0.  Bit-exact copy. */
cp_status_t cp_layout_seq2head_split(int n_ranks, cp_split_t split, const cp_tensor_t* in, cp_tensor_t* out,
                                     void* stream);
/* Exact inverse of cp_layout_seq2head_split: in [B, H, L, d] -> out [B, L, H, d]. */
cp_status_t cp_layout_head2seq_split(int n_ranks, cp_split_t split, const cp_tensor_t* in, cp_tensor_t* out,
                                     void* stream);

/* One ring step of rank `rank` at step `step` (RING plans): the partial attention of query
 * chunk r against KV chunk j = (rank - step) mod n_cp ([CP] ring step 2).
 * q, k, v: the full tensors as for cp_attn_fwd.  o_part [B,Hq,c,d] fp32 receives the
 * normalised partial P V / l, lse_part [B,Hq,c] fp32 its LSE.  A chunk wholly above the
 * causal diagonal yields O = 0, LSE = -inf (the merge identity).  Under a two-shard split
 * rank r's c rows are its two shards (local order) and the KV rows are rank j's two shards;
 * a query shard that sees neither KV shard gets the identity.  Under a two-shard split the
 * second query shard's work runs on a stream the plan owns (created at the first such call
 * on the device, destroyed with the plan), forked from `stream` and joined back into it: work
 * enqueued on `stream` after the call sees both shards' results.  Calls on one plan enqueue
 * one at a time (a lock). */
cp_status_t cp_ring_step(const cp_plan_t* plan, int rank, int step, const cp_tensor_t* q,
                         const cp_tensor_t* k, const cp_tensor_t* v, cp_tensor_t* o_part,
                         cp_tensor_t* lse_part, void* stream);

/* Online-softmax merge of a partial into an accumulator, in place ([CP] ring step 3):
 * m = max(la, lb); wa = e^(la-m); wb = e^(lb-m); LSE = m + ln(wa+wb);
 * O = (wa*Oa + wb*Ob)/(wa+wb); an operand with LSE = -inf is the identity.
 * o_acc, o_part [B,H,c,d] fp32; lse_acc, lse_part [B,H,c] fp32 (same shapes). */
cp_status_t cp_lse_merge(cp_tensor_t* o_acc, cp_tensor_t* lse_acc, const cp_tensor_t* o_part,
                         const cp_tensor_t* lse_part, void* stream);

/* Synchronise `stream`, read and clear the plan's device status word.  Returns CP_OK, or the
 * stored error (CP_ERR_TIMEOUT).  If detail != NULL it receives the raw word: the error code in
 * the low byte and the site of the first expired wait in bits 8..15. */
cp_status_t cp_device_status(const cp_plan_t* plan, void* stream, int* detail);

const char* cp_status_string(cp_status_t status);

/* ---- host-only plan queries (no GPU needed) ---------------------------------------------- */
/* Ring map: at `step`, rank `rank` holds KV chunk *chunk = (rank - step) mod N, which is
 * *kind = 0 (skipped: wholly above the diagonal), 1 (fully visible) or 2 (diagonal, masked).
 * Under a two-shard split *chunk is the KV rank and *kind is 2 at the diagonal step and 1
 * otherwise (some shard pair is visible at every step). */
cp_status_t cp_plan_step_chunk(const cp_plan_t* plan, int rank, int step, int* chunk, int* kind);
/* Algorithmic FLOPs of one forward (4*B*Hq*d*visible pairs) or backward (2.5x forward). */
cp_status_t cp_plan_flops(const cp_plan_t* plan, int backward, double* flops);
/* Number of CTAs (work items) the fused forward kernel launches. */
cp_status_t cp_plan_num_work_items(const cp_plan_t* plan, int64_t* n);
/* Library version string. */
const char* cp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CP_ATTN_H */
