// cp_attn.cu — host side of libcpattn.so: plan construction and validation, TMA tensor-map
// encoding, workspace carving, and the launches behind the C ABI declared in cp_attn.h.
#include "cp_attn.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <vector>

#include "aux_kernels.cuh"
#include "bwd_dq_kernel.cuh"
#include "bwd_kernel.cuh"
#include "fwd_kernel.cuh"
#include "tmap.h"

using namespace cpattn;

// Streams and events of the plan on one device, created at their first use and kept until the
// plan is destroyed: the host-buffer forward's copy streams (e_in / e_comp: one pair per block
// of KV heads), and the side stream on which the two-shard ring step runs its second query
// shard, forked from and joined back into the caller's stream.
struct HostPipe {
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t e_start = nullptr, e_done = nullptr;
  std::vector<cudaEvent_t> e_in, e_comp;
  cudaStream_t s_side = nullptr;
  cudaEvent_t e_fork = nullptr, e_join = nullptr;
};

struct cp_plan {
  cp_attn_config_t cfg;
  int G;
  float scale;
  mutable std::mutex mu;
  mutable std::map<int, int*> status_words;  // per device ordinal
  mutable std::mutex host_mu;                // held while a host-buffer forward enqueues
  mutable std::map<int, HostPipe> host_pipes;  // per device ordinal
};

namespace {

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int elem_bytes(cp_dtype_t t) { return t == CP_BF16 ? 2 : 4; }

// Check a 4-D data tensor: dtype, exact shape, innermost stride 1, other strides x element
// size multiples of 16 bytes, 16-byte aligned base (the TMA / 128-bit vector rules).
cp_status_t check4(const cp_tensor_t* t, cp_dtype_t dt, int64_t s0, int64_t s1, int64_t s2, int64_t s3) {
  if (!t || !t->data) return CP_ERR_INVALID_ARG;
  if (t->ndim != 4 || t->dtype != dt) return CP_ERR_INVALID_ARG;
  if (t->shape[0] != s0 || t->shape[1] != s1 || t->shape[2] != s2 || t->shape[3] != s3) return CP_ERR_INVALID_ARG;
  if (t->stride[3] != 1) return CP_ERR_ALIGNMENT;
  const int eb = elem_bytes(dt);
  for (int i = 0; i < 3; ++i)
    if (t->stride[i] <= 0 || (t->stride[i] * eb) % 16 != 0) return CP_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(t->data) % 16 != 0) return CP_ERR_ALIGNMENT;
  return CP_OK;
}

// Check a 3-D fp32 row-statistics tensor (LSE / D): exact shape, 4-byte aligned, any strides.
cp_status_t check3(const cp_tensor_t* t, int64_t s0, int64_t s1, int64_t s2) {
  if (!t || !t->data) return CP_ERR_INVALID_ARG;
  if (t->ndim != 3 || t->dtype != CP_FP32) return CP_ERR_INVALID_ARG;
  if (t->shape[0] != s0 || t->shape[1] != s1 || t->shape[2] != s2) return CP_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (t->stride[i] < 0) return CP_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(t->data) % 4 != 0) return CP_ERR_ALIGNMENT;
  return CP_OK;
}

#define CP_TRY(expr)                 \
  do {                               \
    cp_status_t st__ = (expr);       \
    if (st__ != CP_OK) return st__;  \
  } while (0)

// ---- device status word -----------------------------------------------------------------
int* status_word(const cp_plan_t* plan, cp_status_t* err) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    *err = CP_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> g(plan->mu);
  auto it = plan->status_words.find(dev);
  if (it != plan->status_words.end()) return it->second;
  int* w = nullptr;
  if (cudaMalloc(&w, sizeof(int)) != cudaSuccess || cudaMemset(w, 0, sizeof(int)) != cudaSuccess) {
    *err = CP_ERR_CUDA;
    return nullptr;
  }
  plan->status_words[dev] = w;
  return w;
}

// A [B, H, L, d] view given either directly (head-major) or as the plain pointer of a
// contiguous head-major workspace buffer.
struct View {
  const void* data;
  int64_t B, H, L, d, sB, sH, sL;
};
View view_of(const cp_tensor_t* t) {
  return View{t->data, t->shape[0], t->shape[1], t->shape[2], t->shape[3], t->stride[0], t->stride[1], t->stride[2]};
}
View contiguous_view(const void* p, int64_t B, int64_t H, int64_t L, int64_t d) {
  return View{p, B, H, L, d, H * L * d, L * d, d};
}

template <int D>
cp_status_t launch_fwd_d(const FwdParams& p, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         int64_t grid, cudaStream_t s) {
  const size_t smem = fwd_smem_bytes(D);
  if (cudaFuncSetAttribute(ring_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return CP_ERR_CUDA;
  ring_fwd_kernel<D><<<(unsigned)grid, kFwdThreads, smem, s>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

struct FwdOut {
  void* o;
  int64_t o_sb, o_sh, o_sl;
  int out_fp32;
  float* lse;
  int64_t l_sb, l_sh, l_sl;
};

// Work decomposition of the fused forward for a ring of n_chunks over [B, H, L, d].
void fill_geometry(const cp_plan_t* plan, int n_chunks, FwdParams& p) {
  const cp_attn_config_t& c = plan->cfg;
  p.B = c.B;
  p.Hq = c.Hq;
  p.Hkv = c.Hkv;
  p.L = c.L;
  p.d = c.d;
  p.G = plan->G;
  p.n_chunks = n_chunks;
  p.chunk_len = c.L / n_chunks;
  p.tiles_per_chunk = (p.chunk_len + kBN - 1) / kBN;
  p.pair_heads = (plan->G % 2 == 0) ? 1 : 0;
  p.pos_per_chunk = p.pair_heads ? p.tiles_per_chunk : (p.tiles_per_chunk + 1) / 2;
  p.n_inner = p.pair_heads ? c.B * c.Hkv * (plan->G / 2) : c.B * c.Hq;
  p.causal = c.causal ? 1 : 0;
  p.scale_log2 = static_cast<float>(static_cast<double>(plan->scale) * 1.4426950408889634);
  p.step_rank = -1;
  p.step_chunk = 0;
  p.step_chunk2 = -1;
  p.out_row_base = 0;
  p.wait_limit_ns = c.wait_limit_ns ? c.wait_limit_ns : kDefaultWaitLimitNs;
  p.debug_fault = c.debug_fault;
}

cp_status_t run_fwd_kernel(const cp_plan_t* plan, FwdParams& p, const View& q, const View& k, const View& v,
                           const FwdOut& out, int64_t grid, cudaStream_t s) {
  cp_status_t err = CP_OK;
  int* sw = status_word(plan, &err);
  if (!sw) return err;
  p.o = out.o;
  p.o_sb = out.o_sb;
  p.o_sh = out.o_sh;
  p.o_sl = out.o_sl;
  p.out_fp32 = out.out_fp32;
  p.lse = out.lse;
  p.l_sb = out.l_sb;
  p.l_sh = out.l_sh;
  p.l_sl = out.l_sl;
  p.status = sw;
  CUtensorMap mq, mk, mv;
  CP_TRY(make_map_bhld(&mq, q.data, q.B, q.H, q.L, q.d, q.sB, q.sH, q.sL));
  CP_TRY(make_map_bhld(&mk, k.data, k.B, k.H, k.L, k.d, k.sB, k.sH, k.sL));
  CP_TRY(make_map_bhld(&mv, v.data, v.B, v.H, v.L, v.d, v.sB, v.sH, v.sL));
  if (grid <= 0) return CP_OK;
  if (p.d == 128) return launch_fwd_d<128>(p, mq, mk, mv, grid, s);
  return launch_fwd_d<64>(p, mq, mk, mv, grid, s);
}

// ---- permute ------------------------------------------------------------------------------
// out[b, y, x, :] = in[b, x, y, :] for in [B, X, Y, d] (element strides given per axis).
cp_status_t launch_permute(const void* in, void* out, int64_t B, int64_t X, int64_t Y, int64_t d, int eb,
                           const int64_t in_str[3], const int64_t out_str_yx[3], cudaStream_t s, int remap = 0,
                           cp_split_t split = CP_SPLIT_CONTIGUOUS, int n_ranks = 1) {
  const int64_t row_bytes = d * eb;
  if (row_bytes % 16 != 0) return CP_ERR_ALIGNMENT;
  PermuteParams p;
  p.in = static_cast<const uint4*>(in);
  p.out = static_cast<uint4*>(out);
  p.vec_per_row = static_cast<int>(row_bytes / 16);
  p.vec_shift = -1;
  for (int sh = 0; sh < 31; ++sh)
    if ((1 << sh) == p.vec_per_row) p.vec_shift = sh;
  // about kPermVecPerPass vectors per block: one pass of kPermVecPerThread loads per thread
  p.rows_per_block = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(kPermMaxRows, kPermVecPerPass / p.vec_per_row)));
  p.X = static_cast<int>(X);
  p.Y = static_cast<int>(Y);
  p.n_rows = B * X * Y;
  const int64_t per = 16 / eb;
  p.in_sb = in_str[0] / per;
  p.in_sx = in_str[1] / per;
  p.in_sy = in_str[2] / per;
  p.out_sb = out_str_yx[0] / per;
  p.out_sy = out_str_yx[1] / per;
  p.out_sx = out_str_yx[2] / per;
  p.remap = (split == CP_SPLIT_CONTIGUOUS) ? 0 : remap;
  p.split = split == CP_SPLIT_ZIGZAG ? 1 : 2;
  p.n_ranks = n_ranks;
  p.shard = 1;
  if (p.remap) {
    const int64_t L = remap == 1 ? X : Y;
    if (n_ranks < 1 || L % (2 * n_ranks) != 0) return CP_ERR_INVALID_ARG;
    p.shard = static_cast<int>(L / (2 * n_ranks));
  }
  if (p.n_rows == 0) return CP_OK;
  const int64_t grid = (p.n_rows + p.rows_per_block - 1) / p.rows_per_block;
  permute_rows_kernel<<<(unsigned)grid, kPermThreads, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

// seq-major [B, L, H, d] tensor (rank-major rows under a two-shard split) -> contiguous
// head-major buffer [B, H, L, d] in position order
cp_status_t seq_to_head_buf(const cp_tensor_t* in, void* buf, cudaStream_t s, cp_split_t split = CP_SPLIT_CONTIGUOUS,
                            int n_ranks = 1) {
  const int64_t B = in->shape[0], L = in->shape[1], H = in->shape[2], d = in->shape[3];
  const int64_t in_str[3] = {in->stride[0], in->stride[1], in->stride[2]};
  const int64_t out_str[3] = {H * L * d, L * d, d};  // (b, y=h, x=l)
  return launch_permute(in->data, buf, B, L, H, d, elem_bytes(in->dtype), in_str, out_str, s, 1, split, n_ranks);
}
// contiguous head-major buffer [B, H, L, d] in position order -> seq-major tensor [B, L, H, d]
cp_status_t head_buf_to_seq(const void* buf, cp_tensor_t* out, cudaStream_t s, cp_split_t split = CP_SPLIT_CONTIGUOUS,
                            int n_ranks = 1) {
  const int64_t B = out->shape[0], L = out->shape[1], H = out->shape[2], d = out->shape[3];
  const int64_t in_str[3] = {H * L * d, L * d, d};                      // (b, x=h, y=l)
  const int64_t out_str[3] = {out->stride[0], out->stride[1], out->stride[2]};  // (b, y=l, x=h)
  return launch_permute(buf, out->data, B, H, L, d, elem_bytes(out->dtype), in_str, out_str, s, 2, split, n_ranks);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

template <int D>
cp_status_t launch_bwd_d(const BwdParams& p, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const CUtensorMap& mdo, int64_t grid, cudaStream_t s) {
  const size_t smem = bwd_smem_bytes(D);
  if (cudaFuncSetAttribute(ring_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return CP_ERR_CUDA;
  ring_bwd_kernel<D><<<(unsigned)grid, kBwdThreads, smem, s>>>(mq, mk, mv, mdo, p);
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

template <int D>
cp_status_t launch_bwd_dq_d(const DqParams& p, const CUtensorMap& mk, const CUtensorMap& mv, int64_t grid,
                            cudaStream_t s) {
  const size_t smem = bwd_dq_smem_bytes(D);
  if (cudaFuncSetAttribute(ring_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return CP_ERR_CUDA;
  ring_bwd_dq_kernel<D><<<(unsigned)grid, kDqThreads, smem, s>>>(mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

// D = rowsum(dO * O) for [b, h, l] rows given by per-axis element strides.
cp_status_t launch_rowdot(const void* o, const int64_t os[3], const void* g, const int64_t gs[3], float* D, int B,
                          int H, int L, int d, cudaStream_t s, cp_split_t split = CP_SPLIT_CONTIGUOUS,
                          int n_ranks = 1) {
  const int sp = split == CP_SPLIT_ZIGZAG ? 1 : (split == CP_SPLIT_STRIPED ? 2 : 0);
  DotParams p{static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(g), D, B, H, L, d,
              os[0], os[1], os[2], gs[0], gs[1], gs[2], (int64_t)H * L, (int64_t)L, 1,
              sp, n_ranks, sp ? L / (2 * n_ranks) : 1};
  const int64_t rows = (int64_t)B * H * L;
  if (rows == 0) return CP_OK;
  const int64_t threads = (rows + kDotRows - 1) / kDotRows * (d / 8);
  rowdot_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

cp_status_t run_backward(const cp_plan_t* plan, const cp_tensor_t* q, const cp_tensor_t* k, const cp_tensor_t* v,
                         const cp_tensor_t* o, const cp_tensor_t* lse, const cp_tensor_t* dout, cp_tensor_t* dq,
                         cp_tensor_t* dk, cp_tensor_t* dv, void* ws, size_t ws_bytes, void* stream) {
  if (!plan) return CP_ERR_INVALID_ARG;
  const cp_attn_config_t& c = plan->cfg;
  const cudaStream_t s = as_stream(stream);
  const bool seq = c.mode != CP_MODE_RING;
  if (!seq) {
    CP_TRY(check4(q, CP_BF16, c.B, c.Hq, c.L, c.d));
    CP_TRY(check4(k, CP_BF16, c.B, c.Hkv, c.L, c.d));
    CP_TRY(check4(v, CP_BF16, c.B, c.Hkv, c.L, c.d));
    CP_TRY(check4(o, CP_BF16, c.B, c.Hq, c.L, c.d));
    CP_TRY(check4(dout, CP_BF16, c.B, c.Hq, c.L, c.d));
    CP_TRY(check4(dq, CP_BF16, c.B, c.Hq, c.L, c.d));
    CP_TRY(check4(dk, CP_BF16, c.B, c.Hkv, c.L, c.d));
    CP_TRY(check4(dv, CP_BF16, c.B, c.Hkv, c.L, c.d));
  } else {
    CP_TRY(check4(q, CP_BF16, c.B, c.L, c.Hq, c.d));
    CP_TRY(check4(k, CP_BF16, c.B, c.L, c.Hkv, c.d));
    CP_TRY(check4(v, CP_BF16, c.B, c.L, c.Hkv, c.d));
    CP_TRY(check4(o, CP_BF16, c.B, c.L, c.Hq, c.d));
    CP_TRY(check4(dout, CP_BF16, c.B, c.L, c.Hq, c.d));
    CP_TRY(check4(dq, CP_BF16, c.B, c.L, c.Hq, c.d));
    CP_TRY(check4(dk, CP_BF16, c.B, c.L, c.Hkv, c.d));
    CP_TRY(check4(dv, CP_BF16, c.B, c.L, c.Hkv, c.d));
  }
  CP_TRY(check3(lse, c.B, c.Hq, c.L));
  size_t need = 0;
  cp_attn_workspace_size(plan, 1, &need);
  if (!ws || ws_bytes < need) return CP_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return CP_ERR_ALIGNMENT;
  cp_status_t err = CP_OK;
  int* sw = status_word(plan, &err);
  if (!sw) return err;

  const size_t nq = (size_t)c.B * c.Hq * c.L * c.d, nkv = (size_t)c.B * c.Hkv * c.L * c.d;
  const size_t nrow = (size_t)c.B * c.Hq * c.L;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* Dvec = reinterpret_cast<float*>(w);
  w += align256(nrow * 4);

  // D = rowsum(dO * O): strides along (b, h, l) of o and dout in either layout
  const int64_t os[3] = {o->stride[0], seq ? o->stride[2] : o->stride[1], seq ? o->stride[1] : o->stride[2]};
  const int64_t gs[3] = {dout->stride[0], seq ? dout->stride[2] : dout->stride[1],
                         seq ? dout->stride[1] : dout->stride[2]};
  CP_TRY(launch_rowdot(o->data, os, dout->data, gs, Dvec, c.B, c.Hq, c.L, c.d, s, seq ? c.split : CP_SPLIT_CONTIGUOUS,
                       c.n_cp));

  View vq, vk, vv, vdo;
  void *dkh = nullptr, *dvh = nullptr, *dqh = nullptr;
  const bool remap = seq && c.split != CP_SPLIT_CONTIGUOUS;
  if (!seq) {
    vq = view_of(q);
    vk = view_of(k);
    vv = view_of(v);
    vdo = view_of(dout);
  } else {
    void* qh = w;
    w += align256(nq * 2);
    void* doh = w;
    w += align256(nq * 2);
    void* kh = w;
    w += align256(nkv * 2);
    void* vh = w;
    w += align256(nkv * 2);
    dkh = w;
    w += align256(nkv * 2);
    dvh = w;
    w += align256(nkv * 2);
    if (remap) dqh = w;  // under a two-shard split dQ goes head-major first, then rank-major
    // all-to-all seq -> head of the inputs and of the upstream gradient (the extra a2a of the
    // backward, "05. 長系列の分散学習（Context Parallelism）" §3)
    CP_TRY(seq_to_head_buf(q, qh, s, c.split, c.n_cp));
    CP_TRY(seq_to_head_buf(k, kh, s, c.split, c.n_cp));
    CP_TRY(seq_to_head_buf(v, vh, s, c.split, c.n_cp));
    CP_TRY(seq_to_head_buf(dout, doh, s, c.split, c.n_cp));
    vq = contiguous_view(qh, c.B, c.Hq, c.L, c.d);
    vk = contiguous_view(kh, c.B, c.Hkv, c.L, c.d);
    vv = contiguous_view(vh, c.B, c.Hkv, c.L, c.d);
    vdo = contiguous_view(doh, c.B, c.Hq, c.L, c.d);
  }

  BwdParams p{};
  p.B = c.B;
  p.Hq = c.Hq;
  p.Hkv = c.Hkv;
  p.L = c.L;
  p.d = c.d;
  p.G = plan->G;
  p.n_chunks = c.mode == CP_MODE_ULYSSES ? 1 : c.n_cp;
  p.chunk_len = c.L / p.n_chunks;
  p.tiles_per_chunk = (p.chunk_len + 127) / 128;
  p.causal = c.causal ? 1 : 0;
  p.scale = plan->scale;
  p.scale_log2 = static_cast<float>(static_cast<double>(plan->scale) * 1.4426950408889634);
  p.lse = static_cast<const float*>(lse->data);
  p.lse_sb = lse->stride[0];
  p.lse_sh = lse->stride[1];
  p.lse_sl = lse->stride[2];
  p.Dvec = Dvec;
  if (!seq) {
    p.dk = static_cast<__nv_bfloat16*>(dk->data);
    p.dk_sb = dk->stride[0];
    p.dk_sh = dk->stride[1];
    p.dk_sl = dk->stride[2];
    p.dv = static_cast<__nv_bfloat16*>(dv->data);
    p.dv_sb = dv->stride[0];
    p.dv_sh = dv->stride[1];
    p.dv_sl = dv->stride[2];
  } else {
    p.dk = static_cast<__nv_bfloat16*>(dkh);
    p.dv = static_cast<__nv_bfloat16*>(dvh);
    p.dk_sb = p.dv_sb = (int64_t)c.Hkv * c.L * c.d;
    p.dk_sh = p.dv_sh = (int64_t)c.L * c.d;
    p.dk_sl = p.dv_sl = c.d;
  }
  p.status = sw;
  p.wait_limit_ns = c.wait_limit_ns ? c.wait_limit_ns : kDefaultWaitLimitNs;
  p.debug_fault = c.debug_fault;
  CUtensorMap mq, mk, mv, mdo;
  CP_TRY(make_map_bhld(&mq, vq.data, vq.B, vq.H, vq.L, vq.d, vq.sB, vq.sH, vq.sL));
  CP_TRY(make_map_bhld(&mk, vk.data, vk.B, vk.H, vk.L, vk.d, vk.sB, vk.sH, vk.sL));
  CP_TRY(make_map_bhld(&mv, vv.data, vv.B, vv.H, vv.L, vv.d, vv.sB, vv.sH, vv.sL));
  CP_TRY(make_map_bhld(&mdo, vdo.data, vdo.B, vdo.H, vdo.L, vdo.d, vdo.sB, vdo.sH, vdo.sL));
  const int64_t grid = (int64_t)p.n_chunks * p.tiles_per_chunk * c.B * c.Hkv;
  if (c.d == 128) {
    CP_TRY(launch_bwd_d<128>(p, mq, mk, mv, mdo, grid, s));
  } else {
    CP_TRY(launch_bwd_d<64>(p, mq, mk, mv, mdo, grid, s));
  }
  // dQ, query-stationary: written once, scaled, as bf16 straight into dq (in the caller's
  // layout: [b, h, l] strides of either the head-major or the sequence-major tensor)
  DqParams qp{};
  qp.B = c.B;
  qp.Hq = c.Hq;
  qp.Hkv = c.Hkv;
  qp.L = c.L;
  qp.d = c.d;
  qp.G = plan->G;
  qp.n_chunks = p.n_chunks;
  qp.chunk_len = p.chunk_len;
  qp.tiles_per_chunk = p.tiles_per_chunk;
  qp.causal = p.causal;
  qp.scale = p.scale;
  qp.scale_log2 = p.scale_log2;
  qp.lse = p.lse;
  qp.lse_sb = p.lse_sb;
  qp.lse_sh = p.lse_sh;
  qp.lse_sl = p.lse_sl;
  qp.Dvec = Dvec;
  // Q and dO rows, read by the kernel's elementwise warps into TMEM (the same views as the maps)
  qp.q = static_cast<const __nv_bfloat16*>(vq.data);
  qp.q_sb = vq.sB;
  qp.q_sh = vq.sH;
  qp.q_sl = vq.sL;
  qp.dout = static_cast<const __nv_bfloat16*>(vdo.data);
  qp.do_sb = vdo.sB;
  qp.do_sh = vdo.sH;
  qp.do_sl = vdo.sL;
  if (remap) {
    qp.dq = static_cast<__nv_bfloat16*>(dqh);
    qp.dq_sb = (int64_t)c.Hq * c.L * c.d;
    qp.dq_sh = (int64_t)c.L * c.d;
    qp.dq_sl = c.d;
  } else {
    qp.dq = static_cast<__nv_bfloat16*>(dq->data);
    qp.dq_sb = dq->stride[0];
    qp.dq_sh = seq ? dq->stride[2] : dq->stride[1];
    qp.dq_sl = seq ? dq->stride[1] : dq->stride[2];
  }
  qp.status = sw;
  qp.wait_limit_ns = p.wait_limit_ns;
  qp.debug_fault = c.debug_fault;
  const int64_t qgrid = (int64_t)qp.n_chunks * qp.tiles_per_chunk * c.B * c.Hq;
  if (c.d == 128) {
    CP_TRY(launch_bwd_dq_d<128>(qp, mk, mv, qgrid, s));
  } else {
    CP_TRY(launch_bwd_dq_d<64>(qp, mk, mv, qgrid, s));
  }
  if (!seq) return CP_OK;
  // all-to-all head -> seq of dK and dV (and of dQ under a two-shard split)
  if (remap) CP_TRY(head_buf_to_seq(dqh, dq, s, c.split, c.n_cp));
  CP_TRY(head_buf_to_seq(dkh, dk, s, c.split, c.n_cp));
  return head_buf_to_seq(dvh, dv, s, c.split, c.n_cp);
}

}  // namespace

// =====================================================================================
extern "C" {

const char* cp_version(void) { return "cpattn 0.1 (sm_100a tcgen05)"; }

const char* cp_status_string(cp_status_t s) {
  switch (s) {
    case CP_OK: return "ok";
    case CP_ERR_INVALID_ARG: return "invalid argument";
    case CP_ERR_UNSUPPORTED: return "unsupported configuration";
    case CP_ERR_ALIGNMENT: return "alignment or stride violation";
    case CP_ERR_WORKSPACE: return "workspace missing or too small";
    case CP_ERR_CUDA: return "CUDA error";
    case CP_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

cp_status_t cp_attn_plan(const cp_attn_config_t* cfg, cp_plan_t** out) {
  if (!cfg || !out) return CP_ERR_INVALID_ARG;
  const cp_attn_config_t& c = *cfg;
  if (c.B < 1 || c.Hq < 1 || c.Hkv < 1 || c.L < 1 || c.d < 1 || c.n_cp < 1 || c.n_hp < 1) return CP_ERR_INVALID_ARG;
  if (c.Hq % c.Hkv != 0) return CP_ERR_INVALID_ARG;
  if (c.causal != 0 && c.causal != 1) return CP_ERR_INVALID_ARG;
  if (!(c.softmax_scale >= 0.f) || std::isinf(c.softmax_scale)) return CP_ERR_INVALID_ARG;
  if (c.split != CP_SPLIT_CONTIGUOUS && c.split != CP_SPLIT_ZIGZAG && c.split != CP_SPLIT_STRIPED)
    return CP_ERR_INVALID_ARG;
  if (c.split != CP_SPLIT_CONTIGUOUS) {
    if (c.mode == CP_MODE_2D) return CP_ERR_UNSUPPORTED;
    if (c.n_cp < 1 || c.L % (2 * c.n_cp) != 0) return CP_ERR_INVALID_ARG;  // two shards per rank
  }
  switch (c.mode) {
    case CP_MODE_RING:
      if (c.n_hp != 1 || c.L % c.n_cp != 0) return CP_ERR_INVALID_ARG;
      break;
    case CP_MODE_ULYSSES:
      if (c.n_hp != 1 || c.L % c.n_cp != 0) return CP_ERR_INVALID_ARG;
      if (c.Hq % c.n_cp != 0 || c.Hkv % c.n_cp != 0) return CP_ERR_INVALID_ARG;
      break;
    case CP_MODE_2D:
      if ((int64_t)c.n_hp * c.n_cp <= 0 || c.L % (c.n_hp * c.n_cp) != 0) return CP_ERR_INVALID_ARG;
      if (c.Hq % c.n_hp != 0 || c.Hkv % c.n_hp != 0) return CP_ERR_INVALID_ARG;
      break;
    default:
      return CP_ERR_INVALID_ARG;
  }
  if (c.d != 64 && c.d != 128) return CP_ERR_UNSUPPORTED;
  if (c.debug_fault < 0 || c.debug_fault > 3) return CP_ERR_INVALID_ARG;
  cp_plan_t* p = new (std::nothrow) cp_plan_t();
  if (!p) return CP_ERR_INVALID_ARG;
  p->cfg = c;
  p->G = c.Hq / c.Hkv;
  p->scale = c.softmax_scale > 0.f ? c.softmax_scale : static_cast<float>(1.0 / std::sqrt((double)c.d));
  *out = p;
  return CP_OK;
}

void cp_attn_plan_destroy(cp_plan_t* plan) {
  if (!plan) return;
  int prev = -1;
  cudaGetDevice(&prev);
  for (auto& kv : plan->status_words) {
    if (cudaSetDevice(kv.first) == cudaSuccess) cudaFree(kv.second);
  }
  for (auto& kv : plan->host_pipes) {
    if (cudaSetDevice(kv.first) != cudaSuccess) continue;
    HostPipe& hp = kv.second;
    for (cudaEvent_t e : hp.e_in) cudaEventDestroy(e);
    for (cudaEvent_t e : hp.e_comp) cudaEventDestroy(e);
    if (hp.e_start) cudaEventDestroy(hp.e_start);
    if (hp.e_done) cudaEventDestroy(hp.e_done);
    if (hp.s_in) cudaStreamDestroy(hp.s_in);
    if (hp.s_out) cudaStreamDestroy(hp.s_out);
    if (hp.e_fork) cudaEventDestroy(hp.e_fork);
    if (hp.e_join) cudaEventDestroy(hp.e_join);
    if (hp.s_side) cudaStreamDestroy(hp.s_side);
  }
  if (prev >= 0) cudaSetDevice(prev);
  delete plan;
}

cp_status_t cp_attn_workspace_size(const cp_plan_t* plan, int backward, size_t* bytes) {
  if (!plan || !bytes) return CP_ERR_INVALID_ARG;
  const cp_attn_config_t& c = plan->cfg;
  const size_t nq = (size_t)c.B * c.Hq * c.L * c.d, nkv = (size_t)c.B * c.Hkv * c.L * c.d;
  const size_t nrow = (size_t)c.B * c.Hq * c.L;
  const bool seq_major = c.mode != CP_MODE_RING;
  size_t ws = 0;
  if (!backward) {
    if (seq_major) ws = 2 * align256(nq * 2) + 2 * align256(nkv * 2);
  } else {
    ws = align256(nrow * 4);                                             // D
    if (seq_major) ws += 2 * align256(nq * 2) + 4 * align256(nkv * 2);  // q, do ; k, v, dk, dv
    if (seq_major && c.split != CP_SPLIT_CONTIGUOUS) ws += align256(nq * 2);  // dq
  }
  *bytes = ws;
  return CP_OK;
}

cp_status_t cp_attn_fwd(const cp_plan_t* plan, const cp_tensor_t* q, const cp_tensor_t* k, const cp_tensor_t* v,
                        cp_tensor_t* o, cp_tensor_t* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!plan) return CP_ERR_INVALID_ARG;
  const cp_attn_config_t& c = plan->cfg;
  const cudaStream_t s = as_stream(stream);
  CP_TRY(check3(lse, c.B, c.Hq, c.L));
  FwdParams p{};
  if (c.mode == CP_MODE_RING) {
    CP_TRY(check4(q, CP_BF16, c.B, c.Hq, c.L, c.d));
    CP_TRY(check4(k, CP_BF16, c.B, c.Hkv, c.L, c.d));
    CP_TRY(check4(v, CP_BF16, c.B, c.Hkv, c.L, c.d));
    CP_TRY(check4(o, CP_BF16, c.B, c.Hq, c.L, c.d));
    fill_geometry(plan, c.n_cp, p);
    const int64_t grid = (int64_t)p.n_chunks * p.pos_per_chunk * p.n_inner;
    FwdOut out{o->data, o->stride[0], o->stride[1], o->stride[2], 0, static_cast<float*>(lse->data),
               lse->stride[0], lse->stride[1], lse->stride[2]};
    return run_fwd_kernel(plan, p, view_of(q), view_of(k), view_of(v), out, grid, s);
  }
  // ULYSSES / TWO_D: sequence-major in and out, head-major in the workspace.
  CP_TRY(check4(q, CP_BF16, c.B, c.L, c.Hq, c.d));
  CP_TRY(check4(k, CP_BF16, c.B, c.L, c.Hkv, c.d));
  CP_TRY(check4(v, CP_BF16, c.B, c.L, c.Hkv, c.d));
  CP_TRY(check4(o, CP_BF16, c.B, c.L, c.Hq, c.d));
  size_t need = 0;
  cp_attn_workspace_size(plan, 0, &need);
  if (!ws || ws_bytes < need) return CP_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return CP_ERR_ALIGNMENT;
  const size_t nq = (size_t)c.B * c.Hq * c.L * c.d, nkv = (size_t)c.B * c.Hkv * c.L * c.d;
  uint8_t* w = static_cast<uint8_t*>(ws);
  void* qh = w;
  w += align256(nq * 2);
  void* kh = w;
  w += align256(nkv * 2);
  void* vh = w;
  w += align256(nkv * 2);
  void* oh = w;
  // step 2 of the Ulysses flow (head-group all-to-all for 2D): seq -> head
  CP_TRY(seq_to_head_buf(q, qh, s, c.split, c.n_cp));
  CP_TRY(seq_to_head_buf(k, kh, s, c.split, c.n_cp));
  CP_TRY(seq_to_head_buf(v, vh, s, c.split, c.n_cp));
  // step 3: attention per head group (Ulysses: one chunk = full sequence; 2D: ring over n_cp)
  fill_geometry(plan, c.mode == CP_MODE_ULYSSES ? 1 : c.n_cp, p);
  const int64_t grid = (int64_t)p.n_chunks * p.pos_per_chunk * p.n_inner;
  FwdOut out{oh, (int64_t)c.Hq * c.L * c.d, (int64_t)c.L * c.d, c.d, 0, static_cast<float*>(lse->data),
             lse->stride[0], lse->stride[1], lse->stride[2]};
  CP_TRY(run_fwd_kernel(plan, p, contiguous_view(qh, c.B, c.Hq, c.L, c.d), contiguous_view(kh, c.B, c.Hkv, c.L, c.d),
                        contiguous_view(vh, c.B, c.Hkv, c.L, c.d), out, grid, s));
  // step 4: head -> seq
  return head_buf_to_seq(oh, o, s, c.split, c.n_cp);
}

namespace {

// A host tensor in canonical contiguous layout with the given shape.
cp_status_t check_host(const cp_tensor_t* t, cp_dtype_t dt, int nd, const int64_t* shape) {
  if (!t || !t->data || t->ndim != nd || t->dtype != dt) return CP_ERR_INVALID_ARG;
  int64_t stride = 1;
  for (int i = nd - 1; i >= 0; --i) {
    if (t->shape[i] != shape[i]) return CP_ERR_INVALID_ARG;
    if (t->stride[i] != stride) return CP_ERR_ALIGNMENT;
    stride *= shape[i];
  }
  return CP_OK;
}

// KV heads per pipelined block: the largest divisor of Hkv that gives at most 8 blocks per
// batch element (enough blocks to hide the transfers, few enough that every launch still fills
// the GPU many times over).
int host_block_heads(int Hkv) {
  for (int nb = 8; nb >= 1; --nb)
    if (Hkv % nb == 0) return Hkv / nb;
  return Hkv;
}

}  // namespace

cp_status_t cp_attn_host_workspace_size(const cp_plan_t* plan, size_t* bytes) {
  if (!plan || !bytes) return CP_ERR_INVALID_ARG;
  const cp_attn_config_t& c = plan->cfg;
  const size_t nq = (size_t)c.B * c.Hq * c.L * c.d, nkv = (size_t)c.B * c.Hkv * c.L * c.d;
  *bytes = 2 * align256(nq * 2) + 2 * align256(nkv * 2) + align256((size_t)c.B * c.Hq * c.L * 4);
  return CP_OK;
}

cp_status_t cp_attn_fwd_host(const cp_plan_t* plan, const cp_tensor_t* q, const cp_tensor_t* k,
                             const cp_tensor_t* v, cp_tensor_t* o, cp_tensor_t* lse, void* ws,
                             size_t ws_bytes, void* stream) {
  if (!plan) return CP_ERR_INVALID_ARG;
  const cp_attn_config_t& c = plan->cfg;
  if (c.mode != CP_MODE_RING) return CP_ERR_UNSUPPORTED;
  const int64_t sq[4] = {c.B, c.Hq, c.L, c.d}, skv[4] = {c.B, c.Hkv, c.L, c.d}, sl[3] = {c.B, c.Hq, c.L};
  CP_TRY(check_host(q, CP_BF16, 4, sq));
  CP_TRY(check_host(k, CP_BF16, 4, skv));
  CP_TRY(check_host(v, CP_BF16, 4, skv));
  CP_TRY(check_host(o, CP_BF16, 4, sq));
  CP_TRY(check_host(lse, CP_FP32, 3, sl));
  size_t need = 0;
  CP_TRY(cp_attn_host_workspace_size(plan, &need));
  if (!ws || ws_bytes < need) return CP_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return CP_ERR_ALIGNMENT;
  const size_t nq = (size_t)c.B * c.Hq * c.L * c.d, nkv = (size_t)c.B * c.Hkv * c.L * c.d;
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint8_t* dq = w;
  w += align256(nq * 2);
  uint8_t* dk = w;
  w += align256(nkv * 2);
  uint8_t* dv = w;
  w += align256(nkv * 2);
  uint8_t* dO = w;
  w += align256(nq * 2);
  float* dl = reinterpret_cast<float*>(w);

  const cudaStream_t s = as_stream(stream);
  const int hb = host_block_heads(c.Hkv);      // KV heads per block
  const int nb = c.Hkv / hb;                   // blocks per batch element
  const int G = plan->G;
  const size_t q_blk = (size_t)hb * G * c.L * c.d * 2, kv_blk = (size_t)hb * c.L * c.d * 2;
  const size_t l_blk = (size_t)hb * G * c.L * 4;
  const int n_parts = c.B * nb;

  cp_status_t st = CP_OK;
  auto cuda_ok = [&](cudaError_t e) {
    if (e != cudaSuccess && st == CP_OK) st = CP_ERR_CUDA;
    return st == CP_OK;
  };
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CP_ERR_CUDA;
  // The plan's streams and events for this device (created at the first call).  The lock is
  // held while this call enqueues: a wait captures an event's latest record when it is
  // enqueued, so concurrent calls may reuse the events, one after the other.
  std::lock_guard<std::mutex> guard(plan->host_mu);
  HostPipe& hp = plan->host_pipes[dev];
  if (!hp.s_in && !cuda_ok(cudaStreamCreateWithFlags(&hp.s_in, cudaStreamNonBlocking))) return st;
  if (!hp.s_out && !cuda_ok(cudaStreamCreateWithFlags(&hp.s_out, cudaStreamNonBlocking))) return st;
  if (!hp.e_start && !cuda_ok(cudaEventCreateWithFlags(&hp.e_start, cudaEventDisableTiming))) return st;
  if (!hp.e_done && !cuda_ok(cudaEventCreateWithFlags(&hp.e_done, cudaEventDisableTiming))) return st;
  while ((int)hp.e_in.size() < n_parts) {
    cudaEvent_t a = nullptr, b2 = nullptr;
    if (!cuda_ok(cudaEventCreateWithFlags(&a, cudaEventDisableTiming))) return st;
    if (!cuda_ok(cudaEventCreateWithFlags(&b2, cudaEventDisableTiming))) {
      cudaEventDestroy(a);
      return st;
    }
    hp.e_in.push_back(a);
    hp.e_comp.push_back(b2);
  }
  const cudaStream_t s_in = hp.s_in, s_out = hp.s_out;
  if (!cuda_ok(cudaEventRecord(hp.e_start, s)) || !cuda_ok(cudaStreamWaitEvent(s_in, hp.e_start, 0)) ||
      !cuda_ok(cudaStreamWaitEvent(s_out, hp.e_start, 0))) {
  } else {
    for (int part = 0; part < n_parts && st == CP_OK; ++part) {
      const int b = part / nb, kb = part - b * nb;
      const size_t qoff = ((size_t)b * c.Hq + (size_t)kb * hb * G) * c.L * c.d * 2;
      const size_t kvoff = ((size_t)b * c.Hkv + (size_t)kb * hb) * c.L * c.d * 2;
      const size_t loff = ((size_t)b * c.Hq + (size_t)kb * hb * G) * c.L * 4;
      const cudaEvent_t e_in = hp.e_in[part], e_comp = hp.e_comp[part];
      // 1) this block's inputs in (behind the previous block's, on s_in)
      cuda_ok(cudaMemcpyAsync(dq + qoff, static_cast<const uint8_t*>(q->data) + qoff, q_blk, cudaMemcpyHostToDevice, s_in));
      cuda_ok(cudaMemcpyAsync(dk + kvoff, static_cast<const uint8_t*>(k->data) + kvoff, kv_blk, cudaMemcpyHostToDevice, s_in));
      cuda_ok(cudaMemcpyAsync(dv + kvoff, static_cast<const uint8_t*>(v->data) + kvoff, kv_blk, cudaMemcpyHostToDevice, s_in));
      cuda_ok(cudaEventRecord(e_in, s_in));
      cuda_ok(cudaStreamWaitEvent(s, e_in, 0));
      // 2) the forward of the block on the caller's stream: the same kernel over the block's
      //    heads (views offset to them; the geometry counts only the block's heads)
      if (st == CP_OK) {
        FwdParams p{};
        fill_geometry(plan, c.n_cp, p);
        p.B = 1;
        p.Hq = hb * G;
        p.Hkv = hb;
        p.n_inner = p.pair_heads ? hb * (G / 2) : hb * G;
        const int64_t grid = (int64_t)p.n_chunks * p.pos_per_chunk * p.n_inner;
        const int64_t hsz = (int64_t)c.L * c.d;
        FwdOut out{dO + qoff, (int64_t)hb * G * hsz, hsz, c.d, 0, reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(dl) + loff),
                   (int64_t)hb * G * c.L, c.L, 1};
        st = run_fwd_kernel(plan, p, contiguous_view(dq + qoff, 1, hb * G, c.L, c.d),
                            contiguous_view(dk + kvoff, 1, hb, c.L, c.d), contiguous_view(dv + kvoff, 1, hb, c.L, c.d),
                            out, grid, s);
      }
      cuda_ok(cudaEventRecord(e_comp, s));
      // 3) its outputs out (on s_out, behind the previous block's)
      cuda_ok(cudaStreamWaitEvent(s_out, e_comp, 0));
      cuda_ok(cudaMemcpyAsync(static_cast<uint8_t*>(o->data) + qoff, dO + qoff, q_blk, cudaMemcpyDeviceToHost, s_out));
      cuda_ok(cudaMemcpyAsync(static_cast<uint8_t*>(lse->data) + loff, reinterpret_cast<uint8_t*>(dl) + loff, l_blk,
                              cudaMemcpyDeviceToHost, s_out));
    }
    // the caller's stream continues only after the last block's outputs have landed
    cuda_ok(cudaEventRecord(hp.e_done, s_out));
    cuda_ok(cudaStreamWaitEvent(s, hp.e_done, 0));
  }
  return st;
}

cp_status_t cp_ring_step(const cp_plan_t* plan, int rank, int step, const cp_tensor_t* q, const cp_tensor_t* k,
                         const cp_tensor_t* v, cp_tensor_t* o_part, cp_tensor_t* lse_part, void* stream) {
  if (!plan) return CP_ERR_INVALID_ARG;
  const cp_attn_config_t& c = plan->cfg;
  if (c.mode != CP_MODE_RING) return CP_ERR_INVALID_ARG;
  const int N = c.n_cp;
  if (rank < 0 || rank >= N || step < 0 || step >= N) return CP_ERR_INVALID_ARG;
  const int ch = c.L / N;
  CP_TRY(check4(q, CP_BF16, c.B, c.Hq, c.L, c.d));
  CP_TRY(check4(k, CP_BF16, c.B, c.Hkv, c.L, c.d));
  CP_TRY(check4(v, CP_BF16, c.B, c.Hkv, c.L, c.d));
  CP_TRY(check4(o_part, CP_FP32, c.B, c.Hq, ch, c.d));
  CP_TRY(check3(lse_part, c.B, c.Hq, ch));
  const cudaStream_t s = as_stream(stream);
  const int j = ((rank - step) % N + N) % N;
  if (c.split != CP_SPLIT_CONTIGUOUS) {
    // Two shards per rank (each w = c/2 rows), chunks of a 2N-chunk split: the query rows are
    // rank's shards (a0, a1) in that order, the KV rows rank j's shards (b0, b1).  One launch
    // per query shard covers both KV shards, merged in the kernel; a query shard that sees
    // neither gets the merge identity.  The second shard's launch runs on the plan's side
    // stream, so the two launches fill each other's last wave; both are ordered after the work
    // already on the caller's stream, and the caller's stream waits for both.
    const int w = ch / 2;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return CP_ERR_CUDA;
    std::lock_guard<std::mutex> guard(plan->host_mu);  // the side stream's events are reused
    HostPipe& hp = plan->host_pipes[dev];
    if (!hp.s_side && cudaStreamCreateWithFlags(&hp.s_side, cudaStreamNonBlocking) != cudaSuccess) return CP_ERR_CUDA;
    if (!hp.e_fork && cudaEventCreateWithFlags(&hp.e_fork, cudaEventDisableTiming) != cudaSuccess) return CP_ERR_CUDA;
    if (!hp.e_join && cudaEventCreateWithFlags(&hp.e_join, cudaEventDisableTiming) != cudaSuccess) return CP_ERR_CUDA;
    if (cudaEventRecord(hp.e_fork, s) != cudaSuccess || cudaStreamWaitEvent(hp.s_side, hp.e_fork, 0) != cudaSuccess)
      return CP_ERR_CUDA;
    cp_status_t st = CP_OK;
    auto shards = [&](int r, int& x0, int& x1) {
      x0 = r;
      x1 = c.split == CP_SPLIT_ZIGZAG ? 2 * N - 1 - r : r + N;
    };
    int a[2], b[2];
    shards(rank, a[0], a[1]);
    shards(j, b[0], b[1]);
    for (int hq = 0; hq < 2 && st == CP_OK; ++hq) {
      const cudaStream_t sh = hq == 0 ? s : hp.s_side;
      int vis[2], nv = 0;
      for (int t = 0; t < 2; ++t)
        if (!c.causal || b[t] <= a[hq]) vis[nv++] = b[t];
      if (nv == 0) {
        const int64_t n = (int64_t)c.B * c.Hq * w * c.d;
        fill_identity_kernel<<<(unsigned)((n + 255) / 256), 256, 0, sh>>>(
            static_cast<float*>(o_part->data) + (int64_t)hq * w * o_part->stride[2],
            static_cast<float*>(lse_part->data) + (int64_t)hq * w * lse_part->stride[2], c.B, c.Hq, w, c.d,
            o_part->stride[0], o_part->stride[1], o_part->stride[2], lse_part->stride[0], lse_part->stride[1],
            lse_part->stride[2]);
        if (cudaGetLastError() != cudaSuccess) st = CP_ERR_CUDA;
        continue;
      }
      FwdParams p{};
      fill_geometry(plan, 2 * N, p);
      p.step_rank = a[hq];
      p.step_chunk = vis[0];
      p.step_chunk2 = nv > 1 ? vis[1] : -1;
      p.out_row_base = (a[hq] - hq) * w;  // query shard a[hq] lands at rows [hq*w, (hq+1)*w)
      const int64_t grid = (int64_t)p.pos_per_chunk * p.n_inner;
      FwdOut out{o_part->data, o_part->stride[0], o_part->stride[1], o_part->stride[2], 1,
                 static_cast<float*>(lse_part->data), lse_part->stride[0], lse_part->stride[1], lse_part->stride[2]};
      st = run_fwd_kernel(plan, p, view_of(q), view_of(k), view_of(v), out, grid, sh);
    }
    // join: the caller's stream waits for the side stream's launch (also after an error, so
    // that nothing is left behind on the side stream)
    if (cudaEventRecord(hp.e_join, hp.s_side) != cudaSuccess || cudaStreamWaitEvent(s, hp.e_join, 0) != cudaSuccess)
      return CP_ERR_CUDA;
    return st;
  }
  if (c.causal && j > rank) {
    const int64_t n = (int64_t)c.B * c.Hq * ch * c.d;
    fill_identity_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
        static_cast<float*>(o_part->data), static_cast<float*>(lse_part->data), c.B, c.Hq, ch, c.d,
        o_part->stride[0], o_part->stride[1], o_part->stride[2], lse_part->stride[0], lse_part->stride[1],
        lse_part->stride[2]);
    return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
  }
  FwdParams p{};
  fill_geometry(plan, N, p);
  p.step_rank = rank;
  p.step_chunk = j;
  p.out_row_base = rank * ch;
  const int64_t grid = (int64_t)p.pos_per_chunk * p.n_inner;
  FwdOut out{o_part->data, o_part->stride[0], o_part->stride[1], o_part->stride[2], 1,
             static_cast<float*>(lse_part->data), lse_part->stride[0], lse_part->stride[1], lse_part->stride[2]};
  return run_fwd_kernel(plan, p, view_of(q), view_of(k), view_of(v), out, grid, s);
}

cp_status_t cp_lse_merge(cp_tensor_t* o_acc, cp_tensor_t* lse_acc, const cp_tensor_t* o_part,
                         const cp_tensor_t* lse_part, void* stream) {
  if (!o_acc) return CP_ERR_INVALID_ARG;
  const int64_t B = o_acc->shape[0], H = o_acc->shape[1], R = o_acc->shape[2], d = o_acc->shape[3];
  if (d != 64 && d != 128) return CP_ERR_UNSUPPORTED;
  CP_TRY(check4(o_acc, CP_FP32, B, H, R, d));
  CP_TRY(check4(o_part, CP_FP32, B, H, R, d));
  CP_TRY(check3(lse_acc, B, H, R));
  CP_TRY(check3(lse_part, B, H, R));
  MergeParams p{static_cast<float*>(o_acc->data), static_cast<float*>(lse_acc->data),
                static_cast<const float*>(o_part->data), static_cast<const float*>(lse_part->data),
                (int)B, (int)H, (int)R, (int)d,
                o_acc->stride[0], o_acc->stride[1], o_acc->stride[2],
                lse_acc->stride[0], lse_acc->stride[1], lse_acc->stride[2],
                o_part->stride[0], o_part->stride[1], o_part->stride[2],
                lse_part->stride[0], lse_part->stride[1], lse_part->stride[2]};
  if (B * H * R == 0) return CP_OK;
  const int64_t rows_per_block = (32 / (d / 4)) * kMergeSlots * (kMergeThreads / 32);
  const dim3 grid((unsigned)((R + rows_per_block - 1) / rows_per_block), (unsigned)std::min<int64_t>(B * H, 65535));
  lse_merge_kernel<<<grid, kMergeThreads, 0, as_stream(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

cp_status_t cp_layout_seq2head(int n_ranks, const cp_tensor_t* in, cp_tensor_t* out, void* stream) {
  if (!in || !out || n_ranks < 1) return CP_ERR_INVALID_ARG;
  const int64_t B = in->shape[0], L = in->shape[1], H = in->shape[2], d = in->shape[3];
  if (in->dtype != out->dtype) return CP_ERR_INVALID_ARG;
  CP_TRY(check4(in, in->dtype, B, L, H, d));
  CP_TRY(check4(out, out->dtype, B, H, L, d));
  if (H % n_ranks != 0 || L % n_ranks != 0) return CP_ERR_INVALID_ARG;
  const int64_t in_str[3] = {in->stride[0], in->stride[1], in->stride[2]};
  const int64_t out_str[3] = {out->stride[0], out->stride[1], out->stride[2]};  // (b, y=h, x=l)
  return launch_permute(in->data, out->data, B, L, H, d, elem_bytes(in->dtype), in_str, out_str, as_stream(stream));
}

cp_status_t cp_layout_head2seq(int n_ranks, const cp_tensor_t* in, cp_tensor_t* out, void* stream) {
  if (!in || !out || n_ranks < 1) return CP_ERR_INVALID_ARG;
  const int64_t B = in->shape[0], H = in->shape[1], L = in->shape[2], d = in->shape[3];
  if (in->dtype != out->dtype) return CP_ERR_INVALID_ARG;
  CP_TRY(check4(in, in->dtype, B, H, L, d));
  CP_TRY(check4(out, out->dtype, B, L, H, d));
  if (H % n_ranks != 0 || L % n_ranks != 0) return CP_ERR_INVALID_ARG;
  const int64_t in_str[3] = {in->stride[0], in->stride[1], in->stride[2]};
  const int64_t out_str[3] = {out->stride[0], out->stride[1], out->stride[2]};  // (b, y=l, x=h)
  return launch_permute(in->data, out->data, B, H, L, d, elem_bytes(in->dtype), in_str, out_str, as_stream(stream));
}

cp_status_t cp_layout_seq2head_split(int n_ranks, cp_split_t split, const cp_tensor_t* in, cp_tensor_t* out,
                                     void* stream) {
  if (!in || !out || n_ranks < 1) return CP_ERR_INVALID_ARG;
  if (split != CP_SPLIT_CONTIGUOUS && split != CP_SPLIT_ZIGZAG && split != CP_SPLIT_STRIPED) return CP_ERR_INVALID_ARG;
  const int64_t B = in->shape[0], L = in->shape[1], H = in->shape[2], d = in->shape[3];
  if (in->dtype != out->dtype) return CP_ERR_INVALID_ARG;
  CP_TRY(check4(in, in->dtype, B, L, H, d));
  CP_TRY(check4(out, out->dtype, B, H, L, d));
  if (H % n_ranks != 0 || L % (split == CP_SPLIT_CONTIGUOUS ? n_ranks : 2 * n_ranks) != 0) return CP_ERR_INVALID_ARG;
  const int64_t in_str[3] = {in->stride[0], in->stride[1], in->stride[2]};
  const int64_t out_str[3] = {out->stride[0], out->stride[1], out->stride[2]};  // (b, y=h, x=l)
  return launch_permute(in->data, out->data, B, L, H, d, elem_bytes(in->dtype), in_str, out_str, as_stream(stream), 1,
                        split, n_ranks);
}

cp_status_t cp_layout_head2seq_split(int n_ranks, cp_split_t split, const cp_tensor_t* in, cp_tensor_t* out,
                                     void* stream) {
  if (!in || !out || n_ranks < 1) return CP_ERR_INVALID_ARG;
  if (split != CP_SPLIT_CONTIGUOUS && split != CP_SPLIT_ZIGZAG && split != CP_SPLIT_STRIPED) return CP_ERR_INVALID_ARG;
  const int64_t B = in->shape[0], H = in->shape[1], L = in->shape[2], d = in->shape[3];
  if (in->dtype != out->dtype) return CP_ERR_INVALID_ARG;
  CP_TRY(check4(in, in->dtype, B, H, L, d));
  CP_TRY(check4(out, out->dtype, B, L, H, d));
  if (H % n_ranks != 0 || L % (split == CP_SPLIT_CONTIGUOUS ? n_ranks : 2 * n_ranks) != 0) return CP_ERR_INVALID_ARG;
  const int64_t in_str[3] = {in->stride[0], in->stride[1], in->stride[2]};
  const int64_t out_str[3] = {out->stride[0], out->stride[1], out->stride[2]};  // (b, y=l, x=h)
  return launch_permute(in->data, out->data, B, H, L, d, elem_bytes(in->dtype), in_str, out_str, as_stream(stream), 2,
                        split, n_ranks);
}

cp_status_t cp_device_status(const cp_plan_t* plan, void* stream, int* detail) {
  if (!plan) return CP_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return CP_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CP_ERR_CUDA;
  int* w = nullptr;
  {
    std::lock_guard<std::mutex> g(plan->mu);
    auto it = plan->status_words.find(dev);
    if (it != plan->status_words.end()) w = it->second;
  }
  int word = 0;
  if (w) {
    if (cudaMemcpy(&word, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return CP_ERR_CUDA;
    if (word != 0 && cudaMemset(w, 0, sizeof(int)) != cudaSuccess) return CP_ERR_CUDA;
  }
  if (detail) *detail = word;
  if (word == 0) return CP_OK;
  return static_cast<cp_status_t>(-(word & 0xff));
}

cp_status_t cp_plan_step_chunk(const cp_plan_t* plan, int rank, int step, int* chunk, int* kind) {
  if (!plan || !chunk || !kind) return CP_ERR_INVALID_ARG;
  const cp_attn_config_t& c = plan->cfg;
  const int N = c.mode == CP_MODE_ULYSSES ? 1 : c.n_cp;
  if (rank < 0 || rank >= N || step < 0 || step >= N) return CP_ERR_INVALID_ARG;
  const int j = ((rank - step) % N + N) % N;
  *chunk = j;
  if (c.split != CP_SPLIT_CONTIGUOUS) {
    // two shards per rank: some shard of rank j is below some shard of `rank` at every step
    *kind = !c.causal ? 1 : (j == rank ? 2 : 1);
    return CP_OK;
  }
  *kind = !c.causal ? 1 : (j > rank ? 0 : (j == rank ? 2 : 1));
  return CP_OK;
}

cp_status_t cp_plan_flops(const cp_plan_t* plan, int backward, double* flops) {
  if (!plan || !flops) return CP_ERR_INVALID_ARG;
  const cp_attn_config_t& c = plan->cfg;
  const double L = c.L;
  const double pairs = c.causal ? L * (L + 1) / 2.0 : L * L;
  const double fwd = 4.0 * c.B * c.Hq * c.d * pairs;
  *flops = backward ? 2.5 * fwd : fwd;
  return CP_OK;
}

cp_status_t cp_plan_num_work_items(const cp_plan_t* plan, int64_t* n) {
  if (!plan || !n) return CP_ERR_INVALID_ARG;
  const cp_attn_config_t& c = plan->cfg;
  FwdParams p{};
  fill_geometry(plan, c.mode == CP_MODE_ULYSSES ? 1 : c.n_cp, p);
  *n = (int64_t)p.n_chunks * p.pos_per_chunk * p.n_inner;
  return CP_OK;
}

cp_status_t cp_attn_bwd(const cp_plan_t* plan, const cp_tensor_t* q, const cp_tensor_t* k, const cp_tensor_t* v,
                        const cp_tensor_t* o, const cp_tensor_t* lse, const cp_tensor_t* dout, cp_tensor_t* dq,
                        cp_tensor_t* dk, cp_tensor_t* dv, void* ws, size_t ws_bytes, void* stream) {
  return run_backward(plan, q, k, v, o, lse, dout, dq, dk, dv, ws, ws_bytes, stream);
}

}  // extern "C"

// =====================================================================================
// Forward without any device allocation by the library (see cp_attn_fwd_noalloc in
// cp_attn.h).  Its scratch is this file-scope array; host code reaches it only through the
// device address that cudaGetSymbolAddress returns for the current device.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB on every device that loads the library
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of the static scratch on the current device, looked up once per process and
// device ordinal and cached from then on (a cudaDeviceReset would invalidate it).
cp_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CP_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return CP_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return CP_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return CP_OK;
}

}  // namespace

extern "C" cp_status_t cp_attn_fwd_noalloc(const cp_plan_t* plan, const cp_tensor_t* q, const cp_tensor_t* k,
                                           const cp_tensor_t* v, cp_tensor_t* o, cp_tensor_t* lse, void* stream) {
  if (!plan) return CP_ERR_INVALID_ARG;
  const cp_attn_config_t& c = plan->cfg;
  if (c.mode != CP_MODE_ULYSSES && c.mode != CP_MODE_2D) return CP_ERR_INVALID_ARG;
  // This path has no status word, so an injected wait expiry could not be reported: each CTA
  // would wait out its full limit and the call would return CP_OK with O/LSE unwritten.
  if (c.debug_fault != 0) return CP_ERR_UNSUPPORTED;
  CP_TRY(check3(lse, c.B, c.Hq, c.L));
  CP_TRY(check4(q, CP_BF16, c.B, c.L, c.Hq, c.d));
  CP_TRY(check4(k, CP_BF16, c.B, c.L, c.Hkv, c.d));
  CP_TRY(check4(v, CP_BF16, c.B, c.L, c.Hkv, c.d));
  CP_TRY(check4(o, CP_BF16, c.B, c.L, c.Hq, c.d));
  size_t need = 0;
  CP_TRY(cp_attn_workspace_size(plan, 0, &need));
  if (need > kNoAllocScratchBytes) return CP_ERR_WORKSPACE;  // problem too large for the static scratch
  void* ws = nullptr;
  CP_TRY(noalloc_scratch(&ws));
  const cudaStream_t s = as_stream(stream);
  const size_t nq = (size_t)c.B * c.Hq * c.L * c.d, nkv = (size_t)c.B * c.Hkv * c.L * c.d;
  uint8_t* w = static_cast<uint8_t*>(ws);
  void* qh = w;
  w += align256(nq * 2);
  void* kh = w;
  w += align256(nkv * 2);
  void* vh = w;
  w += align256(nkv * 2);
  void* oh = w;
  // Every byte of the scratch that is read below is written first in this call, so nothing
  // from an earlier call needs clearing.
  CP_TRY(seq_to_head_buf(q, qh, s, c.split, c.n_cp));
  CP_TRY(seq_to_head_buf(k, kh, s, c.split, c.n_cp));
  CP_TRY(seq_to_head_buf(v, vh, s, c.split, c.n_cp));
  FwdParams p{};
  fill_geometry(plan, c.mode == CP_MODE_ULYSSES ? 1 : c.n_cp, p);
  p.o = oh;
  p.o_sb = (int64_t)c.Hq * c.L * c.d;
  p.o_sh = (int64_t)c.L * c.d;
  p.o_sl = c.d;
  p.out_fp32 = 0;
  p.lse = static_cast<float*>(lse->data);
  p.l_sb = lse->stride[0];
  p.l_sh = lse->stride[1];
  p.l_sl = lse->stride[2];
  p.status = nullptr;  // no status word: it would have to be allocated
  CUtensorMap mq, mk, mv;
  CP_TRY(make_map_bhld(&mq, qh, c.B, c.Hq, c.L, c.d, (int64_t)c.Hq * c.L * c.d, (int64_t)c.L * c.d, c.d));
  CP_TRY(make_map_bhld(&mk, kh, c.B, c.Hkv, c.L, c.d, (int64_t)c.Hkv * c.L * c.d, (int64_t)c.L * c.d, c.d));
  CP_TRY(make_map_bhld(&mv, vh, c.B, c.Hkv, c.L, c.d, (int64_t)c.Hkv * c.L * c.d, (int64_t)c.L * c.d, c.d));
  const int64_t grid = (int64_t)p.n_chunks * p.pos_per_chunk * p.n_inner;
  if (grid > 0) {
    if (c.d == 128) {
      CP_TRY(launch_fwd_d<128>(p, mq, mk, mv, grid, s));
    } else {
      CP_TRY(launch_fwd_d<64>(p, mq, mk, mv, grid, s));
    }
  }
  return head_buf_to_seq(oh, o, s, c.split, c.n_cp);
}
