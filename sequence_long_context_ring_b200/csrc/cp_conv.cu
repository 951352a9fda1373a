// cp_conv.cu — host side of the context-parallel FIR convolution in libcpattn.so: plan
// validation, tensor maps, and the launches of fir_tc_kernel (whole 128-sample blocks on the
// tensor cores) and fir_edge_kernel (a shard's halo boundary and the ragged tail).
#include "cp_conv.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <new>

#include "conv_kernel.cuh"
#include "tmap.h"

using namespace cpattn;

struct cp_conv_plan {
  cp_conv_config_t cfg;
  mutable std::mutex mu;
  mutable std::map<int, int*> status_words;  // per device ordinal
};

namespace {

constexpr uint64_t kConvDefaultWaitLimitNs = 2000000000ull;

#define CV_TRY(expr)                 \
  do {                               \
    cp_status_t st__ = (expr);       \
    if (st__ != CP_OK) return st__;  \
  } while (0)

// x / y: [B, D, len] bf16, sequence innermost, the other strides multiples of 8 elements,
// base 16-byte aligned.
cp_status_t check_seq(const cp_tensor_t* t, int B, int D, int64_t len) {
  if (!t || !t->data || t->ndim != 3 || t->dtype != CP_BF16) return CP_ERR_INVALID_ARG;
  if (t->shape[0] != B || t->shape[1] != D || t->shape[2] != len) return CP_ERR_INVALID_ARG;
  if (t->stride[2] != 1) return CP_ERR_ALIGNMENT;
  for (int i = 0; i < 2; ++i)
    if (t->stride[i] <= 0 || t->stride[i] % 8 != 0) return CP_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(t->data) % 16 != 0) return CP_ERR_ALIGNMENT;
  return CP_OK;
}

cp_status_t check_filter(const cp_tensor_t* t, int D, int lh) {
  if (!t || !t->data || t->ndim != 2 || t->dtype != CP_BF16) return CP_ERR_INVALID_ARG;
  if (t->shape[0] != D || t->shape[1] != lh) return CP_ERR_INVALID_ARG;
  if (t->stride[1] != 1 || t->stride[0] < lh) return CP_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(t->data) % 2 != 0) return CP_ERR_ALIGNMENT;
  return CP_OK;
}

cp_status_t check_halo(const cp_tensor_t* t, int B, int D, int lh) {
  if (!t->data || t->ndim != 3 || t->dtype != CP_BF16) return CP_ERR_INVALID_ARG;
  if (t->shape[0] != B || t->shape[1] != D || t->shape[2] != lh - 1) return CP_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (t->stride[i] < 0) return CP_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(t->data) % 2 != 0) return CP_ERR_ALIGNMENT;
  return CP_OK;
}

int* conv_status_word(const cp_conv_plan_t* plan, cp_status_t* err) {
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

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// Convolve the rows of x [B, D, len] into y; the tensor-core kernel covers the whole
// 128-sample blocks with a zero halo, the edge kernel outputs [0, head) (with `halo`) and
// [tail0, len).
cp_status_t run_conv(const cp_conv_plan_t* plan, const cp_tensor_t* x, const cp_tensor_t* halo,
                     const cp_tensor_t* h, cp_tensor_t* y, int64_t len, cudaStream_t stream) {
  const cp_conv_config_t& c = plan->cfg;
  cp_status_t err = CP_OK;
  int* status = conv_status_word(plan, &err);
  if (!status) return err;
  const int64_t nblk = len / 128;
  if (nblk > 0) {
    CUtensorMap mx, my;
    // input boxes of 136 blocks: a tile's 128 and the 8 before it
    CV_TRY(make_map_bhld(&mx, x->data, c.B, c.D, nblk, 128, x->stride[0], x->stride[1], 128, 128 + kConvLead));
    CV_TRY(make_map_bhld(&my, y->data, c.B, c.D, nblk, 128, y->stride[0], y->stride[1], 128));
    ConvParams p{};
    p.D = c.D;
    p.tiles_per_row = static_cast<int>((nblk + 127) / 128);
    p.n_tiles = static_cast<long long>(c.B) * c.D * p.tiles_per_row;
    p.lh = c.lh;
    p.kk1 = (129 - c.lh) / 16;
    p.h = static_cast<const __nv_bfloat16*>(h->data);
    p.h_sd = h->stride[0];
    p.status = status;
    p.wait_limit_ns = c.wait_limit_ns ? c.wait_limit_ns : kConvDefaultWaitLimitNs;
    p.debug_fault = c.debug_fault;
    const int sms = sm_count();
    if (sms <= 0) return CP_ERR_CUDA;
    const long long grid = p.n_tiles < sms ? p.n_tiles : sms;
    const size_t smem = fir_smem_bytes();
    if (cudaFuncSetAttribute(fir_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return CP_ERR_CUDA;
    fir_tc_kernel<<<(unsigned)grid, kConvThreads, smem, stream>>>(mx, my, p);
    if (cudaGetLastError() != cudaSuccess) return CP_ERR_CUDA;
  }
  const bool with_halo = halo != nullptr && c.lh > 1;
  const int head = (nblk > 0 && with_halo) ? c.lh - 1 : 0;
  const int64_t tail0 = nblk * 128;
  const int64_t n_edge = head + (len - tail0);
  if (n_edge > 0) {
    FirEdgeParams e{};
    e.x = static_cast<const __nv_bfloat16*>(x->data);
    e.x_sb = x->stride[0];
    e.x_sd = x->stride[1];
    if (with_halo) {
      e.halo = static_cast<const __nv_bfloat16*>(halo->data);
      e.g_sb = halo->stride[0];
      e.g_sd = halo->stride[1];
      e.g_st = halo->stride[2];
    }
    e.h = static_cast<const __nv_bfloat16*>(h->data);
    e.h_sd = h->stride[0];
    e.y = static_cast<__nv_bfloat16*>(y->data);
    e.y_sb = y->stride[0];
    e.y_sd = y->stride[1];
    e.D = c.D;
    e.len = static_cast<int>(len);
    e.lh = c.lh;
    e.head = head;
    e.tail0 = static_cast<int>(tail0);
    const dim3 grid(static_cast<unsigned>(static_cast<int64_t>(c.B) * c.D),
                    static_cast<unsigned>((n_edge + kEdgeThreads - 1) / kEdgeThreads));
    fir_edge_kernel<<<grid, kEdgeThreads, 0, stream>>>(e);
    if (cudaGetLastError() != cudaSuccess) return CP_ERR_CUDA;
  }
  return CP_OK;
}

}  // namespace

extern "C" {

cp_status_t cp_conv_plan(const cp_conv_config_t* cfg, cp_conv_plan_t** out) {
  if (!cfg || !out) return CP_ERR_INVALID_ARG;
  *out = nullptr;
  const cp_conv_config_t& c = *cfg;
  if (c.B < 1 || c.D < 1 || c.L < 1 || c.n_cp < 1) return CP_ERR_INVALID_ARG;
  if (c.lh < 1 || c.lh > kConvMaxTaps) return CP_ERR_INVALID_ARG;
  if (c.L % c.n_cp != 0) return CP_ERR_INVALID_ARG;
  if (c.lh - 1 > c.L / c.n_cp) return CP_ERR_INVALID_ARG;
  if (c.debug_fault < 0 || c.debug_fault > 1) return CP_ERR_INVALID_ARG;
  if (static_cast<int64_t>(c.B) * c.D > 0x7fffffffLL) return CP_ERR_INVALID_ARG;
  cp_conv_plan_t* p = new (std::nothrow) cp_conv_plan_t();
  if (!p) return CP_ERR_INVALID_ARG;
  p->cfg = c;
  *out = p;
  return CP_OK;
}

void cp_conv_plan_destroy(cp_conv_plan_t* plan) {
  if (!plan) return;
  int prev = -1;
  cudaGetDevice(&prev);
  for (auto& kv : plan->status_words) {
    if (cudaSetDevice(kv.first) == cudaSuccess) cudaFree(kv.second);
  }
  if (prev >= 0) cudaSetDevice(prev);
  delete plan;
}

cp_status_t cp_conv_fir_fwd(const cp_conv_plan_t* plan, const cp_tensor_t* x, const cp_tensor_t* h,
                            cp_tensor_t* y, void* stream) {
  if (!plan) return CP_ERR_INVALID_ARG;
  const cp_conv_config_t& c = plan->cfg;
  CV_TRY(check_seq(x, c.B, c.D, c.L));
  CV_TRY(check_seq(y, c.B, c.D, c.L));
  CV_TRY(check_filter(h, c.D, c.lh));
  if (x->data == y->data) return CP_ERR_INVALID_ARG;
  return run_conv(plan, x, nullptr, h, y, c.L, reinterpret_cast<cudaStream_t>(stream));
}

cp_status_t cp_conv_fir_shard(const cp_conv_plan_t* plan, int rank, const cp_tensor_t* x,
                              const cp_tensor_t* halo, const cp_tensor_t* h, cp_tensor_t* y, void* stream) {
  if (!plan) return CP_ERR_INVALID_ARG;
  const cp_conv_config_t& c = plan->cfg;
  if (rank < 0 || rank >= c.n_cp) return CP_ERR_INVALID_ARG;
  const int64_t len = c.L / c.n_cp;
  CV_TRY(check_seq(x, c.B, c.D, len));
  CV_TRY(check_seq(y, c.B, c.D, len));
  CV_TRY(check_filter(h, c.D, c.lh));
  if (x->data == y->data) return CP_ERR_INVALID_ARG;
  if (rank == 0 && halo) return CP_ERR_INVALID_ARG;           // no predecessor
  if (rank > 0 && c.lh > 1) {
    if (!halo) return CP_ERR_INVALID_ARG;
    CV_TRY(check_halo(halo, c.B, c.D, c.lh));
  }
  return run_conv(plan, x, c.lh > 1 ? halo : nullptr, h, y, len, reinterpret_cast<cudaStream_t>(stream));
}

cp_status_t cp_conv_device_status(const cp_conv_plan_t* plan, void* stream, int* detail) {
  if (!plan) return CP_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return CP_ERR_CUDA;
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

cp_status_t cp_conv_cost(const cp_conv_plan_t* plan, double* hbm_bytes, double* fmas) {
  if (!plan || !hbm_bytes || !fmas) return CP_ERR_INVALID_ARG;
  const cp_conv_config_t& c = plan->cfg;
  const double rows = static_cast<double>(c.B) * c.D;
  *hbm_bytes = rows * c.L * 2.0 * 2.0 + static_cast<double>(c.D) * c.lh * 2.0;
  // sum over t of min(t + 1, l_h)
  const double L = c.L, lh = c.lh;
  const double taps = L <= lh ? L * (L + 1) / 2 : lh * (lh + 1) / 2 + (L - lh) * lh;
  *fmas = rows * taps;
  return CP_OK;
}

}  // extern "C"
