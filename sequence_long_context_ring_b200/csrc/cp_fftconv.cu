// cp_fftconv.cu — host side of the distributed FFT convolution in libcpattn.so: plan
// validation, workspace layout, and the launches of fftconv_slice_kernel (filter spectra, then
// the signal's slices) and fftconv_inverse_kernel (the cross-rank inverse).
#include "cp_fftconv.h"

#include <cuda_runtime.h>

#include <new>

#include "fftconv_kernel.cuh"

using namespace cpattn;

struct cp_fftconv_plan {
  cp_fftconv_config_t cfg;
  int c, logc;
};

namespace {

#define FC_TRY(expr)                 \
  do {                               \
    cp_status_t st__ = (expr);       \
    if (st__ != CP_OK) return st__;  \
  } while (0)

bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// [s0, s1, len] bf16 (or [s1, len] when s0 < 0), sequence innermost, 2-byte aligned
cp_status_t check_rows(const cp_tensor_t* t, int s0, int s1, int len) {
  const int nd = s0 < 0 ? 2 : 3;
  if (!t || !t->data || t->ndim != nd || t->dtype != CP_BF16) return CP_ERR_INVALID_ARG;
  if (nd == 3 && (t->shape[0] != s0 || t->shape[1] != s1 || t->shape[2] != len)) return CP_ERR_INVALID_ARG;
  if (nd == 2 && (t->shape[0] != s1 || t->shape[1] != len)) return CP_ERR_INVALID_ARG;
  if (t->stride[nd - 1] != 1) return CP_ERR_ALIGNMENT;
  for (int i = 0; i < nd - 1; ++i)
    if (t->stride[i] < 0) return CP_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(t->data) % 2 != 0) return CP_ERR_ALIGNMENT;
  return CP_OK;
}

size_t spec_bytes(const cp_fftconv_config_t& c) { return align256(16ull * c.D * c.L); }
size_t w_bytes(const cp_fftconv_config_t& c) { return align256(16ull * c.B * c.D * c.L); }
size_t tw_bytes(const cp_fftconv_config_t& c) {  // w_2L^m (2L) and w_c^m (c / 2)
  return align256(8ull * 2 * c.L) + align256(8ull * (c.L / c.n_cp) / 2 + 8);
}

template <int NN>
cudaError_t launch_inverse(const FftInvParams& ip, int c, int rows, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>((c + kFftThreads - 1) / kFftThreads), static_cast<unsigned>(rows));
  fftconv_inverse_kernel<NN><<<grid, kFftThreads, 0, st>>>(ip);
  return cudaGetLastError();
}

}  // namespace

extern "C" {

cp_status_t cp_fftconv_plan(const cp_fftconv_config_t* cfg, cp_fftconv_plan_t** out) {
  if (!cfg || !out) return CP_ERR_INVALID_ARG;
  *out = nullptr;
  const cp_fftconv_config_t& c = *cfg;
  if (c.B < 1 || c.D < 1 || c.L < 1 || c.n_cp < 1) return CP_ERR_INVALID_ARG;
  if (c.L % c.n_cp != 0) return CP_ERR_INVALID_ARG;
  if (static_cast<int64_t>(c.B) * c.D > 65535) return CP_ERR_UNSUPPORTED;   // grid.y of the inverse
  const int cl = c.L / c.n_cp;
  if (!pow2(c.n_cp) || c.n_cp > kFftMaxN) return CP_ERR_UNSUPPORTED;
  if (!pow2(cl) || cl < 4 || cl > kFftMaxC) return CP_ERR_UNSUPPORTED;
  cp_fftconv_plan_t* p = new (std::nothrow) cp_fftconv_plan_t();
  if (!p) return CP_ERR_INVALID_ARG;
  p->cfg = c;
  p->c = cl;
  p->logc = 0;
  while ((1 << p->logc) < cl) ++p->logc;
  *out = p;
  return CP_OK;
}

void cp_fftconv_plan_destroy(cp_fftconv_plan_t* plan) { delete plan; }

cp_status_t cp_fftconv_workspace_size(const cp_fftconv_plan_t* plan, size_t* bytes) {
  if (!plan || !bytes) return CP_ERR_INVALID_ARG;
  *bytes = spec_bytes(plan->cfg) + w_bytes(plan->cfg) + tw_bytes(plan->cfg);
  return CP_OK;
}

cp_status_t cp_fftconv_fwd(const cp_fftconv_plan_t* plan, const cp_tensor_t* x, const cp_tensor_t* h,
                           cp_tensor_t* y, void* ws, size_t ws_bytes, void* stream) {
  if (!plan) return CP_ERR_INVALID_ARG;
  const cp_fftconv_config_t& c = plan->cfg;
  FC_TRY(check_rows(x, c.B, c.D, c.L));
  FC_TRY(check_rows(y, c.B, c.D, c.L));
  FC_TRY(check_rows(h, -1, c.D, c.L));
  if (x->data == y->data) return CP_ERR_INVALID_ARG;
  size_t need = 0;
  FC_TRY(cp_fftconv_workspace_size(plan, &need));
  if (!ws || ws_bytes < need) return CP_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return CP_ERR_ALIGNMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  float2* spec = static_cast<float2*>(ws);
  float2* wbuf = reinterpret_cast<float2*>(static_cast<char*>(ws) + spec_bytes(c));
  float2* tw2l = reinterpret_cast<float2*>(static_cast<char*>(ws) + spec_bytes(c) + w_bytes(c));
  float2* twc = tw2l + align256(8ull * 2 * c.L) / 8;
  fftconv_twiddle_kernel<<<static_cast<unsigned>((2 * c.L + 255) / 256), 256, 0, st>>>(tw2l, c.L, twc, plan->c);
  if (cudaGetLastError() != cudaSuccess) return CP_ERR_CUDA;
  const int Q = 2 * c.n_cp;
  const size_t smem = fftconv_smem_bytes(plan->c, c.n_cp);
  if (cudaFuncSetAttribute(fftconv_slice_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(fftconv_slice_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess)
    return CP_ERR_CUDA;

  FftParams p{};
  p.D = c.D;
  p.L = c.L;
  p.N = c.n_cp;
  p.c = plan->c;
  p.logc = plan->logc;
  p.spec = spec;
  p.w = wbuf;
  p.tw2l = tw2l;
  p.twc = twc;
  // filter spectra: one CTA per (channel, slice)
  p.src = static_cast<const __nv_bfloat16*>(h->data);
  p.s_sb = 0;
  p.s_sd = h->stride[0];
  fftconv_slice_kernel<0><<<static_cast<unsigned>(static_cast<int64_t>(c.D) * Q), kFftThreads, smem, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return CP_ERR_CUDA;
  // signal slices: one CTA per (row, slice), the 2N slices of a row adjacent (its x stays in L2)
  p.src = static_cast<const __nv_bfloat16*>(x->data);
  p.s_sb = x->stride[0];
  p.s_sd = x->stride[1];
  fftconv_slice_kernel<1><<<static_cast<unsigned>(static_cast<int64_t>(c.B) * c.D * Q), kFftThreads, smem, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return CP_ERR_CUDA;
  // cross-rank inverse into y
  FftInvParams ip{};
  ip.w = wbuf;
  ip.y = static_cast<__nv_bfloat16*>(y->data);
  ip.y_sb = y->stride[0];
  ip.y_sd = y->stride[1];
  ip.D = c.D;
  ip.L = c.L;
  ip.c = plan->c;
  const int rows = c.B * c.D;
  cudaError_t e;
  switch (c.n_cp) {
    case 1: e = launch_inverse<1>(ip, plan->c, rows, st); break;
    case 2: e = launch_inverse<2>(ip, plan->c, rows, st); break;
    case 4: e = launch_inverse<4>(ip, plan->c, rows, st); break;
    case 8: e = launch_inverse<8>(ip, plan->c, rows, st); break;
    case 16: e = launch_inverse<16>(ip, plan->c, rows, st); break;
    default: e = launch_inverse<32>(ip, plan->c, rows, st); break;
  }
  return e == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

cp_status_t cp_fftconv_cost(const cp_fftconv_plan_t* plan, double* hbm_bytes, double* flops) {
  if (!plan || !hbm_bytes || !flops) return CP_ERR_INVALID_ARG;
  const cp_fftconv_config_t& c = plan->cfg;
  const double B = c.B, D = c.D, L = c.L, N = c.n_cp, Q = 2.0 * c.n_cp, cl = plan->c, lg = plan->logc;
  // filter: h read, spectra written; signal: x and the spectra read, slices written;
  // inverse: slices read, y written
  *hbm_bytes = 2 * D * L + 16 * D * L + B * (2 * D * L + 16 * D * L + 16 * D * L) + B * (16 * D * L + 2 * D * L);
  const double cross = cl * (4 * N + 6);           // N real x complex MACs and a twiddle per sample
  const double fft = 5 * cl * lg;                  // c/2 log2 c butterflies of 10 flops
  *flops = D * Q * (cross + fft) + B * D * Q * (cross + 2 * fft + 12 * cl) + B * D * 8 * N * L;
  return CP_OK;
}

}  // extern "C"
