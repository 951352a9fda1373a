// fftconv_kernel.cuh — causal long convolution by the distributed radix-N DiF FFT
// ("05. 長系列の分散学習（Context Parallelism）" §4 FFT 畳み込み: the convolution theorem, the DiF
// butterfly X = x + y, Y = (x - y) w^j, and the radix-N_cp split in which every rank keeps its
// shard and the spectrum stays in its decimated order).
//
// With x held in N contiguous shards of c = L / N samples and the 2L-point transform that the
// causal (linear) convolution needs, the first DiF stage is radix-2N over the N data shards
// (the N zero shards of the padding add nothing).  Frequency slice q in [0, 2N) holds the
// frequencies 2N k1 + q:
//
//   z_q(n)  = w_2L^(n q) * sum_{r<N} x(n + c r) w_2N^(r q)          cross-rank stage
//   Z_q(k1) = sum_n z_q(n) w_c^(n k1)                                local c-point DFT
//   P_q     = Z_q . H_q                                              spectral product
//   w_q(n)  = w_2L^(-n q) * sum_k1 P_q(k1) w_c^(-n k1)               local inverse DFT
//   y(n + c r) = (1 / 2L) Re sum_{q<2N} w_2N^(-r q) w_q(n)           cross-rank inverse
//
// One CTA per (row, q) runs the cross-rank stage, the local forward FFT, the product and the
// local inverse FFT in shared memory; a second kernel runs the cross-rank inverse.  The local
// forward FFT is decimation in frequency (natural order in, bit-reversed out) and the inverse
// decimation in time with conjugate twiddles (bit-reversed in, natural out): the spectra, and
// the filter's spectra they are multiplied with, stay in the bit-reversed order and are never
// permuted.  Passes of up to 3 radix-2 stages (a radix-8 group per thread) run in registers
// between shared-memory passes.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace cpattn {

constexpr int kFftThreads = 512;
constexpr int kFftMaxC = 8192;     // local transform length: c complex fp32 (+ padding) + c/2 twiddles
constexpr int kFftMaxN = 32;       // ranks: 2N <= 64 frequency slices

struct FftParams {
  const __nv_bfloat16* src;  // rows of x [B, D, L] (signal) or h [D, L] (filter)
  long long s_sb, s_sd;      // strides of src (elements); the sequence is innermost
  int D, L, N, c, logc;
  float2* spec;              // filter spectra [D][2N][c], local order of the forward FFT
  float2* w;                 // signal: w_q(n), [rows][2N][c]
  const float2* tw2l;        // w_2L^m, m < 2L
  const float2* twc;         // w_c^m, m < c / 2
};

__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
__device__ __forceinline__ float2 cmul_conj(float2 a, float2 b) {  // a * conj(b)
  return make_float2(fmaf(a.x, b.x, a.y * b.y), fmaf(a.y, b.x, -a.x * b.y));
}
__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }

// exp(-i pi t) = (cos pi t, -sin pi t).  sincospif takes its argument in units of pi, so the
// dyadic arguments used here (m / 2^k) reach it without rounding.
__device__ __forceinline__ float2 unit_root(float t) {
  float s, c;
  sincospif(t, &s, &c);
  return make_float2(c, -s);
}

// The twiddle tables of one call: w_2L^m for m < 2L and w_c^m for m < c/2 (every CTA reads
// them from L2 instead of evaluating sines).
__global__ void fftconv_twiddle_kernel(float2* tw2l, int L, float2* twc, int c) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < 2 * L) tw2l[i] = unit_root(static_cast<float>(i) / L);
  if (i < c / 2) twc[i] = unit_root(2.0f * i / c);
}

// z * w_M^m for the roots a radix-8 group needs (M = 2^(t+1) <= 8, m < 2^t), exactly:
// w_2^0 = w_4^0 = w_8^0 = 1, w_4^1 = w_8^2 = -i, w_8^1 = (1 - i)/sqrt 2, w_8^3 = -(1 + i)/sqrt 2.
template <int T, int M>
__device__ __forceinline__ float2 rot(float2 z) {
  constexpr float kHalfSqrt2 = 0.70710678118654752440f;
  if constexpr (M == 0) {
    return z;
  } else if constexpr ((T == 1 && M == 1) || (T == 2 && M == 2)) {
    return make_float2(z.y, -z.x);
  } else if constexpr (T == 2 && M == 1) {
    return make_float2((z.x + z.y) * kHalfSqrt2, (z.y - z.x) * kHalfSqrt2);
  } else {  // T == 2 && M == 3
    return make_float2((z.y - z.x) * kHalfSqrt2, -(z.x + z.y) * kHalfSqrt2);
  }
}

// Shared-memory index of element i: one float2 of padding per 16 keeps the power-of-two
// strides of the passes off a single bank.
__device__ __forceinline__ int pidx(int i) { return i + (i >> 4); }

template <int T, int K>
__device__ __forceinline__ float2 stage_twiddle(float2 base) {
  return rot<T, K & ((1 << T) - 1)>(base);
}

// One pass of R (<= 3) decimation-in-frequency radix-2 stages over spans s*2^(R-1), ..., s
// (largest first).  Group g holds the 2^R elements i0 + k s, i0 = (g / s) s 2^R + (g mod s).
// In the stage of span hs = s 2^t the pair (k, k + 2^t) takes w_2hs^(j0 + s m), m = k mod 2^t,
// = w_2hs^j0 * w_(2^(t+1))^m: one table read per stage, times an exact root.
template <int R>
__device__ __forceinline__ void dif_pass(float2* a, const float2* tw, int logc, int logs) {
  const int c = 1 << logc, s = 1 << logs;
  constexpr int E = 1 << R;
  const int groups = c >> R;
  for (int g = threadIdx.x; g < groups; g += kFftThreads) {
    const int j0 = g & (s - 1);
    const int i0 = (g - j0) * E + j0;
    float2 v[E];
#pragma unroll
    for (int k = 0; k < E; ++k) v[k] = a[pidx(i0 + k * s)];
#pragma unroll
    for (int t = R - 1; t >= 0; --t) {
      const float2 base = tw[j0 << (logc - logs - t - 1)];   // w_c^(j0 c / (2 s 2^t))
#pragma unroll
      for (int k = 0; k < E; ++k) {
        if (k & (1 << t)) continue;
        const float2 u = v[k], w = v[k + (1 << t)];
        float2 tf;
        if (t == 0) tf = base;
        else if (t == 1) tf = (k & 1) ? rot<1, 1>(base) : base;
        else tf = (k & 3) == 0 ? base : (k & 3) == 1 ? rot<2, 1>(base) : (k & 3) == 2 ? rot<2, 2>(base) : rot<2, 3>(base);
        v[k] = cadd(u, w);
        v[k + (1 << t)] = cmul(csub(u, w), tf);
      }
    }
#pragma unroll
    for (int k = 0; k < E; ++k) a[pidx(i0 + k * s)] = v[k];
  }
}

// The mirror: decimation-in-time stages of spans s, ..., s*2^(R-1) with conjugate twiddles,
// each the inverse of the DiF butterfly times 2: (X, Y) -> (X + Y conj(w), X - Y conj(w)).
template <int R>
__device__ __forceinline__ void dit_pass(float2* a, const float2* tw, int logc, int logs) {
  const int c = 1 << logc, s = 1 << logs;
  constexpr int E = 1 << R;
  const int groups = c >> R;
  for (int g = threadIdx.x; g < groups; g += kFftThreads) {
    const int j0 = g & (s - 1);
    const int i0 = (g - j0) * E + j0;
    float2 v[E];
#pragma unroll
    for (int k = 0; k < E; ++k) v[k] = a[pidx(i0 + k * s)];
#pragma unroll
    for (int t = 0; t < R; ++t) {
      const float2 base = tw[j0 << (logc - logs - t - 1)];   // w_c^(j0 c / (2 s 2^t))
#pragma unroll
      for (int k = 0; k < E; ++k) {
        if (k & (1 << t)) continue;
        float2 tf;
        if (t == 0) tf = base;
        else if (t == 1) tf = (k & 1) ? rot<1, 1>(base) : base;
        else tf = (k & 3) == 0 ? base : (k & 3) == 1 ? rot<2, 1>(base) : (k & 3) == 2 ? rot<2, 2>(base) : rot<2, 3>(base);
        const float2 u = v[k], w = cmul_conj(v[k + (1 << t)], tf);
        v[k] = cadd(u, w);
        v[k + (1 << t)] = csub(u, w);
      }
    }
#pragma unroll
    for (int k = 0; k < E; ++k) a[pidx(i0 + k * s)] = v[k];
  }
}

// Split log2(c) stages into passes of at most 3 (as even as possible); forward: largest spans
// first; inverse: the same passes in reverse order.
__device__ __forceinline__ int fft_passes(int logc, int* radix) {
  const int np = (logc + 2) / 3;
  int left = logc;
  for (int p = 0; p < np; ++p) {
    radix[p] = (left + (np - p) - 1) / (np - p);
    left -= radix[p];
  }
  return np;
}

__device__ __forceinline__ void run_dif(float2* a, const float2* tw, int logc, int r, int logs) {
  if (r == 1) dif_pass<1>(a, tw, logc, logs);
  else if (r == 2) dif_pass<2>(a, tw, logc, logs);
  else dif_pass<3>(a, tw, logc, logs);
}
__device__ __forceinline__ void run_dit(float2* a, const float2* tw, int logc, int r, int logs) {
  if (r == 1) dit_pass<1>(a, tw, logc, logs);
  else if (r == 2) dit_pass<2>(a, tw, logc, logs);
  else dit_pass<3>(a, tw, logc, logs);
}

// MODE 0: the filter's spectra H_q -> p.spec.  MODE 1: the signal's w_q -> p.w.
template <int MODE>
__global__ void __launch_bounds__(kFftThreads, 2) fftconv_slice_kernel(const FftParams p) {
  extern __shared__ float2 fsm[];
  const int Q = 2 * p.N;
  const int row = blockIdx.x / Q;
  const int q = blockIdx.x - row * Q;
  const int c = p.c;
  float2* a = fsm;                           // c values at pidx(i)
  float2* tw = fsm + c + c / 16;             // c / 2 twiddles w_c^m
  float2* cf = tw + c / 2;                   // N cross-rank coefficients w_2N^(r q)
  float2* ew = cf + kFftMaxN;                // w_2L^(e q), e < 8

#pragma unroll 8
  for (int m = threadIdx.x; m < c / 2; m += kFftThreads) tw[m] = p.twc[m];
  // w_2N^(r q) = w_2L^((r q mod 2N) c); ew[e] = w_2L^(e q)
  for (int r = threadIdx.x; r < p.N; r += kFftThreads) cf[r] = p.tw2l[((r * q) % Q) * c];
  if (threadIdx.x < 8) ew[threadIdx.x] = p.tw2l[(threadIdx.x * q) % (2 * p.L)];
  __syncthreads();

  // cross-rank stage, 8 consecutive samples per thread (16-byte loads of every shard):
  // z_q(n) = w_2L^(n q) sum_r x(n + c r) w_2N^(r q)
  const int b = row / p.D, ch = row - (row / p.D) * p.D;
  const __nv_bfloat16* xr = p.src + b * p.s_sb + ch * p.s_sd;
  const bool vec = (c % 8 == 0) && ((reinterpret_cast<uintptr_t>(xr) & 15) == 0);
  for (int n0 = threadIdx.x * 8; n0 < c; n0 += kFftThreads * 8) {
    float2 acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = make_float2(0.f, 0.f);
    // four shards' loads in flight before their products (the loop bound is a runtime N)
    for (int r0 = 0; r0 < p.N; r0 += 4) {
      uint4 raw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = r0 + u;
        if (r >= p.N) {
          raw[u] = make_uint4(0, 0, 0, 0);
        } else if (vec) {
          raw[u] = *reinterpret_cast<const uint4*>(xr + r * c + n0);
        } else {
          uint16_t e8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) e8[e] = (n0 + e < c) ? __bfloat16_as_ushort(xr[r * c + n0 + e]) : 0;
          raw[u] = make_uint4(e8[0] | (e8[1] << 16), e8[2] | (e8[3] << 16), e8[4] | (e8[5] << 16), e8[6] | (e8[7] << 16));
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (r0 + u >= p.N) break;
        const float2 cr = cf[r0 + u];
        const __nv_bfloat162* pr = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(pr[e]);
          acc[2 * e].x = fmaf(f.x, cr.x, acc[2 * e].x);
          acc[2 * e].y = fmaf(f.x, cr.y, acc[2 * e].y);
          acc[2 * e + 1].x = fmaf(f.y, cr.x, acc[2 * e + 1].x);
          acc[2 * e + 1].y = fmaf(f.y, cr.y, acc[2 * e + 1].y);
        }
      }
    }
    // w_2L^(n q) = w_2L^(n0 q) w_2L^(e q); n0 q < 2N c = 2L
    const float2 t0 = p.tw2l[n0 * q];
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (n0 + e < c) a[pidx(n0 + e)] = cmul(acc[e], cmul(t0, ew[e]));
  }
  __syncthreads();

  int radix[5];
  const int np = fft_passes(p.logc, radix);
  int logs = p.logc;
  for (int i = 0; i < np; ++i) {
    logs -= radix[i];
    run_dif(a, tw, p.logc, radix[i], logs);
    __syncthreads();
  }

  const long long slice = (static_cast<long long>(row) * Q + q) * c;
  if (MODE == 0) {
    for (int k = threadIdx.x; k < c; k += kFftThreads) p.spec[slice + k] = a[pidx(k)];
    return;
  }
  const float2* hq = p.spec + (static_cast<long long>(ch) * Q + q) * c;
  for (int k0 = threadIdx.x; k0 < c; k0 += 4 * kFftThreads) {
    float2 hv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int k = k0 + u * kFftThreads;
      hv[u] = k < c ? hq[k] : make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int k = k0 + u * kFftThreads;
      if (k < c) a[pidx(k)] = cmul(a[pidx(k)], hv[u]);
    }
  }
  __syncthreads();
  logs = 0;
  for (int i = np - 1; i >= 0; --i) {
    run_dit(a, tw, p.logc, radix[i], logs);
    logs += radix[i];
    __syncthreads();
  }
  // w_q(n) = w_2L^(-n q) * (local inverse)
  for (int m0 = threadIdx.x; m0 < c; m0 += 4 * kFftThreads) {
    float2 tv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int n = m0 + u * kFftThreads;
      tv[u] = n < c ? p.tw2l[(n & ~7) * q] : make_float2(1.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int n = m0 + u * kFftThreads;
      if (n < c) p.w[slice + n] = cmul_conj(a[pidx(n)], cmul(tv[u], ew[n & 7]));
    }
  }
}

// Cross-rank inverse: y(n + c r) = (1 / 2L) Re sum_q w_2N^(-r q) w_q(n), rounded to bf16.
struct FftInvParams {
  const float2* w;           // [rows][2N][c]
  __nv_bfloat16* y;          // [B, D, L]
  long long y_sb, y_sd;
  int D, L, c;
};

template <int NN>
__global__ void __launch_bounds__(kFftThreads) fftconv_inverse_kernel(const FftInvParams p) {
  constexpr int Q = 2 * NN;
  __shared__ float2 rt[Q];  // w_2N^(-m) = exp(+pi i m / N), m < 2N
  for (int m = threadIdx.x; m < Q; m += kFftThreads) {
    const float2 u = unit_root(static_cast<float>(m) / NN);
    rt[m] = make_float2(u.x, -u.y);
  }
  __syncthreads();
  const int row = blockIdx.y;
  const int n = blockIdx.x * kFftThreads + threadIdx.x;
  if (n >= p.c) return;
  const float2* wr = p.w + static_cast<long long>(row) * Q * p.c + n;
  float acc[NN];
#pragma unroll
  for (int r = 0; r < NN; ++r) acc[r] = 0.f;
#pragma unroll 4
  for (int q = 0; q < Q; ++q) {
    const float2 wq = wr[static_cast<long long>(q) * p.c];
#pragma unroll
    for (int r = 0; r < NN; ++r) {
      const float2 t = rt[(r * q) & (Q - 1)];
      acc[r] = fmaf(wq.x, t.x, fmaf(-wq.y, t.y, acc[r]));
    }
  }
  const int b = row / p.D, ch = row - (row / p.D) * p.D;
  __nv_bfloat16* yr = p.y + b * p.y_sb + ch * p.y_sd;
  const float inv = 1.0f / (2.0f * p.L);
#pragma unroll
  for (int r = 0; r < NN; ++r) yr[r * p.c + n] = __float2bfloat16_rn(acc[r] * inv);
}

__host__ __device__ constexpr size_t fftconv_smem_bytes(int c, int N) {
  return (static_cast<size_t>(c) + c / 16 + c / 2 + kFftMaxN + 8) * sizeof(float2);
}

}  // namespace cpattn
