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

// Shared-memory index of element i: within each row of 16 float2 (128 bytes, one pass over
// the banks) the position is XORed with 5 x the row number.  A bijection inside every row, so
// no padding; chosen by enumerating the half-warp access patterns of every pass (radix 8 at
// spans 1024/128/16 or 256/32/4, radix 4 at spans 4/1, the cross stage's 8-sample runs, the
// contiguous reads): each lands on 16 distinct bank pairs.
__device__ __forceinline__ int pidx(int i) { return i ^ (((i >> 4) * 5) & 15); }

// The twiddle of stage t (span s 2^t) for group element k: w_2hs^(j0 + s m) = base * w_(2^(t+1))^m,
// m = k mod 2^t, base = w_2hs^j0 (one table read per stage).
template <int T>
__device__ __forceinline__ float2 stage_tf(float2 base, int k) {
  if (T == 0) return base;
  if (T == 1) return (k & 1) ? rot<1, 1>(base) : base;
  const int m = k & 3;
  return m == 0 ? base : m == 1 ? rot<2, 1>(base) : m == 2 ? rot<2, 2>(base) : rot<2, 3>(base);
}

// bases[t] = w_(2 s 2^t)^j0: the pass's table holds the largest-span root per j0 (consecutive
// j0 in consecutive entries: no bank conflicts across a warp), the others are its squares.
template <int R>
__device__ __forceinline__ void stage_bases(float2 (&bases)[R], const float2* tp, int j0) {
  bases[R - 1] = tp[j0];
#pragma unroll
  for (int t = R - 1; t > 0; --t) bases[t - 1] = cmul(bases[t], bases[t]);
}

template <int R>
__device__ __forceinline__ void dif_stages(float2 (&v)[1 << R], const float2 (&bases)[R]) {
#pragma unroll
  for (int t = R - 1; t >= 0; --t) {
    const float2 base = bases[t];
#pragma unroll
    for (int k = 0; k < (1 << R); ++k) {
      if (k & (1 << t)) continue;
      const float2 tf = t == 0 ? stage_tf<0>(base, k) : t == 1 ? stage_tf<1>(base, k) : stage_tf<2>(base, k);
      const float2 u = v[k], w = v[k + (1 << t)];
      v[k] = cadd(u, w);
      v[k + (1 << t)] = cmul(csub(u, w), tf);
    }
  }
}

// The mirror: decimation-in-time stages with conjugate twiddles, each the inverse of the DiF
// butterfly times 2: (X, Y) -> (X + Y conj(w), X - Y conj(w)).
template <int R>
__device__ __forceinline__ void dit_stages(float2 (&v)[1 << R], const float2 (&bases)[R]) {
#pragma unroll
  for (int t = 0; t < R; ++t) {
    const float2 base = bases[t];
#pragma unroll
    for (int k = 0; k < (1 << R); ++k) {
      if (k & (1 << t)) continue;
      const float2 tf = t == 0 ? stage_tf<0>(base, k) : t == 1 ? stage_tf<1>(base, k) : stage_tf<2>(base, k);
      const float2 u = v[k], w = cmul_conj(v[k + (1 << t)], tf);
      v[k] = cadd(u, w);
      v[k + (1 << t)] = csub(u, w);
    }
  }
}

// A pass of R radix-2 stages over spans s 2^(R-1) .. s (s = 2^logs).  Group g holds the 2^R
// elements i0 + k s, i0 = (g - j0) 2^R + j0, j0 = g mod s.  KIND: 0 DiF in shared memory;
// 1 DiT in shared memory; 2 DiF whose result goes to global `out` (the filter's spectrum, last
// pass); 3 the middle of the signal's transform (s = 1): the last DiF pass, the spectral
// product with `hq`, and the first DiT pass, in registers; 4 DiT whose result, times the
// conjugate twiddle w_2L^(-n q) = conj(lo[n mod C1] hi[n / C1]), goes to global `out`.
template <int R, int KIND>
__device__ __forceinline__ void fft_pass(float2* a, const float2* tp, int logc, int logs, float2* out,
                                         const float2* hq, const float2* lo, const float2* hi, int logc1) {
  constexpr int E = 1 << R;
  const int c = 1 << logc, s = 1 << logs;
  const int groups = c >> R;
  for (int g = threadIdx.x; g < groups; g += kFftThreads) {
    const int j0 = g & (s - 1);
    const int i0 = (g - j0) * E + j0;
    float2 v[E];
#pragma unroll
    for (int k = 0; k < E; ++k) v[k] = a[pidx(i0 + k * s)];
    float2 bases[R];
    stage_bases<R>(bases, tp, j0);
    if (KIND == 0 || KIND == 2 || KIND == 3) dif_stages<R>(v, bases);
    if (KIND == 3) {
      // s = 1: the group's elements are contiguous in the spectrum's storage order
#pragma unroll
      for (int k = 0; k < E; ++k) v[k] = cmul(v[k], hq[i0 + k]);
    }
    if (KIND == 1 || KIND == 3 || KIND == 4) dit_stages<R>(v, bases);
    if (KIND == 2) {
#pragma unroll
      for (int k = 0; k < E; ++k) out[i0 + k * s] = v[k];
    } else if (KIND == 4) {
      const int m1 = (1 << logc1) - 1;
#pragma unroll
      for (int k = 0; k < E; ++k) {
        const int n = i0 + k * s;
        out[n] = cmul_conj(v[k], cmul(lo[n & m1], hi[n >> logc1]));
      }
    } else {
#pragma unroll
      for (int k = 0; k < E; ++k) a[pidx(i0 + k * s)] = v[k];
    }
  }
}

template <int KIND>
__device__ __forceinline__ void run_pass(int r, float2* a, const float2* tp, int logc, int logs, float2* out,
                                         const float2* hq, const float2* lo, const float2* hi, int logc1) {
  if (r == 1) fft_pass<1, KIND>(a, tp, logc, logs, out, hq, lo, hi, logc1);
  else if (r == 2) fft_pass<2, KIND>(a, tp, logc, logs, out, hq, lo, hi, logc1);
  else fft_pass<3, KIND>(a, tp, logc, logs, out, hq, lo, hi, logc1);
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

// MODE 0: the filter's spectra H_q -> p.spec.  MODE 1: the signal's w_q -> p.w.
template <int MODE>
__global__ void __launch_bounds__(kFftThreads, 2) fftconv_slice_kernel(const FftParams p) {
  extern __shared__ float2 fsm[];
  const int Q = 2 * p.N;
  const int row = blockIdx.x / Q;
  const int q = blockIdx.x - row * Q;
  const int c = p.c;
  const int logc1 = p.logc < 6 ? p.logc : 6;          // n = n_lo + C1 n_hi, C1 = min(c, 64)
  const int c1 = 1 << logc1;
  int radix[5], toff[6];
  const int np = fft_passes(p.logc, radix);
  float2* a = fsm;                           // c values at pidx(i)
  float2* tpass = fsm + c;                   // per pass p: w_(s_p 2^R_p)^j0, j0 < s_p (<= c / 4 + 1 in all)
  {
    int logs = p.logc, off = 0;
    for (int i = 0; i < np; ++i) {
      logs -= radix[i];
      toff[i] = off;
      // w_(s 2^R)^j0 = w_c^(j0 c / (s 2^R)); s = 2^logs
      for (int j0 = threadIdx.x; j0 < (1 << logs); j0 += kFftThreads)
        tpass[off + j0] = p.twc[j0 << (p.logc - logs - radix[i])];
      off += 1 << logs;
    }
    toff[np] = off;
  }
  float2* cf = tpass + c / 4 + 16;           // N cross-rank coefficients w_2N^(r q)
  float2* lo = cf + kFftMaxN;                // w_2L^(u q), u < C1
  float2* hi = lo + 64;                      // w_2L^(C1 v q), v < c / C1 (<= 128)

  // w_2N^(r q) = w_2L^((r q mod 2N) c); lo/hi: every index below 2L (u q < C1 2N <= 2L, C1 v q < c 2N)
  for (int r = threadIdx.x; r < p.N; r += kFftThreads) cf[r] = p.tw2l[((r * q) % Q) * c];
  if (threadIdx.x < c1) lo[threadIdx.x] = p.tw2l[threadIdx.x * q];
  for (int v = threadIdx.x; v < (c >> logc1); v += kFftThreads) hi[v] = p.tw2l[(v << logc1) * q];
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
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int n = n0 + e;
      if (n < c) a[pidx(n)] = cmul(acc[e], cmul(lo[n & (c1 - 1)], hi[n >> logc1]));
    }
  }
  __syncthreads();

  const long long slice = (static_cast<long long>(row) * Q + q) * c;
  int logs = p.logc;
  for (int i = 0; i + 1 < np; ++i) {
    logs -= radix[i];
    run_pass<0>(radix[i], a, tpass + toff[i], p.logc, logs, nullptr, nullptr, nullptr, nullptr, 0);
    __syncthreads();
  }
  // logs is now radix[np-1]: the last pass has s = 1
  if (MODE == 0) {
    run_pass<2>(radix[np - 1], a, tpass + toff[np - 1], p.logc, 0, p.spec + slice, nullptr, nullptr, nullptr, 0);
    return;
  }
  const float2* hq = p.spec + (static_cast<long long>(ch) * Q + q) * c;
  run_pass<3>(radix[np - 1], a, tpass + toff[np - 1], p.logc, 0, nullptr, hq, nullptr, nullptr, 0);
  __syncthreads();
  logs = radix[np - 1];
  for (int i = np - 2; i >= 1; --i) {
    run_pass<1>(radix[i], a, tpass + toff[i], p.logc, logs, nullptr, nullptr, nullptr, nullptr, 0);
    logs += radix[i];
    __syncthreads();
  }
  if (np >= 2) {
    // the last inverse pass writes w_q(n) = w_2L^(-n q) * (local inverse) straight to global
    run_pass<4>(radix[0], a, tpass + toff[0], p.logc, logs, p.w + slice, nullptr, lo, hi, logc1);
  } else {
    for (int n = threadIdx.x; n < c; n += kFftThreads)
      p.w[slice + n] = cmul_conj(a[pidx(n)], cmul(lo[n & (c1 - 1)], hi[n >> logc1]));
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
  return (static_cast<size_t>(c) + c / 4 + 16 + kFftMaxN + 64 + 128) * sizeof(float2);
}

}  // namespace cpattn
