/*
 * cp_fftconv.h — C ABI of libcpattn.so, long-filter operator: the causal convolution of a
 * context-parallel sequence with a filter as long as the sequence, by the distributed FFT,
 * all virtual ranks on one B200.
 *
 * Source: "05. 長系列の分散学習（Context Parallelism）", homemade-llm StripedHyena 2 series,
 * §4 (FFT 畳み込み：周波数領域の魔法): the convolution theorem x * h = F^-1(F(x) . F(h)); the DFT
 * y(k) = sum_j x(j) w_l^(jk), w_l = exp(-2 pi i / l); the decimation-in-frequency butterfly
 * X = x + y, Y = (x - y) w^j; and its distributed form: the DiF split keeps every shard on its
 * rank, a DiF forward and the mirrored inverse bring the result back in the input's shard
 * layout without an all-to-all, and N_cp > 2 uses radix N = N_cp.
 *
 *   y[b, c, t] = sum_{k<=t} h[c, k] * x[b, c, t - k],   t < L
 *
 * Readings taken: the causal (linear) convolution needs a 2L-point transform, so the first DiF
 * stage is radix 2N over the N data shards and N zero shards; virtual rank r of the sequence
 * holds samples [r c, (r+1) c), c = L / N; frequency slice q in [0, 2N) holds the frequencies
 * 2N k + q of the padded transform (virtual rank r the slices 2r and 2r + 1, i.e. its
 * frequencies k = r mod N of each half); the spectra stay in this decimated order.  Arithmetic
 * in fp32 complex (twiddles from sincospif with exact arguments); x, h, y bf16, y rounded once to
 * nearest even.
 *
 * Conventions are those of cp_attn.h.  Layouts: x, y [B, D, L] and h [D, L] with the sequence
 * innermost (stride 1), other strides free, 2-byte aligned.  Limits: N = n_cp a power of two
 * <= 32, c = L / N a power of two in [4, 8192] (a rank's slice transform stays in one CTA's
 * shared memory).  The workspace holds the filter's spectra [D, 2N, c], the signal's slice
 * results [B, D, 2N, c] (complex fp32, 16 bytes per sample each) and the twiddle tables
 * w_2L^m (m < 2L) and w_c^m (m < c/2).
 */
#ifndef CP_FFTCONV_H
#define CP_FFTCONV_H

#include "cp_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int B, D, L; /* batch, channels, sequence length (= filter length)                     */
  int n_cp;    /* virtual ranks of contiguous shards of c = L / n_cp samples            */
} cp_fftconv_config_t;

typedef struct cp_fftconv_plan cp_fftconv_plan_t;

/* Validate and create a plan (host only).  CP_ERR_INVALID_ARG for a bad shape; CP_ERR_UNSUPPORTED
 * for n_cp or c outside the limits above. */
cp_status_t cp_fftconv_plan(const cp_fftconv_config_t* cfg, cp_fftconv_plan_t** out);
void cp_fftconv_plan_destroy(cp_fftconv_plan_t* plan);

/* Workspace bytes of cp_fftconv_fwd: 16 * D * L + 16 * B * D * L + 16 * L + 4 * c, plus
 * alignment. */
cp_status_t cp_fftconv_workspace_size(const cp_fftconv_plan_t* plan, size_t* bytes);

/* y = x * h over the whole sequence, every virtual rank at once: the filter's spectra, the
 * signal's cross-rank DiF stage + local FFT + spectral product + local inverse FFT per frequency
 * slice, and the cross-rank inverse into the contiguous shards.  x, y [B, D, L] (distinct);
 * h [D, L]; ws of at least cp_fftconv_workspace_size bytes, 256-byte aligned. */
cp_status_t cp_fftconv_fwd(const cp_fftconv_plan_t* plan, const cp_tensor_t* x, const cp_tensor_t* h,
                           cp_tensor_t* y, void* ws, size_t ws_bytes, void* stream);

/* Work of one cp_fftconv_fwd: bytes its three passes move through HBM (x and h read; the
 * spectra and the slice results written and read back; y written) and real floating-point
 * operations of the radix-2 transforms, products and cross-rank sums. */
cp_status_t cp_fftconv_cost(const cp_fftconv_plan_t* plan, double* hbm_bytes, double* flops);

#ifdef __cplusplus
}
#endif

#endif /* CP_FFTCONV_H */
