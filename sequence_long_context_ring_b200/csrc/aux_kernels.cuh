// aux_kernels.cuh — HBM-bound kernels: Ulysses re-layout, step-wise LSE merge, and the
// backward's D = rowsum(dO * O) preprocess.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace cpattn {

// ---- Ulysses all-to-all on one GPU -------------------------------------------------------
// Swaps axes 1 and 2 of a [B, X, Y, d] view: out[b, y, x, :] = in[b, x, y, :].  Rows of d
// elements are contiguous on both sides, so the copy moves whole 16-byte vectors.  A block
// owns a run of consecutive OUTPUT rows (fully sequential writes): it first resolves each row's
// source and destination offsets once (the only divisions, and the split's rank-row map, run
// per row, not per vector), then every thread moves up to kPermVecPerThread vectors whose loads
// are all issued before the first store, so several reads per thread are in flight.
// ("05. 長系列の分散学習（Context Parallelism）" §2: the re-layout [D, L/N_cp] -> [H/N_cp, L];
// "Ulyssesシーケンス並列化の核心" steps 2 and 4.)
struct PermuteParams {
  const uint4* in;
  uint4* out;
  long long n_rows;      // B * Y * X output rows
  int vec_per_row;       // d * elem_bytes / 16
  int vec_shift;         // log2(vec_per_row) when it is a power of two, else -1
  int rows_per_block;    // output rows per block (<= kPermMaxRows)
  int X, Y;              // in is [B, X, Y, row]; out is [B, Y, X, row]
  long long in_sb, in_sx, in_sy;     // strides in 16-byte vectors
  long long out_sb, out_sy, out_sx;
  // Two-shard splits: the sequence axis of the rank-major side is in rank order (rank s's
  // rows at [s*c, (s+1)*c): its first shard, then its second), the other side in position
  // order.  remap 1: the output's x is a position, the input's x its rank-major row;
  // remap 2: the output's y is a rank-major row, the input's y its position.  0: none.
  int remap, split, n_ranks, shard;  // split 1 zig-zag (shards r, 2N-1-r), 2 striped (r, r+N)
};

// Rank-major row of global position pos under a two-shard split (split 1 zig-zag, 2
// striped; n ranks, shard length w = c / 2).
__device__ __forceinline__ int split_rank_row(int pos, int split, int n, int w) {
  const int sh = pos / w, off = pos - sh * w;
  const int hi = sh >= n;  // the rank's second shard
  const int r = hi ? (split == 1 ? 2 * n - 1 - sh : sh - n) : sh;
  return r * 2 * w + hi * w + off;
}
__device__ __forceinline__ int rank_row_of_pos(const PermuteParams& p, int pos) {
  return split_rank_row(pos, p.split, p.n_ranks, p.shard);
}
// Global position of rank-major row u.
__device__ __forceinline__ int pos_of_rank_row(const PermuteParams& p, int u) {
  const int w = p.shard, n = p.n_ranks;
  const int r = u / (2 * w), t = u - r * 2 * w;
  const int hi = t >= w;
  const int sh = hi ? (p.split == 1 ? 2 * n - 1 - r : r + n) : r;
  return sh * w + (t - hi * w);
}

constexpr int kPermThreads = 256;
constexpr int kPermVecPerThread = 4;                                  // per pass of the block
constexpr int kPermVecPerPass = kPermThreads * kPermVecPerThread;     // 1024 vectors (16 KB)
constexpr int kPermMaxRows = 256;

__global__ void __launch_bounds__(kPermThreads) permute_rows_kernel(const PermuteParams p) {
  __shared__ long long src_row[kPermMaxRows];
  __shared__ long long dst_row[kPermMaxRows];
  const long long row0 = static_cast<long long>(blockIdx.x) * p.rows_per_block;
  for (int r = threadIdx.x; r < p.rows_per_block; r += kPermThreads) {
    const long long R = row0 + r;   // output row in (b, y, x) order
    long long src = -1, dst = -1;
    if (R < p.n_rows) {
      const long long by = R / p.X;
      const int x = static_cast<int>(R - by * p.X);
      const long long b = by / p.Y;
      const int y = static_cast<int>(by - b * p.Y);
      const int xi = p.remap == 1 ? rank_row_of_pos(p, x) : x;
      const int yi = p.remap == 2 ? pos_of_rank_row(p, y) : y;
      src = b * p.in_sb + xi * p.in_sx + yi * p.in_sy;
      dst = b * p.out_sb + y * p.out_sy + x * p.out_sx;
    }
    src_row[r] = src;
    dst_row[r] = dst;
  }
  __syncthreads();
  const int total = p.rows_per_block * p.vec_per_row;
  for (int base = 0; base < total; base += kPermVecPerPass) {
    uint4 v[kPermVecPerThread];
    long long dst[kPermVecPerThread];
#pragma unroll
    for (int u = 0; u < kPermVecPerThread; ++u) {
      const int g = base + u * kPermThreads + static_cast<int>(threadIdx.x);
      dst[u] = -1;
      if (g < total) {
        const int r = p.vec_shift >= 0 ? (g >> p.vec_shift) : g / p.vec_per_row;
        const int vec = g - r * p.vec_per_row;
        const long long src = src_row[r];
        if (src >= 0) {
          v[u] = __ldg(p.in + src + vec);
          dst[u] = dst_row[r] + vec;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kPermVecPerThread; ++u)
      if (dst[u] >= 0) p.out[dst[u]] = v[u];
  }
}

// ---- step-wise LSE merge ----------------------------------------------------------------
// (O_acc, LSE_acc) <- (O_acc, LSE_acc) (+) (O_part, LSE_part) in place ("ring attention:
// key/value をリングで回す" step 3):  m = max(l, l'); w = e^(l - m), w' = e^(l' - m);
// O <- (w O + w' O') / (w + w');  l <- m + ln(w + w').  A row of d fp32 is d/4 lanes of 16-byte
// vectors (32 lanes at d = 128, 16 at d = 64).  The grid is (row blocks, (b, h) pairs, strided
// over B * H): a block takes kMergeSlots * 32 / (d/4) rows per warp of one (b, h), and each lane
// issues all its loads (kMergeSlots rows of O, O' and the two LSE values) before the
// arithmetic, so no index division runs per element and several 16-byte reads per lane are in
// flight.
struct MergeParams {
  float* o_acc;
  float* lse_acc;
  const float* o_part;
  const float* lse_part;
  int B, H, R, d;  // rows R per (b, h)
  long long oa_sb, oa_sh, oa_sr, la_sb, la_sh, la_sr;
  long long op_sb, op_sh, op_sr, lp_sb, lp_sh, lp_sr;
};

constexpr int kMergeThreads = 256;
constexpr int kMergeSlots = 4;     // rows (per 32/(d/4) lanes) a lane handles in one pass

__global__ void __launch_bounds__(kMergeThreads) lse_merge_kernel(const MergeParams p) {
  const int lpr = p.d >> 2;                       // lanes per row: 16 or 32
  const int rows_per_slot = 32 / lpr;             // rows a warp covers per slot: 2 or 1
  const int rows_per_warp = rows_per_slot * kMergeSlots;
  const int rows_per_block = rows_per_warp * (kMergeThreads / 32);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int vec = lane & (lpr - 1);
  const int r0 = blockIdx.x * rows_per_block + warp * rows_per_warp + lane / lpr;
  for (int bh = blockIdx.y; bh < p.B * p.H; bh += gridDim.y) {
  const int b = bh / p.H, h = bh - b * p.H;
  float* oa_base = p.o_acc + b * p.oa_sb + h * p.oa_sh;
  const float* op_base = p.o_part + b * p.op_sb + h * p.op_sh;
  float* la_base = p.lse_acc + b * p.la_sb + h * p.la_sh;
  const float* lp_base = p.lse_part + b * p.lp_sb + h * p.lp_sh;
  float4 a[kMergeSlots], o[kMergeSlots];
  float l0[kMergeSlots], l1[kMergeSlots];
#pragma unroll
  for (int k = 0; k < kMergeSlots; ++k) {
    const int r = r0 + k * rows_per_slot;
    if (r < p.R) {
      a[k] = reinterpret_cast<const float4*>(oa_base + r * p.oa_sr)[vec];
      o[k] = __ldg(reinterpret_cast<const float4*>(op_base + r * p.op_sr) + vec);
      l0[k] = la_base[r * p.la_sr];
      l1[k] = __ldg(lp_base + r * p.lp_sr);
    }
  }
  // every lane of a row has read its LSE before the row's first lane overwrites it
  __syncwarp();
#pragma unroll
  for (int k = 0; k < kMergeSlots; ++k) {
    const int r = r0 + k * rows_per_slot;
    if (r < p.R) {
      const float m = fmaxf(l0[k], l1[k]);
      float4 out = make_float4(0.f, 0.f, 0.f, 0.f);
      float lse = -INFINITY;
      if (m != -INFINITY) {
        // one weight is 1; an empty side (LSE = -inf) gets weight 0
        const float wa = __expf(l0[k] - m), wb = __expf(l1[k] - m);
        const float inv = __frcp_rn(wa + wb);
        const float ca = wa * inv, cb = wb * inv;
        out = make_float4(ca * a[k].x + cb * o[k].x, ca * a[k].y + cb * o[k].y, ca * a[k].z + cb * o[k].z,
                          ca * a[k].w + cb * o[k].w);
        lse = m + __logf(wa + wb);
      }
      reinterpret_cast<float4*>(oa_base + r * p.oa_sr)[vec] = out;
      if (vec == 0) la_base[r * p.la_sr] = lse;
    }
  }
  }
}

// ---- backward preprocess: D_i = sum_e dO_ie * O_ie ------------------------------------------
// 16 lanes per row at d = 128 (8 at d = 64), each loading 16 bytes of dO and of O, then a
// butterfly shuffle reduction inside the lane group.  A lane group takes kDotRows consecutive
// rows and issues all their loads before any arithmetic (more bytes in flight per thread).
// Rows are enumerated in the inputs' memory order: heads fastest when o and dout are
// sequence-major (head stride below position stride), positions fastest otherwise, so
// neighbouring lane groups read neighbouring memory.  Output D [B, H, L] fp32 (head-major).
constexpr int kDotRows = 4;

struct DotParams {
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  float* D;
  int B, H, L, d;
  long long o_sb, o_sh, o_sl, g_sb, g_sh, g_sl;  // element strides of o and dout ([b,h,l] axes)
  long long D_sb, D_sh, D_sl;
  // D is in position order; under a two-shard split (split 1 zig-zag, 2 striped) the rows of
  // o and dout are rank-major: position l is read from row split_rank_row(l).  0: same order.
  int split, n_ranks, shard;
};

__global__ void __launch_bounds__(256) rowdot_kernel(const DotParams p) {
  const int lpr = p.d / 8;  // lanes per row (power of two)
  const long long gthread = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long row0 = (gthread / lpr) * kDotRows;
  const int vec = static_cast<int>(gthread % lpr);
  const long long n_rows = static_cast<long long>(p.B) * p.H * p.L;
  uint4 a[kDotRows], g[kDotRows];
  int b[kDotRows], h[kDotRows], l[kDotRows];
  // (fast, slow) index of row0 along the memory order, then carried forward one row at a time
  const bool seq_major = p.o_sh < p.o_sl;
  const int n_fast = seq_major ? p.H : p.L, n_slow = seq_major ? p.L : p.H;
  const long long q1 = row0 / n_fast;
  int fast = static_cast<int>(row0 - q1 * n_fast);
  const long long q2 = q1 / n_slow;
  int slow = static_cast<int>(q1 - q2 * n_slow);
  int bb = static_cast<int>(q2);
#pragma unroll
  for (int u = 0; u < kDotRows; ++u) {
    const long long row = row0 + u;
    h[u] = seq_major ? fast : slow;
    l[u] = seq_major ? slow : fast;
    b[u] = bb;
    a[u] = make_uint4(0u, 0u, 0u, 0u);
    g[u] = a[u];
    if (row < n_rows) {
      const long long lr = p.split ? split_rank_row(l[u], p.split, p.n_ranks, p.shard) : l[u];
      a[u] = reinterpret_cast<const uint4*>(p.o + b[u] * p.o_sb + h[u] * p.o_sh + lr * p.o_sl)[vec];
      g[u] = reinterpret_cast<const uint4*>(p.dout + b[u] * p.g_sb + h[u] * p.g_sh + lr * p.g_sl)[vec];
    }
    if (++fast == n_fast) {
      fast = 0;
      if (++slow == n_slow) {
        slow = 0;
        ++bb;
      }
    }
  }
  float acc[kDotRows];
#pragma unroll
  for (int u = 0; u < kDotRows; ++u) {
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a[u]);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g[u]);
    acc[u] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __bfloat1622float2(a2[e]);
      const float2 y = __bfloat1622float2(g2[e]);
      acc[u] = fmaf(x.x, y.x, acc[u]);
      acc[u] = fmaf(x.y, y.y, acc[u]);
    }
  }
  for (int off = lpr >> 1; off > 0; off >>= 1) {
#pragma unroll
    for (int u = 0; u < kDotRows; ++u) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], off);
  }
  if (vec == 0) {
#pragma unroll
    for (int u = 0; u < kDotRows; ++u)
      if (row0 + u < n_rows) p.D[b[u] * p.D_sb + h[u] * p.D_sh + l[u] * p.D_sl] = acc[u];
  }
}

// ---- fill a step-wise partial with the merge identity (O = 0, LSE = -inf) -------------------
__global__ void fill_identity_kernel(float* o, float* lse, int B, int H, int R, int d, long long o_sb,
                                     long long o_sh, long long o_sr, long long l_sb, long long l_sh,
                                     long long l_sr) {
  const long long n = static_cast<long long>(B) * H * R * d;
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int c = static_cast<int>(i % d);
  long long t = i / d;
  const int r = static_cast<int>(t % R);
  t /= R;
  const int h = static_cast<int>(t % H);
  const int b = static_cast<int>(t / H);
  o[b * o_sb + h * o_sh + r * o_sr + c] = 0.f;
  if (c == 0) lse[b * l_sb + h * l_sh + r * l_sr] = -INFINITY;
}

}  // namespace cpattn
