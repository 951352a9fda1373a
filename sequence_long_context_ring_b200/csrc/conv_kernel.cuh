// conv_kernel.cuh — causal depthwise FIR convolution of a context-parallel sequence
// ("05. 長系列の分散学習（Context Parallelism）" §3 Hyena 演算子をどう分散するか, the p2p
// convolution: a shard's outputs need only its own inputs and the previous rank's last
// l_h - 1 inputs).
//
//   y[b, c, t] = sum_{k < l_h} h[c, k] x[b, c, t - k]      (x = 0 before the halo)
//
// Tensor-core form.  Cut a channel's row into blocks of 128 samples: X[m, j] = x[128 m + j].
// For l_h <= 129 every output of block m reads only blocks m and m - 1:
//
//   Y[m, i] = sum_j X[m, j] T0[i, j] + sum_j X[m - 1, j] T1[i, j]
//   T0[i, j] = h[i - j]        (0 <= i - j < l_h)
//   T1[i, j] = h[i - j + 128]  (i - j + 128 < l_h)
//
// i.e. two dense 128 x 128 x 128 contractions per block tile into one fp32 accumulator, with
// the channel's banded Toeplitz pair as the B operand (built in shared memory once per
// channel) and the input blocks as the A operand (K-major: a block is a contiguous 256-byte
// row).  A stage holds the tile's 128 blocks preceded by 8 more (one 136-row TMA box per
// 64-column half), so the previous-block operand X[m - 1] is the same buffer read one row
// earlier: a descriptor starting 128 bytes before a 1024-byte swizzle atom.  The 128-byte
// swizzle is a function of the absolute shared-memory address on both sides (TMA writes and
// tcgen05 reads), so such a start needs no base offset (checked on the device against the
// oracle: base offset 0 is exact, the other seven phases are not).  Blocks before the row's
// start are outside the tensor map
// and arrive as zeros: the zero halo of rank 0, and the first stage of the page's overlap
// variant.  Half of each Toeplitz pair is zero, which the tensor cores absorb: the kernel
// stays bound by HBM (32 KB in + 32 KB out per tile against at most ~1000 tensor cycles),
// where the direct form at l_h = 128 would need 128 FMAs per output on the CUDA cores,
// several times the HBM time.
//
// Roles (192 threads, one CTA per SM, persistent over a contiguous range of tiles):
//   warp 0      TMA producer: the input rows of each block tile into a stage ring
//   warp 1      TMEM owner and MMA issuer (two 128-column fp32 accumulators)
//   warps 2-5   Toeplitz builder (at each channel change) and epilogue: TMEM -> bf16 ->
//               128B-swizzled staging -> TMA store
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace cpattn {

// ---- bulk stores, proxy fence, named barriers (used by this kernel only) ------------------
// Tiled store shared -> global (bulk-group completion; coordinates past the extent are
// clipped, none may be negative).
__device__ __forceinline__ void tma_store_4d(const void* map, const void* src, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Every committed bulk store of this thread has finished reading its shared-memory source.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Every committed bulk store of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Order this thread's generic-proxy shared-memory writes before later async-proxy reads
// (TMA stores, tcgen05.mma operands).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Named barrier over `count` threads; the second form returns the AND of `pred` over them.
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ bool named_bar_and(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

constexpr int kConvThreads = 192;
constexpr int kConvMaxTaps = 129;                  // l_h - 1 <= 128: the halo fits one block
constexpr int kConvLead = 8;                       // blocks loaded ahead of a tile's first
constexpr uint32_t kConvBox = 128 * 64 * 2;        // 16 KB: 128 rows x 64 bf16, 128B swizzle
constexpr uint32_t kConvInBox = (128 + kConvLead) * 128;   // 17 KB: a 136-row input half
constexpr uint32_t kConvTmemCols = 256;
constexpr int kRevLen = 392;                       // reversed filter copy: 49 x 8 entries
enum : int { kCSiteLoad = 1, kCSiteMmaT = 2, kCSiteMmaX = 3, kCSiteMmaAcc = 4, kCSiteEpi = 5, kCSiteDrain = 7 };

struct ConvParams {
  int D;                     // channels (rows of a batch element)
  int tiles_per_row;         // ceil(nblk / 128), nblk = 128-sample blocks of a row
  long long n_tiles;         // B * D * tiles_per_row
  int lh;                    // filter taps
  int kk1;                   // first K step (16 samples) where T1 has taps: (129 - lh) / 16
  const __nv_bfloat16* h;    // filters [D, lh]
  long long h_sd;            // channel stride of h (elements)
  int* status;
  unsigned long long wait_limit_ns;
  int debug_fault;           // 1: the load warp skips its first tile's load (timeout-path test)
};

// Shared-memory plan.  Three input stages: measured at the full-size workloads, two leave
// HBM idle between tiles and four lose bandwidth to the extra requests in flight.
struct ConvSmem {
  static constexpr int kStages = 3;
  static constexpr uint32_t kStageBytes = 2 * kConvInBox;
  static constexpr uint32_t kRevBytes = 8 * kRevLen * 2;
  static constexpr uint32_t kT0 = 0;
  static constexpr uint32_t kT1 = 2 * kConvBox;
  static constexpr uint32_t kStage0 = kT1 + 2 * kConvBox;
  static constexpr uint32_t kOut = kStage0 + kStages * kStageBytes;
  static constexpr uint32_t kRev = kOut + 2 * kConvBox;          // 2 x 8 shifted reversed filters
  static constexpr uint32_t kFilt = kRev + 2 * kRevBytes;        // 256 bf16, zero-padded filter
  static constexpr uint32_t kBars = kFilt + 512;
  static constexpr uint32_t kBytes = kBars + 256;                // after 1 KB alignment
};

// Shared-memory byte offset of element (r, col) of a 128-row tile held as two 128B-swizzled
// boxes of 64 columns (the layout TMA writes and tcgen05 K-major descriptors read).
__device__ __forceinline__ uint32_t sw128_off(int r, int col) {
  return (col >> 6) * kConvBox + r * 128 + ((((col & 63) >> 3) ^ (r & 7)) << 4) + ((col & 7) << 1);
}

// Wait used only while winding down: ignores the abort flag, keeps its own time limit.
__device__ __forceinline__ void conv_wait_drain(uint64_t* bar, uint32_t parity, const WaitCtl& ctl) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > ctl.limit_ns) {
      if (ctl.status) atomicCAS(ctl.status, 0, kErrTimeout | (kCSiteDrain << 8));
      return;
    }
  }
}

__global__ void __launch_bounds__(kConvThreads, 1)
    fir_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_y,
                  const ConvParams p) {
  using S = ConvSmem;
  constexpr int kStages = S::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint16_t* rev = reinterpret_cast<uint16_t*>(smem + S::kRev);
  uint16_t* filt = reinterpret_cast<uint16_t*>(smem + S::kFilt);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBars);
  // Barriers.  Tile i (local index) uses stage i % kStages and accumulator i & 1.
  //  full[s]    TMA -> MMA: the stage's input rows landed (fill n = i / kStages, parity n & 1)
  //  empty[s]   MMA commit: the stage's MMAs completed, the producer may refill it
  //  tfull[a]   MMA commit: accumulator a holds tile i (parity (i >> 1) & 1)
  //  tempty[a]  epilogue -> MMA: accumulator a drained (one arrival per epilogue warp)
  //  t_ready    builder -> MMA: the Toeplitz pair of the next row's channel is in shared memory
  //  drain      MMA commit at the end: all MMAs complete before TMEM is freed
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* tfull = bars + 2 * kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* t_ready = tempty + 2;
  uint64_t* drain_bar = t_ready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* skip_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  // this CTA's contiguous range of tiles (row-major: tile = row * tiles_per_row + mt)
  const long long t_begin = p.n_tiles * blockIdx.x / gridDim.x;
  const long long t_end = p.n_tiles * (blockIdx.x + 1) / gridDim.x;
  const int n_local = static_cast<int>(t_end - t_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(t_ready, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    // A launch whose status word already holds an error does no work.
    *skip_flag = (p.status != nullptr && *reinterpret_cast<volatile int*>(p.status) != 0) ? 1 : 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (*skip_flag || n_local <= 0) return;  // uniform across the CTA
  if (warp == 1) {
    tmem_alloc(tmem_slot, kConvTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t smem0 = smem_u32(smem);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_y);
      const uint64_t pol = policy_evict_first();
      int issued = 0;
      const int skipped = p.debug_fault == 1 ? 0 : -1;  // tile whose load is left out
      for (int i = 0; i < n_local; ++i) {
        const int s = i % kStages;
        if (i >= kStages && !wait_bounded(&empty[s], ((i / kStages) - 1) & 1, ctl, kCSiteLoad)) break;
        if (i == skipped) {
          ++issued;
          continue;
        }
        const long long t = t_begin + i;
        const int row = static_cast<int>(t / p.tiles_per_row);
        const int m0 = static_cast<int>(t - static_cast<long long>(row) * p.tiles_per_row) * 128;
        const int b = row / p.D, ch = row - b * p.D;
        uint8_t* st = smem + S::kStage0 + s * S::kStageBytes;
        // blocks m0 - 8 .. m0 + 127 (those before the row start arrive as zeros)
        mbar_arrive_expect_tx(&full[s], S::kStageBytes);
        tma_load_4d(st, &tm_x, &full[s], 0, m0 - kConvLead, ch, b, pol);
        tma_load_4d(st + kConvInBox, &tm_x, &full[s], 64, m0 - kConvLead, ch, b, pol);
        ++issued;
      }
      // drain: every load issued has landed before the CTA can exit
      for (int n = (issued > kStages ? issued - kStages : 0); n < issued; ++n)
        if (n != skipped) conv_wait_drain(&full[n % kStages], (n / kStages) & 1, ctl);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc_bf16(128, 128, false);
      const int kk_prev = p.lh > 1 ? p.kk1 : 8;       // K steps of the previous block with taps
      // descriptors built once: stage 0's current-block and previous-block views (the latter
      // one 128-byte row earlier) and the two Toeplitz tiles
      const uint32_t cur0 = smem0 + S::kStage0 + kConvLead * 128;                     // atom-aligned
      const uint32_t cur_d0 = sdesc_lo(cur0, 16), prev_d0 = sdesc_lo(cur0 - 128, 16);
      const uint32_t t0_d = sdesc_lo(smem0 + S::kT0, 16), t1_d = sdesc_lo(smem0 + S::kT1, 16);
      int rebuilds = 0, last_row = -1;
      bool ok = true;
      for (int i = 0; i < n_local && ok; ++i) {
        const int s = i % kStages, a = i & 1;
        const long long t = t_begin + i;
        const int row = static_cast<int>(t / p.tiles_per_row);
        if (row != last_row) {
          if (!wait_bounded(t_ready, rebuilds & 1, ctl, kCSiteMmaT)) { ok = false; break; }
          ++rebuilds;
          last_row = row;
        }
        if (!wait_bounded(&full[s], (i / kStages) & 1, ctl, kCSiteMmaX)) { ok = false; break; }
        if (i >= 2 && !wait_bounded(&tempty[a], ((i >> 1) - 1) & 1, ctl, kCSiteMmaAcc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + a * 128;
        const uint32_t cur_d = sdesc_lo_at(cur_d0, s * S::kStageBytes);
        const uint32_t prev_d = sdesc_lo_at(prev_d0, s * S::kStageBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kConvInBox + (kk & 3) * 32;
          const uint32_t toff = (kk >> 2) * kConvBox + (kk & 3) * 32;
          umma_ss(d, sdesc_lo_at(cur_d, off), sdesc_lo_at(t0_d, toff), idesc, kk > 0 ? 1u : 0u);
        }
        for (int kk = kk_prev; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kConvInBox + (kk & 3) * 32;
          const uint32_t toff = (kk >> 2) * kConvBox + (kk & 3) * 32;
          umma_ss(d, sdesc_lo_at(prev_d, off), sdesc_lo_at(t1_d, toff), idesc, 1u);
        }
        umma_commit(&empty[s]);
        umma_commit(&tfull[a]);
      }
      umma_commit(drain_bar);
      conv_wait_drain(drain_bar, 0, ctl);
    }
    __syncwarp();
  } else {
    // ---------------- Toeplitz builder + epilogue (warps 2-5) ----------------
    const int et = threadIdx.x - 64;             // 0..127
    const int q = warp & 3;                      // TMEM lane quarter this warp may access
    const int m = 32 * q + lane;                 // accumulator row = block within the tile
    uint8_t* out = smem + S::kOut;

    // Toeplitz pair of a channel.  With the reversed filter r[u] = f(255 - u) (f = h padded
    // with zeros), a row chunk T0[i, j0..j0+7] is r[255 - i + j0 ..] and T1[i, j0..j0+7] is
    // r[127 - i + j0 ..]: 8 consecutive entries, copied as one 16-byte vector from the one of
    // 8 shifted copies (rev[s][v] = r[v + s]) in which the run starts 16-byte aligned.  The
    // copies of the next row's channel are prepared in the second buffer while the current
    // row's tiles run, so a channel change costs only the 16-byte copies into T0 and T1.
    auto prep = [&](int row, int rb) {            // filter of `row`'s channel -> rev buffer rb
      named_bar_sync(2, 128);                    // filt and rev[rb] are no longer read
      const int ch = row % p.D;
      for (int k = et; k < 256; k += 128)
        filt[k] = k < p.lh ? __bfloat16_as_ushort(p.h[static_cast<long long>(ch) * p.h_sd + k]) : 0;
      named_bar_sync(2, 128);
      uint16_t* rv = rev + rb * 8 * kRevLen;
      for (int idx = et; idx < 8 * kRevLen; idx += 128) {
        const int sh = idx / kRevLen, v = idx - sh * kRevLen;
        const int k = 255 - (v + sh);
        rv[idx] = k >= 0 ? filt[k] : 0;
      }
    };
    auto build = [&](int rb) {                   // T0, T1 from rev buffer rb
      named_bar_sync(2, 128);                    // rev[rb] complete
      const uint16_t* rv = rev + rb * 8 * kRevLen;
      const int i = et;
#pragma unroll 4
      for (int col = 0; col < 128; col += 8) {
        const int u0 = 255 - i + col, u1 = 127 - i + col;
        *reinterpret_cast<uint4*>(smem + S::kT0 + sw128_off(i, col)) =
            *reinterpret_cast<const uint4*>(rv + (u0 & 7) * kRevLen + (u0 & ~7));
        *reinterpret_cast<uint4*>(smem + S::kT1 + sw128_off(i, col)) =
            *reinterpret_cast<const uint4*>(rv + (u1 & 7) * kRevLen + (u1 & ~7));
      }
      fence_proxy_async_smem();                  // generic writes -> tensor-core reads
      named_bar_sync(2, 128);
      if (et == 0) mbar_arrive(t_ready);
    };

    auto row_of = [&](int i) { return static_cast<int>((t_begin + i) / p.tiles_per_row); };
    const int row_last = row_of(n_local - 1);
    int rb = 0;
    prep(row_of(0), 0);
    build(0);
    if (row_of(0) < row_last) prep(row_of(0) + 1, 1);
    for (int i = 0; i < n_local; ++i) {
      const int a = i & 1;
      // every epilogue thread polls; the AND over the 128 keeps their control flow uniform
      const bool landed = wait_bounded(&tfull[a], (i >> 1) & 1, ctl, kCSiteEpi);
      __syncwarp();
      if (!named_bar_and(3, 128, landed)) break;
      tc_fence_after();
      const int row = row_of(i);
      // the MMAs of tile i were the last readers of this channel's Toeplitz pair; the next
      // row (row + 1: a CTA's tiles are consecutive) has its copies ready in the other buffer
      const bool row_ends = i + 1 < n_local && row_of(i + 1) != row;
      if (row_ends) {
        rb ^= 1;
        build(rb);
      }
      // accumulator row m -> 128 fp32 outputs of block m0 + m (four loads, one wait)
      uint32_t r[128];
      const uint32_t tl = tmem_base + a * 128 + ((32u * q) << 16);
      tmem_ld32(tl, *reinterpret_cast<uint32_t(*)[32]>(r));
      tmem_ld32(tl + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
      tmem_ld32(tl + 64, *reinterpret_cast<uint32_t(*)[32]>(r + 64));
      tmem_ld32(tl + 96, *reinterpret_cast<uint32_t(*)[32]>(r + 96));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[a]);
      uint32_t v[64];
#pragma unroll
      for (int e = 0; e < 128; e += 2) v[e >> 1] = pack_bf16x2(__uint_as_float(r[e]), __uint_as_float(r[e + 1]));
      // staging: the previous tile's store has finished reading it
      if (et == 0) bulk_wait_read_all();
      named_bar_sync(2, 128);
#pragma unroll
      for (int c = 0; c < 16; ++c)
        *reinterpret_cast<uint4*>(out + sw128_off(m, c * 8)) =
            make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
      fence_proxy_async_smem();
      named_bar_sync(2, 128);
      if (et == 0) {
        const long long t = t_begin + i;
        const int m0 = static_cast<int>(t - static_cast<long long>(row) * p.tiles_per_row) * 128;
        const int b = row / p.D, ch = row - b * p.D;
        tma_store_4d(&tm_y, out, 0, m0, ch, b);
        tma_store_4d(&tm_y, out + kConvBox, 64, m0, ch, b);
        bulk_commit_group();
      }
      // off the MMA's path: the copies of the row after next into the freed buffer
      if (row_ends && row + 2 <= row_last) prep(row + 2, rb ^ 1);
    }
    if (et == 0) bulk_wait_all();
  }
  tc_fence_before();
  named_bar_sync(1, kConvThreads);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kConvTmemCols);
  }
}

// ---- direct form on the CUDA cores ----------------------------------------------------------
// Outputs t in [0, head) and [tail0, len) of every row, with an explicit halo: the input at
// t - k < 0 is halo[l_h - 1 + t - k] (zero without a halo).  Serves the per-rank call's
// boundary (the second stage of the overlap variant) and the samples past the last whole
// 128-sample block.
struct FirEdgeParams {
  const __nv_bfloat16* x;   long long x_sb, x_sd;      // [B, D, len], unit innermost stride
  const __nv_bfloat16* halo; long long g_sb, g_sd, g_st;  // [B, D, lh - 1] or null
  const __nv_bfloat16* h;   long long h_sd;            // [D, lh]
  __nv_bfloat16* y;         long long y_sb, y_sd;
  int D, len, lh, head, tail0;
};

constexpr int kEdgeThreads = 128;

__global__ void __launch_bounds__(kEdgeThreads) fir_edge_kernel(const FirEdgeParams p) {
  const int row = blockIdx.x;
  const int b = row / p.D, ch = row - b * p.D;
  const int n = p.head + (p.len - p.tail0);
  const int idx = blockIdx.y * kEdgeThreads + threadIdx.x;
  if (idx >= n) return;
  const int t = idx < p.head ? idx : p.tail0 + (idx - p.head);
  const __nv_bfloat16* xr = p.x + b * p.x_sb + ch * p.x_sd;
  const __nv_bfloat16* hr = p.h + ch * p.h_sd;
  float acc = 0.f;
  for (int k = 0; k < p.lh; ++k) {
    const int u = t - k;
    float xv = 0.f;
    if (u >= 0) xv = __bfloat162float(xr[u]);
    else if (p.halo) xv = __bfloat162float(p.halo[b * p.g_sb + ch * p.g_sd + (p.lh - 1 + u) * p.g_st]);
    acc = fmaf(__bfloat162float(hr[k]), xv, acc);
  }
  p.y[b * p.y_sb + ch * p.y_sd + t] = __float2bfloat16_rn(acc);
}

// Dynamic shared memory of fir_tc_kernel: 1 KB alignment slack + the plan above.
__host__ __device__ constexpr size_t fir_smem_bytes() { return 1024 + ConvSmem::kBytes; }

}  // namespace cpattn
