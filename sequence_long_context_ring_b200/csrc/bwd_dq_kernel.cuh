// bwd_dq_kernel.cuh — dQ of the ring-attention backward for sm_100a (tcgen05 + TMEM + TMA),
// query-stationary, recomputing the probabilities from the forward's stored LSE
// ("スケーラビリティとメモリ管理" in "長いシーケンスのLLMトレーニングの進展": keep only what
// is needed, recompute the rest).  For one 128-row query tile of head h, over every KV tile it
// sees, in ring order (its own chunk r first, then r-1, ..., 0; non-causal: all chunks):
//   S = Q K^T;  P = 2^(S*scale*log2e - LSE*log2e);  dP = dO V^T;  dS = P o (dP - D);
//   dQ += dS K      (D = rowsum(dO o O) from the preprocess kernel)
// dQ accumulates in TMEM over the whole visit and is written once, scaled and rounded to
// bf16: no atomics, and the result does not depend on the order in which CTAs run.
//
// Warp roles (320 threads):
//   warps 0-7  elementwise: warp w handles query rows 32(w%4) .. +31 (thread <-> TMEM lane)
//              and keys [64(w/4), 64(w/4) + 64) -- no row reduction is needed (LSE and D are
//              known), so the two warpgroups split the columns.  Before the loop they copy the
//              tile's Q (warpgroup 0) and dO (warpgroup 1) rows into TMEM, where they serve as
//              the A operand of every S and dP MMA; the epilogue writes dQ (each warpgroup half
//              of the d columns)
//   warp  8    loads: K_i into a 4-slot ring, V_i into a 3-slot ring (TMA)
//   warp  9    MMA issuer (one thread)
// TMEM columns: dQ [0,128)  S [128,256)  dP [256,384)  Q [384, 384+d/2)  dO [384+d/2, 384+d)
// (Q and dO as bf16 pairs, one row per lane).  S and dP take their A operand from TMEM, so each
// of their MMAs reads only the K or V tile from shared memory.  dS of keys [64h, 64h+64)
// (bf16, two per column) overwrites dP columns [64h, 64h+32), which warpgroup h has already
// read.
// Per iteration i: S(i+1) is issued as soon as the warps hold S(i) in registers; dQ(i) once
// dS(i) is in TMEM; then dP(i+1) over dS(i) (the pipe runs one thread's MMAs in order).  The
// warps turn S(i) into P(i) while dQ(i-1) and dP(i) run on the tensor cores.
#pragma once
#include "sm100.cuh"

namespace cpattn {

constexpr int kDqThreads = 320;
constexpr int kDqLoadWarp = 8;
constexpr int kDqMmaWarp = 9;
// K_i is read by S(i) (issued most of an iteration early) and by dQ(i), V_i by dP(i) only, so
// K gets more of the seven slots.
constexpr int kDqKSlots = 4;
constexpr int kDqVSlots = 3;

enum DqSite : int {
  kQSiteLoadK = 33, kQSiteLoadV = 34, kQSiteMmaQ = 35, kQSiteMmaK = 36, kQSiteMmaV = 37, kQSiteMmaSFree = 38,
  kQSiteMmaDs = 39, kQSiteS = 40, kQSiteDp = 41, kQSiteDone = 42, kQSiteDrain = 43,
};

struct DqParams {
  int B, Hq, Hkv, L, d, G;
  int n_chunks, chunk_len, tiles_per_chunk;
  int causal;
  float scale;        // softmax scale (applied to dQ once, in the epilogue)
  float scale_log2;   // scale * log2(e)
  const float* lse;   // [B, Hq, L] natural-log LSE of the forward
  long long lse_sb, lse_sh, lse_sl;
  const float* Dvec;  // [B, Hq, L] rowsum(dO * O), contiguous
  const __nv_bfloat16* q;    // [B, Hq, L, d] by the strides below (rows d-contiguous)
  long long q_sb, q_sh, q_sl;
  const __nv_bfloat16* dout;
  long long do_sb, do_sh, do_sl;
  __nv_bfloat16* dq;  // [B, Hq, L, d] by the strides below
  long long dq_sb, dq_sh, dq_sl;
  int* status;
  unsigned long long wait_limit_ns;
  int debug_fault;    // 3: the warps never report Q/dO in TMEM (a test of the timeout path)
};

struct DqItem {
  int b, h, g, r, row0, q_end, n_diag, n_tiles;
};

// Work items (batch, KV head)-major, then longest first: last chunk, last query tiles (the
// causal work grows with the row).
__device__ __forceinline__ DqItem decode_dq_item(const DqParams& p) {
  DqItem it;
  // (batch, KV head)-major: the CTAs in flight are the query tiles of one KV group's heads and
  // stream that group's K/V tiles, re-read from L2; within it longest first
  const int n_pos = p.n_chunks * p.tiles_per_chunk;
  const int per_bg = n_pos * p.G;
  const int bg = blockIdx.x / per_bg;
  const int rem = blockIdx.x - bg * per_bg;
  const int pos = rem / p.G;
  it.b = bg / p.Hkv;
  it.g = bg - it.b * p.Hkv;
  it.h = it.g * p.G + (rem - pos * p.G);
  it.r = p.n_chunks - 1 - pos / p.tiles_per_chunk;
  const int qpos = p.tiles_per_chunk - 1 - pos % p.tiles_per_chunk;
  const int c0 = it.r * p.chunk_len;
  it.row0 = c0 + qpos * 128;
  it.q_end = min(c0 + p.chunk_len, p.L);
  it.n_diag = qpos + 1;  // tiles of chunk r up to (and including) the one holding the diagonal
  it.n_tiles = p.causal ? it.n_diag + it.r * p.tiles_per_chunk : p.n_chunks * p.tiles_per_chunk;
  return it;
}

// KV tiles of the item in ring visit order, without divisions: chunk j, tile tt, tiles left.
struct DqKvIter {
  int j, tt, left;
  __device__ __forceinline__ DqKvIter(const DqParams& p, const DqItem& it)
      : j(it.r), tt(0), left(p.causal ? it.n_diag : p.tiles_per_chunk) {}
  __device__ __forceinline__ void next(const DqParams& p) {
    ++tt;
    if (--left == 0) {
      tt = 0;
      left = p.tiles_per_chunk;
      j = (j == 0 ? p.n_chunks : j) - 1;
    }
  }
  __device__ __forceinline__ int kv0(const DqParams& p) const { return j * p.chunk_len + tt * 128; }
  __device__ __forceinline__ int kv_end(const DqParams& p) const { return min(j * p.chunk_len + p.chunk_len, p.L); }
};

__device__ __forceinline__ void dq_wait_drain(uint64_t* bar, uint32_t parity, const WaitCtl& ctl) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > ctl.limit_ns) {
      if (ctl.status) atomicCAS(ctl.status, 0, kErrTimeout | (kQSiteDrain << 8));
      return;
    }
  }
}

// Dynamic shared memory: 1 KB alignment slack + 4 K slots + 3 V slots + barriers
// (d = 128: 230,656 bytes).
__host__ __device__ constexpr size_t bwd_dq_smem_bytes(int d) {
  return 1024 + static_cast<size_t>(kDqKSlots + kDqVSlots) * 128 * d * 2 + 256;
}

template <int D>
__global__ void __launch_bounds__(kDqThreads, 1)
    ring_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const DqParams p) {
  static_assert(D == 64 || D == 128, "head dim");
  constexpr int kBoxes = D / 64;
  constexpr uint32_t kBoxBytes = 128 * 64 * 2;
  constexpr uint32_t kTile = kBoxes * kBoxBytes;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* k_s = smem;                              // [kDqKSlots]
  uint8_t* v_s = k_s + kDqKSlots * kTile;           // [kDqVSlots]
  uint64_t* bars = reinterpret_cast<uint64_t*>(v_s + kDqVSlots * kTile);
  // Barriers (a waiter on a two-barrier pair [t & 1] uses parity (t >> 1) & 1; none can run two
  // phases ahead of its waiter, because each next phase needs that waiter's own progress):
  //  qa_full         elementwise -> MMA: Q and dO rows in TMEM (8 warp arrivals)
  //  k_full[kK]      K_i landed in slot i % kK (parity (i / kK) & 1)
  //  v_full[kV]      V_i landed in slot i % kV (parity (i / kV) & 1)
  //  k_free[kK]      MMA commit after dQ(i): slot i % kK (K_i) no longer read
  //  v_free[kV]      MMA commit after dP(i): slot i % kV (V_i) no longer read
  //  s_full          MMA commit after S(i) (parity i & 1)
  //  s_free          elementwise -> MMA: S(i) loaded into registers (8 warp arrivals)
  //  dp_full[2]      MMA commit after dP(i)
  //  ds_full[2]      elementwise -> MMA: dS(i) written to TMEM (8 warp arrivals)
  uint64_t* qa_full = bars + 0;
  uint64_t* k_full = bars + 1;                      // [kK]
  uint64_t* v_full = k_full + kDqKSlots;            // [kV]
  uint64_t* k_free = v_full + kDqVSlots;            // [kK]
  uint64_t* v_free = k_free + kDqKSlots;            // [kV]
  uint64_t* s_full = v_free + kDqVSlots;
  uint64_t* s_free = s_full + 1;
  uint64_t* dp_full = s_free + 1;                   // [2]
  uint64_t* ds_full = dp_full + 2;                  // [2]
  uint64_t* drain_bar = ds_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* skip_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    mbar_init(qa_full, 8);
    for (int s = 0; s < kDqKSlots; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_free[s], 1);
    }
    for (int s = 0; s < kDqVSlots; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_free[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 8);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&dp_full[s], 1);
      mbar_init(&ds_full[s], 8);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *skip_flag = (p.status != nullptr && *reinterpret_cast<volatile int*>(p.status) != 0) ? 1 : 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (*skip_flag) return;
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const DqItem it = decode_dq_item(p);
  const int T = it.n_tiles;
  const uint32_t tDQ = tmem_base, tS = tmem_base + 128, tDP = tmem_base + 256;
  const uint32_t tQa = tmem_base + 384, tDOa = tmem_base + 384 + D / 2;

  if (warp == kDqLoadWarp) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const uint64_t pol_kv = policy_evict_last();
      int nk = 0, nv = 0;  // loads issued
      DqKvIter kvi(p, it);
      for (int i = 0; i < T; ++i, kvi.next(p)) {
        const int kv0 = kvi.kv0(p);
        // K_i takes the slot of K_{i-kK}: free once dQ(i-kK) completed
        if (i >= kDqKSlots &&
            !wait_bounded(&k_free[i % kDqKSlots], ((i / kDqKSlots) - 1) & 1, ctl, kQSiteLoadK)) break;
        {
          uint64_t* full = &k_full[i % kDqKSlots];
          uint8_t* dst = k_s + (i % kDqKSlots) * kTile;
          mbar_arrive_expect_tx(full, kTile);
#pragma unroll
          for (int x = 0; x < kBoxes; ++x) tma_load_4d(dst + x * kBoxBytes, &tm_k, full, x * 64, kv0, it.g, it.b, pol_kv);
          ++nk;
        }
        // V_i takes the slot of V_{i-kV}: free once dP(i-kV) completed
        if (i >= kDqVSlots &&
            !wait_bounded(&v_free[i % kDqVSlots], ((i / kDqVSlots) - 1) & 1, ctl, kQSiteLoadV)) break;
        {
          uint64_t* full = &v_full[i % kDqVSlots];
          uint8_t* dst = v_s + (i % kDqVSlots) * kTile;
          mbar_arrive_expect_tx(full, kTile);
#pragma unroll
          for (int x = 0; x < kBoxes; ++x) tma_load_4d(dst + x * kBoxBytes, &tm_v, full, x * 64, kv0, it.g, it.b, pol_kv);
          ++nv;
        }
      }
      // drain: every load this thread issued has landed before the CTA can exit
      for (int n = (nk > kDqKSlots ? nk - kDqKSlots : 0); n < nk; ++n)
        dq_wait_drain(&k_full[n % kDqKSlots], (n / kDqKSlots) & 1, ctl);
      for (int n = (nv > kDqVSlots ? nv - kDqVSlots : 0); n < nv; ++n)
        dq_wait_drain(&v_full[n % kDqVSlots], (n / kDqVSlots) & 1, ctl);
    }
    __syncwarp();
  } else if (warp == kDqMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_kk = make_idesc_bf16(128, 128, false);  // S, dP: A TMEM, B K-major
      constexpr uint32_t idesc_o = make_idesc_bf16(128, D, true);      // dQ: A TMEM, B (K) N-major
      // Operand descriptors, built once: slot 0 of K and V as K-major tiles, slot 0 of K as the
      // N-major B of dQ; a slot's descriptor is slot 0's plus the slot offset.
      const uint32_t k_d0 = sdesc_lo(smem_u32(k_s), 16), v_d0 = sdesc_lo(smem_u32(v_s), 16);
      const uint32_t kn_d0 = sdesc_lo(smem_u32(k_s), kBoxBytes);
      // X = A B^T over d: A (Q or dO rows) from TMEM, 8 columns per 16 d; B d-contiguous in
      // shared memory; 128 x 128 into TMEM column d_tmem
      auto issue_kk = [=](uint32_t d_tmem, uint32_t a_tmem, uint32_t b) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
          umma_ts(d_tmem, a_tmem + 8u * kk, sdesc_lo_at(b, off), idesc_kk, kk > 0 ? 1u : 0u);
        }
      };
      auto wait_k = [&](int i) { return wait_bounded(&k_full[i % kDqKSlots], (i / kDqKSlots) & 1, ctl, kQSiteMmaK); };
      auto wait_v = [&](int i) {
        return wait_bounded(&v_full[i % kDqVSlots], (i / kDqVSlots) & 1, ctl, kQSiteMmaV);
      };
      auto kdesc = [&](int i) { return sdesc_lo_at(k_d0, (i % kDqKSlots) * kTile); };
      auto vdesc = [&](int i) { return sdesc_lo_at(v_d0, (i % kDqVSlots) * kTile); };
      // dP(i) into the dP columns; V_i's slot is free once it completes
      auto issue_dp = [&](int i) -> bool {
        if (!wait_v(i)) return false;
        issue_kk(tDP, tDOa, vdesc(i));
        umma_commit(&dp_full[i & 1]);
        umma_commit(&v_free[i % kDqVSlots]);
        return true;
      };

      bool ok = wait_bounded(qa_full, 0, ctl, kQSiteMmaQ);
      if (ok && T > 0) {
        tc_fence_after();
        ok = wait_k(0);
        if (ok) {
          issue_kk(tS, tQa, kdesc(0));
          umma_commit(s_full);
          ok = issue_dp(0);
        }
      }
      for (int i = 0; i < T && ok; ++i) {
        // S(i+1) over S(i), once the elementwise warps hold S(i) in registers
        if (i + 1 < T) {
          if (!wait_bounded(s_free, i & 1, ctl, kQSiteMmaSFree)) { ok = false; break; }
          if (!wait_k(i + 1)) { ok = false; break; }
          tc_fence_after();
          issue_kk(tS, tQa, kdesc(i + 1));
          umma_commit(s_full);
        }
        // dQ += dS(i) K(i): A = dS from TMEM (8 columns per 16 keys), B = K N-major
        if (!wait_bounded(&ds_full[i & 1], (i >> 1) & 1, ctl, kQSiteMmaDs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kn = sdesc_lo_at(kn_d0, (i % kDqKSlots) * kTile);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // keys [16 kk, 16 kk + 16): written by warpgroup kk / 4
          umma_ts(tDQ, tDP + 64u * (kk >> 2) + 8u * (kk & 3), sdesc_lo_at(kn, kk * 2048), idesc_o,
                  (i > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&k_free[i % kDqKSlots]);
        // dP(i+1) over dS(i), which dQ(i) (issued before it) reads
        if (i + 1 < T && !issue_dp(i + 1)) { ok = false; break; }
      }
      // drain: all MMAs issued by this thread are complete before TMEM is freed
      umma_commit(drain_bar);
      dq_wait_drain(drain_bar, 0, ctl);
    }
    __syncwarp();
  } else if (warp < 8) {
    // ---------------- elementwise (thread = query row, 64 keys) and the dQ epilogue ----------
    const uint32_t quarter = warp & 3;
    const int hh = static_cast<int>(warp >> 2);  // key half
    const uint32_t lofs = (quarter * 32u) << 16;
    const int q_row = it.row0 + static_cast<int>(quarter * 32 + lane);
    const bool q_live = q_row < it.q_end;
    // This row of Q (warpgroup 0) or dO (warpgroup 1) into TMEM as bf16 pairs: the A operand of
    // S = Q K^T and dP = dO V^T.  Rows past the sequence are zeros; rows past the chunk are
    // read but get probability 0 below.
    {
      const __nv_bfloat16* src = hh == 0 ? p.q + it.b * p.q_sb + it.h * p.q_sh + static_cast<long long>(q_row) * p.q_sl
                                         : p.dout + it.b * p.do_sb + it.h * p.do_sh + static_cast<long long>(q_row) * p.do_sl;
      const bool in_seq = q_row < p.L;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t r[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint4 x = make_uint4(0u, 0u, 0u, 0u);
          if (in_seq) x = *reinterpret_cast<const uint4*>(src + c * 64 + v * 8);
          r[4 * v] = x.x;
          r[4 * v + 1] = x.y;
          r[4 * v + 2] = x.z;
          r[4 * v + 3] = x.w;
        }
        tmem_st32((hh == 0 ? tQa : tDOa) + lofs + c * 32, r);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && p.debug_fault != 3) mbar_arrive(qa_full);
    }
    // rows past the chunk (ragged tail) get LSE = +inf: probability 0, no contribution
    float lse2 = INFINITY, Dr = 0.f;
    if (q_live) {
      lse2 = p.lse[it.b * p.lse_sb + it.h * p.lse_sh + static_cast<long long>(q_row) * p.lse_sl] *
             1.4426950408889634f;
      Dr = p.Dvec[(static_cast<long long>(it.b) * p.Hq + it.h) * p.L + q_row];
    }
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    const uint64_t nl2 = f2_pack(-lse2, -lse2);
    const uint64_t nD2 = f2_pack(-Dr, -Dr);
    bool ok = true;
    DqKvIter kvi(p, it);
    for (int i = 0; i < T; ++i, kvi.next(p)) {
      const uint32_t tSh = tS + lofs + hh * 64, tDPh = tDP + lofs + hh * 64;
      const int kv0 = kvi.kv0(p) + hh * 64;  // first key of this warp's half
      int lim = kvi.kv_end(p) - kv0;
      if (p.causal) lim = min(lim, q_row - kv0 + 1);
      const bool masked = __any_sync(0xffffffffu, lim < 64);
      if (!__all_sync(0xffffffffu, wait_bounded(s_full, i & 1, ctl, kQSiteS))) { ok = false; break; }
      tc_fence_after();
      uint32_t sa[32], sb[32];
      tmem_ld32(tSh + 0, sa);
      tmem_ld32(tSh + 32, sb);
      tmem_wait_ld();
      // S(i) is in registers: the MMA may write S(i+1)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      // P = 2^(S * scale * log2(e) - LSE * log2(e)) of one 32-key chunk, in place (fp32 bits),
      // computed while dP(i) is still on its way; the mask code exists only in the masked
      // instance
      auto p_chunk = [&](uint32_t (&r)[32], int cc, auto with_mask) {
        if constexpr (decltype(with_mask)::value) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (cc * 32 + e >= lim) r[e] = __float_as_uint(-INFINITY);
        }
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(r[2 * e2]), __uint_as_float(r[2 * e2 + 1])), sl2x2, nl2), x0, x1);
          r[2 * e2] = __float_as_uint(ex2_approx(x0));
          r[2 * e2 + 1] = __float_as_uint(ex2_approx(x1));
        }
      };
      if (masked) {
        p_chunk(sa, 0, Flag<true>{});
        p_chunk(sb, 1, Flag<true>{});
      } else {
        p_chunk(sa, 0, Flag<false>{});
        p_chunk(sb, 1, Flag<false>{});
      }
      if (!__all_sync(0xffffffffu, wait_bounded(&dp_full[i & 1], (i >> 1) & 1, ctl, kQSiteDp))) { ok = false; break; }
      tc_fence_after();
      uint32_t dpa[32], dpb[32];
      tmem_ld32(tDPh, dpa);
      tmem_ld32(tDPh + 32, dpb);
      tmem_wait_ld();
      // dS = P (dP - D) of one 32-key chunk -> 16 packed bf16 columns over dP (already read)
      auto ds_chunk = [&](const uint32_t (&pr)[32], const uint32_t (&g)[32], int cc) {
        uint32_t pk[16];
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          const uint64_t dd = f2_add(f2_pack(__uint_as_float(g[2 * e2]), __uint_as_float(g[2 * e2 + 1])), nD2);
          float d0, d1;
          f2_unpack(f2_mul(f2_pack(__uint_as_float(pr[2 * e2]), __uint_as_float(pr[2 * e2 + 1])), dd), d0, d1);
          pk[e2] = pack_bf16x2(d0, d1);
        }
        tmem_st16(tDPh + cc * 16, pk);
      };
      ds_chunk(sa, dpa, 0);
      ds_chunk(sb, dpb, 1);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ds_full[i & 1]);
    }
    // epilogue: dQ * scale -> bf16, d columns of this warpgroup's half
    if (ok && T > 0 &&
        __all_sync(0xffffffffu,
                   wait_bounded(&k_free[(T - 1) % kDqKSlots], ((T - 1) / kDqKSlots) & 1, ctl, kQSiteDone))) {
      tc_fence_after();
      __nv_bfloat16* dst = p.dq + it.b * p.dq_sb + it.h * p.dq_sh + static_cast<long long>(q_row) * p.dq_sl;
#pragma unroll
      for (int c2 = 0; c2 < D / 64; ++c2) {
        const int cc = hh * (D / 64) + c2;
        uint32_t r[32];
        tmem_ld32(tDQ + lofs + cc * 32, r);
        tmem_wait_ld();
        if (q_live) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 v4;
            v4.x = pack_bf16x2(__uint_as_float(r[e]) * p.scale, __uint_as_float(r[e + 1]) * p.scale);
            v4.y = pack_bf16x2(__uint_as_float(r[e + 2]) * p.scale, __uint_as_float(r[e + 3]) * p.scale);
            v4.z = pack_bf16x2(__uint_as_float(r[e + 4]) * p.scale, __uint_as_float(r[e + 5]) * p.scale);
            v4.w = pack_bf16x2(__uint_as_float(r[e + 6]) * p.scale, __uint_as_float(r[e + 7]) * p.scale);
            *reinterpret_cast<uint4*>(dst + cc * 32 + e) = v4;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace cpattn
