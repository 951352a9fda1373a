// fwd_kernel.cuh — fused ring-attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes ("ring attention: key/value をリングで回す", steps 1-4, in "05. 長系列の分散
// 学習（Context Parallelism）"): virtual rank r keeps its query chunk; at ring step s it holds
// KV chunk j = (r - s) mod N and computes the partial attention of its queries against that
// chunk; the partials are combined by the online-softmax (LSE) merge.  Chunks wholly above
// the causal diagonal (j > r) are skipped; the diagonal chunk (j = r) is masked key <= query.
//
// One CTA owns two 128-row query tiles (A, B) that stream the same KV tiles:
//   * GQA (G even): two query heads of one KV group at the same rows;
//   * otherwise:    two consecutive 128-row tiles of one head inside one chunk.
// The KV chunks are visited in ascending order (0, 1, ..., the diagonal chunk r last), the same
// for every rank, so concurrent CTAs share K/V tiles in L2.
// Within a work item the running (max, sum, O) state is carried across tiles, so the merge
// of a finished chunk's partial into the accumulator happens at every chunk boundary as the
// same rescale-and-add that joins two tiles: (O, LSE) (+) (O', LSE') with weights e^(LSE-m).
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax for tile A (thread t <-> query row t <-> TMEM lane t)
//   warps 4-7  softmax for tile B
//   warp  8    TMA producer: Q tiles once, then K_0, V_0, K_1, V_1, ... into a 5-slot
//              shared-memory ring (one 128-row K or V tile per slot, each with its own
//              barrier), issued two iterations ahead of their use
//   warp  9    MMA issuer (one thread): S = Q K^T into TMEM, O += P V with P read from TMEM
//   warps 10-11 idle (they complete the producer warpgroup for the register rebalance)
// TMEM (512 columns x 128 lanes x 32 bit): S_A [0,128) O_A [128,256) S_B [256,384)
// O_B [384,512).  P (bf16, packed two per column) overwrites the first 64 columns of S.
//
// Every wait is bounded (WaitCtl): on expiry the kernel records CP_ERR_TIMEOUT with the wait
// site in the status word, drains its in-flight copies and MMAs, frees TMEM and returns.
#pragma once
#include <type_traits>
#include "sm100.cuh"

namespace cpattn {

constexpr int kBM = 128;       // query rows per tile
constexpr int kBN = 128;       // keys per KV tile
constexpr int kKvSlots = 5;    // shared-memory ring: K_i is item 2i, V_i item 2i+1, slot = item % 5
constexpr int kFwdThreads = 384;  // three warpgroups
// Registers per thread after the warpgroups rebalance (setmaxnreg): the launch gives every
// thread 168 (384 x 168 = 64,512 of the SM's 65,536); the producer warpgroup (load, MMA, two
// idle warps) gives back down to 72 and each softmax warpgroup grows to 216:
// 2 x 128 x 216 + 128 x 72 = 64,512, the launch's total.  Per SMSP (one warp of each
// warpgroup): 216 + 216 + 72 = 504 registers x 32 lanes = 16,128 of 16,384.
constexpr int kSoftmaxRegs = 216;
constexpr int kProducerRegs = 72;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kProducerRegs <= kFwdThreads * 168, "register split");
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;
// Largest exponent (log2) an unnormalised probability may reach against a row's offset before
// the offset is moved (and O, l rescaled).
constexpr float kStaleLimit = 64.0f;
constexpr float kStaleLimitPow = 18446744073709551616.0f;  // 2^64
#ifndef CPATTN_EMU_PAIRS
#define CPATTN_EMU_PAIRS 0
#endif
// Of every 16 exponential pairs of a 32-column chunk, this many run on the FMA pipe.
constexpr int kEmuPairs = CPATTN_EMU_PAIRS;

enum WaitSite : int {
  kSiteLoadEmpty = 1, kSiteMmaQ = 2, kSiteMmaKV = 3, kSiteMmaP = 4,
  kSiteSoftS = 5, kSiteSoftO = 6, kSiteDrain = 7,
};

struct FwdParams {
  int B, Hq, Hkv, L, d, G;
  int n_chunks, chunk_len;   // ring size N and chunk length c
  int tiles_per_chunk;       // ceil(c / 128)
  int pos_per_chunk;         // work-item positions along the query axis of one chunk
  int pair_heads;            // 1: A/B are heads (2p, 2p+1) of a KV group; 0: consecutive tiles
  int n_inner;               // work items per query position
  int causal;
  float scale_log2;          // softmax scale * log2(e)
  int step_rank;             // -1: fused over all ranks and steps; else one step: query chunk
  int step_chunk;            // step_rank against KV chunk step_chunk and, when step_chunk2 >= 0,
  int step_chunk2;           // also chunk step_chunk2 (the two shards a rank holds under a
                             // two-shard split), merged in the kernel
  int out_row_base;          // subtracted from the global row when writing o / lse
  void* o;                   // bf16 or fp32 output, [B, Hq, rows, d]
  long long o_sb, o_sh, o_sl;
  int out_fp32;
  float* lse;                // [B, Hq, rows]
  long long l_sb, l_sh, l_sl;
  int* status;
  unsigned long long wait_limit_ns;
  int debug_fault;
};

struct Item {
  int b, g, headA, headB, rowA, rowB, r, q_end, n_tiles, n_diag;
};

// KV tiles of chunk b that the query tiles of item it (in chunk it.r) see in one step.
__device__ __forceinline__ int step_tiles(const FwdParams& p, int r, int n_diag, int b) {
  if (b < 0) return 0;
  if (!p.causal) return p.tiles_per_chunk;
  return b < r ? p.tiles_per_chunk : (b == r ? n_diag : 0);
}

__device__ __forceinline__ Item decode_item(const FwdParams& p) {
  Item it;
  const int idx = blockIdx.x;
  // items of one KV head: a pair of query heads (pair_heads) or one query head (else)
  const int ig = p.pair_heads ? (p.G >> 1) : p.G;
  int pos, bg, w, qpos;
  if (p.step_rank >= 0) {
    pos = idx / p.n_inner;
    const int inner = idx - pos * p.n_inner;
    bg = inner / ig;
    w = inner - bg * ig;
    it.r = p.step_rank;
    qpos = p.pos_per_chunk - 1 - pos;
  } else {
    // KV-head-major: all of one (batch, KV head)'s items before the next, so the CTAs in flight
    // walk the same K/V chunks (in ascending order) and re-read them from L2, not DRAM; within
    // a KV head, longest first: last chunk, last query tiles first (the causal work grows with
    // the row)
    const int per_bg = p.n_chunks * p.pos_per_chunk * ig;
    bg = idx / per_bg;
    const int rem = idx - bg * per_bg;
    pos = rem / ig;
    w = rem - pos * ig;
    it.r = p.n_chunks - 1 - pos / p.pos_per_chunk;
    qpos = p.pos_per_chunk - 1 - pos % p.pos_per_chunk;
  }
  const int c0 = it.r * p.chunk_len;
  it.q_end = min(c0 + p.chunk_len, p.L);
  int last;  // last valid query row of the item
  it.b = bg / p.Hkv;
  it.g = bg - it.b * p.Hkv;
  if (p.pair_heads) {
    it.headA = it.g * p.G + 2 * w;
    it.headB = it.headA + 1;
    it.rowA = c0 + qpos * kBM;
    it.rowB = it.rowA;
    last = min(it.rowA + kBM, it.q_end) - 1;
  } else {
    it.headA = it.g * p.G + w;
    it.headB = it.headA;
    it.rowA = c0 + (2 * qpos) * kBM;
    it.rowB = it.rowA + kBM;
    last = min(it.rowB + kBM, it.q_end) - 1;
  }
  it.n_diag = (last - c0) / kBN + 1;
  if (p.step_rank >= 0) {
    it.n_tiles = step_tiles(p, it.r, it.n_diag, p.step_chunk) + step_tiles(p, it.r, it.n_diag, p.step_chunk2);
  } else if (p.causal) {
    it.n_tiles = it.n_diag + it.r * p.tiles_per_chunk;
  } else {
    it.n_tiles = p.n_chunks * p.tiles_per_chunk;
  }
  return it;
}

// The KV tiles of an item in visit order, walked without divisions (this runs once per tile
// on the softmax critical path): chunk j, tile tt inside it, tiles left in the chunk.
//   fused, causal:     chunks 0, 1, ..., r-1 (all tiles), then the diagonal chunk r (its first
//                      n_diag tiles)
//   fused, non-causal: chunks 0, 1, ..., N-1
//   one ring step:     chunk step_chunk, then chunk step_chunk2 if set (each only as far as
//                      the causal mask lets the item's query tiles see it)
// Every rank visits the chunks in the same ascending order (a ring schedule in which the
// chunk that arrives at step s is chunk s; the merged result does not depend on the order),
// so CTAs that start together stream the same K/V tiles at the same time and share them
// through L2.
struct KvIter {
  int j, tt, left, last, last_len, second, second_len;
  __device__ __forceinline__ KvIter(const FwdParams& p, const Item& it) {
    tt = 0;
    second = -1;
    second_len = 0;
    if (p.step_rank >= 0) {
      const int t1 = step_tiles(p, it.r, it.n_diag, p.step_chunk);
      const int t2 = step_tiles(p, it.r, it.n_diag, p.step_chunk2);
      if (t1 > 0) {
        j = p.step_chunk;
        left = t1;
        if (t2 > 0) {
          second = p.step_chunk2;
          second_len = t2;
        }
      } else {
        j = p.step_chunk2;
        left = t2;
      }
      last = -1;
      last_len = 0;
    } else {
      j = 0;
      last = p.causal ? it.r : -1;
      last_len = it.n_diag;
      left = (last == 0) ? last_len : p.tiles_per_chunk;
    }
  }
  __device__ __forceinline__ void next(const FwdParams& p) {
    ++tt;
    if (--left == 0) {
      tt = 0;
      if (second >= 0) {
        j = second;
        left = second_len;
        second = -1;
      } else {
        ++j;
        left = (j == last) ? last_len : p.tiles_per_chunk;
      }
    }
  }
  __device__ __forceinline__ int kv0(const FwdParams& p) const { return j * p.chunk_len + tt * kBN; }
  __device__ __forceinline__ int kv_end(const FwdParams& p) const { return min(j * p.chunk_len + p.chunk_len, p.L); }
};

// Wait used only while winding down: ignores the abort flag, keeps its own time limit.
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity, const WaitCtl& ctl) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > ctl.limit_ns) {
      if (ctl.status) atomicCAS(ctl.status, 0, kErrTimeout | (kSiteDrain << 8));
      return;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    ring_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  static_assert(D == 64 || D == 128, "head dim");
  constexpr int kBoxes = D / 64;                 // 64-column (128-byte) TMA boxes per row
  constexpr uint32_t kBoxBytes = 128 * 64 * 2;   // 16 KB
  constexpr uint32_t kTileBytes = kBoxes * kBoxBytes;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = smem;                                  // 2 tiles
  uint8_t* kv_smem = smem + 2 * kTileBytes;                // kKvSlots tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(kv_smem + kKvSlots * kTileBytes);
  uint64_t* q_full = bars + 0;
  // Barriers.  Ring item n (K_i: n = 2i, V_i: n = 2i+1) lives in slot n % 5.
  //  kv_full[slot] TMA -> MMA: the item landed (phase parity (n / 5) & 1)
  //  kv_free[t&1]  MMA commit after S_B(t): K_t and V_{t-1} are no longer read, and S_B(t) is
  //                in TMEM (softmax B waits on it too) -- one commit serves both.  The loads
  //                of iteration t+2 wait for it: K_{t+2} reuses the slot of V_{t-1}, V_{t+2}
  //                the slot of K_t.
  //  s_full_a      MMA commit after S_A(t)
  //  p_half[ab]    softmax -> MMA: P of keys [0, 64) of tile ab written to TMEM (4 arrivals)
  //  p_full[ab]    softmax -> MMA: P of keys [64, 128) written (4 warp arrivals)
  // A waiter on a two-barrier pair uses parity (t >> 1) & 1; no barrier can run two phases
  // ahead of its waiter because each next phase needs that waiter's own progress first.
  uint64_t* kv_full = bars + 1;                  // [kKvSlots]
  uint64_t* kv_free = bars + 1 + kKvSlots;       // [2]
  uint64_t* s_full_a = kv_free + 2;
  uint64_t* p_half = s_full_a + 1;               // [2]
  uint64_t* p_full = p_half + 2;                 // [2]
  uint64_t* o_full = p_full + 2;
  uint64_t* drain_bar = o_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* skip_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kKvSlots; ++s) mbar_init(&kv_full[s], 1);
    for (int s = 0; s < 2; ++s) mbar_init(&kv_free[s], 1);
    mbar_init(s_full_a, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&p_half[s], 4);
      mbar_init(&p_full[s], 4);
    }
    mbar_init(o_full, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    // A launch whose status word already holds an error does no work: after one expired
    // wait the remaining CTAs end at once instead of each running into its own limit.
    *skip_flag = (p.status != nullptr && *reinterpret_cast<volatile int*>(p.status) != 0) ? 1 : 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (*skip_flag) return;  // uniform across the CTA (read after the barrier)
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const Item it = decode_item(p);

  // Each role branch sets its register budget (warpgroup-wide) and ends at the named barrier
  // 1 that every warp reaches once its TMEM and shared-memory work is done; warp 0 then frees
  // TMEM.  The branches never rejoin.
  if (warp >= 8) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
  if (warp == kLoadWarp) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      const bool load_q = (p.debug_fault != 1);
      if (load_q) {
        mbar_arrive_expect_tx(q_full, 2 * kTileBytes);
#pragma unroll
        for (int x = 0; x < kBoxes; ++x) {
          tma_load_4d(q_smem + x * kBoxBytes, &tm_q, q_full, x * 64, it.rowA, it.headA, it.b, pol_q);
          tma_load_4d(q_smem + kTileBytes + x * kBoxBytes, &tm_q, q_full, x * 64, it.rowB, it.headB, it.b, pol_q);
        }
      }
      int issued = 0;  // ring items issued
      KvIter kvi(p, it);
      for (int i = 0; i < it.n_tiles; ++i, kvi.next(p)) {
        // K_i and V_i take the slots of V_{i-3} and K_{i-2}: both free once the MMAs of
        // iteration i-2 up to S_B(i-2) have completed (PV_B(i-3) precedes S_B(i-2))
        if (i >= 2 && !wait_bounded(&kv_free[i & 1], ((i - 2) >> 1) & 1, ctl, kSiteLoadEmpty)) break;
        const int kv0 = kvi.kv0(p);
#pragma unroll
        for (int kv = 0; kv < 2; ++kv) {
          const int n = 2 * i + kv;
          uint64_t* full = &kv_full[n % kKvSlots];
          uint8_t* dst = kv_smem + (n % kKvSlots) * kTileBytes;
          mbar_arrive_expect_tx(full, kTileBytes);
#pragma unroll
          for (int x = 0; x < kBoxes; ++x)
            tma_load_4d(dst + x * kBoxBytes, kv == 0 ? &tm_k : &tm_v, full, x * 64, kv0, it.g, it.b, pol_kv);
        }
        issued += 2;
      }
      // drain: every load this thread issued has landed before the CTA can exit (the last
      // fill of each slot is the only phase of its barrier still pending)
      if (load_q) wait_drain(q_full, 0, ctl);
      for (int n = (issued > kKvSlots ? issued - kKvSlots : 0); n < issued; ++n)
        wait_drain(&kv_full[n % kKvSlots], (n / kKvSlots) & 1, ctl);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc_bf16(128, kBN, false);
      constexpr uint32_t idesc_o = make_idesc_bf16(128, D, true);
      // Operand descriptors, built once: the two Q tiles and ring slot 0 as K-major tiles, ring
      // slot 0 as an N-major tile (V); a slot's descriptor is slot 0's plus the slot offset.
      const uint32_t q_d0 = sdesc_lo(smem_u32(q_smem), 16);
      const uint32_t kv_k0 = sdesc_lo(smem_u32(kv_smem), 16);
      const uint32_t kv_n0 = sdesc_lo(smem_u32(kv_smem), kBoxBytes);

      // S_ab = Q_ab K^T: M=128, N=128, K=D in steps of 16 (32 bytes inside a 128-byte swizzled row)
      auto issue_s = [=](int ab, int st) {
        const uint32_t kd = sdesc_lo_at(kv_k0, st * kTileBytes);
        const uint32_t qd = sdesc_lo_at(q_d0, ab * kTileBytes);
        const uint32_t d_tmem = tmem_base + ab * 256;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3) * 32;
          umma_ss(d_tmem, sdesc_lo_at(qd, off), sdesc_lo_at(kd, off), idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      // O_ab += P_ab V over keys [64 h, 64 h + 64): A = P from TMEM (8 columns per 16 keys),
      // B = V N-major (d contiguous)
      auto issue_pv = [=](int ab, int st, int h, bool acc) {
        const uint32_t vd = sdesc_lo_at(kv_n0, st * kTileBytes);
        const uint32_t p_tmem = tmem_base + ab * 256;
        const uint32_t o_tmem = tmem_base + 128 + ab * 256;
#pragma unroll
        for (int kk = 4 * h; kk < 4 * h + 4; ++kk) {
          umma_ts(o_tmem, p_tmem + kk * 8, sdesc_lo_at(vd, kk * 2048), idesc_o, (acc || kk > 0) ? 1u : 0u);
        }
      };
      // both halves of PV_ab, each after its half of P is in TMEM
      auto wait_issue_pv = [&](int ab, int st, int t) {
        if (!wait_bounded(&p_half[ab], t & 1, ctl, kSiteMmaP)) return false;
        tc_fence_after();
        issue_pv(ab, st, 0, t > 0);
        if (!wait_bounded(&p_full[ab], t & 1, ctl, kSiteMmaP)) return false;
        tc_fence_after();
        issue_pv(ab, st, 1, true);
        return true;
      };

      // TMA-filled operands need no tcgen05 fence (the mbarrier wait orders them); P written
      // by the softmax threads with tcgen05.st does (after_thread_sync after the wait).
      bool ok = wait_bounded(q_full, 0, ctl, kSiteMmaQ);
      const int T = it.n_tiles;
      int vslot_prev = 0;
      for (int i = 0; i < T && ok; ++i) {
        const int nk = 2 * i, nv = 2 * i + 1;
        const int kslot = nk % kKvSlots, vslot = nv % kKvSlots;
        if (!wait_bounded(&kv_full[kslot], (nk / kKvSlots) & 1, ctl, kSiteMmaKV)) { ok = false; break; }
        issue_s(0, kslot);
        umma_commit(s_full_a);
        if (i > 0 && !wait_issue_pv(1, vslot_prev, i - 1)) { ok = false; break; }
        issue_s(1, kslot);
        umma_commit(&kv_free[i & 1]);
        if (!wait_bounded(&kv_full[vslot], (nv / kKvSlots) & 1, ctl, kSiteMmaKV)) { ok = false; break; }
        if (!wait_issue_pv(0, vslot, i)) { ok = false; break; }
        vslot_prev = vslot;
      }
      if (ok && T > 0 && wait_issue_pv(1, vslot_prev, T - 1)) umma_commit(o_full);
      // drain: all MMAs issued by this thread are complete before TMEM is freed
      umma_commit(drain_bar);
      wait_drain(drain_bar, 0, ctl);
    }
    __syncwarp();
  }
  tc_fence_before();
  asm volatile("bar.sync 1, %0;" ::"n"(kFwdThreads) : "memory");
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ---------------- softmax / correction / epilogue (warps 0-7) ----------------
    const int ab = warp >> 2;                       // 0: tile A, 1: tile B
    const uint32_t lane_base = (warp & 3) * 32;     // TMEM lane window of this warp
    const int row_in_tile = lane_base + lane;
    const int q_row = (ab == 0 ? it.rowA : it.rowB) + row_in_tile;
    const int head = ab == 0 ? it.headA : it.headB;
    const uint32_t tS = tmem_base + (ab ? 256u : 0u) + (lane_base << 16);
    const uint32_t tO = tmem_base + (ab ? 384u : 128u) + (lane_base << 16);
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    // Exponent offset of the row (log2 units of the scaled scores): the exact max of the first
    // tile, then kept.  Exponentials are 2^(s*sl2 - m_run); while they stay below 2^kStaleLimit
    // nothing overflows (O, l < 2^(64+18+16) in fp32) and the result is exact, because the
    // final normalisation and the LSE use the same offset.  A tile that would pass the limit
    // moves the offset to its own max and rescales O and l by 2^(old - new).
    float m_run = -INFINITY;
    float l_run = 0.f;        // running sum of 2^(s*sl2 - m_run)
    bool ok = true;

    // Masked key columns (c >= lim) of one 32-column chunk of the S row -> -inf.
    auto mask_chunk = [](uint32_t (&r)[32], int c0, int lim) {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (c0 + e >= lim) r[e] = __float_as_uint(-INFINITY);
    };
    // Row max of one chunk as two interleaved 3-input chains (depth 8 each).
    auto max_chunk = [](const uint32_t (&r)[32]) {
      float a = fmax3(__uint_as_float(r[0]), __uint_as_float(r[1]), __uint_as_float(r[2]));
      float b = fmax3(__uint_as_float(r[3]), __uint_as_float(r[4]), __uint_as_float(r[5]));
#pragma unroll
      for (int e = 6; e < 30; e += 4) {
        a = fmax3(a, __uint_as_float(r[e]), __uint_as_float(r[e + 1]));
        b = fmax3(b, __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
      }
      return fmax3(a, b, fmaxf(__uint_as_float(r[30]), __uint_as_float(r[31])));
    };
    // 2^(s*sl2 - m) of one 32-column chunk -> 16 packed bf16 columns of P written over S
    // columns already read (P columns [16cc, 16cc+16)); returns the chunk's sum.  All the
    // chunk's exponentials are issued before their results are summed (two chains) and packed:
    // consuming each result at once stalled the warp on the MUFU latency.  emu: a share of the
    // pairs runs on the FMA pipe (only for chunks without masked columns, whose exponentials
    // must be exact zeros).
    auto exp_chunk = [&](const uint32_t (&r)[32], int cc, uint64_t negm2, bool emu) {
      float pv[32];
#pragma unroll
      for (int e2 = 0; e2 < 16; ++e2) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(r[2 * e2]), __uint_as_float(r[2 * e2 + 1])), sl2x2, negm2), x0,
                  x1);
        if (kEmuPairs > 0 && emu && (e2 * kEmuPairs) % 16 < kEmuPairs) {
          ex2_fma2(x0, x1, pv[2 * e2], pv[2 * e2 + 1]);
        } else {
          pv[2 * e2] = ex2_approx(x0);
          pv[2 * e2 + 1] = ex2_approx(x1);
        }
      }
      uint64_t s0 = f2_pack(0.f, 0.f), s1 = s0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int e2 = h * 8 + e;
          const uint64_t pp = f2_pack(pv[2 * e2], pv[2 * e2 + 1]);
          if (e & 1) s1 = f2_add(s1, pp); else s0 = f2_add(s0, pp);
          pk[e] = pack_bf16x2(pv[2 * e2], pv[2 * e2 + 1]);
        }
        tmem_st8(tS + cc * 16 + h * 8, pk);
      }
      float a0, a1, b0, b1;
      f2_unpack(s0, a0, a1);
      f2_unpack(s1, b0, b1);
      return (a0 + a1) + (b0 + b1);
    };
    // all stores of this thread's P are in TMEM before one lane of the warp arrives
    auto publish = [&](uint64_t* bar) {
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };

    KvIter kvi(p, it);
    for (int i = 0; i < it.n_tiles; ++i, kvi.next(p)) {
      // warp-uniform decisions only: the TMEM loads and stores below are .sync.aligned
      uint64_t* s_bar = ab == 0 ? s_full_a : &kv_free[i & 1];
      const uint32_t s_par = ab == 0 ? (i & 1) : ((i >> 1) & 1);
      if (!__all_sync(0xffffffffu, wait_bounded(s_bar, s_par, ctl, kSiteSoftS))) { ok = false; break; }
      tc_fence_after();
      const int kv0 = kvi.kv0(p);
      int lim = kvi.kv_end(p) - kv0;
      if (p.causal) lim = min(lim, q_row - kv0 + 1);
      const bool masked = __any_sync(0xffffffffu, lim < kBN);
      // The rest of the tile, instantiated with and without the mask code: only tiles at the
      // diagonal or at a ragged chunk end take the masked instance, the others carry no
      // per-element tests.
      auto tile = [&](auto with_mask) {
        constexpr bool kMasked = decltype(with_mask)::value;
        const bool emu = !kMasked;

        // The whole S row stays in registers until the tile is settled (a rare recompute needs
        // it; P overwrites the first 64 columns of S in TMEM).  Chunks 2 and 3 load while the
        // exponentials of chunks 0 and 1 run.
        uint32_t ra[32], rb[32], rc[32], rd[32];
        tmem_ld32(tS + 0, ra);
        tmem_ld32(tS + 32, rb);
        tmem_wait_ld();
        tmem_ld32(tS + 64, rc);
        tmem_ld32(tS + 96, rd);
        if constexpr (kMasked) {
          mask_chunk(ra, 0, lim);
          mask_chunk(rb, 32, lim);
        }
        if (i == 0) {
          // first tile: the exact row max before any exponential
          tmem_wait_ld();
          if constexpr (kMasked) {
            mask_chunk(rc, 64, lim);
            mask_chunk(rd, 96, lim);
          }
          m_run = fmaxf(fmaxf(max_chunk(ra), max_chunk(rb)), fmaxf(max_chunk(rc), max_chunk(rd))) * sl2;
        }
        uint64_t negm2;
        {
          const float m_off = (m_run == -INFINITY) ? 0.f : m_run;
          negm2 = f2_pack(-m_off, -m_off);
        }
        float l_tile = exp_chunk(ra, 0, negm2, emu);
        l_tile += exp_chunk(rb, 1, negm2, emu);
        if (i > 0) {
          tmem_wait_ld();
          if constexpr (kMasked) {
            mask_chunk(rc, 64, lim);
            mask_chunk(rd, 96, lim);
          }
        }
        // Before the first half of P is released: the offset must keep every exponential of the
        // tile below 2^kStaleLimit (keys [0,64) by their sum, [64,128) by their max).
        const float m23 = fmaxf(max_chunk(rc), max_chunk(rd)) * sl2;
        const bool over = !(l_tile <= kStaleLimitPow) || m23 > m_run + kStaleLimit;
        if (__any_sync(0xffffffffu, over)) {
          // rare: move the offset of the rows that need it to their tile max, rescale O and l
          // (O holds the previous tiles' sum: PV of the previous tile has completed because S of
          // this tile was issued after it), and recompute the whole tile's P; rows whose offset
          // did not move recompute the same values
          float alpha = 1.f;
          if (over) {
            const float m_new = fmaxf(fmaxf(max_chunk(ra), max_chunk(rb)) * sl2, m23);
            if (m_new > m_run) {
              alpha = ex2_approx(m_run - m_new);  // 0 when m_run = -inf
              m_run = m_new;
            }
          }
          const float m_off = (m_run == -INFINITY) ? 0.f : m_run;
          negm2 = f2_pack(-m_off, -m_off);
          tmem_wait_st();
          l_tile = exp_chunk(ra, 0, negm2, false);
          l_tile += exp_chunk(rb, 1, negm2, false);
          l_tile += exp_chunk(rc, 2, negm2, false);
          l_tile += exp_chunk(rd, 3, negm2, false);
          l_run = l_run * alpha + l_tile;
  #pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t r[32];
            tmem_ld32(tO + cc * 32, r);
            tmem_wait_ld();
  #pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(tO + cc * 32, r);
          }
          publish(&p_half[ab]);
          publish(&p_full[ab]);
        } else {
          publish(&p_half[ab]);
          l_tile += exp_chunk(rc, 2, negm2, emu);
          l_tile += exp_chunk(rd, 3, negm2, emu);
          l_run += l_tile;
          publish(&p_full[ab]);
        }
      };
      if (masked) {
        tile(Flag<true>{});
      } else {
        tile(Flag<false>{});
      }
    }

    // ---------------- epilogue: O / l, LSE ----------------
    if (ok && it.n_tiles > 0 && __all_sync(0xffffffffu, wait_bounded(o_full, 0, ctl, kSiteSoftO))) {
      tc_fence_after();
      const bool valid = (q_row < it.q_end) && (ab == 0 || p.pair_heads || it.rowB < it.q_end);
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      const long long orow = static_cast<long long>(q_row - p.out_row_base);
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tO + cc * 32, r);
        tmem_wait_ld();
        if (valid) {
          if (p.out_fp32) {
            float* dst = reinterpret_cast<float*>(p.o) + it.b * p.o_sb + head * p.o_sh + orow * p.o_sl + cc * 32;
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              float4 v4 = make_float4(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l,
                                      __uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
              *reinterpret_cast<float4*>(dst + e) = v4;
            }
          } else {
            __nv_bfloat16* dst =
                reinterpret_cast<__nv_bfloat16*>(p.o) + it.b * p.o_sb + head * p.o_sh + orow * p.o_sl + cc * 32;
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 v4;
              v4.x = pack_bf16x2(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l);
              v4.y = pack_bf16x2(__uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
              v4.z = pack_bf16x2(__uint_as_float(r[e + 4]) * inv_l, __uint_as_float(r[e + 5]) * inv_l);
              v4.w = pack_bf16x2(__uint_as_float(r[e + 6]) * inv_l, __uint_as_float(r[e + 7]) * inv_l);
              *reinterpret_cast<uint4*>(dst + e) = v4;
            }
          }
        }
      }
      if (valid) {
        const float lse = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994530942f : -INFINITY;
        p.lse[it.b * p.l_sb + head * p.l_sh + orow * p.l_sl] = lse;
      }
    }

    tc_fence_before();
    asm volatile("bar.sync 1, %0;" ::"n"(kFwdThreads) : "memory");
    if (warp == 0) {
      tc_fence_after();
      tmem_dealloc(tmem_base, kTmemCols);
    }
  }
}

// Dynamic shared memory: 1 KB alignment slack + Q (2 tiles) + KV ring + barriers
// (d = 128: 230,656 bytes of the 232,448 a CTA may use).
__host__ __device__ constexpr size_t fwd_smem_bytes(int d) {
  return 1024 + static_cast<size_t>(2 + kKvSlots) * 128 * d * 2 + 256;
}

}  // namespace cpattn
