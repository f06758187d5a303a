// Fused bidirectional multi-head self-attention forward for sm_100a.
//
// Computes, per image b and head h of a packed [B, N, 3, H, d] bf16 QKV
// buffer, O = softmax(Q K^T * scale) V over all N tokens and writes O as
// [B, N, H, d] bf16.  This is the ViT-backbone multi-head self-attention that
// the Pi0 Flash Attention tutorial fuses ("Pi0 VLA deployment tutorial: Flash
// Attention for the vision encoder", section 1: reorder the computation,
// stay aware of the memory hierarchy, fuse -- so the N x N score matrix never
// goes to memory; section 3.2: the qkv linear feeds the attention module).
//
// Blackwell mapping (one persistent CTA per SM, 384 threads = 3 warpgroups):
//   warp 1      TMA producer: Q tiles (128 query rows) into one or two
//               buffers per Q slot (with two, the next round's tile loads
//               while the current round runs), K and V blocks (BK keys) into
//               a ring of `ring` slots.  With `reuse`, a head's K/V blocks are
//               loaded once and serve all of that head's Q tiles.
//   warp 0      tcgen05 issuer of S = Q K^T into tensor memory (SS MMA, M=128,
//               N=keys of the block, K=16 steps over d).
//   warp 2      tcgen05 issuer of O += P V with P read from tensor memory (TS
//               MMA, N=64, plus N=16 for d=72).
//   warps 4-11  softmax, one warpgroup per Q slot, one thread per query row
//               (= tensor-memory lane): online softmax in fp32 with exp2 and a
//               pre-scaled log2(e), P as bf16 pairs in its own tensor-memory
//               columns, O rescaled in tensor memory only when the running
//               maximum grows by more than 2^8, epilogue O / l -> bf16 into
//               a per-warp shared-memory buffer written out by one TMA store
//               of the warp's 32 rows (whole 128-byte rows per transaction),
//               or, where the staging's space is needed for a longer K/V ring,
//               by 16-byte row stores.
//   warp 3      idle.
//
// Schedule.  A round holds up to two 128-row Q tiles, one per Q slot and
// softmax warpgroup.  With fewer heads than SMs a CTA takes single tiles or
// single rounds; with more, whole heads, loading a head's K/V once for all its
// rounds when they fit the ring.  When a head has an odd number of Q tiles
// (577 tokens make 5), whole-head rounds would end every head with a half
// round, so instead a CTA walks the tiles of its heads two at a time across
// head boundaries: the round that pairs the last tile of one head with the
// first of the next streams both heads' K/V blocks through the ring (one load
// per slot and block), the others one load per block shared by both slots;
// when a head's blocks fit the ring, consecutive rounds of one head load them
// once (`carry`).
//
// Pipelining.  A softmax thread signals "S consumed" as soon as it has the S
// row of block j in registers, so the tensor core computes S of block j+1
// while block j is being exponentiated; P V of block j follows as soon as P
// is stored.  A full round holds two Q tiles of one head (slots 0 and 1, one
// per softmax warpgroup) whose exponentials share the special-function pipe.
// A half round (a lone last tile) has slot 0 only.
//
// Tensor memory (512 columns): slot s owns columns [256 s, 256 s + 256):
// S at +0 (BK fp32 columns), O at +BK (DP = 64 or 80 fp32 columns), P at
// +BK+DP (BK/2 columns of bf16 pairs).  d=64 uses BK=128 (128+64+64 = 256),
// d=72 uses BK=112 (112+80+56 = 248).
//
// Shared memory: Q buffers, the K/V ring, the output staging (8 warps x 32
// rows, 128-byte swizzled), barriers.  A tile row holds channels 0..63 in a
// 128-byte-swizzled region (TMA box {64,1,1,rows,1}); for d=72 channels
// 64..79 (72..79 zero-filled by TMA) sit in a 32-byte-swizzled region.  Q and
// K are read K-major by the MMA, V MN-major.
//
// Every mbarrier wait is bounded; a wait that runs out sets a shared abort
// flag and the device status word, every role then leaves its loop, the
// producer waits (bounded) for its own TMA copies, the MMA thread waits
// (bounded) for its own tensor-core work, and the tensor memory is freed.
// Every barrier has one consumer role that waits on each of its phases in
// order, and no barrier can complete twice before its consumer has waited,
// so a parity wait never confuses two phases.  The one barrier whose waiter
// skips phases, "P V issued" (waited on only before a round's first S), is
// never more than one phase past the phase waited for (see mma_role).
#pragma once

#include <cuda_bf16.h>
#include <math.h>

#include "ptx.cuh"

namespace vla {

constexpr int kQRows = 128;  // query rows per tile = TMEM lanes = MMA M
constexpr int kMmaWarp = 0;    // S = Q K^T issuer; also allocates tensor memory
constexpr int kLoadWarp = 1;   // TMA producer
constexpr int kPvWarp = 2;     // O += P V issuer
constexpr int kSoftmaxWarp0 = 4;
constexpr int kThreads = 384;
constexpr int kMaxRing = 6;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxQBuf = 2;  // Q buffers per slot
constexpr int kNumBarriers = 16 + 4 * kMaxRing + 5;
constexpr uint32_t kBarrierRegionBytes = 512;  // barriers + tmem address + abort flag
constexpr uint32_t kAlignSlack = 1024;
constexpr unsigned long long kDrainLimitNs = 100000000ull;

// Device status codes (the first wait that ran out records its site).
enum : int {
  kSiteLoadQ = 1, kSiteLoadK = 2, kSiteLoadV = 3,
  kSiteMmaQ = 11, kSiteMmaK = 12, kSiteMmaV = 13, kSiteMmaP = 14, kSiteMmaFree = 15,
  kSiteMmaPvIssued = 16,
  kSiteSoftS = 21, kSiteSoftO = 22,
  kSiteDrain = 31,
  kSiteTestStall = 41,
};

__device__ int g_vla_attn_status;  // 0 = ok, else 1000 + site of the first timed-out wait

// Timeline hooks for diagnostic builds: a translation unit may define these
// before including this header to record when each role reaches the points
// below; by default they compile to nothing.
enum : int {
  kTrMmaS = 1, kTrMmaPV = 2, kTrMmaSDone = 3, kTrMmaPVDone = 4, kTrMmaFree = 5, kTrMmaP = 6,
  kTrMmaV = 7, kTrMmaK = 8,
  kTrSoftS = 10, kTrSoftMax = 11, kTrSoftExp = 13, kTrSoftP = 14,
  kTrSoftEpi = 15,
};
#ifndef VLA_TRACE_EVENT
#define VLA_TRACE_EVENT(kind, slot, block) ((void)0)
#endif
#ifndef VLA_TRACE_INIT
#define VLA_TRACE_INIT() ((void)0)
#endif
#ifndef VLA_TRACE_END
#define VLA_TRACE_END() ((void)0)
#endif

template <int D>
struct Geom {
  static_assert(D == 64 || D == 72, "head dimension must be 64 or 72");
  static constexpr bool kHasTail = D > 64;
  static constexpr int BK = kHasTail ? 112 : 128;  // keys per block
  static constexpr int DP = kHasTail ? 80 : 64;    // MMA N of P V (d padded to 16)
  // Q tile: 128 rows x 128 B (SW128) [+ 128 rows x 32 B (SW32)].
  static constexpr uint32_t kQTail = 128 * 128;
  static constexpr uint32_t kQBytes = kQTail + (kHasTail ? 128 * 32 : 0);
  // K / V block: BK rows x 128 B (SW128) [+ BK rows x 32 B (SW32)], stride a
  // multiple of 1024 B so every region keeps its swizzle alignment.
  static constexpr uint32_t kKVTail = BK * 128;
  static constexpr uint32_t kKVBytes = kKVTail + (kHasTail ? BK * 32 : 0);
  static constexpr uint32_t kKVStride = (kKVBytes + 1023u) & ~1023u;
  // Output staging: per softmax warp 32 rows x 128 B (128-byte swizzled)
  // [+ 32 rows x 16 B for channels 64..71 of d=72], written by TMA stores.
  static constexpr uint32_t kStageWarp = 32 * 128;
  static constexpr uint32_t kStageTailWarp = 32 * 16;
  static constexpr uint32_t kStageBytes = 8 * kStageWarp + (kHasTail ? 8 * kStageTailWarp : 0);
  // Tensor-memory columns within a slot.
  static constexpr uint32_t kColO = BK;
  static constexpr uint32_t kColP = BK + DP;
  static_assert(BK + DP + BK / 2 <= 256, "slot does not fit its 256 TMEM columns");
};

struct AttnParams {
  CUtensorMap tm_q;        // 128B-swizzled box {64, 1, 1, 128, 1} (Q tiles)
  CUtensorMap tm_q_tail;   // 32B-swizzled box {16, 1, 1, 128, 1}, channels 64..79 (d = 72)
  CUtensorMap tm_kv;       // 128B-swizzled box {64, 1, 1, BK, 1} (K / V blocks)
  CUtensorMap tm_kv_tail;  // 32B-swizzled box {16, 1, 1, BK, 1} (d = 72)
  CUtensorMap tm_o;        // O as [B, N, H, d]: 128B-swizzled box {64, 1, 32, 1}
  CUtensorMap tm_o_tail;   // unswizzled box {8, 1, 32, 1} at channel 64 (d = 72)
  int B, N, H;
  int num_kblocks;         // ceil(N / BK)
  int num_qtiles;          // ceil(N / 128)
  int rounds_per_head;     // ceil(num_qtiles / 2): a round = up to two Q tiles
  int rounds_per_unit;     // rounds_per_head (whole head) or 1
  int tile_units;          // 1: a unit is one Q tile (slot 0 only), for batches whose
                           // tiles all fit on the SMs at once
  int units_per_head;
  int num_units;
  int ring;                // K/V ring slots (<= kMaxRing)
  int reuse;               // 1 when num_kblocks <= ring (not stream mode): a unit loads
                           // its K/V once
  float c;                 // scale * log2(e)
  unsigned long long wait_limit_ns;
  int test_stall;          // testing hook: softmax warps wait on a barrier nothing completes
  int stream;              // 1: a CTA pairs its heads' Q tiles across head boundaries
                           // (whole heads with an odd tile count), K/V streamed
  int qbuf;                // Q buffers per slot (1 or 2): with 2 the next round's Q tile
                           // loads while the current round runs
  int carry;               // stream mode with a head's K/V blocks fitting the ring: rounds
                           // of one head in a row load those blocks once
  __nv_bfloat16* o;        // [B, N, H, d] (the row stores of the kernel without staging)
};

template <int D>
__host__ __device__ constexpr uint32_t smem_bytes_for(int ring, int qbuf, bool stage_out) {
  return 2u * static_cast<uint32_t>(qbuf) * Geom<D>::kQBytes +
         2u * static_cast<uint32_t>(ring) * Geom<D>::kKVStride +
         (stage_out ? Geom<D>::kStageBytes : 0u) + kBarrierRegionBytes + kAlignSlack;
}

struct Barriers {
  uint32_t base;
  // Q buffer i = slot * qbuf + (the slot's Q load count mod qbuf).
  __device__ uint32_t q_full(int i) const { return base + 8u * (0 + i); }
  __device__ uint32_t q_empty(int i) const { return base + 8u * (4 + i); }
  __device__ uint32_t s_full(int s) const { return base + 8u * (8 + s); }   // S in TMEM
  __device__ uint32_t s_free(int s) const { return base + 8u * (10 + s); }  // S read out
  __device__ uint32_t p_full(int s) const { return base + 8u * (12 + s); }  // P in TMEM
  __device__ uint32_t o_prog(int s) const { return base + 8u * (14 + s); }  // each P V done
  __device__ uint32_t k_full(int i) const { return base + 8u * (16 + i); }
  __device__ uint32_t k_empty(int i) const { return base + 8u * (16 + kMaxRing + i); }
  __device__ uint32_t v_full(int i) const { return base + 8u * (16 + 2 * kMaxRing + i); }
  __device__ uint32_t v_empty(int i) const { return base + 8u * (16 + 3 * kMaxRing + i); }
  __device__ uint32_t drain(int i) const { return base + 8u * (16 + 4 * kMaxRing + i); }
  // Never arrived at: the testing hook's wait runs out on it.
  __device__ uint32_t never() const { return base + 8u * (16 + 4 * kMaxRing + 2); }
  // One phase per P V group issued (not completed) for slot s.
  __device__ uint32_t pv_issued(int s) const { return base + 8u * (16 + 4 * kMaxRing + 3 + s); }
};

// Bounded wait for the phase of `bar` with the given parity, executed by a
// whole converged warp; the result is the same in every lane.  Returns false
// when the CTA has aborted or this wait ran out (which aborts the CTA).
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity,
                                             volatile int* abort_flag,
                                             unsigned long long limit_ns, int site) {
  bool done = mbar_try_wait(bar, parity);
  if (__all_sync(0xffffffffu, done)) return true;
  if (!done) {
    const uint64_t t0 = global_timer_ns();
    while (true) {
      if (mbar_try_wait(bar, parity)) {
        done = true;
        break;
      }
      if (*abort_flag) break;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        atomicCAS(&g_vla_attn_status, 0, 1000 + site);
        break;
      }
    }
  }
  return __all_sync(0xffffffffu, done);
}

// Wait used while draining: ignores the abort flag, gives up after limit_ns.
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity,
                                           unsigned long long limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) {
      atomicCAS(&g_vla_attn_status, 0, 1000 + kSiteDrain);
      return;
    }
  }
}

// Keys of block j rounded up to the MMA granularity of 16.
template <int BK>
__device__ __forceinline__ int block_cols(int N, int j) {
  const int rem = N - j * BK;
  const int n16 = (rem + 15) & ~15;
  return n16 < BK ? n16 : BK;
}

// One round of the schedule (up to two Q tiles, one per slot), identical for
// every role.  Both slots belong to one head except in stream mode.
struct Round {
  int b0, b1, h0, h1, t0, t1;  // image, head and Q tile of slot 0 / slot 1
  int nslots;                  // 2 = both slots, 1 = slot 0 only
  bool shared_kv;              // both slots read one head's K/V: one K/V event per key block
  bool first;                  // first round of its unit
  bool last;                   // last round of its unit
  // Per-slot fields by selects (no runtime-indexed arrays, which would live
  // in local memory).
  __device__ __forceinline__ int b(int s) const { return s ? b1 : b0; }
  __device__ __forceinline__ int h(int s) const { return s ? h1 : h0; }
  __device__ __forceinline__ int tile(int s) const { return s ? t1 : t0; }
};

// Walks this CTA's rounds: whole units (u strided by the grid, rounds rr of
// each), or in stream mode the Q tiles of its heads two at a time.
struct Cursor {
  int u, rr;      // unit and round within it
  int tq;         // stream mode: tile of head u for slot 0 of the next round
};

__device__ __forceinline__ Cursor cursor_start() {
  return Cursor{static_cast<int>(blockIdx.x), 0, 0};
}

__device__ __forceinline__ bool cursor_more(const AttnParams& p, const Cursor& c) {
  return c.u < p.num_units;
}

__device__ __forceinline__ Round next_round(const AttnParams& p, Cursor& c) {
  Round x;
  if (p.stream) {
    // Slot 0: tile tq of head u; slot 1: the next tile, possibly of the next head.
    int ub = c.u, tb = c.tq + 1;
    if (tb == p.num_qtiles) {
      ub = c.u + static_cast<int>(gridDim.x);
      tb = 0;
    }
    x.nslots = ub < p.num_units ? 2 : 1;
    if (x.nslots == 1) {
      ub = c.u;
      tb = c.tq;
    }
    x.b0 = c.u / p.H;
    x.h0 = c.u - x.b0 * p.H;
    x.t0 = c.tq;
    if (ub == c.u) {
      x.b1 = x.b0;
      x.h1 = x.h0;
    } else {
      x.b1 = ub / p.H;
      x.h1 = ub - x.b1 * p.H;
    }
    x.t1 = tb;
    x.shared_kv = ub == c.u;
    // Consecutive rounds whose two tiles share a head (tiles 0-1, 2-3, ...)
    // form a run: with `carry` the run loads its K/V blocks once and its later
    // rounds read them from the ring; a round that pairs two heads, or a lone
    // last tile, is a run of its own.
    x.first = !(x.shared_kv && x.nslots == 2 && x.t0 >= 2);
    x.last = !(x.shared_kv && x.nslots == 2 && x.t0 + 3 < p.num_qtiles);
    // Advance two tiles.
    c.u = ub;
    c.tq = tb + 1;
    if (x.nslots == 1 || c.tq == p.num_qtiles) {
      c.u = x.nslots == 1 ? p.num_units : ub + static_cast<int>(gridDim.x);
      c.tq = 0;
    }
    return x;
  }
  const int bh = c.u / p.units_per_head;
  const int r = (c.u - bh * p.units_per_head) * p.rounds_per_unit + c.rr;
  int t0;
  if (p.tile_units) {
    t0 = r;
    x.nslots = 1;
  } else {
    t0 = 2 * r;
    x.nslots = (2 * r + 1 < p.num_qtiles) ? 2 : 1;
  }
  x.b0 = x.b1 = bh / p.H;
  x.h0 = x.h1 = bh - x.b0 * p.H;
  x.t0 = t0;
  x.t1 = t0 + 1;
  x.shared_kv = true;
  x.first = c.rr == 0;
  x.last = c.rr == p.rounds_per_unit - 1;
  if (++c.rr == p.rounds_per_unit) {
    c.rr = 0;
    c.u += static_cast<int>(gridDim.x);
  }
  return x;
}

// Position of a K/V load event in the ring: slot index and the parity of
// the number of times the ring has wrapped (the phase its barriers are in).
struct RingPos {
  int slot;
  uint32_t phase;
  __device__ __forceinline__ void advance(int R) {
    if (++slot == R) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

// ------------------------------------------------------------ producer
template <int D>
__device__ void load_role(const AttnParams& p, uint32_t sQ, uint32_t sK, uint32_t sV,
                          const Barriers& bar, volatile int* abort_flag) {
  using G = Geom<D>;
  const int R = p.ring;
  const int nb = p.num_kblocks;
  uint32_t nq0 = 0, nq1 = 0;  // Q loads issued for slot 0 / 1
  uint32_t kv_ev = 0;         // K/V load events issued
  RingPos pos{0, 0u};         // ring position of the next K/V event
  bool ok = true;

  // The whole warp runs this loop and waits together; one lane issues.
  auto load_q = [&](int s, const Round& x) -> bool {
    const uint32_t nq = s == 0 ? nq0 : nq1;
    const uint32_t qb = static_cast<uint32_t>(p.qbuf);
    const int qi = s * p.qbuf + static_cast<int>(nq % qb);  // Q buffer of this load
    if (!wait_bounded(bar.q_empty(qi), ((nq / qb) & 1u) ^ 1u, abort_flag, p.wait_limit_ns,
                      kSiteLoadQ))
      return false;
    if (elect_one()) {
      const uint32_t dst = sQ + qi * G::kQBytes;
      const int row0 = x.tile(s) * kQRows;
      mbar_arrive_expect_tx(bar.q_full(qi), G::kQBytes);
      tma_load_5d(dst, &p.tm_q, bar.q_full(qi), 0, x.h(s), 0, row0, x.b(s));
      if (G::kHasTail)
        tma_load_5d(dst + G::kQTail, &p.tm_q_tail, bar.q_full(qi), 64, x.h(s), 0, row0, x.b(s));
    }
    __syncwarp();
    if (s == 0) ++nq0; else ++nq1;
    return true;
  };
  auto load_kv = [&](uint32_t dst, uint32_t mbar, int w, int j, int b, int hh) {
    if (elect_one()) {
      mbar_arrive_expect_tx(mbar, G::kKVBytes);
      tma_load_5d(dst, &p.tm_kv, mbar, 0, hh, w, j * G::BK, b);
      if (G::kHasTail)
        tma_load_5d(dst + G::kKVTail, &p.tm_kv_tail, mbar, 64, hh, w, j * G::BK, b);
    }
    __syncwarp();
  };

  for (Cursor cu = cursor_start(); ok && cursor_more(p, cu);) {
    const Round x = next_round(p, cu);
    const bool reuse = p.reuse || (p.carry && x.shared_kv);
    if (!reuse || x.first) {
      const int E = x.shared_kv ? nb : 2 * nb;
      for (int e = 0; ok && e < E; ++e) {
        const int se = x.shared_kv ? 0 : (e & 1);
        const int j = x.shared_kv ? e : (e >> 1);
        const int slot = pos.slot;
        if (!wait_bounded(bar.k_empty(slot), pos.phase ^ 1u, abort_flag, p.wait_limit_ns,
                          kSiteLoadK) ||
            !wait_bounded(bar.v_empty(slot), pos.phase ^ 1u, abort_flag, p.wait_limit_ns,
                          kSiteLoadV)) {
          ok = false;
          break;
        }
        load_kv(sK + slot * G::kKVStride, bar.k_full(slot), 1, j, x.b(se), x.h(se));
        if (j == 0) {
          // Q tiles right after their first K block so S(0) can start early.
          if (x.shared_kv) {
            for (int s = 0; ok && s < x.nslots; ++s) ok = load_q(s, x);
          } else {
            ok = load_q(se, x);
          }
        }
        load_kv(sV + slot * G::kKVStride, bar.v_full(slot), 2, j, x.b(se), x.h(se));
        ++kv_ev;
        pos.advance(R);
      }
    } else {
      for (int s = 0; ok && s < x.nslots; ++s) ok = load_q(s, x);
    }
  }
  // Wait (bounded) until every copy this thread issued has landed.
  for (int s = 0; s < 2; ++s) {
    for (int k = 0; k < p.qbuf; ++k) {
      const uint32_t loads = ((s == 0 ? nq0 : nq1) + static_cast<uint32_t>(p.qbuf - 1 - k)) /
                             static_cast<uint32_t>(p.qbuf);  // loads into buffer s * qbuf + k
      if (loads > 0) wait_drain(bar.q_full(s * p.qbuf + k), (loads - 1u) & 1u, kDrainLimitNs);
    }
  }
  for (int i = 0; i < R; ++i) {
    const uint32_t arms = kv_ev / R + (static_cast<uint32_t>(i) < kv_ev % R ? 1u : 0u);
    if (arms > 0) {
      wait_drain(bar.k_full(i), (arms - 1u) & 1u, kDrainLimitNs);
      wait_drain(bar.v_full(i), (arms - 1u) & 1u, kDrainLimitNs);
    }
  }
}

// ------------------------------------------------------------ MMA issuers
// Two warps issue tensor-core work: the score warp issues S = Q K^T (waiting
// for each slot to have read its previous S), the value warp issues
// O += P V (waiting for each slot's P).  Issue blocks the issuing thread for
// about the duration of the MMA, so separate issuers keep each chain
// responsive.  They touch disjoint tensor-memory columns (S vs P / O).
// Shared-memory descriptors are built once; a K step only moves the start
// address field (bits [0,14), in 16-byte units), so each step is one add.
template <int D>
__device__ void mma_role(const AttnParams& p, uint32_t tmem, uint32_t sQ, uint32_t sK,
                         uint32_t sV, const Barriers& bar, volatile int* abort_flag,
                         bool score_warp) {
  using G = Geom<D>;
  const int R = p.ring;
  const int nb = p.num_kblocks;
  const unsigned long long lim = p.wait_limit_ns;
  uint32_t nq0 = 0, nq1 = 0;  // Q tiles consumed per slot
  int qi0 = 0, qi1 = 0;       // Q buffer of the current round per slot
  uint32_t nf0 = 0, nf1 = 0;  // s_free phases consumed per slot
  uint32_t np0 = 0, np1 = 0;  // p_full phases consumed per slot
  RingPos pos{0, 0u};         // ring position of the next unit / round's first K/V event
  uint32_t npv0 = 0, npv1 = 0;  // score warp: P V groups of each slot in earlier rounds

  const uint64_t q_desc0 = smem_desc(sQ, 16, 1024, kSwizzle128);
  const uint64_t q_tail0 = smem_desc(sQ + G::kQTail, 16, 256, kSwizzle32);
  const uint64_t k_desc0 = smem_desc(sK, 16, 1024, kSwizzle128);
  const uint64_t k_tail0 = smem_desc(sK + G::kKVTail, 16, 256, kSwizzle32);
  const uint64_t v_desc0 = smem_desc(sV, G::kKVTail, 1024, kSwizzle128);
  const uint64_t v_tail0 = smem_desc(sV + G::kKVTail, 32 * G::BK, 256, kSwizzle32);
  constexpr uint64_t kQStep = G::kQBytes >> 4;     // next Q buffer
  constexpr uint64_t kKVStep = G::kKVStride >> 4;  // next ring slot
  constexpr uint32_t kIdescPV = idesc_bf16_m128(64u, 1u);
  constexpr uint32_t kIdescPVTail = idesc_bf16_m128(16u, 1u);

  auto wait_k = [&](const RingPos& e) -> bool {
    if (!wait_bounded(bar.k_full(e.slot), e.phase, abort_flag, lim, kSiteMmaK)) return false;
    tc_fence_after();
    return true;
  };
  auto wait_v = [&](const RingPos& e) -> bool {
    if (!wait_bounded(bar.v_full(e.slot), e.phase, abort_flag, lim, kSiteMmaV)) return false;
    VLA_TRACE_EVENT(kTrMmaV, 0, 0);
    tc_fence_after();
    return true;
  };
  auto wait_q = [&](int s) -> bool {
    const uint32_t nq = s == 0 ? nq0 : nq1;
    const uint32_t qb = static_cast<uint32_t>(p.qbuf);
    const int qi = s * p.qbuf + static_cast<int>(nq % qb);
    if (!wait_bounded(bar.q_full(qi), (nq / qb) & 1u, abort_flag, lim, kSiteMmaQ)) return false;
    if (s == 0) {
      ++nq0;
      qi0 = qi;
    } else {
      ++nq1;
      qi1 = qi;
    }
    tc_fence_after();
    return true;
  };
  auto wait_free = [&](int s) -> bool {
    const uint32_t nf = s == 0 ? nf0 : nf1;
    if (!wait_bounded(bar.s_free(s), nf & 1u, abort_flag, lim, kSiteMmaFree)) return false;
    VLA_TRACE_EVENT(kTrMmaFree, s, 0);
    if (s == 0) ++nf0; else ++nf1;
    tc_fence_after();
    return true;
  };
  auto wait_p = [&](int s) -> bool {
    const uint32_t np = s == 0 ? np0 : np1;
    if (!wait_bounded(bar.p_full(s), np & 1u, abort_flag, lim, kSiteMmaP)) return false;
    VLA_TRACE_EVENT(kTrMmaP, s, 0);
    if (s == 0) ++np0; else ++np1;
    tc_fence_after();
    return true;
  };
  // The whole warp runs the issue loop and waits together; one lane issues
  // the tensor-core instructions and commits.
  auto commit = [&](uint32_t mbar) {
    if (elect_one()) mma_commit(mbar);
    __syncwarp();
  };
  // S of Q slot s against key block j held in ring slot `kslot`.
  auto scores = [&](int s, int j, int kslot) {
    VLA_TRACE_EVENT(kTrMmaS, s, j);
    const uint32_t idesc = idesc_bf16_m128(static_cast<uint32_t>(block_cols<G::BK>(p.N, j)), 0u);
    const uint32_t d_tmem = tmem + s * 256;
    const int qi = s == 0 ? qi0 : qi1;
    const uint64_t qd = q_desc0 + qi * kQStep;
    const uint64_t kd = k_desc0 + kslot * kKVStep;
    if (elect_one()) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss(d_tmem, qd + 2 * kk, kd + 2 * kk, idesc, kk > 0 ? 1u : 0u);  // 16 ch = 32 B
      if (G::kHasTail)
        mma_ss(d_tmem, q_tail0 + qi * kQStep, k_tail0 + kslot * kKVStep, idesc, 1u);
      mma_commit(bar.s_full(s));
    }
    __syncwarp();
    VLA_TRACE_EVENT(kTrMmaSDone, s, j);
  };
  // O_s (+)= P_s V_j, V_j in ring slot `vslot`.
  auto values = [&](int s, int j, int vslot) {
    VLA_TRACE_EVENT(kTrMmaPV, s, j);
    const int ksteps = block_cols<G::BK>(p.N, j) / 16;
    const uint32_t o_tmem = tmem + s * 256 + G::kColO;
    const uint32_t p_tmem = tmem + s * 256 + G::kColP;
    const uint64_t vd = v_desc0 + vslot * kKVStep;
    const uint64_t vt = v_tail0 + vslot * kKVStep;
    if (elect_one()) {
      for (int kk = 0; kk < ksteps; ++kk) {
        const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
        mma_ts(o_tmem, p_tmem + kk * 8, vd + kk * 128, kIdescPV, acc);  // 16 keys x 128 B
        if (G::kHasTail) mma_ts(o_tmem + 64, p_tmem + kk * 8, vt + kk * 32, kIdescPVTail, acc);
      }
      mma_commit(bar.o_prog(s));
      mbar_arrive(bar.pv_issued(s));
    }
    __syncwarp();
    VLA_TRACE_EVENT(kTrMmaPVDone, s, j);
  };

  bool ok = true;
  RingPos unit_pos = pos;
  for (Cursor cu = cursor_start(); ok && cursor_more(p, cu);) {
    const Round x = next_round(p, cu);
    if (x.first) unit_pos = pos;
    const int ns = x.nslots;
    const bool sh = x.shared_kv;
    const bool reuse = p.reuse || (p.carry && x.shared_kv);
    const bool release = !reuse || x.last;
    RingPos cur = reuse ? unit_pos : pos;  // K/V event of the next (block, slot)
    if (score_warp) {
      // S of block j for slot s as soon as slot s has read S of block j-1.
      // A round's first S waits until the slot's last P V of the previous
      // round has been issued: the tensor pipe runs in issue order, and that
      // P V gates the slot's epilogue, which comes before the new S is needed.
      for (int j = 0; ok && j < nb; ++j) {
        for (int s = 0; ok && s < ns; ++s) {
          if ((!sh || s == 0) && !(ok = wait_k(cur))) break;
          if (j == 0) {
            // No later P V of slot s can be issued before this S, so the
            // barrier is at most one phase ahead of the one waited for.
            const uint32_t npv = s == 0 ? npv0 : npv1;
            if (npv > 0 && !(ok = wait_bounded(bar.pv_issued(s), (npv - 1u) & 1u, abort_flag,
                                               lim, kSiteMmaPvIssued)))
              break;
          }
          if (!(ok = (j == 0 ? wait_q(s) : wait_free(s)))) break;
          scores(s, j, cur.slot);
          if (j == nb - 1) commit(bar.q_empty(s == 0 ? qi0 : qi1));
          if (!sh) {
            if (release) commit(bar.k_empty(cur.slot));
            cur.advance(R);
          }
        }
        if (!ok) break;
        if (sh) {
          if (release) commit(bar.k_empty(cur.slot));
          cur.advance(R);
        }
      }
      if (!ok) break;
      for (int s = 0; ok && s < ns; ++s) ok = wait_free(s);  // last block read out
      if (!ok) break;
      npv0 += static_cast<uint32_t>(nb);
      if (ns == 2) npv1 += static_cast<uint32_t>(nb);
    } else {
      // P V of block j for slot s as soon as slot s has stored P of block j.
      for (int j = 0; ok && j < nb; ++j) {
        for (int s = 0; ok && s < ns; ++s) {
          if ((!sh || s == 0) && !(ok = wait_v(cur))) break;
          if (!(ok = wait_p(s))) break;
          values(s, j, cur.slot);
          if (!sh) {
            if (release) commit(bar.v_empty(cur.slot));
            cur.advance(R);
          }
        }
        if (!ok) break;
        if (sh) {
          if (release) commit(bar.v_empty(cur.slot));
          cur.advance(R);
        }
      }
      if (!ok) break;
    }
    pos = cur;  // first event after this round (reuse: after the unit)
  }
  // Every tensor-core operation this warp issued must finish before the
  // tensor memory is freed.
  const uint32_t drain = bar.drain(score_warp ? 0 : 1);
  commit(drain);
  wait_drain(drain, 0u, kDrainLimitNs);
}

// ------------------------------------------------------------ softmax
struct SoftState {
  float m_run;  // running maximum (raw logits) used for the exponent
  float l_run;  // running sum of weights
};

// One pair of exponentials in kPolyEvery (0: none) is evaluated on the FMA pipe
// instead of the special-function unit, the limit of this kernel, sharing its
// work at the cost of more issued instructions.
constexpr int kPolyEvery = 16;

// One key block for one query row.  Reads S (NC columns at compile time,
// nvalid valid at run time), signals that S has been read, updates the
// running max / sum and leaves P (bf16 pairs, zero past NC) in pk.  Returns
// whether the warp must rescale O by alpha (warp-uniform).
template <int D, int NC>
__device__ __forceinline__ bool softmax_block(const AttnParams& p, SoftState& st, uint32_t tS,
                                              int nvalid, int j, const Barriers& bar, int s,
                                              int lane, uint32_t (&pk)[64], float& alpha) {
  const float c = p.c;
  float x[NC];
  {
    uint32_t sr[128];
    tmem_ld128(tS, sr);
#pragma unroll
    for (int i = 0; i < NC; ++i) x[i] = __uint_as_float(sr[i]);
  }
  // S is in registers: the tensor core may overwrite it with the next block.
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar.s_free(s));
  if (nvalid < NC) {
#pragma unroll
    for (int i = 0; i < NC; ++i)
      if (i >= nvalid) x[i] = -INFINITY;
  }
  float mx[4] = {x[0], x[1], x[2], x[3]};
  if constexpr (NC > 4) {
#pragma unroll
    for (int i = 4; i + 8 <= NC; i += 8) {
      mx[0] = fmax3(mx[0], x[i + 0], x[i + 4]);
      mx[1] = fmax3(mx[1], x[i + 1], x[i + 5]);
      mx[2] = fmax3(mx[2], x[i + 2], x[i + 6]);
      mx[3] = fmax3(mx[3], x[i + 3], x[i + 7]);
    }
    if constexpr (((NC - 4) % 8) != 0) {
#pragma unroll
      for (int i = NC - 4; i < NC; ++i) mx[i & 3] = fmaxf(mx[i & 3], x[i]);
    }
  }
  const float m_blk = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
  // Keep a stale maximum unless the block's maximum exceeds it by more than 8
  // in log2 units: the final O / l cancels the common factor, and the weights
  // stay below 2^8.
  const bool grow = (m_blk - st.m_run) * c > 8.0f;
  const bool rescale = __any_sync(0xffffffffu, grow);
  alpha = 1.0f;
  if (rescale) {
    const float m_new = fmaxf(st.m_run, m_blk);
    alpha = ex2_approx((st.m_run - m_new) * c);
    st.m_run = m_new;
    st.l_run *= alpha;
  }
  const float mc = st.m_run * c;
  VLA_TRACE_EVENT(kTrSoftMax, s, j);
  // Exponent arguments and running sums in packed fp32 pairs.
  const uint64_t c2 = f32x2_pack(c, c);
  const uint64_t nmc2 = f32x2_pack(-mc, -mc);
  uint64_t acc2[2] = {0ull, 0ull};
#pragma unroll
  for (int i = 0; i < NC / 2; ++i) {
    const uint64_t a = f32x2_fma(f32x2_pack(x[2 * i], x[2 * i + 1]), c2, nmc2);
    float p0, p1;
    if (kPolyEvery > 0 && i % kPolyEvery == kPolyEvery - 1) {
      exp2_fma_pair(a, p0, p1);  // FMA pipe
    } else {
      float a0, a1;
      f32x2_unpack(a, a0, a1);
      p0 = ex2_approx(a0);       // special-function unit
      p1 = ex2_approx(a1);
    }
    acc2[i & 1] = f32x2_add(acc2[i & 1], f32x2_pack(p0, p1));
    pk[i] = pack_bf16x2(p0, p1);
  }
  float lsum[4];
  f32x2_unpack(acc2[0], lsum[0], lsum[1]);
  f32x2_unpack(acc2[1], lsum[2], lsum[3]);
#pragma unroll
  for (int i = NC / 2; i < 64; ++i) pk[i] = 0u;
  VLA_TRACE_EVENT(kTrSoftExp, s, j);
  st.l_run += (lsum[0] + lsum[1]) + (lsum[2] + lsum[3]);
  return rescale;
}

template <int D>
__device__ __forceinline__ bool softmax_block_dispatch(const AttnParams& p, SoftState& st,
                                                       uint32_t tS, int ncols, int nvalid, int j,
                                                       const Barriers& bar, int s, int lane,
                                                       uint32_t (&pk)[64], float& alpha) {
#define VLA_SB(NC) return softmax_block<D, NC>(p, st, tS, nvalid, j, bar, s, lane, pk, alpha)
  if (ncols >= Geom<D>::BK) VLA_SB(Geom<D>::BK);
  switch (ncols) {
    case 112: VLA_SB(112);
    case 96: VLA_SB(96);
    case 80: VLA_SB(80);
    case 64: VLA_SB(64);
    case 48: VLA_SB(48);
    case 32: VLA_SB(32);
    default: VLA_SB(16);
  }
#undef VLA_SB
}

// Where a finished round's output goes: image, head and first row of this
// warp's 32 rows, and 1 / l for this thread's row.
struct OutRow {
  int b, h, row0;
  float inv_l;
};

// O / l -> bf16 for this warp's 32 rows: with kStageOut through its
// shared-memory staging buffer (128-byte swizzle: 16-byte chunk t of row r
// at chunk t ^ (r mod 8), so the eight rows of a store phase hit distinct
// banks), then one TMA store of the 32 x d box, rows past N falling outside
// the tensor; without, each thread's row by 16-byte stores.  The
// tensor-memory loads are warp-collective.
template <int D, bool kStageOut>
__device__ __forceinline__ void store_output(const AttnParams& p, uint32_t tO, const OutRow& r,
                                             uint32_t stage, uint32_t stage_tail, int lane) {
  using G = Geom<D>;
  uint32_t ob[64];
  tmem_ld64(tO, ob);
  uint32_t ot[16];
  if (G::DP > 64) tmem_ld16(tO + 64, ot);
  if (r.row0 >= p.N) return;  // warp-uniform: no row of this warp is a token
  if constexpr (!kStageOut) {
    // 16-byte stores of this thread's row (rows past N are not written).
    const int row = r.row0 + (lane & 31);
    if (row < p.N) {
      uint4* d4 = reinterpret_cast<uint4*>(
          p.o + ((static_cast<size_t>(r.b) * p.N + row) * p.H + r.h) * D);
#pragma unroll
      for (int t = 0; t < D / 8; ++t) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int ch = 8 * t + e;
          v[e] = __uint_as_float(ch < 64 ? ob[ch] : ot[ch - 64]) * r.inv_l;
        }
        d4[t] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                           pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
      }
    }
    return;
  }
  // The previous store from this buffer must have finished reading it.
  if (lane == 0) bulk_wait_read<0>();
  __syncwarp();
  const uint32_t row_s = stage + static_cast<uint32_t>(lane) * 128u;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(ob[8 * t + e]) * r.inv_l;
    st_shared_v4(row_s + ((static_cast<uint32_t>(t) ^ (lane & 7u)) << 4), pack_bf16x2(v[0], v[1]),
                 pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
  }
  if (G::kHasTail) {
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(ot[e]) * r.inv_l;
    st_shared_v4(stage_tail + static_cast<uint32_t>(lane) * 16u, pack_bf16x2(v[0], v[1]),
                 pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
  }
  fence_async_shared();
  __syncwarp();
  if (lane == 0) {
    tma_store_4d(&p.tm_o, stage, 0, r.h, r.row0, r.b);
    if (G::kHasTail) tma_store_4d(&p.tm_o_tail, stage_tail, 64, r.h, r.row0, r.b);
    bulk_commit();
  }
}

// Softmax warpgroup of Q slot s.  Per key block: read S, exponentials, then
// (after the previous P V has finished with the P columns) store P; after a
// round's last block, O / l of its Q tile to the output.

template <int D, bool kStageOut>
__device__ void softmax_loop(const AttnParams& p, uint32_t tmem, const Barriers& bar,
                             volatile int* abort_flag, int warp, int lane, uint32_t stage,
                             uint32_t stage_tail) {
  using G = Geom<D>;
  const int s = (warp - kSoftmaxWarp0) >> 2;  // Q slot of this warpgroup
  const int quad = warp & 3;
  const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
  const uint32_t tS = tmem + lane_bits + s * 256;
  const uint32_t tO = tS + G::kColO;
  const uint32_t tP = tS + G::kColP;
  const int nb = p.num_kblocks;
  uint32_t ns = 0;   // s_full phases consumed
  uint32_t nop = 0;  // o_prog phases consumed
  if (p.test_stall) {
    // Testing hook: a wait that nothing completes runs out after the bound,
    // which takes the whole CTA down the error path.
    (void)wait_bounded(bar.never(), 0u, abort_flag, p.wait_limit_ns, kSiteTestStall);
    return;
  }
  auto wait_pv = [&]() -> bool {
    if (!wait_bounded(bar.o_prog(s), nop & 1u, abort_flag, p.wait_limit_ns, kSiteSoftO))
      return false;
    ++nop;
    tc_fence_after();
    return true;
  };

  for (Cursor cu = cursor_start(); cursor_more(p, cu);) {
    const Round x = next_round(p, cu);
    const bool full = x.nslots == 2;
    if (!full && s == 1) continue;
    SoftState st{-INFINITY, 0.0f};
    for (int j = 0; j < nb; ++j) {
      if (!wait_bounded(bar.s_full(s), ns & 1u, abort_flag, p.wait_limit_ns, kSiteSoftS))
        return;
      ++ns;
      tc_fence_after();
      VLA_TRACE_EVENT(kTrSoftS, s, j);
      uint32_t pk[64];
      float alpha;
      const bool rescale = softmax_block_dispatch<D>(p, st, tS, block_cols<G::BK>(p.N, j),
                                                     min(G::BK, p.N - j * G::BK), j, bar, s,
                                                     lane, pk, alpha);
      // P V of the previous block must be done before P is overwritten and
      // before O is touched (this observes every phase of o_prog in order).
      if (j > 0) {
        if (!wait_pv()) return;
      }
      tmem_st64(tP, pk);
      if (j > 0 && rescale) {
        uint32_t ob[64];
        tmem_ld64(tO, ob);
#pragma unroll
        for (int i = 0; i < 64; ++i) ob[i] = __float_as_uint(__uint_as_float(ob[i]) * alpha);
        tmem_st64(tO, ob);
        if (G::DP > 64) {
          uint32_t ot[16];
          tmem_ld16(tO + 64, ot);
#pragma unroll
          for (int i = 0; i < 16; ++i) ot[i] = __float_as_uint(__uint_as_float(ot[i]) * alpha);
          tmem_st16(tO + 64, ot);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.p_full(s));
      VLA_TRACE_EVENT(kTrSoftP, s, j);
    }
    // Epilogue: the last P V, then O / l.
    if (!wait_pv()) return;
    VLA_TRACE_EVENT(kTrSoftEpi, s, 0);
    const OutRow r{x.b(s), x.h(s), x.tile(s) * kQRows + quad * 32, 1.0f / st.l_run};
    store_output<D, kStageOut>(p, tO, r, stage, stage_tail, lane);
  }
}

template <int D, bool kStageOut>
__device__ void softmax_role(const AttnParams& p, uint32_t tmem, const Barriers& bar,
                             volatile int* abort_flag, int warp, int lane, uint32_t stage,
                             uint32_t stage_tail) {
  softmax_loop<D, kStageOut>(p, tmem, bar, abort_flag, warp, lane, stage, stage_tail);
  // This warp's output stores must have read the staging buffer before the
  // CTA ends, on every path out of the loop (their writes are visible to
  // whatever follows the grid once it has completed).
  if (lane == 0) bulk_wait_read<0>();
  __syncwarp();
}

// ------------------------------------------------------------ kernel
// kStageOut: the output through shared-memory staging and TMA stores (else
// 16-byte row stores, leaving the staging's space to the K/V ring).
template <int D, bool kStageOut>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using G = Geom<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t sQ = base;
  const uint32_t sK = sQ + 2 * p.qbuf * G::kQBytes;
  const uint32_t sV = sK + p.ring * G::kKVStride;
  const uint32_t sStage = sV + p.ring * G::kKVStride;
  const uint32_t sBar = sStage + (kStageOut ? G::kStageBytes : 0u);
  uint8_t* bar_generic = smem_raw + (sBar - raw);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_generic + 8 * kNumBarriers);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_generic + 8 * kNumBarriers + 4);
  const Barriers bar{sBar};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * kMaxQBuf; ++i) {
      mbar_init(bar.q_full(i), 1);
      mbar_init(bar.q_empty(i), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar.s_full(s), 1);
      mbar_init(bar.s_free(s), 4);
      mbar_init(bar.p_full(s), 4);
      mbar_init(bar.o_prog(s), 1);
    }
    for (int i = 0; i < kMaxRing; ++i) {
      mbar_init(bar.k_full(i), 1);
      mbar_init(bar.k_empty(i), 1);
      mbar_init(bar.v_full(i), 1);
      mbar_init(bar.v_empty(i), 1);
    }
    mbar_init(bar.drain(0), 1);
    mbar_init(bar.drain(1), 1);
    mbar_init(bar.never(), 1);
    mbar_init(bar.pv_issued(0), 1);
    mbar_init(bar.pv_issued(1), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  VLA_TRACE_INIT();
  if (warp == kLoadWarp && lane == 0) {
    prefetch_tmap(&p.tm_q);
    prefetch_tmap(&p.tm_kv);
    if (kStageOut) prefetch_tmap(&p.tm_o);
    if (G::kHasTail) {
      prefetch_tmap(&p.tm_q_tail);
      prefetch_tmap(&p.tm_kv_tail);
      if (kStageOut) prefetch_tmap(&p.tm_o_tail);
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The prologue above (barriers, tensor memory, tensor-map prefetch) may
  // overlap the previous kernel; global memory is touched only after it.
  grid_dep_wait();
  grid_dep_launch();

  if (warp == kLoadWarp) {
    load_role<D>(p, sQ, sK, sV, bar, abort_flag);
    __syncwarp();
  } else if (warp == kMmaWarp || warp == kPvWarp) {
    mma_role<D>(p, tmem, sQ, sK, sV, bar, abort_flag, warp == kMmaWarp);
    __syncwarp();
  } else if (warp >= kSoftmaxWarp0) {
    const int ws = warp - kSoftmaxWarp0;  // staging buffer of this warp
    softmax_role<D, kStageOut>(p, tmem, bar, abort_flag, warp, lane, sStage + ws * G::kStageWarp,
                    sStage + 8 * G::kStageWarp + ws * G::kStageTailWarp);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  VLA_TRACE_END();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace vla
