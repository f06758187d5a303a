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
//   warp 9      TMA producer: Q tiles (128 query rows) into two Q slots, K and
//               V blocks (128 keys) into a ring of `ring` slots.  With
//               `reuse`, a head's K/V blocks are loaded once and serve all of
//               that head's Q tiles.
//   warp 8      tcgen05 issuer (one thread): S = Q K^T into tensor memory
//               (SS MMA, M=128, N=keys of the block, K=16 steps over d), then
//               O += P V with P read from tensor memory (TS MMA, N=64 or
//               64+16).
//   warps 0-7   softmax, one warpgroup per Q slot, one thread per query row
//               (= tensor-memory lane): online softmax in fp32 with exp2 and a
//               pre-scaled log2(e), P packed to bf16 pairs and stored back over
//               its own S columns, O rescaled in tensor memory only when the
//               running maximum grows by more than 2^8, epilogue O / l -> bf16
//               with 16-byte stores.
//   warps 10-11 idle.
//
// Work is a sequence of rounds.  A full round holds two Q tiles of one head:
// slot s owns S buffer s and O accumulator s, the tensor core works on one
// slot while the other slot's softmax runs, and the two softmax warpgroups
// take turns on the exp2 unit (an mbarrier token passed back and forth), so
// the special-function pipe stays busy instead of both groups stalling on it
// at once.  A half round (the odd last tile of a head) has only slot 0; it
// then uses both S buffers in turn so S of the next key block is computed
// while the current one is being exponentiated.
//
// Tensor memory (512 columns): S buffer b at columns [256 b, 256 b + 128)
// (fp32; overwritten in place by P as bf16 pairs in its first 64 columns);
// O accumulator s at [256 s + 128, 256 s + 128 + 80).
//
// Shared memory per 128-row tile: channels 0..63 as a 128-byte-swizzled
// 128 x 128 B region (TMA box {64,1,1,128,1}); for d = 72 the channels 64..79
// (72..79 zero-filled by TMA) as a 32-byte-swizzled 128 x 32 B region.
// Q and K are read K-major by the MMA, V MN-major.
//
// Every mbarrier wait is bounded; a wait that runs out sets a shared abort
// flag and the device status word, every role then leaves its loop, the
// producer waits (bounded) for its own TMA copies, the MMA thread waits
// (bounded) for its own tensor-core work, and the tensor memory is freed.
// Each barrier is waited on in phase order by every thread that waits on it,
// or it cannot complete twice without an intervening wait, so a parity wait
// never confuses two phases.
#pragma once

#include <cuda_bf16.h>
#include <math.h>

#include "ptx.cuh"

namespace vla {

constexpr int kTileRows = 128;  // query rows per tile = keys per block = TMEM lanes
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kThreads = 384;
constexpr int kMaxRing = 6;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kMainRegionBytes = 128 * 128;  // 128 rows x 64 bf16 channels
constexpr uint32_t kTailRegionBytes = 128 * 32;   // 128 rows x 16 bf16 channels
constexpr int kNumBarriers = 14 + 4 * kMaxRing + 1;
constexpr uint32_t kBarrierRegionBytes = 512;     // barriers + tmem address + abort flag
constexpr uint32_t kAlignSlack = 1024;
constexpr unsigned long long kDrainLimitNs = 100000000ull;

// Device status codes (the first wait that ran out records its site).
enum : int {
  kSiteLoadQ = 1, kSiteLoadK = 2, kSiteLoadV = 3,
  kSiteMmaQ = 11, kSiteMmaK = 12, kSiteMmaV = 13, kSiteMmaP = 14,
  kSiteSoftS = 21, kSiteSoftO = 22, kSiteSoftTok = 23,
  kSiteDrain = 31,
};

__device__ int g_vla_attn_status;  // 0 = ok, else 1000 + site of the first timed-out wait

// Timeline hook for diagnostic builds: a translation unit may define
// VLA_TRACE_EVENT(kind, slot, block) before including this header to record
// when each role reaches the points below; by default it compiles to nothing.
enum : int {
  kTrMmaS = 1, kTrMmaPV = 2,
  kTrSoftS = 10, kTrSoftMax = 11, kTrSoftTok = 12, kTrSoftExp = 13, kTrSoftP = 14,
  kTrSoftEpi = 15,
};
#ifndef VLA_TRACE_EVENT
#define VLA_TRACE_EVENT(kind, slot, block) ((void)0)
#endif
#ifndef VLA_TRACE_INIT
#define VLA_TRACE_INIT() ((void)0)
#endif

template <int D>
struct TileGeom {
  static_assert(D == 64 || D == 72, "head dimension must be 64 or 72");
  static constexpr bool kHasTail = D > 64;
  static constexpr uint32_t kBytes = kMainRegionBytes + (kHasTail ? kTailRegionBytes : 0);
};

struct AttnParams {
  CUtensorMap tm_main;  // 128B-swizzled box {64, 1, 1, 128, 1} over the packed QKV
  CUtensorMap tm_tail;  // 32B-swizzled box {16, 1, 1, 128, 1}, channels 64..79 (d = 72)
  __nv_bfloat16* o;     // [B, N, H, d]
  int B, N, H;
  int num_kblocks;      // ceil(N / 128)
  int num_qtiles;       // ceil(N / 128)
  int rounds_per_head;  // ceil(num_qtiles / 2): a round = up to two Q tiles
  int rounds_per_unit;  // rounds_per_head (whole head) or 1
  int units_per_head;
  int num_units;
  int ring;             // K/V ring slots (<= kMaxRing)
  int reuse;            // 1 when num_kblocks <= ring: a unit loads its K/V once
  float c;              // scale * log2(e)
  unsigned long long wait_limit_ns;
};

template <int D>
__host__ __device__ constexpr uint32_t smem_bytes_for_ring(int ring) {
  return (2u + 2u * static_cast<uint32_t>(ring)) * TileGeom<D>::kBytes + kBarrierRegionBytes +
         kAlignSlack;
}

struct Barriers {
  uint32_t base;
  __device__ uint32_t q_full(int s) const { return base + 8u * (0 + s); }
  __device__ uint32_t q_empty(int s) const { return base + 8u * (2 + s); }
  // S ready / P ready, per "channel": 0 = buffer 0 (slot 0), 1 = buffer 1 used
  // by slot 1 in full rounds, 2 = buffer 1 used by slot 0 in half rounds.
  // Each channel has exactly one consumer warpgroup, which waits on every phase.
  __device__ uint32_t s_full(int ch) const { return base + 8u * (4 + ch); }
  __device__ uint32_t p_full(int ch) const { return base + 8u * (7 + ch); }
  __device__ uint32_t o_prog(int s) const { return base + 8u * (10 + s); }  // per O slot, every PV
  __device__ uint32_t tok(int s) const { return base + 8u * (12 + s); }     // exp2 turn of slot s
  __device__ uint32_t k_full(int i) const { return base + 8u * (14 + i); }
  __device__ uint32_t k_empty(int i) const { return base + 8u * (14 + kMaxRing + i); }
  __device__ uint32_t v_full(int i) const { return base + 8u * (14 + 2 * kMaxRing + i); }
  __device__ uint32_t v_empty(int i) const { return base + 8u * (14 + 3 * kMaxRing + i); }
  __device__ uint32_t drain() const { return base + 8u * (14 + 4 * kMaxRing); }
};

// Bounded wait for the phase of `bar` with the given parity.  Returns false
// when the CTA has aborted or this wait ran out (which aborts the CTA).
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity,
                                             volatile int* abort_flag,
                                             unsigned long long limit_ns, int site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicCAS(&g_vla_attn_status, 0, 1000 + site);
      return false;
    }
  }
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

__device__ __forceinline__ int block_cols(int N, int j) {
  const int rem = N - j * kTileRows;
  const int n16 = (rem + 15) & ~15;
  return n16 < kTileRows ? n16 : kTileRows;
}

// One (unit, round) step of the schedule, identical for every role.
struct Round {
  int b, h, r;      // image, head, round index within the head
  int nslots;       // 2 = full round (tiles 2r, 2r+1), 1 = half round (tile 2r only)
  bool first;       // first round of its unit
  bool last;        // last round of its unit
};

__device__ __forceinline__ Round make_round(const AttnParams& p, int u, int rr) {
  Round x;
  const int bh = u / p.units_per_head;
  x.r = (u % p.units_per_head) * p.rounds_per_unit + rr;
  x.b = bh / p.H;
  x.h = bh % p.H;
  x.nslots = (2 * x.r + 1 < p.num_qtiles) ? 2 : 1;
  x.first = rr == 0;
  x.last = rr == p.rounds_per_unit - 1;
  return x;
}

// ------------------------------------------------------------ producer
template <int D>
__device__ void load_role(const AttnParams& p, uint32_t sQ, uint32_t sK, uint32_t sV,
                          const Barriers& bar, volatile int* abort_flag) {
  constexpr uint32_t kTile = TileGeom<D>::kBytes;
  const int R = p.ring;
  const int nb = p.num_kblocks;
  uint32_t nq0 = 0, nq1 = 0;  // Q loads issued into slot 0 / 1
  uint32_t kv_ev = 0;         // K/V load events issued
  bool ok = true;

  auto load_tile = [&](uint32_t dst, uint32_t mbar, int w, int row0, int b, int h) {
    tma_load_5d(dst, &p.tm_main, mbar, 0, h, w, row0, b);
    if (TileGeom<D>::kHasTail) tma_load_5d(dst + kMainRegionBytes, &p.tm_tail, mbar, 64, h, w,
                                           row0, b);
  };
  auto load_q = [&](int s, const Round& x) -> bool {
    const uint32_t nq = s == 0 ? nq0 : nq1;
    if (!wait_bounded(bar.q_empty(s), (nq & 1u) ^ 1u, abort_flag, p.wait_limit_ns, kSiteLoadQ))
      return false;
    mbar_arrive_expect_tx(bar.q_full(s), kTile);
    load_tile(sQ + s * kTile, bar.q_full(s), 0, (2 * x.r + s) * kTileRows, x.b, x.h);
    if (s == 0) ++nq0; else ++nq1;
    return true;
  };

  for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
    for (int rr = 0; ok && rr < p.rounds_per_unit; ++rr) {
      const Round x = make_round(p, u, rr);
      if (!p.reuse || x.first) {
        for (int j = 0; ok && j < nb; ++j) {
          const int slot = static_cast<int>(kv_ev % R);
          const uint32_t n = kv_ev / R;
          if (!wait_bounded(bar.k_empty(slot), (n & 1u) ^ 1u, abort_flag, p.wait_limit_ns,
                            kSiteLoadK)) {
            ok = false;
            break;
          }
          if (!wait_bounded(bar.v_empty(slot), (n & 1u) ^ 1u, abort_flag, p.wait_limit_ns,
                            kSiteLoadV)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar.k_full(slot), kTile);
          load_tile(sK + slot * kTile, bar.k_full(slot), 1, j * kTileRows, x.b, x.h);
          if (j == 0) {
            // Q tiles right after the first K block so S(0) can start early.
            for (int s = 0; ok && s < x.nslots; ++s) ok = load_q(s, x);
          }
          mbar_arrive_expect_tx(bar.v_full(slot), kTile);
          load_tile(sV + slot * kTile, bar.v_full(slot), 2, j * kTileRows, x.b, x.h);
          ++kv_ev;
        }
      } else {
        for (int s = 0; ok && s < x.nslots; ++s) ok = load_q(s, x);
      }
    }
  }
  // Wait (bounded) until every copy this thread issued has landed.
  if (nq0 > 0) wait_drain(bar.q_full(0), (nq0 - 1u) & 1u, kDrainLimitNs);
  if (nq1 > 0) wait_drain(bar.q_full(1), (nq1 - 1u) & 1u, kDrainLimitNs);
  for (int i = 0; i < R; ++i) {
    const uint32_t arms = kv_ev / R + (static_cast<uint32_t>(i) < kv_ev % R ? 1u : 0u);
    if (arms > 0) {
      wait_drain(bar.k_full(i), (arms - 1u) & 1u, kDrainLimitNs);
      wait_drain(bar.v_full(i), (arms - 1u) & 1u, kDrainLimitNs);
    }
  }
}

// ------------------------------------------------------------ MMA issuer
template <int D>
__device__ __forceinline__ void issue_scores(uint32_t tmem_s, uint32_t q_addr, uint32_t k_addr,
                                             int ncols) {
  const uint32_t idesc = idesc_bf16_m128(static_cast<uint32_t>(ncols), 0u);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    mma_ss(tmem_s, smem_desc(q_addr + kk * 32, 16, 1024, kSwizzle128),
           smem_desc(k_addr + kk * 32, 16, 1024, kSwizzle128), idesc, kk > 0 ? 1u : 0u);
  }
  if (TileGeom<D>::kHasTail) {
    mma_ss(tmem_s, smem_desc(q_addr + kMainRegionBytes, 16, 256, kSwizzle32),
           smem_desc(k_addr + kMainRegionBytes, 16, 256, kSwizzle32), idesc, 1u);
  }
}

template <int D>
__device__ __forceinline__ void issue_values(uint32_t tmem_o, uint32_t tmem_p, uint32_t v_addr,
                                             int ncols, bool accumulate) {
  constexpr uint32_t idesc_main = idesc_bf16_m128(64u, 1u);
  constexpr uint32_t idesc_tail = idesc_bf16_m128(16u, 1u);
  const int ksteps = ncols / 16;
  for (int kk = 0; kk < ksteps; ++kk) {
    const uint32_t acc = (accumulate || kk > 0) ? 1u : 0u;
    mma_ts(tmem_o, tmem_p + kk * 8,
           smem_desc(v_addr + kk * 16 * 128, kMainRegionBytes, 1024, kSwizzle128), idesc_main,
           acc);
    if (TileGeom<D>::kHasTail) {
      mma_ts(tmem_o + 64, tmem_p + kk * 8,
             smem_desc(v_addr + kMainRegionBytes + kk * 16 * 32, kTailRegionBytes, 256,
                       kSwizzle32),
             idesc_tail, acc);
    }
  }
}

template <int D>
__device__ void mma_role(const AttnParams& p, uint32_t tmem, uint32_t sQ, uint32_t sK,
                         uint32_t sV, const Barriers& bar, volatile int* abort_flag) {
  constexpr uint32_t kTile = TileGeom<D>::kBytes;
  const int R = p.ring;
  const int nb = p.num_kblocks;
  uint32_t nq0 = 0, nq1 = 0;  // q_full phases consumed per Q slot
  uint32_t np0 = 0, np1 = 0, np2 = 0;  // p_full phases consumed per channel
  uint32_t kv_ev = 0;
  const unsigned long long lim = p.wait_limit_ns;

  auto wait_k = [&](uint32_t ev) -> bool {
    if (!wait_bounded(bar.k_full(static_cast<int>(ev % R)), (ev / R) & 1u, abort_flag, lim,
                      kSiteMmaK))
      return false;
    tc_fence_after();
    return true;
  };
  auto wait_v = [&](uint32_t ev) -> bool {
    if (!wait_bounded(bar.v_full(static_cast<int>(ev % R)), (ev / R) & 1u, abort_flag, lim,
                      kSiteMmaV))
      return false;
    tc_fence_after();
    return true;
  };
  auto wait_q = [&](int s) -> bool {
    const uint32_t nq = s == 0 ? nq0 : nq1;
    if (!wait_bounded(bar.q_full(s), nq & 1u, abort_flag, lim, kSiteMmaQ)) return false;
    if (s == 0) ++nq0; else ++nq1;
    tc_fence_after();
    return true;
  };
  auto wait_p = [&](int ch) -> bool {
    const uint32_t np = ch == 0 ? np0 : (ch == 1 ? np1 : np2);
    if (!wait_bounded(bar.p_full(ch), np & 1u, abort_flag, lim, kSiteMmaP)) return false;
    if (ch == 0) ++np0; else if (ch == 1) ++np1; else ++np2;
    tc_fence_after();
    return true;
  };
  // S into buffer `buf` for Q slot `s` and key block j (event ev), signalled
  // on channel `ch`.
  auto scores = [&](int s, int buf, int ch, int j, uint32_t ev) {
    VLA_TRACE_EVENT(kTrMmaS, s, j);
    issue_scores<D>(tmem + buf * 256, sQ + s * kTile, sK + static_cast<int>(ev % R) * kTile,
                    block_cols(p.N, j));
    mma_commit(bar.s_full(ch));
  };
  auto values = [&](int s, int buf, int j, uint32_t ev) {
    VLA_TRACE_EVENT(kTrMmaPV, s, j);
    issue_values<D>(tmem + s * 256 + 128, tmem + buf * 256, sV + static_cast<int>(ev % R) * kTile,
                    block_cols(p.N, j), j > 0);
    mma_commit(bar.o_prog(s));
  };

  bool ok = true;
  for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
    const uint32_t unit_ev0 = kv_ev;
    for (int rr = 0; ok && rr < p.rounds_per_unit; ++rr) {
      const Round x = make_round(p, u, rr);
      const uint32_t ev0 = p.reuse ? unit_ev0 : kv_ev;
      const bool release = !p.reuse || x.last;
      if (x.nslots == 2) {
        if (!(ok = wait_k(ev0))) break;
        for (int s = 0; s < 2; ++s) {
          if (!(ok = wait_q(s))) break;
          scores(s, s, s, 0, ev0);
          if (nb == 1) mma_commit(bar.q_empty(s));
        }
        if (!ok) break;
        if (release) mma_commit(bar.k_empty(static_cast<int>(ev0 % R)));
        for (int j = 0; ok && j < nb; ++j) {
          const uint32_t ev = ev0 + j;
          if (!(ok = wait_v(ev))) break;
          for (int s = 0; s < 2; ++s) {
            if (!(ok = wait_p(s))) break;
            values(s, s, j, ev);
            if (j + 1 < nb) {
              if (s == 0 && !(ok = wait_k(ev + 1))) break;
              scores(s, s, s, j + 1, ev + 1);
              if (j + 1 == nb - 1) mma_commit(bar.q_empty(s));
            }
          }
          if (!ok) break;
          if (release) {
            mma_commit(bar.v_empty(static_cast<int>(ev % R)));
            if (j + 1 < nb) mma_commit(bar.k_empty(static_cast<int>((ev + 1) % R)));
          }
        }
      } else {
        // Half round: slot 0 alone, S alternating between buffers 0 and 1
        // (channels 0 and 2).
        if (!(ok = wait_q(0))) break;
        for (int j = 0; j < 2 && j < nb; ++j) {
          if (!(ok = wait_k(ev0 + j))) break;
          scores(0, j, 2 * j, j, ev0 + j);
          if (j == nb - 1) mma_commit(bar.q_empty(0));
          if (release) mma_commit(bar.k_empty(static_cast<int>((ev0 + j) % R)));
        }
        for (int j = 0; ok && j < nb; ++j) {
          const uint32_t ev = ev0 + j;
          const int buf = j & 1;
          if (!(ok = wait_v(ev))) break;
          if (!(ok = wait_p(2 * buf))) break;
          values(0, buf, j, ev);
          if (release) mma_commit(bar.v_empty(static_cast<int>(ev % R)));
          if (j + 2 < nb) {
            if (!(ok = wait_k(ev + 2))) break;
            scores(0, buf, 2 * buf, j + 2, ev + 2);
            if (j + 2 == nb - 1) mma_commit(bar.q_empty(0));
            if (release) mma_commit(bar.k_empty(static_cast<int>((ev + 2) % R)));
          }
        }
      }
      if (!p.reuse) kv_ev += nb;
    }
    if (p.reuse) kv_ev += nb;
  }
  // Every tensor-core operation issued above must finish before the tensor
  // memory is freed.
  mma_commit(bar.drain());
  wait_drain(bar.drain(), 0u, kDrainLimitNs);
}

// ------------------------------------------------------------ softmax
struct SoftState {
  float m_run;  // running maximum (raw logits) used for the exponent
  float l_run;  // running sum of weights
};

// One key block for one query row: S (fp32, NC valid columns at compile time,
// nvalid at run time) -> running max / sum, P (bf16 pairs) into the S buffer,
// O rescaled when the maximum grows.  Returns false on abort.
template <int D, int NC>
__device__ __forceinline__ bool softmax_block(const AttnParams& p, SoftState& st, uint32_t tS,
                                              uint32_t tO, int nvalid, bool first_block,
                                              bool use_token, uint32_t tok_wait_bar,
                                              uint32_t tok_wait_parity, uint32_t tok_arrive_bar,
                                              uint32_t o_prog_bar, uint32_t o_prog_parity,
                                              volatile int* abort_flag, int lane) {
  constexpr int DP = TileGeom<D>::kHasTail ? 80 : 64;
  const float c = p.c;
  uint32_t sr[128];
  tmem_ld128(tS, sr);
  float x[NC];
#pragma unroll
  for (int i = 0; i < NC; ++i) x[i] = __uint_as_float(sr[i]);
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
  float alpha = 1.0f;
  if (rescale) {
    const float m_new = fmaxf(st.m_run, m_blk);
    alpha = ex2_approx((st.m_run - m_new) * c);
    st.m_run = m_new;
    st.l_run *= alpha;
  }
  const float mc = st.m_run * c;
  VLA_TRACE_EVENT(kTrSoftMax, 0, 0);
  if (use_token) {
    if (!wait_bounded(tok_wait_bar, tok_wait_parity, abort_flag, p.wait_limit_ns, kSiteSoftTok))
      return false;
  }
  VLA_TRACE_EVENT(kTrSoftTok, 0, 0);
  float lsum[4] = {0.f, 0.f, 0.f, 0.f};
  uint32_t pk[64];
#pragma unroll
  for (int i = 0; i < NC / 2; ++i) {
    const float p0 = ex2_approx(fmaf(x[2 * i], c, -mc));
    const float p1 = ex2_approx(fmaf(x[2 * i + 1], c, -mc));
    lsum[i & 3] += p0 + p1;
    pk[i] = pack_bf16x2(p0, p1);
  }
#pragma unroll
  for (int i = NC / 2; i < 64; ++i) pk[i] = 0u;
  VLA_TRACE_EVENT(kTrSoftExp, 0, 0);
  if (use_token) {
    __syncwarp();
    if (lane == 0) mbar_arrive(tok_arrive_bar);
  }
  st.l_run += (lsum[0] + lsum[1]) + (lsum[2] + lsum[3]);
  tmem_st64(tS, pk);
  if (!first_block) {
    // P V of the previous block has to be complete before O is touched (and
    // this observes every phase of the O progress barrier in order).
    if (!wait_bounded(o_prog_bar, o_prog_parity, abort_flag, p.wait_limit_ns, kSiteSoftO))
      return false;
    tc_fence_after();
    if (rescale) {
      uint32_t ob[64];
      tmem_ld64(tO, ob);
#pragma unroll
      for (int i = 0; i < 64; ++i) ob[i] = __float_as_uint(__uint_as_float(ob[i]) * alpha);
      tmem_st64(tO, ob);
      if (DP > 64) {
        uint32_t ot[16];
        tmem_ld16(tO + 64, ot);
#pragma unroll
        for (int i = 0; i < 16; ++i) ot[i] = __float_as_uint(__uint_as_float(ot[i]) * alpha);
        tmem_st16(tO + 64, ot);
      }
    }
  }
  tmem_wait_st();
  return true;
}

template <int D>
__device__ __forceinline__ bool softmax_block_dispatch(
    const AttnParams& p, SoftState& st, uint32_t tS, uint32_t tO, int ncols, int nvalid,
    bool first_block, bool use_token, uint32_t tw, uint32_t twp, uint32_t ta, uint32_t ob,
    uint32_t obp, volatile int* abort_flag, int lane) {
#define VLA_SB(NC)                                                                          \
  return softmax_block<D, NC>(p, st, tS, tO, nvalid, first_block, use_token, tw, twp, ta, ob, \
                              obp, abort_flag, lane)
  switch (ncols) {
    case 128: VLA_SB(128);
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

template <int D>
__device__ void softmax_role(const AttnParams& p, uint32_t tmem, const Barriers& bar,
                             volatile int* abort_flag, int warp, int lane) {
  constexpr int DP = TileGeom<D>::kHasTail ? 80 : 64;
  const int s = warp >> 2;  // Q slot of this warpgroup
  const int quad = warp & 3;
  const int row_in_tile = quad * 32 + lane;
  const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
  const uint32_t tO = tmem + lane_bits + s * 256 + 128;
  const int nb = p.num_kblocks;
  uint32_t ns0 = 0, ns1 = 0, ns2 = 0;  // s_full phases consumed per channel
  uint32_t npv = 0;           // completions of o_prog[s] accounted for
  uint32_t ntok = 0;          // exp2 turns taken by this warpgroup

  for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
    for (int rr = 0; rr < p.rounds_per_unit; ++rr) {
      const Round x = make_round(p, u, rr);
      const bool full = x.nslots == 2;
      if (!full && s == 1) continue;
      const int tile = 2 * x.r + s;
      SoftState st{-INFINITY, 0.0f};
      for (int j = 0; j < nb; ++j) {
        const int buf = full ? s : (j & 1);
        const int ch = full ? s : 2 * buf;
        const uint32_t ns = ch == 0 ? ns0 : (ch == 1 ? ns1 : ns2);
        if (!wait_bounded(bar.s_full(ch), ns & 1u, abort_flag, p.wait_limit_ns, kSiteSoftS))
          return;
        if (ch == 0) ++ns0; else if (ch == 1) ++ns1; else ++ns2;
        VLA_TRACE_EVENT(kTrSoftS, s, j);
        tc_fence_after();
        const uint32_t tS = tmem + lane_bits + buf * 256;
        // Slot 0 takes exp2 turns 0, 1, 2, ... after slot 1's turns -1, 0, 1, ...
        const uint32_t tw = bar.tok(s);
        const uint32_t twp = s == 0 ? ((ntok & 1u) ^ 1u) : (ntok & 1u);
        const bool ok = softmax_block_dispatch<D>(
            p, st, tS, tO, block_cols(p.N, j), min(kTileRows, p.N - j * kTileRows), j == 0, full,
            tw, twp, bar.tok(1 - s), bar.o_prog(s), (npv + j - 1) & 1u, abort_flag, lane);
        if (!ok) return;
        if (full) ++ntok;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar.p_full(ch));
        VLA_TRACE_EVENT(kTrSoftP, s, j);
      }
      // Epilogue: wait for the last P V, then O / l -> bf16, 16-byte stores.
      if (!wait_bounded(bar.o_prog(s), (npv + nb - 1) & 1u, abort_flag, p.wait_limit_ns,
                        kSiteSoftO))
        return;
      npv += nb;
      tc_fence_after();
      VLA_TRACE_EVENT(kTrSoftEpi, s, 0);
      const float inv_l = 1.0f / st.l_run;
      uint32_t ob[64];
      tmem_ld64(tO, ob);
      uint32_t ot[16];
      if (DP > 64) tmem_ld16(tO + 64, ot);
      const int row = tile * kTileRows + row_in_tile;
      if (row < p.N) {
        uint4* dst = reinterpret_cast<uint4*>(
            p.o + ((static_cast<size_t>(x.b) * p.N + row) * p.H + x.h) * D);
#pragma unroll
        for (int t = 0; t < D / 8; ++t) {
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int ch = 8 * t + e;
            v[e] = __uint_as_float(ch < 64 ? ob[ch] : ot[ch - 64]) * inv_l;
          }
          uint4 w;
          w.x = pack_bf16x2(v[0], v[1]);
          w.y = pack_bf16x2(v[2], v[3]);
          w.z = pack_bf16x2(v[4], v[5]);
          w.w = pack_bf16x2(v[6], v[7]);
          dst[t] = w;
        }
      }
    }
  }
}

// ------------------------------------------------------------ kernel
template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  constexpr uint32_t kTile = TileGeom<D>::kBytes;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t sQ = base;
  const uint32_t sK = sQ + 2 * kTile;
  const uint32_t sV = sK + p.ring * kTile;
  const uint32_t sBar = sV + p.ring * kTile;
  uint8_t* bar_generic = smem_raw + (sBar - raw);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_generic + 8 * kNumBarriers);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_generic + 8 * kNumBarriers + 4);
  const Barriers bar{sBar};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar.q_full(s), 1);
      mbar_init(bar.q_empty(s), 1);
      mbar_init(bar.o_prog(s), 1);
      mbar_init(bar.tok(s), 4);
    }
    for (int ch = 0; ch < 3; ++ch) {
      mbar_init(bar.s_full(ch), 1);
      mbar_init(bar.p_full(ch), 4);
    }
    for (int i = 0; i < kMaxRing; ++i) {
      mbar_init(bar.k_full(i), 1);
      mbar_init(bar.k_empty(i), 1);
      mbar_init(bar.v_full(i), 1);
      mbar_init(bar.v_empty(i), 1);
    }
    mbar_init(bar.drain(), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  VLA_TRACE_INIT();
  if (warp == kLoadWarp && lane == 0) {
    prefetch_tmap(&p.tm_main);
    if (TileGeom<D>::kHasTail) prefetch_tmap(&p.tm_tail);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kLoadWarp) {
    if (lane == 0) load_role<D>(p, sQ, sK, sV, bar, abort_flag);
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if (lane == 0) mma_role<D>(p, tmem, sQ, sK, sV, bar, abort_flag);
    __syncwarp();
  } else if (warp < 8) {
    softmax_role<D>(p, tmem, bar, abort_flag, warp, lane);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace vla
