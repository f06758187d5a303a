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
// Blackwell mapping (one persistent CTA per SM, 320 threads):
//   warp 9      TMA producer: Q tiles (128 query rows) into two Q slots, K and
//               V blocks (128 keys) into a ring of `ring` slots.  With
//               `reuse`, a head's K/V blocks are loaded once and serve all of
//               that head's Q tiles.
//   warp 8      tcgen05 issuer (one thread): S = Q K^T into tensor memory
//               (SS MMA, M=128, N=keys of the block, K=16 steps over d), then
//               O += P V with P read from tensor memory (TS MMA, N=64 or
//               64+16).  Two Q tiles ("slots") are interleaved so the tensor
//               core works on one slot while the other slot's softmax runs.
//   warps 0-7   softmax, one warpgroup per slot, one thread per query row
//               (= tensor-memory lane): online softmax in fp32 with exp2 and a
//               pre-scaled log2(e), P packed to bf16 pairs and stored back over
//               its own S columns, O rescaled in tensor memory only when the
//               running maximum grows by more than 2^8, epilogue O / l -> bf16
//               with 16-byte stores.
//
// Tensor memory (512 columns): slot s uses columns [256 s, 256 s + 128) for
// S (fp32) -- later overwritten in place by P (bf16 pairs, 64 columns) -- and
// [256 s + 128, 256 s + 128 + 80) for the fp32 O accumulator.
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
#pragma once

#include <cuda_bf16.h>
#include <math.h>

#include "ptx.cuh"

namespace vla {

constexpr int kTileRows = 128;  // query rows per tile = keys per block = TMEM lanes
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kThreads = 320;
constexpr int kMaxRing = 6;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kMainRegionBytes = 128 * 128;  // 128 rows x 64 bf16 channels
constexpr uint32_t kTailRegionBytes = 128 * 32;   // 128 rows x 16 bf16 channels
constexpr int kNumBarriers = 10 + 4 * kMaxRing + 1;
constexpr uint32_t kBarrierRegionBytes = 512;     // barriers + tmem address + abort flag
constexpr uint32_t kAlignSlack = 1024;

// Device status codes (the first wait that ran out records its site).
enum : int {
  kSiteLoadQ = 1, kSiteLoadK = 2, kSiteLoadV = 3,
  kSiteMmaQ = 11, kSiteMmaK = 12, kSiteMmaV = 13, kSiteMmaP = 14,
  kSiteSoftS = 21, kSiteSoftO = 22,
  kSiteDrain = 31,
};

__device__ int g_vla_attn_status;  // 0 = ok, else 1000 + site of the first timed-out wait

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
  __device__ uint32_t s_full(int s) const { return base + 8u * (4 + s); }
  __device__ uint32_t p_full(int s) const { return base + 8u * (6 + s); }
  __device__ uint32_t o_full(int s) const { return base + 8u * (8 + s); }
  __device__ uint32_t k_full(int i) const { return base + 8u * (10 + i); }
  __device__ uint32_t k_empty(int i) const { return base + 8u * (10 + kMaxRing + i); }
  __device__ uint32_t v_full(int i) const { return base + 8u * (10 + 2 * kMaxRing + i); }
  __device__ uint32_t v_empty(int i) const { return base + 8u * (10 + 3 * kMaxRing + i); }
  __device__ uint32_t drain() const { return base + 8u * (10 + 4 * kMaxRing); }
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

// ------------------------------------------------------------ producer
template <int D>
__device__ void load_role(const AttnParams& p, uint32_t sQ, uint32_t sK, uint32_t sV,
                          const Barriers& bar, volatile int* abort_flag) {
  constexpr uint32_t kTile = TileGeom<D>::kBytes;
  const int R = p.ring;
  const int nb = p.num_kblocks;
  uint32_t nq[2] = {0u, 0u};
  uint32_t kv_ev = 0;
  for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
    const int bh = u / p.units_per_head;
    const int r0 = (u % p.units_per_head) * p.rounds_per_unit;
    const int b = bh / p.H, h = bh % p.H;
    for (int rr = 0; rr < p.rounds_per_unit; ++rr) {
      const int r = r0 + rr;
      const int nslots = (2 * r + 1 < p.num_qtiles) ? 2 : 1;
      if (!p.reuse || rr == 0) {
        for (int j = 0; j < nb; ++j) {
          const int slot = static_cast<int>(kv_ev % R);
          const uint32_t n = kv_ev / R;
          if (!wait_bounded(bar.k_empty(slot), (n & 1u) ^ 1u, abort_flag, p.wait_limit_ns,
                            kSiteLoadK))
            goto drain;
          mbar_arrive_expect_tx(bar.k_full(slot), kTile);
          tma_load_5d(sK + slot * kTile, &p.tm_main, bar.k_full(slot), 0, h, 1, j * kTileRows, b);
          if (TileGeom<D>::kHasTail)
            tma_load_5d(sK + slot * kTile + kMainRegionBytes, &p.tm_tail, bar.k_full(slot), 64, h,
                        1, j * kTileRows, b);
          if (j == 0) {
            // Q tiles go right after the first K block so S(0) can start early.
            for (int s = 0; s < nslots; ++s) {
              if (!wait_bounded(bar.q_empty(s), (nq[s] & 1u) ^ 1u, abort_flag, p.wait_limit_ns,
                                kSiteLoadQ))
                goto drain_k;
              mbar_arrive_expect_tx(bar.q_full(s), kTile);
              const int row0 = (2 * r + s) * kTileRows;
              tma_load_5d(sQ + s * kTile, &p.tm_main, bar.q_full(s), 0, h, 0, row0, b);
              if (TileGeom<D>::kHasTail)
                tma_load_5d(sQ + s * kTile + kMainRegionBytes, &p.tm_tail, bar.q_full(s), 64, h,
                            0, row0, b);
              ++nq[s];
            }
          }
          if (!wait_bounded(bar.v_empty(slot), (n & 1u) ^ 1u, abort_flag, p.wait_limit_ns,
                            kSiteLoadV))
            goto drain_k;
          mbar_arrive_expect_tx(bar.v_full(slot), kTile);
          tma_load_5d(sV + slot * kTile, &p.tm_main, bar.v_full(slot), 0, h, 2, j * kTileRows, b);
          if (TileGeom<D>::kHasTail)
            tma_load_5d(sV + slot * kTile + kMainRegionBytes, &p.tm_tail, bar.v_full(slot), 64, h,
                        2, j * kTileRows, b);
          ++kv_ev;
          continue;
        drain_k:
          // K of this event was issued but V was not: count K as armed only.
          wait_drain(bar.k_full(slot), n & 1u, 100000000ull);
          goto drain;
        }
      } else {
        for (int s = 0; s < nslots; ++s) {
          if (!wait_bounded(bar.q_empty(s), (nq[s] & 1u) ^ 1u, abort_flag, p.wait_limit_ns,
                            kSiteLoadQ))
            goto drain;
          mbar_arrive_expect_tx(bar.q_full(s), kTile);
          const int row0 = (2 * r + s) * kTileRows;
          tma_load_5d(sQ + s * kTile, &p.tm_main, bar.q_full(s), 0, h, 0, row0, b);
          if (TileGeom<D>::kHasTail)
            tma_load_5d(sQ + s * kTile + kMainRegionBytes, &p.tm_tail, bar.q_full(s), 64, h, 0,
                        row0, b);
          ++nq[s];
        }
      }
    }
  }
drain:
  // Wait (bounded) until every copy this thread issued has landed.
  for (int s = 0; s < 2; ++s)
    if (nq[s] > 0) wait_drain(bar.q_full(s), (nq[s] - 1u) & 1u, 100000000ull);
  for (int i = 0; i < R; ++i) {
    const uint32_t arms = kv_ev / R + (static_cast<uint32_t>(i) < kv_ev % R ? 1u : 0u);
    if (arms > 0) {
      wait_drain(bar.k_full(i), (arms - 1u) & 1u, 100000000ull);
      wait_drain(bar.v_full(i), (arms - 1u) & 1u, 100000000ull);
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
  uint32_t nq[2] = {0u, 0u};
  uint32_t np[2] = {0u, 0u};
  uint32_t kv_ev = 0;
  for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
    const int r0 = (u % p.units_per_head) * p.rounds_per_unit;
    const uint32_t unit_ev0 = kv_ev;
    for (int rr = 0; rr < p.rounds_per_unit; ++rr) {
      const int r = r0 + rr;
      const int nslots = (2 * r + 1 < p.num_qtiles) ? 2 : 1;
      const uint32_t ev0 = p.reuse ? unit_ev0 : kv_ev;
      const bool last_use = !p.reuse || rr == p.rounds_per_unit - 1;
      // First key block: S for every slot of the round.
      {
        const int slot = static_cast<int>(ev0 % R);
        if (!wait_bounded(bar.k_full(slot), (ev0 / R) & 1u, abort_flag, p.wait_limit_ns,
                          kSiteMmaK))
          goto drain;
        for (int s = 0; s < nslots; ++s) {
          if (!wait_bounded(bar.q_full(s), nq[s] & 1u, abort_flag, p.wait_limit_ns, kSiteMmaQ))
            goto drain;
          ++nq[s];
          tc_fence_after();
          issue_scores<D>(tmem + s * 256, sQ + s * kTile, sK + slot * kTile, block_cols(p.N, 0));
          mma_commit(bar.s_full(s));
          if (nb == 1) mma_commit(bar.q_empty(s));
        }
        if (last_use) mma_commit(bar.k_empty(slot));
      }
      for (int j = 0; j < nb; ++j) {
        const uint32_t ev = ev0 + j;
        const int vslot = static_cast<int>(ev % R);
        if (!wait_bounded(bar.v_full(vslot), (ev / R) & 1u, abort_flag, p.wait_limit_ns,
                          kSiteMmaV))
          goto drain;
        const bool has_next = j + 1 < nb;
        const uint32_t evn = ev + 1;
        const int kslot = static_cast<int>(evn % R);
        for (int s = 0; s < nslots; ++s) {
          if (!wait_bounded(bar.p_full(s), np[s] & 1u, abort_flag, p.wait_limit_ns, kSiteMmaP))
            goto drain;
          ++np[s];
          tc_fence_after();
          issue_values<D>(tmem + s * 256 + 128, tmem + s * 256, sV + vslot * kTile,
                          block_cols(p.N, j), j > 0);
          if (!has_next) mma_commit(bar.o_full(s));
          if (has_next) {
            if (s == 0) {
              if (!wait_bounded(bar.k_full(kslot), (evn / R) & 1u, abort_flag, p.wait_limit_ns,
                                kSiteMmaK))
                goto drain;
              tc_fence_after();
            }
            issue_scores<D>(tmem + s * 256, sQ + s * kTile, sK + kslot * kTile,
                            block_cols(p.N, j + 1));
            mma_commit(bar.s_full(s));
            if (j + 1 == nb - 1) mma_commit(bar.q_empty(s));
          }
        }
        if (last_use) {
          mma_commit(bar.v_empty(vslot));
          if (has_next) mma_commit(bar.k_empty(kslot));
        }
      }
      if (!p.reuse) kv_ev += nb;
    }
    if (p.reuse) kv_ev += nb;
  }
drain:
  // Every tensor-core operation issued above must finish before the tensor
  // memory is freed.
  mma_commit(bar.drain());
  wait_drain(bar.drain(), 0u, 100000000ull);
}

// ------------------------------------------------------------ softmax
template <int D>
__device__ void softmax_role(const AttnParams& p, uint32_t tmem, const Barriers& bar,
                             volatile int* abort_flag, int warp, int lane) {
  constexpr int DP = TileGeom<D>::kHasTail ? 80 : 64;
  const int s = warp >> 2;
  const int quad = warp & 3;
  const int row_in_tile = quad * 32 + lane;
  const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
  const uint32_t tS = tmem + lane_bits + s * 256;
  const uint32_t tO = tS + 128;
  const int nb = p.num_kblocks;
  const float c = p.c;
  uint32_t ns = 0, no = 0;

  for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
    const int bh = u / p.units_per_head;
    const int r0 = (u % p.units_per_head) * p.rounds_per_unit;
    const int b = bh / p.H, h = bh % p.H;
    for (int rr = 0; rr < p.rounds_per_unit; ++rr) {
      const int r = r0 + rr;
      const int tile = 2 * r + s;
      if (tile >= p.num_qtiles) continue;
      float m_run = -INFINITY;
      float l_run = 0.0f;
      for (int j = 0; j < nb; ++j) {
        if (!wait_bounded(bar.s_full(s), ns & 1u, abort_flag, p.wait_limit_ns, kSiteSoftS))
          return;
        ++ns;
        tc_fence_after();
        const int nvalid = min(kTileRows, p.N - j * kTileRows);
        float x[128];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t rbuf[32];
          tmem_ld32(tS + ch * 32, rbuf);
#pragma unroll
          for (int i = 0; i < 32; ++i) x[ch * 32 + i] = __uint_as_float(rbuf[i]);
        }
        if (nvalid < kTileRows) {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= nvalid) x[i] = -INFINITY;
        }
        float mx[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
        for (int i = 4; i < 128; i += 4) {
          mx[0] = fmaxf(mx[0], x[i + 0]);
          mx[1] = fmaxf(mx[1], x[i + 1]);
          mx[2] = fmaxf(mx[2], x[i + 2]);
          mx[3] = fmaxf(mx[3], x[i + 3]);
        }
        const float m_blk = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        // Keep a stale maximum unless the block's maximum exceeds it by more
        // than 8 in log2 units: the final O / l cancels the common factor, and
        // weights stay below 2^8.
        const bool grow = (m_blk - m_run) * c > 8.0f;
        const bool rescale = __any_sync(0xffffffffu, grow);
        float alpha = 1.0f;
        if (rescale) {
          const float m_new = fmaxf(m_run, m_blk);
          alpha = ex2_approx((m_run - m_new) * c);
          m_run = m_new;
          l_run *= alpha;
        }
        const float mc = m_run * c;
        float lsum[4] = {0.f, 0.f, 0.f, 0.f};
        {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float p0 = ex2_approx(fmaf(x[2 * i], c, -mc));
            const float p1 = ex2_approx(fmaf(x[2 * i + 1], c, -mc));
            lsum[i & 3] += p0 + p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
          tmem_st32(tS, pk);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float p0 = ex2_approx(fmaf(x[64 + 2 * i], c, -mc));
            const float p1 = ex2_approx(fmaf(x[64 + 2 * i + 1], c, -mc));
            lsum[i & 3] += p0 + p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
          tmem_st32(tS + 32, pk);
        }
        l_run += (lsum[0] + lsum[1]) + (lsum[2] + lsum[3]);
        if (rescale && j > 0) {
          // O holds P V of blocks < j (that MMA completed before S of block j
          // was signalled); scale it by alpha in place.
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t ob[32];
            tmem_ld32(tO + ch * 32, ob);
#pragma unroll
            for (int i = 0; i < 32; ++i) ob[i] = __float_as_uint(__uint_as_float(ob[i]) * alpha);
            tmem_st32(tO + ch * 32, ob);
          }
          if (DP > 64) {
            uint32_t ob[16];
            tmem_ld16(tO + 64, ob);
#pragma unroll
            for (int i = 0; i < 16; ++i) ob[i] = __float_as_uint(__uint_as_float(ob[i]) * alpha);
            tmem_st16(tO + 64, ob);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar.p_full(s));
      }
      // Epilogue: O / l -> bf16, one 16-byte store per 8 channels.
      if (!wait_bounded(bar.o_full(s), no & 1u, abort_flag, p.wait_limit_ns, kSiteSoftO)) return;
      ++no;
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      uint32_t ob[DP];
      {
        uint32_t t32[32];
        tmem_ld32(tO, t32);
#pragma unroll
        for (int i = 0; i < 32; ++i) ob[i] = t32[i];
        tmem_ld32(tO + 32, t32);
#pragma unroll
        for (int i = 0; i < 32; ++i) ob[32 + i] = t32[i];
        if (DP > 64) {
          uint32_t t16[16];
          tmem_ld16(tO + 64, t16);
#pragma unroll
          for (int i = 0; i < 16; ++i) ob[64 + i] = t16[i];
        }
      }
      const int row = tile * kTileRows + row_in_tile;
      if (row < p.N) {
        uint4* dst = reinterpret_cast<uint4*>(
            p.o + ((static_cast<size_t>(b) * p.N + row) * p.H + h) * D);
#pragma unroll
        for (int t = 0; t < D / 8; ++t) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(ob[8 * t + 0]) * inv_l,
                            __uint_as_float(ob[8 * t + 1]) * inv_l);
          v.y = pack_bf16x2(__uint_as_float(ob[8 * t + 2]) * inv_l,
                            __uint_as_float(ob[8 * t + 3]) * inv_l);
          v.z = pack_bf16x2(__uint_as_float(ob[8 * t + 4]) * inv_l,
                            __uint_as_float(ob[8 * t + 5]) * inv_l);
          v.w = pack_bf16x2(__uint_as_float(ob[8 * t + 6]) * inv_l,
                            __uint_as_float(ob[8 * t + 7]) * inv_l);
          dst[t] = v;
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
      mbar_init(bar.s_full(s), 1);
      mbar_init(bar.p_full(s), 4);
      mbar_init(bar.o_full(s), 1);
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
  } else {
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
