// Linear layer y = act(x w^T + bias) (+ res) for sm_100a: a persistent
// tcgen05 GEMM with its epilogue fused, for the layers around the attention
// core of a ViT encoder layer (the qkv projection, the output projection with
// the residual add, the MLP's fc1 with GELU and fc2 with the residual add).
//
// The pages' fused operators: "FluxVLA docs, inference acceleration",
// section 1 (Triton fused kernels: matrix multiply + bias + activation) and
// section 3 (CUDA custom operators: a GEMM + bias, and GEMM + bias + residual,
// in one launch); "Pi0 VLA deployment tutorial", section 3.2 (the block's qkv
// linear feeds the attention).  For the qkv linear (N = 3 H d) the row-major
// output [M, N] is exactly the packed [B, tokens, 3, H, d] input of the
// attention kernel, so no layout change is needed.
//
// Arithmetic: bf16 x and w, fp32 accumulation on the tensor cores, the
// epilogue in fp32 (bias, GELU, residual), one rounding to bf16 (nearest even)
// on store.  GELU is the tanh form a/2 (1 + tanh(sqrt(2/pi) (a + 0.044715
// a^3))) with the hardware tanh approximation.
//
// Blackwell mapping (one persistent CTA per SM, 384 threads):
//   warp 0      TMA producer: per k-step a 128 x 64 tile of x and a BN x 64
//               tile of w (both K-major, 128-byte swizzle) into a ring of
//               stages.
//   warp 1      tcgen05 issuer: per k-step 4 MMAs (M=128, N=BN, K=16) into
//               one of two fp32 accumulators in tensor memory (2 x BN
//               columns), so the epilogue of one tile overlaps the next
//               tile's MMAs.
//   warps 4-11  epilogue: one thread per output row (= tensor-memory lane),
//               two warps per 32-row quarter taking alternate 64-column
//               chunks, each chunk staged in shared memory (the residual
//               brought in by a TMA load) and written by a TMA store.
//   warps 2-3   idle.
// Split K: with few output tiles the K range is cut into `splits` parts; each
// part's CTA writes fp32 partial sums to the caller's workspace, and for each
// 32-row quarter of a tile the last epilogue warp to arrive (an arrival
// counter per quarter in the same workspace) adds the parts up in split order
// and runs the epilogue, so the result does not depend on which part finishes
// first.
//
// Every mbarrier wait is bounded (same helpers and abort protocol as the
// attention kernel): a wait that runs out records its site in the device
// status word, every role leaves its loop, the producer waits for its own
// copies, the issuer for its own tensor-core work, and the tensor memory is
// freed.
#pragma once

#include <cuda_bf16.h>

#include "attn_kernel.cuh"
#include "ptx.cuh"

namespace vla {
namespace gemm {

constexpr int kBM = 128;     // rows per tile = tensor-memory lanes = MMA M
constexpr int kBK = 64;      // K per stage: one 128-byte swizzle atom of bf16
// Epilogue warps: two per SM sub-partition (warps 4-7 and 8-11, the same
// tensor-memory lanes), taking alternate 64-column chunks of a tile, with one
// staging buffer each.  One warp per sub-partition with two buffers and the
// residual prefetched a chunk ahead measured 11 % slower on the output
// projection and 10 % slower on fc1 with GELU (the epilogue, not the MMAs, set
// the pace there).
constexpr int kEpiWarps = 8;
constexpr int kThreads = 128 + 32 * kEpiWarps;
constexpr int kLoadWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kEpiWarp0 = 4;
constexpr int kMaxStages = 8;
// Barriers: per stage full / empty, per accumulator full / empty, two drain
// barriers, and one per residual staging buffer; then the tensor-memory
// address and the abort flag.
constexpr int kNumBarriers = 2 * kMaxStages + 6 + 8;
constexpr uint32_t kBarrierBytes = 512;
static_assert(8 * kNumBarriers + 8 <= kBarrierBytes, "barrier region");
// Output staging of the epilogue: per epilogue warp one buffer of 32 rows x 64
// columns of bf16 (4 KB, 128-byte swizzle) that TMA stores to y (and that a
// TMA load fills with the residual first).
constexpr uint32_t kStageOutBytes = 32 * 128;
constexpr uint32_t kStagingBytes = kEpiWarps * kStageOutBytes;
static_assert(2 * kMaxStages + 6 + kEpiWarps <= kNumBarriers,
              "every residual barrier lies below the tensor-memory address slot");

enum : int { kActNone = 0, kActGelu = 1 };

enum : int {
  kSiteLoad = 51, kSiteMmaFull = 52, kSiteMmaAcc = 53, kSiteEpi = 54, kSiteSplit = 55,
  kSiteDrain = 56,
};

struct GemmParams {
  CUtensorMap tm_a;              // x [M, K] bf16, box {64, 128}
  CUtensorMap tm_b;              // w [N, K] bf16, box {64, BN}
  CUtensorMap tm_y;              // y [M, N] bf16, box {64, 32} (epilogue stores)
  CUtensorMap tm_res;            // res [M, N] bf16, box {64, 32} (when res is given)
  const __nv_bfloat16* bias;     // [N] or null
  const __nv_bfloat16* res;      // [M, N] or null (may be y itself)
  __nv_bfloat16* y;              // [M, N]
  float* partial;                // split K: [splits][tiles][128 x BN] fp32
  unsigned int* counters;        // split K: arrivals per (tile, 32-row quarter), zeroed before
                                 // the launch
  int M, N, K;
  int tiles_m, tiles_n;          // output tiles
  int splits;                    // parts of the K range (1 = no split)
  int ksteps_per_split;          // k-steps of 64 per part (the last part may have fewer)
  int ksteps;                    // k-steps of the whole K range
  int num_work;                  // tiles_m * tiles_n * splits
  int stages;
  int act;
  unsigned long long wait_limit_ns;
};

template <int BN>
struct GemmGeom {
  static_assert(BN == 64 || BN == 128 || BN == 256, "tile N must be 64, 128 or 256");
  static constexpr uint32_t kABytes = kBM * kBK * 2;  // 16 KB
  static constexpr uint32_t kBBytes = BN * kBK * 2;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kTmemCols = 2 * BN;       // two accumulators
};

template <int BN>
__host__ __device__ constexpr uint32_t gemm_smem_bytes(int stages) {
  return static_cast<uint32_t>(stages) * GemmGeom<BN>::kStageBytes + kStagingBytes +
         kBarrierBytes + 1024u;
}

struct GemmBarriers {
  uint32_t base;
  __device__ uint32_t full(int s) const { return base + 8u * s; }
  __device__ uint32_t empty(int s) const { return base + 8u * (kMaxStages + s); }
  __device__ uint32_t acc_full(int b) const { return base + 8u * (2 * kMaxStages + b); }
  __device__ uint32_t acc_empty(int b) const { return base + 8u * (2 * kMaxStages + 2 + b); }
  __device__ uint32_t drain(int i) const { return base + 8u * (2 * kMaxStages + 4 + i); }
  // Residual tile landed in the staging buffer of epilogue warp e.
  __device__ uint32_t res_full(int e) const { return base + 8u * (2 * kMaxStages + 6 + e); }
};

// Tiled 2-D store of a shared-memory box to global memory (bulk group).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(src)
               : "memory");
}

// 2-D tiled load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// The k-th work item of this CTA -> output tile and K part; false when the CTA
// has no k-th item.  Items w = blockIdx.x + k G of the list ordered split, then
// M row, then N tile: the CTAs running at one time cover a few rows of tiles,
// all N tiles of each, so a row block of x is read from DRAM about once and
// w (at most a few MB for these layers) stays in L2.
struct Work {
  int mt, nt, split;
  int k0, k1;  // k-steps [k0, k1)
};

__device__ __forceinline__ bool work_at(const GemmParams& p, int k, Work& r) {
  const int w = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
  if (w >= p.num_work) return false;
  const int tiles = p.tiles_m * p.tiles_n;
  r.split = w / tiles;
  const int t = w - r.split * tiles;
  r.mt = t / p.tiles_n;
  r.nt = t - r.mt * p.tiles_n;
  r.k0 = r.split * p.ksteps_per_split;
  r.k1 = min(p.ksteps, r.k0 + p.ksteps_per_split);
  return true;
}

template <int BN>
__device__ __forceinline__ void gemm_load_role(const GemmParams& p, uint32_t sbase,
                                               const GemmBarriers& bar,
                                               volatile int* abort_flag) {
  using G = GemmGeom<BN>;
  int stage = 0;
  uint32_t phase = 0;
  uint32_t issued = 0;
  bool ok = true;
  Work wk;
  for (int k = 0; ok && work_at(p, k, wk); ++k) {
    for (int ks = wk.k0; ks < wk.k1; ++ks) {
      if (!wait_bounded(bar.empty(stage), phase ^ 1u, abort_flag, p.wait_limit_ns, kSiteLoad)) {
        ok = false;
        break;
      }
      if (elect_one()) {
        const uint32_t dst = sbase + stage * G::kStageBytes;
        mbar_arrive_expect_tx(bar.full(stage), G::kStageBytes);
        tma_load_2d(dst, &p.tm_a, bar.full(stage), ks * kBK, wk.mt * kBM);
        tma_load_2d(dst + G::kABytes, &p.tm_b, bar.full(stage), ks * kBK, wk.nt * BN);
      }
      __syncwarp();
      ++issued;
      if (++stage == p.stages) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  // Wait (bounded) until every copy issued has landed: the last phase of each
  // stage that was armed.
  for (int s = 0; s < p.stages; ++s) {
    const uint32_t arms = issued / p.stages + (static_cast<uint32_t>(s) < issued % p.stages);
    if (arms > 0) wait_drain(bar.full(s), (arms - 1u) & 1u, kDrainLimitNs);
  }
}

template <int BN>
__device__ __forceinline__ void gemm_mma_role(const GemmParams& p, uint32_t tmem, uint32_t sbase,
                                              const GemmBarriers& bar,
                                              volatile int* abort_flag) {
  using G = GemmGeom<BN>;
  constexpr uint32_t kIdesc = idesc_bf16_m128(static_cast<uint32_t>(BN), 0u);
  const uint64_t a0 = smem_desc(sbase, 16, 1024, kSwizzle128);
  const uint64_t b0 = smem_desc(sbase + G::kABytes, 16, 1024, kSwizzle128);
  constexpr uint64_t kStageStep = G::kStageBytes >> 4;
  int stage = 0;
  uint32_t phase = 0;
  bool ok = true;
  Work wk;
  for (int i = 0; ok && work_at(p, i, wk); ++i) {  // i: work items of this CTA
    const int buf = i & 1;
    // The epilogue must have read this accumulator's previous tile.
    if (!wait_bounded(bar.acc_empty(buf), ((i >> 1) & 1) ^ 1, abort_flag, p.wait_limit_ns,
                      kSiteMmaAcc)) {
      ok = false;
      break;
    }
    tc_fence_after();
    const uint32_t d = tmem + static_cast<uint32_t>(buf * BN);
    for (int ks = wk.k0; ks < wk.k1; ++ks) {
      if (!wait_bounded(bar.full(stage), phase, abort_flag, p.wait_limit_ns, kSiteMmaFull)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
        const uint64_t ad = a0 + stage * kStageStep;
        const uint64_t bd = b0 + stage * kStageStep;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          mma_ss(d, ad + 2 * kk, bd + 2 * kk, kIdesc, (ks > wk.k0 || kk > 0) ? 1u : 0u);
        mma_commit(bar.empty(stage));  // stage free once these MMAs have read it
      }
      __syncwarp();
      if (++stage == p.stages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (!ok) break;
    if (elect_one()) mma_commit(bar.acc_full(buf));
    __syncwarp();
  }
  if (elect_one()) mma_commit(bar.drain(0));
  __syncwarp();
  wait_drain(bar.drain(0), 0u, kDrainLimitNs);
}

__device__ __forceinline__ float gelu_tanh(float a) {
  // a/2 (1 + tanh(sqrt(2/pi) (a + 0.044715 a^3)))
  const float k0 = 0.7978845608028654f;  // sqrt(2 / pi)
  const float k1 = 0.044715f;
  const float u = k0 * fmaf(k1 * a, a * a, a);
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(u));
  const float h = 0.5f * a;
  return fmaf(h, t, h);
}

// Epilogue of 8 consecutive columns of one row: v = acc (+ bias) -> act (+ res)
// -> bf16, one 16-byte store.
__device__ __forceinline__ void store8(const GemmParams& p, const float (&acc)[8], int row, int n) {
  float v[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = acc[e];
  if (p.bias != nullptr) {
    const uint4 bb = *reinterpret_cast<const uint4*>(p.bias + n);
    const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] += __uint_as_float(bw[e] << 16);
      v[2 * e + 1] += __uint_as_float(bw[e] & 0xFFFF0000u);
    }
  }
  if (p.act == kActGelu) {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = gelu_tanh(v[e]);
  }
  const size_t off = static_cast<size_t>(row) * p.N + n;
  if (p.res != nullptr) {
    const uint4 rb = *reinterpret_cast<const uint4*>(p.res + off);
    const uint32_t rw[4] = {rb.x, rb.y, rb.z, rb.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] += __uint_as_float(rw[e] << 16);
      v[2 * e + 1] += __uint_as_float(rw[e] & 0xFFFF0000u);
    }
  }
  uint4 o;
  o.x = pack_bf16x2(v[0], v[1]);
  o.y = pack_bf16x2(v[2], v[3]);
  o.z = pack_bf16x2(v[4], v[5]);
  o.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p.y + off) = o;
}

// Epilogue of 8 consecutive columns n.. of one row from fp32 accumulators:
// (+ bias) -> act (+ the residual's 8 bf16 values) -> 4 packed bf16 pairs.
__device__ __forceinline__ uint4 epi8(const GemmParams& p, const uint32_t* acc, int n,
                                      const uint4* res8) {
  float v[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(acc[e]);
  if (p.bias != nullptr && n < p.N) {
    const uint4 bb = *reinterpret_cast<const uint4*>(p.bias + n);
    const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] += __uint_as_float(bw[e] << 16);
      v[2 * e + 1] += __uint_as_float(bw[e] & 0xFFFF0000u);
    }
  }
  if (p.act == kActGelu) {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = gelu_tanh(v[e]);
  }
  if (res8 != nullptr) {
    const uint32_t rw[4] = {res8->x, res8->y, res8->z, res8->w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[2 * e] += __uint_as_float(rw[e] << 16);
      v[2 * e + 1] += __uint_as_float(rw[e] & 0xFFFF0000u);
    }
  }
  uint4 o;
  o.x = pack_bf16x2(v[0], v[1]);
  o.y = pack_bf16x2(v[2], v[3]);
  o.z = pack_bf16x2(v[4], v[5]);
  o.w = pack_bf16x2(v[6], v[7]);
  return o;
}

// Residual loads of one epilogue warp: how many were issued, and whether the
// last one has not been waited for.
struct EpiRes {
  uint32_t issued = 0;
  bool pending = false;
};

template <int BN>
__device__ __forceinline__ void gemm_epilogue_loop(const GemmParams& p, uint32_t tmem,
                                                   const GemmBarriers& bar,
                                                   volatile int* abort_flag, int warp, int lane,
                                                   uint32_t buf_s, EpiRes& rs) {
  const int quad = warp & 3;
  const int ew = warp - kEpiWarp0;  // epilogue warp
  const int set = ew >> 2;          // its 64-column chunks: set, set + 2, ...
  const int r_in = quad * 32 + lane;
  const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
  const size_t tile_elems = static_cast<size_t>(kBM) * BN;
  const int tiles = p.tiles_m * p.tiles_n;
  // The residual of this warp's chunk c of tile (mt, nt) into its buffer, once
  // the store that last read the buffer is done reading it.
  auto load_res = [&](const Work& w, int c) {
    if (lane == 0) {
      bulk_wait_read<0>();
      mbar_arrive_expect_tx(bar.res_full(ew), kStageOutBytes);
      tma_load_2d(buf_s, &p.tm_res, bar.res_full(ew), w.nt * BN + 64 * c, w.mt * kBM + quad * 32);
    }
    __syncwarp();
    rs.pending = true;
  };
  const bool res_tiles = p.res != nullptr && p.splits == 1 && set < BN / 64;
  Work wk;
  for (int i = 0; work_at(p, i, wk); ++i) {
    const int buf = i & 1;
    // The first chunk's residual does not depend on the accumulator: its load
    // runs while the tile's MMAs do.
    if (res_tiles) load_res(wk, set);
    if (!wait_bounded(bar.acc_full(buf), (i >> 1) & 1, abort_flag, p.wait_limit_ns, kSiteEpi))
      return;
    tc_fence_after();
    const uint32_t t = tmem + lane_bits + static_cast<uint32_t>(buf * BN);
    const int row = wk.mt * kBM + r_in;
    const int n_base = wk.nt * BN;
    if (p.splits > 1 && set > 0) {
      // Split K: the first set of epilogue warps does all of it.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.acc_empty(buf));
      continue;
    }
    if (p.splits > 1) {
      // Partial sums of this K part to the workspace (row-major within the tile).
      const int tile = wk.mt * p.tiles_n + wk.nt;
      float* part = p.partial + (static_cast<size_t>(wk.split) * tiles + tile) * tile_elems +
                    static_cast<size_t>(r_in) * BN;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t a[32];
        tmem_ld32(t + 32 * c, a);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          reinterpret_cast<uint4*>(part + 32 * c)[q] =
              make_uint4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar.acc_empty(buf));
      // Each warp owns 32 rows of the tile: the warp that is last to arrive at
      // its (tile, rows) counter adds all parts of those rows in split order.
      __threadfence();
      __syncwarp();
      unsigned int prev = 0;
      if (lane == 0) prev = atomicAdd(p.counters + 4 * tile + quad, 1u);
      prev = __shfl_sync(0xffffffffu, prev, 0);
      if (prev != static_cast<unsigned int>(p.splits - 1)) continue;
      __threadfence();
      // Coalesced: BN / 8 lanes cover one row (8 columns each), 32 / (BN / 8) rows per
      // pass; every split's partial sums of a lane are loaded before they are added.
      constexpr int kLanesPerRow = BN / 8 < 32 ? BN / 8 : 32;
      constexpr int kRowsPerPass = 32 / kLanesPerRow;
      constexpr int kColPasses = BN / 8 / kLanesPerRow;  // 1, except 256-wide tiles: 1
      const int col = (lane % kLanesPerRow) * 8;
      const float* tile_part = p.partial + static_cast<size_t>(tile) * tile_elems;
      const size_t split_stride = static_cast<size_t>(tiles) * tile_elems;
      // Four passes at a time: all their partial-sum loads are in flight together.
      constexpr int kPasses = 32 / kRowsPerPass;
      constexpr int kGroup = kPasses < 4 ? kPasses : 4;
      static_assert(kColPasses == 1, "one column pass per row");
#pragma unroll 1
      for (int pg = 0; pg < kPasses; pg += kGroup) {
        float acc[kGroup][8];
#pragma unroll
        for (int g = 0; g < kGroup; ++g)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[g][e] = 0.0f;
#pragma unroll 2
        for (int sp = 0; sp < p.splits; ++sp) {
          float4 u[kGroup], v[kGroup];
#pragma unroll
          for (int g = 0; g < kGroup; ++g) {
            const int rl = quad * 32 + (pg + g) * kRowsPerPass + lane / kLanesPerRow;
            const float4* q = reinterpret_cast<const float4*>(
                tile_part + sp * split_stride + static_cast<size_t>(rl) * BN + col);
            u[g] = __ldcg(q);
            v[g] = __ldcg(q + 1);
          }
#pragma unroll
          for (int g = 0; g < kGroup; ++g) {
            acc[g][0] += u[g].x; acc[g][1] += u[g].y; acc[g][2] += u[g].z; acc[g][3] += u[g].w;
            acc[g][4] += v[g].x; acc[g][5] += v[g].y; acc[g][6] += v[g].z; acc[g][7] += v[g].w;
          }
        }
#pragma unroll
        for (int g = 0; g < kGroup; ++g) {
          const int rl = quad * 32 + (pg + g) * kRowsPerPass + lane / kLanesPerRow;
          const int grow = wk.mt * kBM + rl;
          const int n = n_base + col;
          if (grow < p.M && n < p.N) store8(p, acc[g], grow, n);
        }
      }
      continue;
    }
    // 64 columns at a time: the residual (if any) arrives in a staging buffer by
    // TMA, each thread writes its row's 64 results into the buffer (128-byte
    // swizzle: 16-byte piece j of row r at piece j ^ (r % 8)), and one TMA
    // store writes the 32 x 64 box; rows >= M and columns >= N are clipped.
    const int row0 = wk.mt * kBM + quad * 32;
#pragma unroll 1
    for (int c = set; c < BN / 64; c += 2) {
      const int n0 = n_base + 64 * c;
      if (p.res != nullptr) {
        if (c != set) load_res(wk, c);
        if (!wait_bounded(bar.res_full(ew), rs.issued & 1u, abort_flag, p.wait_limit_ns,
                          kSiteEpi))
          return;
        rs.pending = false;
        ++rs.issued;
      } else {
        // The store that last read this warp's buffer must be done reading it.
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
      }
      uint32_t a[64];
      tmem_ld32(t + 64 * c, reinterpret_cast<uint32_t(&)[32]>(a[0]));
      tmem_ld32(t + 64 * c + 32, reinterpret_cast<uint32_t(&)[32]>(a[32]));
      const uint32_t row_s = buf_s + static_cast<uint32_t>(lane) * 128u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t piece = row_s + static_cast<uint32_t>((j ^ (lane & 7)) * 16);
        uint4 r8;
        if (p.res != nullptr) {
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(r8.x), "=r"(r8.y), "=r"(r8.z), "=r"(r8.w)
                       : "r"(piece));
        }
        const uint4 o = epi8(p, a + 8 * j, n0 + 8 * j, p.res != nullptr ? &r8 : nullptr);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(piece), "r"(o.x),
                     "r"(o.y), "r"(o.z), "r"(o.w)
                     : "memory");
      }
      fence_async_shared();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&p.tm_y, buf_s, n0, row0);
        bulk_commit();
      }
    }
    (void)row;
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar.acc_empty(buf));
  }
}

template <int BN>
__device__ __forceinline__ void gemm_epilogue_role(const GemmParams& p, uint32_t tmem,
                                                   const GemmBarriers& bar,
                                                   volatile int* abort_flag, int warp, int lane,
                                                   uint32_t staging) {
  const int ew = warp - kEpiWarp0;
  EpiRes rs;
  gemm_epilogue_loop<BN>(p, tmem, bar, abort_flag, warp, lane,
                         staging + static_cast<uint32_t>(ew) * kStageOutBytes, rs);
  // On every way out: a residual load not waited for must land, and every TMA
  // store of this warp must have read its staging buffer, before the CTA
  // exits (the stores' writes are visible once the grid has completed).
  if (rs.pending) wait_drain(bar.res_full(ew), rs.issued & 1u, kDrainLimitNs);
  if (lane == 0) bulk_wait_read<0>();
  __syncwarp();
}

__device__ __forceinline__ void gemm_teardown_sync() {
  tc_fence_before();
  asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory");
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1) linear_kernel(const __grid_constant__ GemmParams p) {
  using G = GemmGeom<BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  const uint32_t staging = sbase + static_cast<uint32_t>(p.stages) * G::kStageBytes;
  const uint32_t sbar = staging + kStagingBytes;
  uint8_t* bar_generic = smem_raw + (sbar - raw);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_generic + 8 * kNumBarriers);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const GemmBarriers bar{sbar};
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(bar.full(s), 1);
      mbar_init(bar.empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar.acc_full(b), 1);
      mbar_init(bar.acc_empty(b), kEpiWarps);
      mbar_init(bar.drain(b), 1);
    }
    for (int e = 0; e < kEpiWarps; ++e) {
      mbar_init(bar.res_full(e), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kLoadWarp && lane == 0) {
    prefetch_tmap(&p.tm_a);
    prefetch_tmap(&p.tm_b);
    prefetch_tmap(&p.tm_y);
    if (p.res != nullptr) prefetch_tmap(&p.tm_res);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), G::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The prologue may overlap the previous kernel (programmatic dependent
  // launch); global memory is touched only after this wait.
  grid_dep_wait();
  grid_dep_launch();

  if (warp == kLoadWarp) {
    gemm_load_role<BN>(p, sbase, bar, abort_flag);
  } else if (warp == kMmaWarp) {
    gemm_mma_role<BN>(p, tmem, sbase, bar, abort_flag);
  } else if (warp >= kEpiWarp0) {
    gemm_epilogue_role<BN>(p, tmem, bar, abort_flag, warp, lane, staging);
  }
  __syncwarp();
  gemm_teardown_sync();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, G::kTmemCols);
  }
}

}  // namespace gemm
}  // namespace vla
