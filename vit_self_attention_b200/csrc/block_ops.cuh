// The layers around the attention core in a ViT encoder layer: the
// LayerNorms (plain, or fused with the residual add), the linear layers (qkv
// projection, output projection with the residual add, the MLP's fc1 with
// its GELU and fc2 with the residual add).
//
//   LayerNorm over the last dimension (width W) of every row, biased
//   variance, fp32 statistics:
//     y[m,i] = (x[m,i] - mean_m) / sqrt(var_m + eps) * gamma[i] + beta[i]
//   ("FluxVLA docs, inference acceleration", Triton fused kernels: norm
//   fusion, residual add + LayerNorm in one kernel.)  A hand-written kernel:
//   one warp per row, 16-byte loads, the row kept in registers between the
//   mean, the variance and the output pass, so x is read once and y written
//   once (HBM-bound).  The fused variant first forms the residual stream
//   s = bf16(x + r), stores it, and normalises the stored values, so that it
//   gives exactly what a separate add and LayerNorm give.
//
//   Linear layer with bias and optional residual, nn.Linear weight layout
//   [N, K] (the pages' weight(K,N) transposed):
//     y[m,n] = act(sum_k x[m,k] * w[n,k] + bias[n]) + res[m,n]
//   (same page, section 3, CUDA custom operators: GEMM + bias (+ residual)
//   in one launch; section 1: matrix multiply + bias + activation; "Pi0 VLA
//   deployment tutorial", section 3.2: the block's qkv linear feeds the
//   attention.)  The hand-written tcgen05 GEMM of gemm_kernel.cuh with the
//   bias, the GELU (tanh form) and the residual add in its epilogue.  For the
//   qkv linear, N = 3 H d and y is exactly the packed [B, tokens, 3, H, d]
//   input of the attention kernel.
//
// This header is included by vla_attn.cu after its host helpers (device
// checks, pointer-range checks) and shares them.
#pragma once

#include <algorithm>

#include "gemm_kernel.cuh"

namespace vla {

constexpr int kLnMaxChunks = 8;  // 8 chunks of 256 elements: W <= 2048

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// One warp per row; lane l holds elements [256 c + 8 l, 256 c + 8 l + 8) of
// chunk c < NCH (elements at or past W are skipped).  8 rows per block.
// ADD: the row is first the residual sum s = bf16(x + r), stored to `s` and
// then normalised (the stream as stored, so the fusion changes no result).
// A row is entirely in registers before any of its outputs is written, and
// rows belong to one warp each, so an output may be the very buffer x or r.
template <int NCH, bool ADD>
__global__ void __launch_bounds__(256) layernorm_kernel(const __nv_bfloat16* x,
                                                        const __nv_bfloat16* r,
                                                        const __nv_bfloat16* __restrict__ gamma,
                                                        const __nv_bfloat16* __restrict__ beta,
                                                        __nv_bfloat16* s, __nv_bfloat16* y,
                                                        long long M, int W, float eps) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + warp;
  grid_dep_wait();  // the previous kernel's output is this kernel's input
  grid_dep_launch();
  if (row >= M) return;
  const __nv_bfloat16* xr = x + row * W;
  float v[NCH][8];
  uint4 sum_bits[ADD ? NCH : 1];
  if constexpr (ADD) {
    const __nv_bfloat16* rr = r + row * W;
    uint4 xb[NCH], rb[NCH];
#pragma unroll
    for (int c = 0; c < NCH; ++c) {  // all loads of the row first
      const int e = c * 256 + lane * 8;
      if (e < W) {
        xb[c] = *reinterpret_cast<const uint4*>(xr + e);
        rb[c] = *reinterpret_cast<const uint4*>(rr + e);
      }
    }
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      if (c * 256 + lane * 8 < W) {
        float a[8], b[8];
        unpack8(xb[c], a);
        unpack8(rb[c], b);
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] = pack_bf16x2(a[2 * i] + b[2 * i], a[2 * i + 1] + b[2 * i + 1]);
        sum_bits[c] = make_uint4(o[0], o[1], o[2], o[3]);
        unpack8(sum_bits[c], v[c]);
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int e = c * 256 + lane * 8;
      if (e < W) unpack8(*reinterpret_cast<const uint4*>(xr + e), v[c]);
    }
  }
  float sum = 0.0f;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    if (c * 256 + lane * 8 < W) {
#pragma unroll
      for (int i = 0; i < 8; ++i) sum += v[c][i];
    }
  }
  const float mean = warp_sum(sum) / static_cast<float>(W);
  float ss = 0.0f;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    if (c * 256 + lane * 8 < W) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float dv = v[c][i] - mean;
        ss += dv * dv;
      }
    }
  }
  const float rstd = rsqrtf(warp_sum(ss) / static_cast<float>(W) + eps);
  __nv_bfloat16* yr = y + row * W;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int e = c * 256 + lane * 8;
    if (e < W) {
      if constexpr (ADD) *reinterpret_cast<uint4*>(s + row * W + e) = sum_bits[c];
      float g[8], b[8];
      unpack8(*reinterpret_cast<const uint4*>(gamma + e), g);
      unpack8(*reinterpret_cast<const uint4*>(beta + e), b);
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float y0 = (v[c][2 * i] - mean) * rstd * g[2 * i] + b[2 * i];
        const float y1 = (v[c][2 * i + 1] - mean) * rstd * g[2 * i + 1] + b[2 * i + 1];
        o[i] = pack_bf16x2(y0, y1);
      }
      *reinterpret_cast<uint4*>(yr + e) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace vla

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(uintptr_t a_lo, uintptr_t a_hi, uintptr_t b_lo, uintptr_t b_hi) {
  return a_lo < b_hi && b_lo < a_hi;
}

template <int NCH, bool ADD>
int launch_layernorm(const void* x, const void* r, const void* gamma, const void* beta, void* s,
                     void* y, long long M, int W, float eps, cudaStream_t stream) {
  const long long blocks = (M + 7) / 8;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  set_dependent_launch(&cfg, attr);
  if (cudaLaunchKernelEx(&cfg, vla::layernorm_kernel<NCH, ADD>,
                         static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(r),
                         static_cast<const __nv_bfloat16*>(gamma),
                         static_cast<const __nv_bfloat16*>(beta), static_cast<__nv_bfloat16*>(s),
                         static_cast<__nv_bfloat16*>(y), M, W, eps) != cudaSuccess) {
    (void)cudaGetLastError();
    return VLA_ATTN_ERR_CUDA;
  }
  g_launches.fetch_add(1);
  return VLA_ATTN_OK;
}

template <bool ADD>
int dispatch_layernorm(const void* x, const void* r, const void* gamma, const void* beta, void* s,
                       void* y, long long M, int W, float eps, cudaStream_t st) {
  switch ((W + 255) / 256) {
    case 1: return launch_layernorm<1, ADD>(x, r, gamma, beta, s, y, M, W, eps, st);
    case 2: return launch_layernorm<2, ADD>(x, r, gamma, beta, s, y, M, W, eps, st);
    case 3: return launch_layernorm<3, ADD>(x, r, gamma, beta, s, y, M, W, eps, st);
    case 4: return launch_layernorm<4, ADD>(x, r, gamma, beta, s, y, M, W, eps, st);
    case 5: return launch_layernorm<5, ADD>(x, r, gamma, beta, s, y, M, W, eps, st);
    case 6: return launch_layernorm<6, ADD>(x, r, gamma, beta, s, y, M, W, eps, st);
    case 7: return launch_layernorm<7, ADD>(x, r, gamma, beta, s, y, M, W, eps, st);
    default: return launch_layernorm<8, ADD>(x, r, gamma, beta, s, y, M, W, eps, st);
  }
}

// ---------------------------------------------------------------- linear
// 2-D tensor map of a row-major [rows, K] bf16 matrix, box {64, box_rows},
// 128-byte swizzle (the K-major operand layout of the GEMM's MMAs, and the
// epilogue's 64-column staging tiles of y and the residual).
int encode_2d(const DriverFns& fns, CUtensorMap* map, const void* base, int K, int rows,
              uint32_t box_rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2ull};
  const cuuint32_t box[2] = {64u, box_rows};
  const cuuint32_t elem_strides[2] = {1u, 1u};
  const CUresult rc = fns.encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
                                 dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? VLA_ATTN_OK : VLA_ATTN_ERR_CUDA;
}

// How a linear layer is cut into work: tile width BN and K parts.
struct LinearPlan {
  int bn = 256;
  int splits = 1;
  int tiles_m = 0, tiles_n = 0, ksteps = 0, ksteps_per_split = 0;
  size_t workspace_needed = 0;  // partial sums + arrival counters (0 without split K)
};

// Tile width: the fewest waves of tiles over the SMs weighted by a tile's cost,
// its MMA time (proportional to BN) plus its 128-row tile of x (loaded whatever
// BN is), wider tiles on ties (more reuse per byte loaded).  Split K when the
// tiles fill at most a quarter of the SMs, the caller's workspace holds the
// partial sums, and the main-loop time the split saves exceeds its fixed cost:
// the counters' memset ahead of the launch, which also forgoes the overlap with
// the previous kernel, and the partial sums' round trip, about 7 us (measured:
// split calls of the 50- to 591-token encoder shapes, K <= 4096, ran at twice
// the time of the same shapes unsplit).
constexpr long long kSplitFixedCycles = 14000;

LinearPlan plan_linear(int M, int K, int N, int sm_count, size_t workspace_bytes) {
  LinearPlan pl;
  pl.tiles_m = (M + vla::gemm::kBM - 1) / vla::gemm::kBM;
  pl.ksteps = (K + vla::gemm::kBK - 1) / vla::gemm::kBK;
  long long best = -1;
  for (int bn : {256, 128, 64}) {
    const long long tiles = static_cast<long long>(pl.tiles_m) * ((N + bn - 1) / bn);
    // Per tile: MMA time ~ BN, plus the 128-row tile of x it loads whatever BN is.
    const long long cost = ((tiles + sm_count - 1) / sm_count) * (bn + 128);
    if (best < 0 || cost < best) {
      best = cost;
      pl.bn = bn;
    }
  }
  pl.tiles_n = (N + pl.bn - 1) / pl.bn;
  const long long tiles = static_cast<long long>(pl.tiles_m) * pl.tiles_n;
  pl.ksteps_per_split = pl.ksteps;
  // Cycles per k-step of one tile: its MMAs or its loads, whichever is longer.
  const long long step = std::max(2ll * pl.bn, 128ll + pl.bn);
  if (4 * tiles <= sm_count && pl.ksteps >= 8) {
    int splits = static_cast<int>(sm_count / tiles);
    splits = std::min(splits, pl.ksteps / 4);
    splits = std::min(splits, 16);
    while (splits > 1) {
      const int per = (pl.ksteps + splits - 1) / splits;
      const int used = (pl.ksteps + per - 1) / per;  // no empty part
      const size_t need = static_cast<size_t>(used) * tiles * vla::gemm::kBM * pl.bn * 4u +
                          static_cast<size_t>(tiles) * 4u * sizeof(unsigned int);
      const long long saved = static_cast<long long>(pl.ksteps - per) * step;
      if (saved <= kSplitFixedCycles) break;  // fewer parts save less
      if (need <= workspace_bytes) {
        pl.splits = used;
        pl.ksteps_per_split = per;
        pl.workspace_needed = need;
        break;
      }
      --splits;
    }
  }
  return pl;
}

template <int BN>
int launch_linear_bn(const DriverFns& fns, const DeviceInfo& di, int dev, const LinearPlan& pl,
                     const void* x, const void* w, const void* bias, const void* res, void* y,
                     int M, int K, int N, int act, void* workspace, cudaStream_t stream) {
  using G = vla::gemm::GemmGeom<BN>;
  vla::gemm::GemmParams prm;
  std::memset(&prm, 0, sizeof(prm));
  int rc = encode_2d(fns, &prm.tm_a, x, K, M, vla::gemm::kBM);
  if (rc != VLA_ATTN_OK) return rc;
  rc = encode_2d(fns, &prm.tm_b, w, K, N, static_cast<uint32_t>(BN));
  if (rc != VLA_ATTN_OK) return rc;
  rc = encode_2d(fns, &prm.tm_y, y, N, M, 32u);
  if (rc != VLA_ATTN_OK) return rc;
  if (res != nullptr) {
    rc = encode_2d(fns, &prm.tm_res, res, N, M, 32u);
    if (rc != VLA_ATTN_OK) return rc;
  }
  int stages = (di.max_smem_optin - static_cast<int>(vla::gemm::kStagingBytes +
                                                     vla::gemm::kBarrierBytes + 1024u)) /
               static_cast<int>(G::kStageBytes);
  if (stages > vla::gemm::kMaxStages) stages = vla::gemm::kMaxStages;
  if (stages < 2) return VLA_ATTN_ERR_DEVICE;
  const uint32_t smem = vla::gemm::gemm_smem_bytes<BN>(stages);
  {
    static int attr[kMaxDevices] = {};
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (attr[dev] < static_cast<int>(smem)) {
      if (cudaFuncSetAttribute(vla::gemm::linear_kernel<BN>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem)) != cudaSuccess)
        return VLA_ATTN_ERR_CUDA;
      attr[dev] = static_cast<int>(smem);
    }
  }
  prm.bias = static_cast<const __nv_bfloat16*>(bias);
  prm.res = static_cast<const __nv_bfloat16*>(res);
  prm.y = static_cast<__nv_bfloat16*>(y);
  prm.M = M;
  prm.N = N;
  prm.K = K;
  prm.tiles_m = pl.tiles_m;
  prm.tiles_n = pl.tiles_n;
  prm.splits = pl.splits;
  prm.ksteps = pl.ksteps;
  prm.ksteps_per_split = pl.ksteps_per_split;
  prm.num_work = pl.tiles_m * pl.tiles_n * pl.splits;
  prm.stages = stages;
  prm.act = act;
  const unsigned long long lim = g_wait_limit_ns.load();
  prm.wait_limit_ns = lim == 0 ? kDefaultWaitLimitNs : lim;
  if (pl.splits > 1) {
    // Partial sums first, then the arrival counters, which must start at zero.
    const size_t tiles = static_cast<size_t>(pl.tiles_m) * pl.tiles_n;
    const size_t part_bytes =
        static_cast<size_t>(pl.splits) * tiles * vla::gemm::kBM * BN * 4u;
    prm.partial = static_cast<float*>(workspace);
    prm.counters = reinterpret_cast<unsigned int*>(static_cast<char*>(workspace) + part_bytes);
    if (cudaMemsetAsync(prm.counters, 0, tiles * 4u * sizeof(unsigned int), stream) !=
        cudaSuccess)
      return VLA_ATTN_ERR_CUDA;
  }
  const int grid = prm.num_work < di.sm_count ? prm.num_work : di.sm_count;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(vla::gemm::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // A split launch follows the memset of its counters: ordinary stream order.
  cudaLaunchAttribute attr[1];
  if (pl.splits == 1) set_dependent_launch(&cfg, attr);
  if (cudaLaunchKernelEx(&cfg, vla::gemm::linear_kernel<BN>, prm) != cudaSuccess) {
    (void)cudaGetLastError();
    return VLA_ATTN_ERR_CUDA;
  }
  g_launches.fetch_add(1);
  return VLA_ATTN_OK;
}

constexpr size_t kLinearWorkspaceBytes = 32u << 20;

// Fixed workspace of vla_linear_fwd_static (split-K partial sums and arrival
// counters): one per device context.
constexpr size_t kStaticWorkspaceBytes = 8u << 20;
__device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

std::mutex g_static_ws_mutex;
void* g_static_ws_addr[kMaxDevices] = {};
CUcontext g_static_ws_ctx[kMaxDevices] = {};

// Device address of this device's static workspace.  A module global's address belongs
// to the context the module is loaded in, so the address is cached together with the
// context that was current when it was looked up, and looked up again whenever another
// context is current (a non-primary context, or the primary one after a device reset).
int static_workspace(int dev, void** out) {
  const DriverFns& fns = driver_fns();
  if (fns.ctx_current == nullptr) return VLA_ATTN_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (fns.ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return VLA_ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_ws_mutex);
  if (g_static_ws_addr[dev] == nullptr || g_static_ws_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return VLA_ATTN_ERR_CUDA;
    }
    g_static_ws_addr[dev] = p;
    g_static_ws_ctx[dev] = ctx;
  }
  *out = g_static_ws_addr[dev];
  return VLA_ATTN_OK;
}

// y = act(x . w^T + bias) (+ res) through one launch of the GEMM; argument checks
// of vla_linear_fwd.
int linear_impl(const void* x, const void* w, const void* bias, const void* res, void* y, int M,
                int K, int N, void* workspace, size_t workspace_bytes, void* stream, bool gelu) {
  if (x == nullptr || w == nullptr || y == nullptr) return VLA_ATTN_ERR_NULL;
  if (workspace == nullptr && workspace_bytes != 0) return VLA_ATTN_ERR_NULL;
  if (M < 1 || K < 1 || N < 1) return VLA_ATTN_ERR_SHAPE;
  if (K % 8 != 0 || N % 8 != 0) return VLA_ATTN_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y) || (bias && !aligned16(bias)) ||
      (res && !aligned16(res)) || (workspace && !aligned16(workspace)))
    return VLA_ATTN_ERR_ALIGN;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VLA_ATTN_ERR_CUDA;
  DeviceInfo di;
  int rc = device_info(dev, &di);
  if (rc != VLA_ATTN_OK) return rc;
  const DriverFns& fns = driver_fns();
  if (fns.ptr_attr == nullptr) return VLA_ATTN_ERR_CUDA;
  uintptr_t xl, xh, wl, wh, yl, yh, bl = 0, bh = 0, rl = 0, rh = 0, sl = 0, sh = 0;
  const size_t mn = static_cast<size_t>(M) * N * 2u;
  if ((rc = check_device_range(fns, x, static_cast<size_t>(M) * K * 2u, dev, &xl, &xh)) !=
      VLA_ATTN_OK)
    return rc;
  if ((rc = check_device_range(fns, w, static_cast<size_t>(N) * K * 2u, dev, &wl, &wh)) !=
      VLA_ATTN_OK)
    return rc;
  if ((rc = check_device_range(fns, y, mn, dev, &yl, &yh)) != VLA_ATTN_OK) return rc;
  if (bias && (rc = check_device_range(fns, bias, N * 2u, dev, &bl, &bh)) != VLA_ATTN_OK)
    return rc;
  if (res && (rc = check_device_range(fns, res, mn, dev, &rl, &rh)) != VLA_ATTN_OK) return rc;
  if (workspace_bytes &&
      (rc = check_device_range(fns, workspace, workspace_bytes, dev, &sl, &sh)) != VLA_ATTN_OK)
    return rc;
  // y may be res itself (in-place residual add); it must not overlap anything else.
  if (overlaps(xl, xh, yl, yh) || overlaps(wl, wh, yl, yh) || (bias && overlaps(bl, bh, yl, yh)) ||
      (res && res != y && overlaps(rl, rh, yl, yh)) ||
      (workspace_bytes && overlaps(sl, sh, yl, yh)))
    return VLA_ATTN_ERR_MEMORY;

  const DriverFns& f2 = driver_fns();
  if (f2.encode == nullptr) return VLA_ATTN_ERR_CUDA;
  const LinearPlan pl = plan_linear(M, K, N, di.sm_count, workspace_bytes);
  const int act = gelu ? vla::gemm::kActGelu : vla::gemm::kActNone;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (pl.bn) {
    case 256:
      return launch_linear_bn<256>(f2, di, dev, pl, x, w, bias, res, y, M, K, N, act, workspace,
                                   st);
    case 128:
      return launch_linear_bn<128>(f2, di, dev, pl, x, w, bias, res, y, M, K, N, act, workspace,
                                   st);
    default:
      return launch_linear_bn<64>(f2, di, dev, pl, x, w, bias, res, y, M, K, N, act, workspace,
                                  st);
  }
}

}  // namespace

extern "C" {

int vla_layernorm_fwd(const void* x, const void* gamma, const void* beta, void* y, int M, int W,
                      float eps, void* stream) {
  if (x == nullptr || gamma == nullptr || beta == nullptr || y == nullptr) return VLA_ATTN_ERR_NULL;
  if (M < 1 || W < 1) return VLA_ATTN_ERR_SHAPE;
  if (W % 8 != 0 || W > 256 * vla::kLnMaxChunks) return VLA_ATTN_ERR_UNSUPPORTED;
  if (!std::isfinite(eps) || eps < 0.0f) return VLA_ATTN_ERR_SCALE;
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(beta) || !aligned16(y))
    return VLA_ATTN_ERR_ALIGN;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VLA_ATTN_ERR_CUDA;
  DeviceInfo di;
  int rc = device_info(dev, &di);
  if (rc != VLA_ATTN_OK) return rc;
  const DriverFns& fns = driver_fns();
  if (fns.ptr_attr == nullptr) return VLA_ATTN_ERR_CUDA;
  const size_t bytes = static_cast<size_t>(M) * W * 2u;
  uintptr_t xl, xh, yl, yh, gl, gh, bl, bh;
  if ((rc = check_device_range(fns, x, bytes, dev, &xl, &xh)) != VLA_ATTN_OK) return rc;
  if ((rc = check_device_range(fns, y, bytes, dev, &yl, &yh)) != VLA_ATTN_OK) return rc;
  if ((rc = check_device_range(fns, gamma, W * 2u, dev, &gl, &gh)) != VLA_ATTN_OK) return rc;
  if ((rc = check_device_range(fns, beta, W * 2u, dev, &bl, &bh)) != VLA_ATTN_OK) return rc;
  // In place (y == x) is allowed: a row is in registers before it is written.
  if ((y != x && overlaps(xl, xh, yl, yh)) || overlaps(gl, gh, yl, yh) || overlaps(bl, bh, yl, yh))
    return VLA_ATTN_ERR_MEMORY;
  return dispatch_layernorm<false>(x, nullptr, gamma, beta, nullptr, y, M, W, eps,
                                   static_cast<cudaStream_t>(stream));
}

int vla_add_layernorm_fwd(const void* x, const void* r, const void* gamma, const void* beta,
                          void* s, void* y, int M, int W, float eps, void* stream) {
  if (x == nullptr || r == nullptr || gamma == nullptr || beta == nullptr || s == nullptr ||
      y == nullptr)
    return VLA_ATTN_ERR_NULL;
  if (M < 1 || W < 1) return VLA_ATTN_ERR_SHAPE;
  if (W % 8 != 0 || W > 256 * vla::kLnMaxChunks) return VLA_ATTN_ERR_UNSUPPORTED;
  if (!std::isfinite(eps) || eps < 0.0f) return VLA_ATTN_ERR_SCALE;
  if (!aligned16(x) || !aligned16(r) || !aligned16(gamma) || !aligned16(beta) || !aligned16(s) ||
      !aligned16(y))
    return VLA_ATTN_ERR_ALIGN;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VLA_ATTN_ERR_CUDA;
  DeviceInfo di;
  int rc = device_info(dev, &di);
  if (rc != VLA_ATTN_OK) return rc;
  const DriverFns& fns = driver_fns();
  if (fns.ptr_attr == nullptr) return VLA_ATTN_ERR_CUDA;
  const size_t bytes = static_cast<size_t>(M) * W * 2u;
  uintptr_t xl, xh, rl, rh, sl, sh, yl, yh, gl, gh, bl, bh;
  if ((rc = check_device_range(fns, x, bytes, dev, &xl, &xh)) != VLA_ATTN_OK) return rc;
  if ((rc = check_device_range(fns, r, bytes, dev, &rl, &rh)) != VLA_ATTN_OK) return rc;
  if ((rc = check_device_range(fns, s, bytes, dev, &sl, &sh)) != VLA_ATTN_OK) return rc;
  if ((rc = check_device_range(fns, y, bytes, dev, &yl, &yh)) != VLA_ATTN_OK) return rc;
  if ((rc = check_device_range(fns, gamma, W * 2u, dev, &gl, &gh)) != VLA_ATTN_OK) return rc;
  if ((rc = check_device_range(fns, beta, W * 2u, dev, &bl, &bh)) != VLA_ATTN_OK) return rc;
  // Each output is either exactly x or r, or disjoint from them; the two
  // outputs are disjoint; gamma and beta are disjoint from both outputs.
  const void* outs[2] = {s, y};
  const uintptr_t olo[2] = {sl, yl}, ohi[2] = {sh, yh};
  for (int i = 0; i < 2; ++i) {
    if ((outs[i] != x && overlaps(xl, xh, olo[i], ohi[i])) ||
        (outs[i] != r && overlaps(rl, rh, olo[i], ohi[i])) || overlaps(gl, gh, olo[i], ohi[i]) ||
        overlaps(bl, bh, olo[i], ohi[i]))
      return VLA_ATTN_ERR_MEMORY;
  }
  if (overlaps(sl, sh, yl, yh)) return VLA_ATTN_ERR_MEMORY;
  return dispatch_layernorm<true>(x, r, gamma, beta, s, y, M, W, eps,
                                  static_cast<cudaStream_t>(stream));
}

size_t vla_linear_workspace_bytes(void) { return kLinearWorkspaceBytes; }

size_t vla_linear_static_workspace_bytes(void) { return kStaticWorkspaceBytes; }

int vla_linear_fwd_static(const void* x, const void* w, const void* bias, const void* res, void* y,
                          int M, int K, int N, void* stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VLA_ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return VLA_ATTN_ERR_DEVICE;
  void* ws = nullptr;
  const int rc = static_workspace(dev, &ws);
  if (rc != VLA_ATTN_OK) return rc;
  return vla_linear_fwd(x, w, bias, res, y, M, K, N, ws, kStaticWorkspaceBytes, stream);
}

int vla_linear_fwd(const void* x, const void* w, const void* bias, const void* res, void* y,
                   int M, int K, int N, void* workspace, size_t workspace_bytes, void* stream) {
  return linear_impl(x, w, bias, res, y, M, K, N, workspace, workspace_bytes, stream, false);
}

int vla_linear_gelu_fwd(const void* x, const void* w, const void* bias, void* y, int M, int K,
                        int N, void* workspace, size_t workspace_bytes, void* stream) {
  return linear_impl(x, w, bias, nullptr, y, M, K, N, workspace, workspace_bytes, stream, true);
}

}  // extern "C"
