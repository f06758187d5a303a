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
//     y[m,n] = sum_k x[m,k] * w[n,k] + bias[n] + res[m,n]
//   (same page, section 3, CUDA custom operators: cublasLt fused GEMM + bias
//   (+ residual) in one launch; "Pi0 VLA deployment tutorial", section 3.2:
//   the block's qkv linear feeds the attention.)  A plain GEMM with a bias
//   epilogue, so it is a cuBLASLt call (tensor cores, bias in the epilogue,
//   residual as C with beta = 1); the row-major product is computed as the
//   column-major y^T = w . x^T.  For the qkv linear, N = 3 H d and y is
//   exactly the packed [B, tokens, 3, H, d] input of the attention kernel.
//   The MLP's first layer applies GELU (the tanh form) in the same epilogue
//   (same page, Triton fused kernels: matrix multiply + bias + activation).
//
// This header is included by vla_attn.cu after its host helpers (device
// checks, pointer-range checks) and shares them.
#pragma once

#include <cublasLt.h>

#include <map>
#include <tuple>

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
  vla::layernorm_kernel<NCH, ADD><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(r),
      static_cast<const __nv_bfloat16*>(gamma), static_cast<const __nv_bfloat16*>(beta),
      static_cast<__nv_bfloat16*>(s), static_cast<__nv_bfloat16*>(y), M, W, eps);
  if (cudaGetLastError() != cudaSuccess) return VLA_ATTN_ERR_CUDA;
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

// cuBLASLt state: one handle per process, one plan (descriptors + heuristic
// algorithm) per shape, device and epilogue.
struct LtPlan {
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t a = nullptr, b = nullptr, c = nullptr;
  cublasLtMatmulAlgo_t algo{};
};

std::mutex g_lt_mutex;
cublasLtHandle_t g_lt = nullptr;
std::map<std::tuple<int, int, int, int, int, int, int, size_t>, LtPlan> g_lt_plans;

// Builds (once) the plan of y^T[N, M] = act(w[N, K] . x^T[K, M] (+ bias)) (+ res^T),
// act = GELU (cuBLASLt's epilogue, the tanh form) or the identity.
int lt_plan(int dev, int M, int K, int N, bool bias, bool res, bool gelu, size_t ws,
            LtPlan** out) {
  if (g_lt == nullptr && cublasLtCreate(&g_lt) != CUBLAS_STATUS_SUCCESS) return VLA_ATTN_ERR_CUDA;
  const auto key = std::make_tuple(dev, M, K, N, bias ? 1 : 0, res ? 1 : 0, gelu ? 1 : 0, ws);
  auto it = g_lt_plans.find(key);
  if (it != g_lt_plans.end()) {
    *out = &it->second;
    return VLA_ATTN_OK;
  }
  LtPlan pl;
  bool ok = cublasLtMatmulDescCreate(&pl.op, CUBLAS_COMPUTE_32F, CUDA_R_32F) ==
            CUBLAS_STATUS_SUCCESS;
  const cublasOperation_t ta = CUBLAS_OP_T, tb = CUBLAS_OP_N;
  const cublasLtEpilogue_t epi =
      gelu ? (bias ? CUBLASLT_EPILOGUE_GELU_BIAS : CUBLASLT_EPILOGUE_GELU)
           : (bias ? CUBLASLT_EPILOGUE_BIAS : CUBLASLT_EPILOGUE_DEFAULT);
  const cudaDataType_t bias_type = CUDA_R_16BF;
  ok = ok && cublasLtMatmulDescSetAttribute(pl.op, CUBLASLT_MATMUL_DESC_TRANSA, &ta,
                                            sizeof(ta)) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatmulDescSetAttribute(pl.op, CUBLASLT_MATMUL_DESC_TRANSB, &tb,
                                            sizeof(tb)) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatmulDescSetAttribute(pl.op, CUBLASLT_MATMUL_DESC_EPILOGUE, &epi,
                                            sizeof(epi)) == CUBLAS_STATUS_SUCCESS;
  if (bias)
    ok = ok && cublasLtMatmulDescSetAttribute(pl.op, CUBLASLT_MATMUL_DESC_BIAS_DATA_TYPE,
                                              &bias_type, sizeof(bias_type)) ==
                   CUBLAS_STATUS_SUCCESS;
  // w as stored ([N, K] row-major) is a column-major K x N matrix (ld K);
  // x ([M, K] row-major) a column-major K x M one; y and res column-major N x M.
  ok = ok && cublasLtMatrixLayoutCreate(&pl.a, CUDA_R_16BF, K, N, K) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatrixLayoutCreate(&pl.b, CUDA_R_16BF, K, M, K) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatrixLayoutCreate(&pl.c, CUDA_R_16BF, N, M, N) == CUBLAS_STATUS_SUCCESS;
  if (ok) {
    cublasLtMatmulPreference_t pref = nullptr;
    ok = cublasLtMatmulPreferenceCreate(&pref) == CUBLAS_STATUS_SUCCESS &&
         cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws,
                                              sizeof(ws)) == CUBLAS_STATUS_SUCCESS;
    cublasLtMatmulHeuristicResult_t h{};
    int found = 0;
    ok = ok && cublasLtMatmulAlgoGetHeuristic(g_lt, pl.op, pl.a, pl.b, pl.c, pl.c, pref, 1, &h,
                                              &found) == CUBLAS_STATUS_SUCCESS &&
         found > 0;
    if (pref != nullptr) cublasLtMatmulPreferenceDestroy(pref);
    if (ok) pl.algo = h.algo;
  }
  if (!ok) {
    if (pl.op) cublasLtMatmulDescDestroy(pl.op);
    if (pl.a) cublasLtMatrixLayoutDestroy(pl.a);
    if (pl.b) cublasLtMatrixLayoutDestroy(pl.b);
    if (pl.c) cublasLtMatrixLayoutDestroy(pl.c);
    return VLA_ATTN_ERR_CUDA;
  }
  auto ins = g_lt_plans.emplace(key, pl);
  *out = &ins.first->second;
  return VLA_ATTN_OK;
}

constexpr size_t kLinearWorkspaceBytes = 32u << 20;

// Fixed cuBLASLt workspace of vla_linear_fwd_static: one per device context.
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

// y = act(x . w^T + bias) (+ res) through one cuBLASLt matmul; argument checks
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

  std::lock_guard<std::mutex> lock(g_lt_mutex);
  LtPlan* pl = nullptr;
  rc = lt_plan(dev, M, K, N, bias != nullptr, res != nullptr, gelu, workspace_bytes, &pl);
  if (rc != VLA_ATTN_OK) return rc;
  if (bias != nullptr &&
      cublasLtMatmulDescSetAttribute(pl->op, CUBLASLT_MATMUL_DESC_BIAS_POINTER, &bias,
                                     sizeof(bias)) != CUBLAS_STATUS_SUCCESS)
    return VLA_ATTN_ERR_CUDA;
  const float alpha = 1.0f;
  const float beta = res != nullptr ? 1.0f : 0.0f;
  const void* c = res != nullptr ? res : y;
  if (cublasLtMatmul(g_lt, pl->op, &alpha, w, pl->a, x, pl->b, &beta, c, pl->c, y, pl->c,
                     &pl->algo, workspace, workspace_bytes,
                     static_cast<cudaStream_t>(stream)) != CUBLAS_STATUS_SUCCESS)
    return VLA_ATTN_ERR_CUDA;
  return VLA_ATTN_OK;
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
