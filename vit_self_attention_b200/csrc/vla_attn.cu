// Host side of the C ABI declared in include/vla_attn.h: argument checks,
// TMA tensor maps over the packed [B, N, 3, H, d] bf16 QKV buffer, work
// decomposition and the launch of the sm_100a attention kernel.
#include "vla_attn.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn_kernel.cuh"

namespace {

// Longest sequence accepted.  577 (ViT-L/14 at 336 px) keeps a head's K/V
// resident in shared memory for all its query tiles; longer sequences (e.g.
// 730 at 384 px, 1025 at 448 px) stream K/V through the ring per round of two
// query tiles once a head's blocks exceed it (d=64: N > 768; d=72: N > 560).
constexpr int kMaxTokens = 16384;
constexpr unsigned long long kDefaultWaitLimitNs = 1000000000ull;
constexpr int kMaxDevices = 64;

std::atomic<uint64_t> g_launches{0};
std::atomic<unsigned long long> g_wait_limit_ns{0};
std::atomic<int> g_test_stall{0};

struct DriverFns {
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  PFN_cuPointerGetAttribute_v4000 ptr_attr = nullptr;
  PFN_cuCtxGetCurrent_v4000 ctx_current = nullptr;
  PFN_cuPointerGetAttributes_v7000 ptr_attrs = nullptr;
};

const DriverFns& driver_fns() {
  static DriverFns fns;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuPointerGetAttribute", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.ptr_attr = reinterpret_cast<PFN_cuPointerGetAttribute_v4000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuPointerGetAttributes", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.ptr_attrs = reinterpret_cast<PFN_cuPointerGetAttributes_v7000>(fn);
  });
  return fns;
}

struct DeviceInfo {
  bool ready = false;
  bool supported = false;
  int sm_count = 0;
  int max_smem_optin = 0;
  int attr[2][2] = {{0, 0}, {0, 0}};  // dynamic shared memory limit set per kernel
                                      // [d = 72][staging] (0 = not yet)
};

std::mutex g_dev_mutex;
DeviceInfo g_dev[kMaxDevices];

int device_info(int dev, DeviceInfo* out) {
  if (dev < 0 || dev >= kMaxDevices) return VLA_ATTN_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& di = g_dev[dev];
  if (!di.ready) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&di.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                               dev) != cudaSuccess)
      return VLA_ATTN_ERR_CUDA;
    di.supported = (major == 10 && minor == 0);
    di.ready = true;
  }
  *out = di;
  return di.supported ? VLA_ATTN_OK : VLA_ATTN_ERR_DEVICE;
}

// Programmatic dependent launch for a kernel launch: the kernel may start (and
// run its prologue) while the previous kernel on the stream finishes; every
// kernel of this library waits for that kernel (griddepcontrol.wait) before it
// touches global memory, so stream order is kept for all data.
void set_dependent_launch(cudaLaunchConfig_t* cfg, cudaLaunchAttribute (&attr)[1]) {
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg->attrs = attr;
  cfg->numAttrs = 1;
}

// Copy-out stream and fork / join events of the pipelined host-buffer entry,
// one set per device, created on first use (guarded by g_pipe_mutex, which
// the caller holds for the whole enqueue sequence).
struct HostPipe {
  cudaStream_t in = nullptr;   // input copies, back to back
  cudaStream_t out = nullptr;  // result copies
  cudaEvent_t start = nullptr;    // `stream`'s earlier work -> copy-in stream
  cudaEvent_t loaded = nullptr;   // a chunk's input copy -> its kernel on `stream`
  cudaEvent_t fork = nullptr;     // a chunk's kernel -> its result copy
  cudaEvent_t join = nullptr;     // copy-out stream -> `stream`
  cudaEvent_t in_join = nullptr;  // copy-in stream -> `stream`
};

std::mutex g_pipe_mutex;
HostPipe g_pipe[kMaxDevices];

int host_pipe(int dev, HostPipe** out) {
  HostPipe& p = g_pipe[dev];
  if (p.out == nullptr) {
    HostPipe n;
    bool ok = cudaStreamCreateWithFlags(&n.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&n.out, cudaStreamNonBlocking) == cudaSuccess;
    cudaEvent_t* evs[5] = {&n.start, &n.loaded, &n.fork, &n.join, &n.in_join};
    for (cudaEvent_t* e : evs)
      ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
      for (cudaEvent_t* e : evs)
        if (*e != nullptr) cudaEventDestroy(*e);
      if (n.in != nullptr) cudaStreamDestroy(n.in);
      if (n.out != nullptr) cudaStreamDestroy(n.out);
      return VLA_ATTN_ERR_CUDA;
    }
    p = n;
  }
  *out = &p;
  return VLA_ATTN_OK;
}

// Raises the kernel's dynamic shared-memory limit to at least `smem` bytes.
template <int D, bool kStageOut>
int ensure_smem_attr(int dev, int smem) {
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  int& cur = g_dev[dev].attr[D == 72 ? 1 : 0][kStageOut ? 1 : 0];
  if (cur < smem) {
    if (cudaFuncSetAttribute(vla::attn_fwd_kernel<D, kStageOut>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return VLA_ATTN_ERR_CUDA;
    cur = smem;
  }
  return VLA_ATTN_OK;
}

// Static shared memory (0 for the product build) and registers per thread of
// the kernel instantiation, read once.
struct KernelAttrs {
  int static_smem = 0;
  int regs = 0;
  bool ok = false;
};

template <int D>
const KernelAttrs& kernel_attrs() {
  static KernelAttrs a;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, vla::attn_fwd_kernel<D, true>) == cudaSuccess) {
      a.static_smem = static_cast<int>(fa.sharedSizeBytes);
      a.regs = fa.numRegs;
      a.ok = true;
    } else {
      (void)cudaGetLastError();
    }
  });
  return a;
}

// Checks that [p, p + bytes) lies inside one device allocation of `dev` (the four
// pointer attributes in one driver query).
int check_device_range(const DriverFns& fns, const void* p, size_t bytes, int dev,
                       uintptr_t* range_lo, uintptr_t* range_hi) {
  const CUdeviceptr dp = reinterpret_cast<CUdeviceptr>(p);
  unsigned int mem_type = 0;
  int ordinal = -1;
  CUdeviceptr start = 0;
  size_t size = 0;
  if (fns.ptr_attrs != nullptr) {
    CUpointer_attribute attrs[4] = {CU_POINTER_ATTRIBUTE_MEMORY_TYPE,
                                    CU_POINTER_ATTRIBUTE_DEVICE_ORDINAL,
                                    CU_POINTER_ATTRIBUTE_RANGE_START_ADDR,
                                    CU_POINTER_ATTRIBUTE_RANGE_SIZE};
    void* data[4] = {&mem_type, &ordinal, &start, &size};
    // Not an error for a pointer the driver does not know: the attributes stay
    // at their defaults (memory type 0), which the checks below refuse.
    if (fns.ptr_attrs(4, attrs, data, dp) != CUDA_SUCCESS) return VLA_ATTN_ERR_MEMORY;
  } else {
    if (fns.ptr_attr == nullptr) return VLA_ATTN_ERR_CUDA;
    if (fns.ptr_attr(&mem_type, CU_POINTER_ATTRIBUTE_MEMORY_TYPE, dp) != CUDA_SUCCESS ||
        fns.ptr_attr(&ordinal, CU_POINTER_ATTRIBUTE_DEVICE_ORDINAL, dp) != CUDA_SUCCESS ||
        fns.ptr_attr(&start, CU_POINTER_ATTRIBUTE_RANGE_START_ADDR, dp) != CUDA_SUCCESS ||
        fns.ptr_attr(&size, CU_POINTER_ATTRIBUTE_RANGE_SIZE, dp) != CUDA_SUCCESS)
      return VLA_ATTN_ERR_MEMORY;
  }
  if (mem_type != CU_MEMORYTYPE_DEVICE || ordinal != dev) return VLA_ATTN_ERR_MEMORY;
  const uintptr_t lo = static_cast<uintptr_t>(dp);
  if (lo < start || bytes > size || lo - start > size - bytes) return VLA_ATTN_ERR_MEMORY;
  *range_lo = lo;
  *range_hi = lo + bytes;
  return VLA_ATTN_OK;
}

int encode_map(const DriverFns& fns, CUtensorMap* map, const void* qkv, int B, int N, int H,
               int d, uint32_t box_c, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  const cuuint64_t dims[5] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), 3u,
                              static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
  const cuuint64_t tok = 3ull * H * d * 2ull;
  const cuuint64_t strides[4] = {static_cast<cuuint64_t>(d) * 2ull,
                                 static_cast<cuuint64_t>(H) * d * 2ull, tok,
                                 tok * static_cast<cuuint64_t>(N)};
  const cuuint32_t box[5] = {box_c, 1u, 1u, box_rows, 1u};
  const cuuint32_t elem_strides[5] = {1u, 1u, 1u, 1u, 1u};
  const CUresult rc = fns.encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(qkv),
                                 dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                 swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? VLA_ATTN_OK : VLA_ATTN_ERR_CUDA;
}

// O as a 4-D tensor [B, N, H, d] (d innermost) for the kernel's output
// stores: box {box_c, 1, 32, 1} (32 rows of one head) at a channel offset.
int encode_out_map(const DriverFns& fns, CUtensorMap* map, const void* o, int B, int N, int H,
                   int d, uint32_t box_c, CUtensorMapSwizzle swizzle) {
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
  const cuuint64_t row = static_cast<cuuint64_t>(H) * d * 2ull;
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2ull, row,
                                 row * static_cast<cuuint64_t>(N)};
  const cuuint32_t box[4] = {box_c, 1u, 32u, 1u};
  const cuuint32_t elem_strides[4] = {1u, 1u, 1u, 1u};
  const CUresult rc = fns.encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(o),
                                 dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                 swizzle, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? VLA_ATTN_OK : VLA_ATTN_ERR_CUDA;
}

int check_args(const void* q, const void* k, const void* v, const void* o, int B, int N, int H,
               int d, float scale) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return VLA_ATTN_ERR_NULL;
  if (B < 1 || N < 1 || H < 1) return VLA_ATTN_ERR_SHAPE;
  if (d != 64 && d != 72) return VLA_ATTN_ERR_UNSUPPORTED;
  if (N > kMaxTokens) return VLA_ATTN_ERR_UNSUPPORTED;
  const uintptr_t qa = reinterpret_cast<uintptr_t>(q);
  const uintptr_t hd_bytes = static_cast<uintptr_t>(H) * d * 2u;
  if (reinterpret_cast<uintptr_t>(k) != qa + hd_bytes ||
      reinterpret_cast<uintptr_t>(v) != qa + 2u * hd_bytes)
    return VLA_ATTN_ERR_SHAPE;
  if ((qa & 15u) != 0 || (reinterpret_cast<uintptr_t>(o) & 15u) != 0) return VLA_ATTN_ERR_ALIGN;
  if (!std::isfinite(scale) || !(scale > 0.0f)) return VLA_ATTN_ERR_SCALE;
  // TMA extents are 32-bit per dimension; element counts must fit size_t math below.
  const unsigned long long total = 3ull * B * N * H * d;
  if (total > (1ull << 46)) return VLA_ATTN_ERR_SHAPE;
  return VLA_ATTN_OK;
}

// Tensor maps of recent calls, in static host memory: direct-mapped tables keyed by
// everything the maps encode (base address, shape, head dimension), one for the QKV
// input and one for the output.  A hit skips the encodings of a call; the maps hold
// no pointer other than the base, so a buffer freed and reallocated at the same
// address with the same shape reuses valid maps.
struct MapSet {
  bool valid = false;
  const void* base = nullptr;
  int B = 0, N = 0, H = 0, d = 0;
  CUtensorMap m0, m1, m2, m3;  // QKV: q, kv, q_tail, kv_tail; output: o, o_tail
};
constexpr int kMapCacheSlots = 64;
std::mutex g_map_mutex;
MapSet g_map_cache[kMapCacheSlots];
MapSet g_out_map_cache[kMapCacheSlots];

MapSet& map_slot(MapSet* table, const void* base, int B, int N, int H, int D) {
  const uint64_t h = (reinterpret_cast<uintptr_t>(base) >> 4) * 0x9E3779B97F4A7C15ull ^
                     (static_cast<uint64_t>(B) * 73856093ull) ^ (static_cast<uint64_t>(N) << 20) ^
                     (static_cast<uint64_t>(H) << 40) ^ static_cast<uint64_t>(D);
  return table[(h >> 32) % kMapCacheSlots];
}

template <int D>
int tensor_maps(const DriverFns& fns, const void* q, const void* o, int B, int N, int H,
                vla::AttnParams* prm) {
  using G = vla::Geom<D>;
  std::lock_guard<std::mutex> lock(g_map_mutex);
  MapSet& e = map_slot(g_map_cache, q, B, N, H, D);
  if (!(e.valid && e.base == q && e.B == B && e.N == N && e.H == H && e.d == D)) {
    e.valid = false;
    int rc = encode_map(fns, &e.m0, q, B, N, H, D, 64u, vla::kQRows, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != VLA_ATTN_OK) return rc;
    rc = encode_map(fns, &e.m1, q, B, N, H, D, 64u, G::BK, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != VLA_ATTN_OK) return rc;
    if (G::kHasTail) {
      rc = encode_map(fns, &e.m2, q, B, N, H, D, 16u, vla::kQRows, CU_TENSOR_MAP_SWIZZLE_32B);
      if (rc != VLA_ATTN_OK) return rc;
      rc = encode_map(fns, &e.m3, q, B, N, H, D, 16u, G::BK, CU_TENSOR_MAP_SWIZZLE_32B);
      if (rc != VLA_ATTN_OK) return rc;
    }
    e.base = q;
    e.B = B;
    e.N = N;
    e.H = H;
    e.d = D;
    e.valid = true;
  }
  MapSet& f = map_slot(g_out_map_cache, o, B, N, H, D);
  if (!(f.valid && f.base == o && f.B == B && f.N == N && f.H == H && f.d == D)) {
    f.valid = false;
    int rc = encode_out_map(fns, &f.m0, o, B, N, H, D, 64u, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != VLA_ATTN_OK) return rc;
    if (G::kHasTail) {
      rc = encode_out_map(fns, &f.m1, o, B, N, H, D, 8u, CU_TENSOR_MAP_SWIZZLE_NONE);
      if (rc != VLA_ATTN_OK) return rc;
    }
    f.base = o;
    f.B = B;
    f.N = N;
    f.H = H;
    f.d = D;
    f.valid = true;
  }
  prm->tm_q = e.m0;
  prm->tm_kv = e.m1;
  prm->tm_o = f.m0;
  if (G::kHasTail) {
    prm->tm_q_tail = e.m2;
    prm->tm_kv_tail = e.m3;
    prm->tm_o_tail = f.m1;
  }
  return VLA_ATTN_OK;
}

template <int D>
int launch(const void* q, void* o, int B, int N, int H, float scale, cudaStream_t stream,
           const DeviceInfo& di, int dev, const DriverFns& fns) {
  using G = vla::Geom<D>;
  vla::AttnParams prm;
  std::memset(&prm, 0, sizeof(prm));
  int rc = tensor_maps<D>(fns, q, o, B, N, H, &prm);
  if (rc != VLA_ATTN_OK) return rc;
  const int nb = (N + G::BK - 1) / G::BK;
  const int nq = (N + vla::kQRows - 1) / vla::kQRows;
  const KernelAttrs& ka = kernel_attrs<D>();
  if (!ka.ok) return VLA_ATTN_ERR_CUDA;
  const int max_smem = di.max_smem_optin - ka.static_smem;
  // Shared memory: Q buffers (qbuf per slot), the K/V ring, and the output
  // staging when the output leaves by TMA stores (stage_out).  The default is
  // staging with two Q buffers (the next round's Q tile loads during the
  // current round) while that leaves a ring of four blocks, else one; stream
  // mode takes one Q buffer and the deeper ring (below).  When a
  // head's K/V blocks fit a ring only without the staging (whole-head units
  // with 5 or 6 blocks), the output goes by row stores instead and the head's
  // K/V stay resident for all its rounds.
  auto ring_for = [&](int qbuf, bool staged) {
    const int r = (max_smem - static_cast<int>(2 * qbuf * G::kQBytes +
                                               (staged ? G::kStageBytes : 0u) +
                                               vla::kBarrierRegionBytes + vla::kAlignSlack)) /
                  static_cast<int>(2 * G::kKVStride);
    return r > vla::kMaxRing ? vla::kMaxRing : r;
  };
  const long long heads_total = static_cast<long long>(B) * H;
  const bool whole_heads = heads_total >= di.sm_count;
  const bool streams = whole_heads && nq > 1 && (nq & 1);
  constexpr int kMinRingQ2 = 4;
  bool stage_out = true;
  int qbuf = vla::kMaxQBuf;
  int ring = ring_for(qbuf, true);
  if (ring < kMinRingQ2) {
    qbuf = 1;
    ring = ring_for(qbuf, true);
  }
  // Stream mode streams every round's K/V blocks through the ring: a ring
  // that holds a whole round's blocks (one Q buffer per slot; 5 blocks at
  // d = 64) measured 1-2 % faster than keeping a second Q buffer to load the
  // next round's tile early (577 tokens at B = 128 and 256, 1025 at B = 64).
  if (streams) {
    qbuf = 1;
    ring = ring_for(1, true);
  }
  if (whole_heads && !streams && nb > ring) {
    if (nb <= ring_for(1, true)) {
      qbuf = 1;
      ring = ring_for(1, true);
    } else if (nb <= ring_for(1, false)) {
      stage_out = false;
      qbuf = 1;
      ring = ring_for(1, false);
    }
  }
  if (ring < 2) return VLA_ATTN_ERR_DEVICE;
  const uint32_t smem = vla::smem_bytes_for<D>(ring, qbuf, stage_out);

  prm.B = B;
  prm.N = N;
  prm.H = H;
  prm.num_kblocks = nb;
  prm.num_qtiles = nq;
  // Work units: whole heads (K/V loaded once per head) when there are enough
  // heads to fill the SMs; otherwise single Q tiles if all of them fit on the
  // SMs at once (shortest per-CTA chain), else single rounds of two tiles.
  // Whole heads with an odd tile count run in stream mode: the CTA pairs its
  // heads' tiles across head boundaries (no half rounds) and streams K/V.
  prm.rounds_per_head = (nq + 1) / 2;
  const long long heads = static_cast<long long>(B) * H;
  prm.rounds_per_unit = heads >= di.sm_count ? prm.rounds_per_head : 1;
  prm.tile_units = (heads < di.sm_count && nq > 1 && heads * nq <= di.sm_count) ? 1 : 0;
  prm.stream = (heads >= di.sm_count && nq > 1 && (nq & 1)) ? 1 : 0;
  prm.units_per_head = prm.tile_units ? nq : prm.rounds_per_head / prm.rounds_per_unit;
  const long long units = heads * prm.units_per_head;
  if (units > 0x7FFFFFFFll) return VLA_ATTN_ERR_SHAPE;
  prm.num_units = static_cast<int>(units);
  prm.ring = ring;
  prm.qbuf = qbuf;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.reuse = (nb <= ring && !prm.stream) ? 1 : 0;
  prm.carry = (nb <= ring && prm.stream) ? 1 : 0;
  prm.c = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  const unsigned long long lim = g_wait_limit_ns.load();
  prm.wait_limit_ns = lim == 0 ? kDefaultWaitLimitNs : lim;
  prm.test_stall = g_test_stall.load();

  rc = stage_out ? ensure_smem_attr<D, true>(dev, static_cast<int>(smem))
                 : ensure_smem_attr<D, false>(dev, static_cast<int>(smem));
  if (rc != VLA_ATTN_OK) return rc;

  const int grid = static_cast<int>(units < di.sm_count ? units : di.sm_count);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(vla::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  set_dependent_launch(&cfg, attr);
  const cudaError_t le = stage_out ? cudaLaunchKernelEx(&cfg, vla::attn_fwd_kernel<D, true>, prm)
                                   : cudaLaunchKernelEx(&cfg, vla::attn_fwd_kernel<D, false>, prm);
  if (le != cudaSuccess) {
    (void)cudaGetLastError();
    return VLA_ATTN_ERR_CUDA;
  }
  g_launches.fetch_add(1);
  return VLA_ATTN_OK;
}

}  // namespace

extern "C" {

int vla_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int N, int H,
                 int d, float scale, void* stream) {
  int rc = check_args(q, k, v, o, B, N, H, d, scale);
  if (rc != VLA_ATTN_OK) return rc;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return VLA_ATTN_ERR_CUDA;
  DeviceInfo di;
  rc = device_info(dev, &di);
  if (rc != VLA_ATTN_OK) return rc;
  const DriverFns& fns = driver_fns();
  if (fns.encode == nullptr || fns.ptr_attr == nullptr) return VLA_ATTN_ERR_CUDA;
  const size_t in_bytes = 3ull * B * N * H * d * 2ull;
  const size_t out_bytes = 1ull * B * N * H * d * 2ull;
  uintptr_t in_lo = 0, in_hi = 0, out_lo = 0, out_hi = 0;
  rc = check_device_range(fns, q, in_bytes, dev, &in_lo, &in_hi);
  if (rc != VLA_ATTN_OK) return rc;
  rc = check_device_range(fns, o, out_bytes, dev, &out_lo, &out_hi);
  if (rc != VLA_ATTN_OK) return rc;
  if (out_lo < in_hi && in_lo < out_hi) return VLA_ATTN_ERR_MEMORY;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 64) return launch<64>(q, o, B, N, H, scale, st, di, dev, fns);
  return launch<72>(q, o, B, N, H, scale, st, di, dev, fns);
}

int vla_attn_fwd_host(const void* qkv_host, void* o_host, void* qkv_dev, void* o_dev, int B,
                      int N, int H, int d, float scale, void* stream) {
  if (qkv_host == nullptr || o_host == nullptr || qkv_dev == nullptr || o_dev == nullptr)
    return VLA_ATTN_ERR_NULL;
  const char* qd = static_cast<const char*>(qkv_dev);
  const size_t hd_bytes = static_cast<size_t>(H > 0 ? H : 0) * (d > 0 ? d : 0) * 2u;
  int rc = check_args(qd, qd + hd_bytes, qd + 2 * hd_bytes, o_dev, B, N, H, d, scale);
  if (rc != VLA_ATTN_OK) return rc;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VLA_ATTN_ERR_CUDA;
  DeviceInfo di;
  if ((rc = device_info(dev, &di)) != VLA_ATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t img_out = static_cast<size_t>(N) * H * d * 2u;  // bytes of one image's O
  const size_t img_in = 3u * img_out;                           // and of its packed QKV
  // The device buffers must hold the whole batch and must not overlap, checked before
  // the first copy is enqueued (as vla_attn_fwd checks its buffers before its launch).
  {
    const DriverFns& fns = driver_fns();
    if (fns.encode == nullptr || fns.ptr_attr == nullptr) return VLA_ATTN_ERR_CUDA;
    uintptr_t in_lo = 0, in_hi = 0, out_lo = 0, out_hi = 0;
    if ((rc = check_device_range(fns, qkv_dev, img_in * B, dev, &in_lo, &in_hi)) != VLA_ATTN_OK)
      return rc;
    if ((rc = check_device_range(fns, o_dev, img_out * B, dev, &out_lo, &out_hi)) != VLA_ATTN_OK)
      return rc;
    if (out_lo < in_hi && in_lo < out_hi) return VLA_ATTN_ERR_MEMORY;
  }
  // Chunks of whole images with at least one head per SM: a chunk's kernel
  // is far shorter than the next chunk's input copy, so its efficiency does
  // not matter, while a small last chunk keeps short the part of the step
  // that nothing overlaps (its kernel and result copy).  A batch smaller than
  // two chunks goes in one.
  const long long min_heads = di.sm_count;
  const int chunk = static_cast<int>((min_heads + H - 1) / H);
  if (B < 2 * chunk) {
    if (cudaMemcpyAsync(qkv_dev, qkv_host, img_in * B, cudaMemcpyHostToDevice, st) != cudaSuccess)
      return VLA_ATTN_ERR_CUDA;
    rc = vla_attn_fwd(qd, qd + hd_bytes, qd + 2 * hd_bytes, o_dev, B, N, H, d, scale, stream);
    if (rc != VLA_ATTN_OK) return rc;
    if (cudaMemcpyAsync(o_host, o_dev, img_out * B, cudaMemcpyDeviceToHost, st) != cudaSuccess)
      return VLA_ATTN_ERR_CUDA;
    return VLA_ATTN_OK;
  }
  // Pipelined: the input copies run back to back on the device's copy-in
  // stream (after `stream`'s earlier work), chunk i's kernel on `stream` once
  // its copy has landed, its result copy on the copy-out stream once the
  // kernel is done; the two directions use separate copy engines.  `stream`
  // waits for both side streams at the end.
  std::lock_guard<std::mutex> lock(g_pipe_mutex);
  HostPipe* pipe = nullptr;
  if ((rc = host_pipe(dev, &pipe)) != VLA_ATTN_OK) return rc;
  const char* hin = static_cast<const char*>(qkv_host);
  char* hout = static_cast<char*>(o_host);
  char* din = static_cast<char*>(qkv_dev);
  char* dout = static_cast<char*>(o_dev);
  bool forked = false;
  if (cudaEventRecord(pipe->start, st) != cudaSuccess ||
      cudaStreamWaitEvent(pipe->in, pipe->start, 0) != cudaSuccess)
    return VLA_ATTN_ERR_CUDA;
  bool loading = false;
  for (int b0 = 0; b0 < B && rc == VLA_ATTN_OK; b0 += chunk) {
    const int nbi = B - b0 < chunk ? B - b0 : chunk;
    const size_t in_off = img_in * b0, out_off = img_out * b0;
    loading = true;
    if (cudaMemcpyAsync(din + in_off, hin + in_off, img_in * nbi, cudaMemcpyHostToDevice,
                        pipe->in) != cudaSuccess ||
        cudaEventRecord(pipe->loaded, pipe->in) != cudaSuccess ||
        cudaStreamWaitEvent(st, pipe->loaded, 0) != cudaSuccess) {
      rc = VLA_ATTN_ERR_CUDA;
      break;
    }
    const char* q = din + in_off;
    rc = vla_attn_fwd(q, q + hd_bytes, q + 2 * hd_bytes, dout + out_off, nbi, N, H, d, scale,
                      stream);
    if (rc != VLA_ATTN_OK) break;
    if (cudaEventRecord(pipe->fork, st) != cudaSuccess ||
        cudaStreamWaitEvent(pipe->out, pipe->fork, 0) != cudaSuccess) {
      rc = VLA_ATTN_ERR_CUDA;
      break;
    }
    forked = true;
    if (cudaMemcpyAsync(hout + out_off, dout + out_off, img_out * nbi, cudaMemcpyDeviceToHost,
                        pipe->out) != cudaSuccess)
      rc = VLA_ATTN_ERR_CUDA;
  }
  // Join even after an error, so that work already on the side streams is
  // ordered before anything later on `stream`.
  if (forked && (cudaEventRecord(pipe->join, pipe->out) != cudaSuccess ||
                 cudaStreamWaitEvent(st, pipe->join, 0) != cudaSuccess))
    rc = VLA_ATTN_ERR_CUDA;
  if (loading && (cudaEventRecord(pipe->in_join, pipe->in) != cudaSuccess ||
                  cudaStreamWaitEvent(st, pipe->in_join, 0) != cudaSuccess))
    rc = VLA_ATTN_ERR_CUDA;
  return rc;
}

const char* vla_attn_strerror(int status) {
  switch (status) {
    case VLA_ATTN_OK: return "ok";
    case VLA_ATTN_ERR_NULL: return "a required pointer is NULL";
    case VLA_ATTN_ERR_SHAPE:
      return "bad shape: B, N, H must be >= 1 and q/k/v must point into one packed [B,N,3,H,d] "
             "buffer (k = q + H*d, v = q + 2*H*d elements)";
    case VLA_ATTN_ERR_UNSUPPORTED:
      return "unsupported: head dimension must be 64 or 72 and N at most vla_attn_max_tokens(d)";
    case VLA_ATTN_ERR_ALIGN: return "q and o must be 16-byte aligned";
    case VLA_ATTN_ERR_SCALE: return "scale must be finite and > 0";
    case VLA_ATTN_ERR_CUDA: return "a CUDA runtime or driver call failed";
    case VLA_ATTN_ERR_TIMEOUT: return "a bounded wait inside the attention kernel ran out";
    case VLA_ATTN_ERR_DEVICE: return "the current device is not an sm_100 (B200-class) GPU";
    case VLA_ATTN_ERR_MEMORY:
      return "a pointer is not device memory of the current device, its allocation is too "
             "small for the shape, or the output overlaps the input";
    default: return "unknown vla_attn status";
  }
}

int vla_attn_last_device_status(void* stream, int* site) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int word = 0;
  if (cudaMemcpyFromSymbolAsync(&word, vla::g_vla_attn_status, sizeof(int), 0,
                                cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return VLA_ATTN_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return VLA_ATTN_ERR_CUDA;
  if (site != nullptr) *site = word == 0 ? 0 : word - 1000;
  return word == 0 ? VLA_ATTN_OK : VLA_ATTN_ERR_TIMEOUT;
}

int vla_attn_reset_device_status(void* stream) {
  static const int zero = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyToSymbolAsync(vla::g_vla_attn_status, &zero, sizeof(int), 0,
                              cudaMemcpyHostToDevice, st) != cudaSuccess)
    return VLA_ATTN_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return VLA_ATTN_ERR_CUDA;
  return VLA_ATTN_OK;
}

int vla_attn_max_tokens(int d) { return (d == 64 || d == 72) ? kMaxTokens : 0; }

uint64_t vla_attn_launch_count(void) { return g_launches.load(); }

void vla_attn_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns); }

void vla_attn_set_test_stall(int enable) { g_test_stall.store(enable ? 1 : 0); }

}  // extern "C"

// LayerNorm and the linear layers around the attention core (same host
// helpers: device and pointer-range checks, launch counter).
#include "block_ops.cuh"
