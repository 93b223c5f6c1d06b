// Host side of libttc05: the C ABI declared in include/gemm_f16.h.
//
// Argument validation, per-device context (SM count, status word), TMA
// tensor-map encoding, the choice between the tile kernels and the small-M
// kernel, the small-M workspace cache and the status/self-test entry points.
// The computation itself is the fused GEMM + ReLU of "Writing high-performance
// kernels in TileLang" (atlascloud.ai blog), section "Escribamos un GEMM".
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdlib>
#include <mutex>
#include <vector>

#include "../../include/gemm_f16.h"
#include "internal.h"
#include "sm100.cuh"

namespace ttc {

// One status word per device (first device-side error wins; 0 = none).
__device__ int g_device_status;

namespace {

constexpr uint64_t kDefaultTimeoutNs = 1000ull * 1000ull * 1000ull;  // 1 s per wait
constexpr int kMaxDevices = 64;

struct DeviceEntry {
  bool ready = false;
  bool supported = false;
  int sm_count = 0;
  int* status = nullptr;
};

std::mutex g_mutex;
DeviceEntry g_devices[kMaxDevices];

struct Workspace {
  int device;
  cudaStream_t stream;
  void* ptr;
  size_t bytes;
};
std::vector<Workspace> g_workspaces;

// ------------------------------------------------------ driver entry points ---
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
typedef CUresult (*AddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);
typedef CUresult (*PointerAttrsFn)(unsigned int, CUpointer_attribute*, void**, CUdeviceptr);

EncodeTiledFn g_encode = nullptr;
AddressRangeFn g_addr_range = nullptr;
PointerAttrsFn g_ptr_attrs = nullptr;
std::once_flag g_entry_once;

void load_entry_points() {
  std::call_once(g_entry_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_addr_range = reinterpret_cast<AddressRangeFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuPointerGetAttributes", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ptr_attrs = reinterpret_cast<PointerAttrsFn>(fn);
  });
}

// ------------------------------------------------------------ device state ---
int get_device(DeviceCtx* ctx) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GEMM_ERR_LAUNCH;
  if (dev < 0 || dev >= kMaxDevices) return GEMM_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceEntry& e = g_devices[dev];
  if (!e.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return GEMM_ERR_LAUNCH;
    e.supported = (major == 10 && minor == 0);
    e.sm_count = sms;
    if (e.supported) {
      // The symbol's device address for this device (host code cannot use the
      // symbol itself as a pointer).
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return GEMM_ERR_LAUNCH;
      e.status = static_cast<int*>(p);
    }
    e.ready = true;
  }
  if (!e.supported) return GEMM_ERR_UNSUPPORTED_DEVICE;
  ctx->device = dev;
  ctx->sm_count = e.sm_count;
  ctx->status = e.status;
  ctx->timeout_ns = kDefaultTimeoutNs;
  return GEMM_OK;
}

// Device memory of the current device (or managed memory) only.
bool is_device_pointer(const void* p, int device) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error state of this query
    return false;
  }
  if (attr.type == cudaMemoryTypeManaged) return true;
  return attr.type == cudaMemoryTypeDevice && attr.device == device;
}

// The bytes [p, p + (rows-1)*ld*2 + cols*2) lie in one allocation.
bool extent_in_allocation(const void* p, int64_t rows, int64_t cols, int64_t ld) {
  if (g_addr_range == nullptr) return true;  // cannot check; TMA bounds still apply
  CUdeviceptr base = 0;
  size_t size = 0;
  if (g_addr_range(&base, &size, reinterpret_cast<CUdeviceptr>(p)) != CUDA_SUCCESS) return false;
  const uint64_t start = reinterpret_cast<uint64_t>(p);
  const uint64_t span = (static_cast<uint64_t>(rows - 1) * static_cast<uint64_t>(ld) +
                         static_cast<uint64_t>(cols)) * 2u;
  return start >= base && start - base + span <= size;
}

// One driver query for memory type, owning device and allocation range.
// Returns -1 when the query itself is unavailable (caller falls back).
int query_pointer(const void* p, int device, int64_t rows, int64_t cols, int64_t ld) {
  if (g_ptr_attrs == nullptr) return -1;
  unsigned int mem_type = 0;
  int ordinal = -1;
  unsigned int managed = 0;
  CUdeviceptr base = 0;
  size_t size = 0;
  CUpointer_attribute attrs[5] = {CU_POINTER_ATTRIBUTE_MEMORY_TYPE,
                                  CU_POINTER_ATTRIBUTE_DEVICE_ORDINAL,
                                  CU_POINTER_ATTRIBUTE_IS_MANAGED,
                                  CU_POINTER_ATTRIBUTE_RANGE_START_ADDR,
                                  CU_POINTER_ATTRIBUTE_RANGE_SIZE};
  void* data[5] = {&mem_type, &ordinal, &managed, &base, &size};
  if (g_ptr_attrs(5, attrs, data, reinterpret_cast<CUdeviceptr>(p)) != CUDA_SUCCESS) return 0;
  const bool on_device = (mem_type == CU_MEMORYTYPE_DEVICE && ordinal == device) || managed != 0;
  if (!on_device || size == 0) return 0;
  const uint64_t start = reinterpret_cast<uint64_t>(p);
  const uint64_t span = (static_cast<uint64_t>(rows - 1) * static_cast<uint64_t>(ld) +
                         static_cast<uint64_t>(cols)) * 2u;
  return (start >= base && start - base + span <= size) ? 1 : 0;
}

int check_matrix(const void* p, int64_t rows, int64_t cols, int64_t ld, int device) {
  if (p == nullptr) return GEMM_ERR_INVALID_ARG;
  if (ld < cols || ld < 1) return GEMM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(p) & 15u) != 0 || (ld & 7) != 0) return GEMM_ERR_ALIGNMENT;
  if (static_cast<uint64_t>(ld) * 2u >= (1ull << 40)) return GEMM_ERR_INVALID_ARG;
  const int q = query_pointer(p, device, rows, cols, ld);
  if (q == 0) return GEMM_ERR_INVALID_ARG;
  if (q < 0) {
    if (!is_device_pointer(p, device)) return GEMM_ERR_INVALID_ARG;
    if (!extent_in_allocation(p, rows, cols, ld)) return GEMM_ERR_INVALID_ARG;
  }
  return GEMM_OK;
}

int get_workspace(const DeviceCtx& d, cudaStream_t stream, void** ptr, size_t* bytes) {
  const size_t need = skinny_workspace_bytes(d.sm_count, 64);
  std::lock_guard<std::mutex> lock(g_mutex);
  for (const Workspace& w : g_workspaces) {
    if (w.device == d.device && w.stream == stream) {
      *ptr = w.ptr;
      *bytes = w.bytes;
      return GEMM_OK;
    }
  }
  void* p = nullptr;
  if (cudaMalloc(&p, need) != cudaSuccess) {
    cudaGetLastError();
    return GEMM_ERR_WORKSPACE;
  }
  // the counters start at zero and every call leaves them at zero
  if (cudaMemsetAsync(p, 0, need, stream) != cudaSuccess) {
    cudaFree(p);
    return GEMM_ERR_WORKSPACE;
  }
  g_workspaces.push_back({d.device, stream, p, need});
  *ptr = p;
  *bytes = need;
  return GEMM_OK;
}

__global__ void zero_fill_kernel(__half* C, int64_t M, int64_t N, int64_t ldc) {
  const int64_t total = M * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / N, c = i - r * N;
    C[r * ldc + c] = __ushort_as_half(0);
  }
}

template <int ACT>
__global__ void bias_act_fill_kernel(__half* C, const __half* bias, int64_t M, int64_t N,
                                     int64_t ldc) {
  const int64_t total = M * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / N, c = i - r * N;
    C[r * ldc + c] = __float2half_rn(activate<ACT>(__half2float(bias[c])));
  }
}

template <int ACT>
__global__ void activation_f32_kernel(const float* x, float* y, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    y[i] = activate<ACT>(x[i]);
}

__global__ void wait_probe_kernel(int* status, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on `bar`: the wait must give up on its own
    if (!mbar_wait(&bar, 0, &abort_flag, timeout_ns))
      raise_abort(status, &abort_flag, kStatusTimeoutBase | (kRoleProbe << 4) | 1);
  }
}

// Streaming-read probe: the grid reads n16 16-byte words once, each thread
// four independent streaming (evict-first) loads per step strided by the
// whole grid, and folds them with XOR so no load is dead; one atomic XOR per
// warp into *sink.
__global__ void __launch_bounds__(512) read_probe_kernel(const uint4* __restrict__ src,
                                                         int64_t n16, unsigned* sink) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  unsigned acc = 0;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    const uint4 v0 = __ldcs(src + i);
    const uint4 v1 = __ldcs(src + i + stride);
    const uint4 v2 = __ldcs(src + i + 2 * stride);
    const uint4 v3 = __ldcs(src + i + 3 * stride);
    acc ^= v0.x ^ v0.y ^ v0.z ^ v0.w ^ v1.x ^ v1.y ^ v1.z ^ v1.w;
    acc ^= v2.x ^ v2.y ^ v2.z ^ v2.w ^ v3.x ^ v3.y ^ v3.z ^ v3.w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = __ldcs(src + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
  acc = __reduce_xor_sync(0xffffffffu, acc);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, acc);
}

int read_and_clear_status(const DeviceCtx& d, cudaStream_t stream, int* out) {
  int host = 0;
  if (cudaMemcpyAsync(&host, d.status, sizeof(int), cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return GEMM_ERR_LAUNCH;
  if (host != 0) {
    if (cudaMemsetAsync(d.status, 0, sizeof(int), stream) != cudaSuccess)
      return GEMM_ERR_LAUNCH;
    // a kernel that gave up may have left split-K arrival counters non-zero
    std::lock_guard<std::mutex> lock(g_mutex);
    for (const Workspace& w : g_workspaces)
      if (w.device == d.device && cudaMemsetAsync(w.ptr, 0, w.bytes, stream) != cudaSuccess)
        return GEMM_ERR_LAUNCH;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GEMM_ERR_LAUNCH;
  }
  *out = host;
  return GEMM_OK;
}

}  // namespace

int encode_tmap_f16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t ld, uint32_t box_inner, uint32_t box_outer) {
  load_entry_points();
  if (g_encode == nullptr) return GEMM_ERR_LAUNCH;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {ld * 2u};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estrides[2] = {1, 1};
  // (L2 promotion none / 128 B / 256 B measured alike on the pair kernels:
  // the same DRAM bytes and time)
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base),
                              dims, strides, box, estrides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GEMM_OK : GEMM_ERR_INVALID_ARG;
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* s = std::getenv("TTC_PDL");
    return !(s != nullptr && s[0] == '0');
  }();
  return on;
}

int pdl_attribute(cudaLaunchAttribute* attr) {
  if (!pdl_enabled()) return 0;
  attr->id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr->val.programmaticStreamSerializationAllowed = 1;
  return 1;
}

int launch_bias_act_fill(const GemmProblem& p) {
  const int64_t total = p.M * p.N;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  __half* C = static_cast<__half*>(p.C);
  const __half* bias = static_cast<const __half*>(p.bias);
  const int g = static_cast<int>(blocks);
  if (p.act == kActRelu)
    bias_act_fill_kernel<kActRelu><<<g, 256, 0, p.stream>>>(C, bias, p.M, p.N, p.ldc);
  else if (p.act == kActGelu)
    bias_act_fill_kernel<kActGelu><<<g, 256, 0, p.stream>>>(C, bias, p.M, p.N, p.ldc);
  else
    bias_act_fill_kernel<kActNone><<<g, 256, 0, p.stream>>>(C, bias, p.M, p.N, p.ldc);
  return cudaGetLastError() == cudaSuccess ? GEMM_OK : GEMM_ERR_LAUNCH;
}

int launch_zero_fill(const GemmProblem& p) {
  const int64_t total = p.M * p.N;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  zero_fill_kernel<<<static_cast<int>(blocks), 256, 0, p.stream>>>(static_cast<__half*>(p.C),
                                                                     p.M, p.N, p.ldc);
  return cudaGetLastError() == cudaSuccess ? GEMM_OK : GEMM_ERR_LAUNCH;
}

}  // namespace ttc

using namespace ttc;

extern "C" {

int gemm_abi_version(void) { return 10300; }

namespace ttc {
namespace {

// Fraction of the SM-pair slots the last wave keeps busy, averaged: tiles /
// (pairs * waves).
double wave_efficiency(int64_t tiles, int64_t pairs) {
  const int64_t waves = (tiles + pairs - 1) / pairs;
  return waves > 0 ? static_cast<double>(tiles) / static_cast<double>(waves * pairs) : 0.0;
}

// The kernel chosen for a shape on a GPU with `sm_count` SMs.  The 512 x 256
// pair tile stages 25 % fewer bytes per MAC than the 256 x 256 one, but its
// single accumulator leaves part of each tile's epilogue exposed, which costs
// more the shorter the main loop and the longer the epilogue.  Measured
// (30-launch bursts and 2-second runs under the power cap, both tiles with
// 4096-row panels, the 256-row tile with 6 stages, waves sweeping K both ways):
//   8192 x 8192 x 8192, ReLU:    512-row tile 0.723 / 0.832 ms, 256-row 0.771 / 0.886
//   8192 x 14336 x 4096, ReLU:   512-row tile 0.643 / 0.750 ms, 256-row 0.649 / 0.766
//   8192 x 14336 x 4096, GELU:   512-row tile 0.695 / 0.806 ms, 256-row 0.682 / 0.798
// So the 512-row tile is taken from K = 4096 with ReLU or no activation and
// from K = 6144 with GELU (its epilogue is the longest), unless its last wave
// wastes more than 6 points more of the SM pairs than the 256-row tiling's.
int select_path_for(int64_t M, int64_t N, int64_t K, int sm_count, int activation) {
  if (M >= 1 && M <= 64) return GEMM_PATH_SKINNY;
  const int64_t pairs = sm_count / 2 > 0 ? sm_count / 2 : 1;
  const int64_t col_tiles = (N + 255) / 256;
  const int64_t tiles256 = ((M + 255) / 256) * col_tiles;
  if (tiles256 < 64) return GEMM_PATH_TILE;
  if (K < (activation == GEMM_ACT_GELU ? 6144 : 4096)) return GEMM_PATH_TILE_PAIR;
  const int64_t tiles512 = ((M + 511) / 512) * col_tiles;
  return wave_efficiency(tiles512, pairs) >= wave_efficiency(tiles256, pairs) - 0.06
             ? GEMM_PATH_TILE_PAIR_TALL
             : GEMM_PATH_TILE_PAIR;
}

int default_stages(int kernel, int block_n) {
  switch (kernel) {
    case GEMM_PATH_TILE:
      return block_n == 256 ? kDefaultStagesTile256
                            : (block_n == 64 ? kDefaultStagesTile64 : kDefaultStagesTile128);
    case GEMM_PATH_TILE_PAIR: return kDefaultStagesPair;
    case GEMM_PATH_TILE_PAIR_TALL: return kDefaultStagesTall;
    case GEMM_PATH_SKINNY: return block_n == 128 ? kDefaultStagesSkinnyNarrow : kDefaultStagesSkinny;
    case GEMM_PATH_SKINNY_EVEN: return block_n == 256 ? kDefaultStagesEven4 : kDefaultStagesEven;
    default: return 0;
  }
}

// Fills the fields of `c` left at 0 with what GEMM_PATH_AUTO would use for an
// M x N output and checks the rest (the stage count is checked against the
// compiled kernels at launch).  Returns GEMM_OK or GEMM_ERR_CONFIG.
int resolve_config(KernelConfig& c, int64_t M, int64_t N, int64_t K, int sm_count) {
  if (c.stages < 0 || c.splits < 0) return GEMM_ERR_CONFIG;
  switch (c.kernel) {
    case GEMM_PATH_TILE:
      if (c.block_n == 0) {
        // 128 x 256 tiles when there are enough of them to fill the GPU,
        // otherwise 128 x 128 tiles (twice as many CTAs for small problems),
        // or 128 x 64 tiles when even those would fill at most half the SMs
        const int64_t tiles256 = ((M + 127) / 128) * ((N + 255) / 256);
        const int64_t tiles128 = ((M + 127) / 128) * ((N + 127) / 128);
        c.block_n = tiles256 >= sm_count ? 256 : (2 * tiles128 <= sm_count ? 64 : 128);
      }
      if (c.block_n != 64 && c.block_n != 128 && c.block_n != 256) return GEMM_ERR_CONFIG;
      break;
    case GEMM_PATH_TILE_PAIR:
    case GEMM_PATH_TILE_PAIR_TALL:
      if (c.block_n == 0) c.block_n = 256;
      if (c.block_n != 256) return GEMM_ERR_CONFIG;
      break;
    case GEMM_PATH_SKINNY:
      if (c.block_n == 0) c.block_n = (N + 127) / 128 <= sm_count ? 128 : 256;
      if (c.block_n != 128 && c.block_n != 256) return GEMM_ERR_CONFIG;
      break;
    case GEMM_PATH_SKINNY_EVEN: {
      const EvenPlan plan = even_plan(N, K, sm_count);
      if (plan.q == 0) return GEMM_ERR_CONFIG;
      if (c.block_n == 0) c.block_n = 64 * plan.q;
      if (c.block_n != 64 * plan.q) return GEMM_ERR_CONFIG;
      break;
    }
    default:
      return GEMM_ERR_CONFIG;
  }
  if (c.stages == 0) c.stages = default_stages(c.kernel, c.block_n);
  if (c.kernel == GEMM_PATH_SKINNY_EVEN) {
    if (c.group_rows != 0 || c.splits != 0 || skinny_m_pad(M) == 0) return GEMM_ERR_CONFIG;
  } else if (c.kernel == GEMM_PATH_SKINNY) {
    if (c.group_rows != 0 || skinny_m_pad(M) == 0) return GEMM_ERR_CONFIG;
  } else {
    if (c.splits != 0) return GEMM_ERR_CONFIG;
    if (c.group_rows == 0)
      c.group_rows = c.kernel == GEMM_PATH_TILE ? kDefaultGroupRows : kDefaultGroupRowsPair;
  }
  return GEMM_OK;
}

// The entry points' common body: validation, then the kernel of `cfg`, or of
// `path` when `cfg` is null.
int run_gemm(const void* A, const void* B, const void* bias, void* C, int64_t M, int64_t N,
             int64_t K, int64_t lda, int64_t ldb, int64_t ldc, int trans_a, int trans_b,
             int activation, int path, const gemm_config* cfg, gemm_stream_t stream) {
  if (M < 0 || N < 0 || K < 0) return GEMM_ERR_INVALID_ARG;
  if ((trans_a != 0 && trans_a != 1) || (trans_b != 0 && trans_b != 1))
    return GEMM_ERR_INVALID_ARG;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return GEMM_ERR_INVALID_ARG;
  if (activation != GEMM_ACT_NONE && activation != GEMM_ACT_RELU &&
      activation != GEMM_ACT_GELU)
    return GEMM_ERR_INVALID_ARG;
  if (cfg == nullptr && path != GEMM_PATH_AUTO && path != GEMM_PATH_TILE &&
      path != GEMM_PATH_SKINNY && path != GEMM_PATH_TILE_PAIR &&
      path != GEMM_PATH_TILE_PAIR_TALL && path != GEMM_PATH_SKINNY_EVEN)
    return GEMM_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return GEMM_OK;
  DeviceCtx d;
  int rc = get_device(&d);
  if (rc != GEMM_OK) return rc;
  KernelConfig kc{};
  if (cfg != nullptr) {
    kc = KernelConfig{cfg->kernel, cfg->block_n, cfg->stages, cfg->group_rows, cfg->splits};
    rc = resolve_config(kc, M, N, K, d.sm_count);
    if (rc != GEMM_OK) return rc;
  } else {
    if (path == GEMM_PATH_AUTO) path = select_path_for(M, N, K, d.sm_count, activation);
    kc = KernelConfig{path, 0, 0, 0, 0};
    if (resolve_config(kc, M, N, K, d.sm_count) != GEMM_OK) return GEMM_ERR_INVALID_ARG;
  }
  load_entry_points();
  rc = check_matrix(C, M, N, ldc, d.device);
  if (rc != GEMM_OK) return rc;
  if (bias != nullptr) {
    // one row of N fp16 values, 16-byte aligned
    rc = check_matrix(bias, 1, N, (N + 7) / 8 * 8, d.device);
    if (rc != GEMM_OK) return rc;
  }
  const int layout = (trans_a ? kLayoutTransA : 0) | (trans_b ? kLayoutTransB : 0);
  GemmProblem p{A, B, C, M, N, K, lda, ldb, ldc, activation, bias, layout, stream};
  if (K == 0) {
    // the empty sum is +0: C = act(bias), or +0 without a bias (act(0) = +0)
    return bias != nullptr ? launch_bias_act_fill(p) : launch_zero_fill(p);
  }
  // stored shapes: A is K x M when transposed, B is N x K when transposed
  rc = trans_a ? check_matrix(A, K, M, lda, d.device) : check_matrix(A, M, K, lda, d.device);
  if (rc == GEMM_OK)
    rc = trans_b ? check_matrix(B, N, K, ldb, d.device) : check_matrix(B, K, N, ldb, d.device);
  if (rc != GEMM_OK) return rc;
  if (kc.kernel == GEMM_PATH_SKINNY || kc.kernel == GEMM_PATH_SKINNY_EVEN) {
    void* ws = nullptr;
    size_t ws_bytes = 0;
    rc = get_workspace(d, stream, &ws, &ws_bytes);
    if (rc != GEMM_OK) return rc;
    if (kc.kernel == GEMM_PATH_SKINNY_EVEN) return launch_skinny_even(p, d, ws, ws_bytes, kc);
    return launch_skinny_gemm(p, d, ws, ws_bytes, kc);
  }
  return launch_tile_gemm(p, d, kc);
}

}  // namespace
}  // namespace ttc

int gemm_select_path(int64_t M, int64_t N, int64_t K) {
  return select_path_for(M, N, K, 148, GEMM_ACT_RELU);  // a B200 has 148 SMs
}

const char* gemm_status_string(int status) {
  switch (status) {
    case GEMM_OK: return "ok";
    case GEMM_ERR_INVALID_ARG: return "invalid argument (size, leading dimension or pointer)";
    case GEMM_ERR_ALIGNMENT: return "pointer not 16-byte aligned or leading dimension not a multiple of 8";
    case GEMM_ERR_UNSUPPORTED_DEVICE: return "current device is not an sm_100 (B200) GPU";
    case GEMM_ERR_LAUNCH: return "CUDA runtime call or kernel launch failed";
    case GEMM_ERR_WORKSPACE: return "small-M workspace allocation failed";
    case GEMM_ERR_DEVICE_TIMEOUT: return "a device-side wait ran out of time";
    case GEMM_ERR_SCRATCH_LIMIT:
      return "problem too large for the fixed scratch of gemm_relu_f16_noalloc (needs M <= 32)";
    case GEMM_ERR_CONFIG:
      return "kernel configuration not compiled, or not valid for this problem";
    default: return "unknown status";
  }
}

int gemm_f16_general(const void* A, const void* B, const void* bias, void* C, int64_t M,
                     int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc, int trans_a,
                     int trans_b, int activation, int path, gemm_stream_t stream) {
  return run_gemm(A, B, bias, C, M, N, K, lda, ldb, ldc, trans_a, trans_b, activation, path,
                  nullptr, stream);
}

int gemm_f16_config(const void* A, const void* B, const void* bias, void* C, int64_t M,
                    int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc, int trans_a,
                    int trans_b, int activation, const gemm_config* cfg, gemm_stream_t stream) {
  if (cfg == nullptr) return GEMM_ERR_INVALID_ARG;
  return run_gemm(A, B, bias, C, M, N, K, lda, ldb, ldc, trans_a, trans_b, activation,
                  GEMM_PATH_AUTO, cfg, stream);
}

int gemm_config_smem_bytes(const gemm_config* cfg) {
  if (cfg == nullptr) return GEMM_ERR_INVALID_ARG;
  int block_n = cfg->block_n;
  if (block_n == 0 && cfg->kernel != GEMM_PATH_TILE && cfg->kernel != GEMM_PATH_SKINNY &&
      cfg->kernel != GEMM_PATH_SKINNY_EVEN)
    block_n = 256;
  const int stages = cfg->stages != 0 ? cfg->stages : default_stages(cfg->kernel, block_n);
  int bytes = -1;
  if (cfg->kernel == GEMM_PATH_SKINNY)
    bytes = skinny_config_smem_bytes(block_n, stages);
  else if (cfg->kernel == GEMM_PATH_SKINNY_EVEN)
    bytes = even_config_smem_bytes(block_n, stages);
  else
    bytes = tile_config_smem_bytes(cfg->kernel, block_n, stages);
  return bytes > 0 ? bytes : GEMM_ERR_CONFIG;
}

int gemm_config_list(gemm_config* out, int capacity) {
  KernelConfig all[64];
  int n = tile_configs_built(all, 64);
  n += skinny_configs_built(all + n, 64 - n);
  n += even_configs_built(all + n, 64 - n);
  for (int i = 0; i < n && i < capacity && out != nullptr; ++i)
    out[i] = gemm_config{all[i].kernel, all[i].block_n, all[i].stages, 0, 0};
  return n;
}

int gemm_auto_config(int64_t M, int64_t N, int64_t K, int activation, gemm_config* out) {
  if (out == nullptr || M < 1 || N < 1 || K < 0 || M > INT32_MAX || N > INT32_MAX ||
      K > INT32_MAX)
    return GEMM_ERR_INVALID_ARG;
  if (activation != GEMM_ACT_NONE && activation != GEMM_ACT_RELU &&
      activation != GEMM_ACT_GELU)
    return GEMM_ERR_INVALID_ARG;
  DeviceCtx d;
  const int rc = get_device(&d);
  if (rc != GEMM_OK) return rc;
  KernelConfig c{select_path_for(M, N, K, d.sm_count, activation), 0, 0, 0, 0};
  if (resolve_config(c, M, N, K, d.sm_count) != GEMM_OK) return GEMM_ERR_INVALID_ARG;
  *out = gemm_config{c.kernel, c.block_n, c.stages, c.group_rows, c.splits};
  return GEMM_OK;
}

int gemm_bias_act_f16(const void* A, const void* B, const void* bias, void* C, int64_t M,
                      int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc,
                      int activation, int path, gemm_stream_t stream) {
  return gemm_f16_general(A, B, bias, C, M, N, K, lda, ldb, ldc, 0, 0, activation, path,
                          stream);
}

int gemm_f16_ex(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K,
                int64_t lda, int64_t ldb, int64_t ldc, int relu, int path,
                gemm_stream_t stream) {
  if (relu != 0 && relu != 1) return GEMM_ERR_INVALID_ARG;
  return gemm_bias_act_f16(A, B, nullptr, C, M, N, K, lda, ldb, ldc,
                           relu ? GEMM_ACT_RELU : GEMM_ACT_NONE, path, stream);
}

int gemm_relu_f16(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K,
                  int64_t lda, int64_t ldb, int64_t ldc, gemm_stream_t stream) {
  return gemm_f16_ex(A, B, C, M, N, K, lda, ldb, ldc, 1, GEMM_PATH_AUTO, stream);
}

int gemm_f16(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K,
             int64_t lda, int64_t ldb, int64_t ldc, gemm_stream_t stream) {
  return gemm_f16_ex(A, B, C, M, N, K, lda, ldb, ldc, 0, GEMM_PATH_AUTO, stream);
}

// The allocation-free entry point: the same validation as gemm_f16_ex, then
// the small-M kernel with the library's fixed scratch array (see the header).
int gemm_relu_f16_noalloc(const void* A, const void* B, void* C, int64_t M, int64_t N,
                          int64_t K, int64_t lda, int64_t ldb, int64_t ldc,
                          gemm_stream_t stream) {
  if (M < 0 || N < 0 || K < 0) return GEMM_ERR_INVALID_ARG;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return GEMM_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return GEMM_OK;
  if (M > 32) return GEMM_ERR_SCRATCH_LIMIT;
  DeviceCtx d;
  int rc = get_device(&d);
  if (rc != GEMM_OK) return rc;
  load_entry_points();
  rc = check_matrix(C, M, N, ldc, d.device);
  if (rc != GEMM_OK) return rc;
  GemmProblem p{A, B, C, M, N, K, lda, ldb, ldc, GEMM_ACT_RELU, nullptr, 0, stream};
  if (K == 0) return launch_zero_fill(p);
  rc = check_matrix(A, M, K, lda, d.device);
  if (rc == GEMM_OK) rc = check_matrix(B, K, N, ldb, d.device);
  if (rc != GEMM_OK) return rc;
  return launch_skinny_gemm_noalloc(p, d);
}

int gemm_activation_f32(const void* x, void* y, int64_t n, int activation,
                        gemm_stream_t stream) {
  if (n < 0 || (activation != GEMM_ACT_NONE && activation != GEMM_ACT_RELU &&
                activation != GEMM_ACT_GELU))
    return GEMM_ERR_INVALID_ARG;
  if (n == 0) return GEMM_OK;
  if (x == nullptr || y == nullptr) return GEMM_ERR_INVALID_ARG;
  DeviceCtx d;
  int rc = get_device(&d);
  if (rc != GEMM_OK) return rc;
  load_entry_points();
  // n floats = n / 2 rows... checked as one row of 2n fp16-sized elements
  if (query_pointer(x, d.device, 1, 2 * n, 2 * n) != 1 ||
      query_pointer(y, d.device, 1, 2 * n, 2 * n) != 1)
    return GEMM_ERR_INVALID_ARG;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  const float* xf = static_cast<const float*>(x);
  float* yf = static_cast<float*>(y);
  const int g = static_cast<int>(blocks);
  if (activation == GEMM_ACT_RELU)
    activation_f32_kernel<kActRelu><<<g, 256, 0, stream>>>(xf, yf, n);
  else if (activation == GEMM_ACT_GELU)
    activation_f32_kernel<kActGelu><<<g, 256, 0, stream>>>(xf, yf, n);
  else
    activation_f32_kernel<kActNone><<<g, 256, 0, stream>>>(xf, yf, n);
  return cudaGetLastError() == cudaSuccess ? GEMM_OK : GEMM_ERR_LAUNCH;
}

int gemm_release(void) {
  int rc = GEMM_OK;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    int prev = 0;
    if (cudaGetDevice(&prev) != cudaSuccess) return GEMM_ERR_LAUNCH;
    uint64_t synced = 0;
    for (const Workspace& w : g_workspaces) {
      if (cudaSetDevice(w.device) != cudaSuccess) {
        rc = GEMM_ERR_LAUNCH;
        continue;
      }
      // the stream the workspace served may be gone: wait for the whole device
      const uint64_t bit = 1ull << (w.device & 63);
      if (!(synced & bit)) {
        if (cudaDeviceSynchronize() != cudaSuccess) rc = GEMM_ERR_LAUNCH;
        synced |= bit;
      }
      if (cudaFree(w.ptr) != cudaSuccess) rc = GEMM_ERR_LAUNCH;
    }
    g_workspaces.clear();
    cudaSetDevice(prev);
  }
  const int h = gemm_host_release();
  return rc != GEMM_OK ? rc : h;
}

int gemm_get_device_status(gemm_stream_t stream, int* device_status) {
  if (device_status == nullptr) return GEMM_ERR_INVALID_ARG;
  DeviceCtx d;
  const int rc = get_device(&d);
  if (rc != GEMM_OK) return rc;
  return read_and_clear_status(d, stream, device_status);
}

int gemm_selftest_wait_timeout(int64_t timeout_ns, gemm_stream_t stream, int* device_status) {
  if (device_status == nullptr || timeout_ns <= 0 || timeout_ns > 10ll * 1000 * 1000 * 1000)
    return GEMM_ERR_INVALID_ARG;
  DeviceCtx d;
  int rc = get_device(&d);
  if (rc != GEMM_OK) return rc;
  wait_probe_kernel<<<1, 32, 0, stream>>>(d.status, static_cast<uint64_t>(timeout_ns));
  if (cudaGetLastError() != cudaSuccess) return GEMM_ERR_LAUNCH;
  return read_and_clear_status(d, stream, device_status);
}

int gemm_read_probe(const void* src, int64_t n_bytes, void* sink, gemm_stream_t stream) {
  if (n_bytes < 0 || (n_bytes & 15) != 0 || sink == nullptr) return GEMM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(src) & 15) != 0 || (reinterpret_cast<uintptr_t>(sink) & 3) != 0)
    return GEMM_ERR_ALIGNMENT;
  DeviceCtx d;
  int rc = get_device(&d);
  if (rc != GEMM_OK) return rc;
  load_entry_points();
  // the sink: one 4-byte word; the source: n_bytes as one row
  if (query_pointer(sink, d.device, 1, 2, 2) != 1) return GEMM_ERR_INVALID_ARG;
  if (n_bytes > 0 && query_pointer(src, d.device, 1, n_bytes / 2, n_bytes / 2) != 1)
    return GEMM_ERR_INVALID_ARG;
  if (cudaMemsetAsync(sink, 0, sizeof(unsigned), stream) != cudaSuccess) return GEMM_ERR_LAUNCH;
  if (n_bytes == 0) return GEMM_OK;
  const int grid = 4 * d.sm_count;  // 4 blocks of 512 threads fill an SM's 2048 threads
  read_probe_kernel<<<grid, 512, 0, stream>>>(static_cast<const uint4*>(src), n_bytes / 16,
                                               static_cast<unsigned*>(sink));
  return cudaGetLastError() == cudaSuccess ? GEMM_OK : GEMM_ERR_LAUNCH;
}

}  // extern "C"
