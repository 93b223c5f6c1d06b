// Small-M (decode-shaped) path of C = ReLU(A @ B) for sm_100a.
//
// With few rows in A the product is bound by reading B from HBM, and one
// output tile per CTA leaves most SMs idle.  "Writing high-performance kernels
// in TileLang" (atlascloud.ai blog), section "La parte buena: las
// optimizaciones son de una sola línea cada una", answers that case for
// attention decode by splitting the reduction axis across SMs and merging the
// pieces afterwards (split-KV / FlashDecoding).  The same idea is applied here
// to the K axis of the GEMM:
//
//   * swap-AB: the kernel computes C^T = B^T A^T, so a 128-wide slab of B's
//     columns is the MMA M dimension (B^T is MN-major in shared memory, read
//     straight from row-major B) and the few rows of A are the MMA N
//     dimension (MP = M rounded up to 32 or 64; A^T is K-major);
//   * stream-K: the (N-tile, 64-deep k-block) units are split evenly over a
//     persistent grid, so every SM streams the same number of bytes of B;
//   * a CTA that covers a whole tile applies ReLU and stores it; one that
//     covers part of a tile writes its fp32 partial tile to a workspace and
//     bumps the tile's arrival counter.  Whichever contributor arrives last
//     sums all partials in a fixed order (by contributor index), then applies
//     ReLU only after the full K reduction and stores fp16.  No CTA ever waits
//     for another one, and the result does not depend on arrival order.
#include <atomic>
#include <mutex>

#include "../../include/gemm_f16.h"
#include "internal.h"
#include "sm100.cuh"

namespace ttc {
namespace {

constexpr int kTN = 128;       // columns of B per tile (MMA M)
constexpr int kBK = 64;        // k-block
constexpr int kUmmaK = 16;
constexpr int kThreads = 192;  // producer, MMA, 4 epilogue warps
constexpr int kEpiWarps = 4;

template <int MP, int STAGES>
struct SkCfg {
  static constexpr int kBBytes = kBK * kTN * 2;    // 16 KiB: two 64-column slabs
  static constexpr int kBChunk = kBK * 64 * 2;     // 8 KiB
  static constexpr int kABytes = MP * kBK * 2;     // MP rows x 128 bytes
  static constexpr int kStageBytes = kBBytes + kABytes;
  static constexpr int kNumBars = 2 * STAGES + 5;
  static constexpr int kSmemBytes = 1024 + STAGES * kStageBytes + kNumBars * 8 + 16;
  static constexpr uint32_t kTmemCols = (2 * MP < 32) ? 32 : 2 * MP;
  static constexpr uint32_t kIdesc = idesc_f16_f32(kTN, MP, /*A MN-major*/ true,
                                                   /*B MN-major*/ false);
  static_assert(MP == 32 || MP == 64, "MP");
  static_assert(kABytes % 1024 == 0, "A tile alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Unit range [begin(c), begin(c+1)) of CTA c when `total` units are split
// over G CTAs as evenly as possible.
__host__ __device__ __forceinline__ int64_t sk_begin(int64_t c, int64_t total, int64_t G) {
  return c * total / G;
}

// The CTA whose range contains unit u.
__device__ __forceinline__ int sk_owner(int64_t u, int64_t total, int G) {
  int c = static_cast<int>((u * G) / total);
  while (c + 1 < G && sk_begin(c + 1, total, G) <= u) ++c;
  return c;
}

// End (exclusive) of a CTA's k-range inside a tile: the tile's end or the
// end of the CTA's units, whichever comes first.
__device__ __forceinline__ int seg_end(int KB, int kb0, int64_t left) {
  const int64_t e = kb0 + left;
  return e < KB ? static_cast<int>(e) : KB;
}

__device__ __forceinline__ float4 ld_cg_f4(const float* p) {
  return __ldcg(reinterpret_cast<const float4*>(p));
}

template <int MP, bool RELU>
__device__ __forceinline__ void store_column(const float (&v)[MP], __half* C, int M, int N,
                                             int64_t ldc, int n) {
  if (n >= N) return;
#pragma unroll
  for (int m = 0; m < MP; ++m) {
    if (m < M) {
      const float x = RELU ? relu_f32(v[m]) : v[m];
      C[static_cast<int64_t>(m) * ldc + n] = __float2half_rn(x);
    }
  }
}

template <int MP, int STAGES, bool RELU>
__global__ void __launch_bounds__(kThreads, 1)
    streamk_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, __half* __restrict__ C, int M,
                        int N, int K, int64_t ldc, float* __restrict__ partials,
                        int* __restrict__ counters, int* status, uint64_t timeout_ns) {
  using Cfg = SkCfg<MP, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* smB = smem;
  uint8_t* smA = smem + STAGES * Cfg::kBBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = bars + 2 * STAGES + 2;
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int cta = blockIdx.x;
  const int KB = (K + kBK - 1) / kBK;
  const int T = (N + kTN - 1) / kTN;
  const int64_t total = static_cast<int64_t>(T) * KB;
  const int64_t ub = sk_begin(cta, total, G);
  const int64_t ue = sk_begin(cta + 1, total, G);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish_alloc_permit();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer ---
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      bool ok = true;
      for (int64_t u = ub; u < ue && ok;) {
        const int t = static_cast<int>(u / KB);
        const int kb0 = static_cast<int>(u - static_cast<int64_t>(t) * KB);
        const int kb1 = seg_end(KB, kb0, ue - u);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], Cfg::kStageBytes);
          uint8_t* bdst = smB + stage * Cfg::kBBytes;
          tma_load_2d(&tmB, &full[stage], bdst, t * kTN, kb * kBK);
          tma_load_2d(&tmB, &full[stage], bdst + Cfg::kBChunk, t * kTN + 64, kb * kBK);
          tma_load_2d(&tmA, &full[stage], smA + stage * Cfg::kABytes, kb * kBK, 0);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        u += kb1 - kb0;
      }
      if (!ok) {
        raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleProducer << 4) | 2);
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s))
            (void)mbar_wait(&full[s], (armed_parity >> s) & 1u, nullptr, timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer ---
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      int site = 0;
      for (int64_t u = ub; u < ue && ok;) {
        const int t = static_cast<int>(u / KB);
        const int kb0 = static_cast<int>(u - static_cast<int64_t>(t) * KB);
        const int kb1 = seg_end(KB, kb0, ue - u);
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag, timeout_ns)) {
          ok = false;
          site = 3;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * MP);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, timeout_ns)) {
            ok = false;
            site = 4;
            break;
          }
          tc_fence_after_sync();
          const uint32_t b_addr = smem_u32(smB + stage * Cfg::kBBytes);
          const uint32_t a_addr = smem_u32(smA + stage * Cfg::kABytes);
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k) {
            // MMA A operand = B^T tile (N-major): advance 16 k-rows of 128 bytes
            const uint64_t adesc =
                smem_desc_sw128(b_addr + k * (kUmmaK * 128), Cfg::kBChunk, 1024);
            // MMA B operand = A^T tile (K-major): advance 32 bytes along the row
            const uint64_t bdesc = smem_desc_sw128(a_addr + k * (kUmmaK * 2), 16, 1024);
            umma_f16(d_tmem, adesc, bdesc, Cfg::kIdesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
        u += kb1 - kb0;
      }
      if (!ok) {
        raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleMma << 4) | site);
        umma_commit(drain);
        (void)mbar_wait(drain, 0, nullptr, timeout_ns);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue ---
    const int q = warp & 3;
    const int row = q * 32 + lane;  // column of C inside the tile
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t u = ub; u < ue;) {
      const int t = static_cast<int>(u / KB);
      const int kb0 = static_cast<int>(u - static_cast<int64_t>(t) * KB);
      const int kb1 = seg_end(KB, kb0, ue - u);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&acc_full[acc], acc_phase, abort_flag, timeout_ns) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      // the four epilogue warps meet at named barriers below: they must all
      // continue or all stop
      ok = named_bar_and(1, kEpiWarps * 32, ok);
      if (!ok) {
        if (lane == 0)
          raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleEpilogue << 4) | 2);
        break;
      }
      tc_fence_after_sync();
      float v[MP];
      {
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>(acc * MP);
#pragma unroll
        for (int j = 0; j < MP / 32; ++j) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(taddr + j * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[j * 32 + i] = __uint_as_float(r[i]);
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);

      const int n = t * kTN + row;
      if (kb0 == 0 && kb1 == KB) {
        store_column<MP, RELU>(v, C, M, N, ldc, n);  // this CTA covered the whole tile
      } else {
        // partial tile: slot 0 = this CTA's first tile, slot 1 = its last
        const int slot = (u == ub) ? 0 : 1;
        float* dst = partials + ((static_cast<int64_t>(cta) * 2 + slot) * kTN + row) * MP;
#pragma unroll
        for (int m = 0; m < MP; m += 4)
          *reinterpret_cast<float4*>(dst + m) = make_float4(v[m], v[m + 1], v[m + 2], v[m + 3]);
        __threadfence();
        named_bar_sync(1, kEpiWarps * 32);
        const int c_first = sk_owner(static_cast<int64_t>(t) * KB, total, G);
        const int c_last = sk_owner(static_cast<int64_t>(t) * KB + KB - 1, total, G);
        if (threadIdx.x == 64) {
          const int prev = atomicAdd(&counters[c_first], 1);
          const int is_last = (prev == c_last - c_first) ? 1 : 0;
          if (is_last) atomicExch(&counters[c_first], 0);  // ready for the next call
          *last_flag = is_last;
        }
        named_bar_sync(1, kEpiWarps * 32);
        const int is_last = *last_flag;
        named_bar_sync(1, kEpiWarps * 32);  // everyone has read the flag
        if (is_last) {
          __threadfence();
          float s[MP];
          for (int cc = c_first; cc <= c_last; ++cc) {
            if (cc == cta) {
#pragma unroll
              for (int m = 0; m < MP; ++m) s[m] = (cc == c_first) ? v[m] : s[m] + v[m];
            } else {
              const int first_tile_cc = static_cast<int>(sk_begin(cc, total, G) / KB);
              const int slot_cc = (t == first_tile_cc) ? 0 : 1;
              const float* src =
                  partials + ((static_cast<int64_t>(cc) * 2 + slot_cc) * kTN + row) * MP;
#pragma unroll
              for (int m = 0; m < MP; m += 4) {
                const float4 p = ld_cg_f4(src + m);
                if (cc == c_first) {
                  s[m] = p.x; s[m + 1] = p.y; s[m + 2] = p.z; s[m + 3] = p.w;
                } else {
                  s[m] += p.x; s[m + 1] += p.y; s[m + 2] += p.z; s[m + 3] += p.w;
                }
              }
            }
          }
          store_column<MP, RELU>(s, C, M, N, ldc, n);
        }
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
      u += kb1 - kb0;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

bool ensure_smem_attr_sk(const void* func, int bytes, int device, std::atomic<uint64_t>& done) {
  const uint64_t bit = 1ull << (device & 63);
  if (done.load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  done.fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

constexpr size_t kCounterBytes(int sm_count) {
  return (static_cast<size_t>(sm_count) * sizeof(int) + 255) & ~static_cast<size_t>(255);
}

template <int MP, int STAGES, bool RELU>
int launch_impl(const GemmProblem& p, const DeviceCtx& d, void* ws, size_t ws_bytes) {
  using Cfg = SkCfg<MP, STAGES>;
  static std::atomic<uint64_t> attr_done{0};
  const int64_t KB = (p.K + kBK - 1) / kBK;
  const int64_t T = (p.N + kTN - 1) / kTN;
  const int64_t total = KB * T;
  const int grid = static_cast<int>(total < d.sm_count ? total : d.sm_count);
  if (ws_bytes < kCounterBytes(d.sm_count) +
                     static_cast<size_t>(grid) * 2 * kTN * MP * sizeof(float))
    return GEMM_ERR_WORKSPACE;
  CUtensorMap tA, tB;
  int rc = encode_tmap_f16_2d(&tA, p.A, p.K, p.M, p.lda, kBK, MP);
  if (rc == 0) rc = encode_tmap_f16_2d(&tB, p.B, p.N, p.K, p.ldb, 64, kBK);
  if (rc != 0) return rc;
  auto kern = streamk_gemm_kernel<MP, STAGES, RELU>;
  if (!ensure_smem_attr_sk(reinterpret_cast<const void*>(kern), Cfg::kSmemBytes, d.device,
                           attr_done))
    return GEMM_ERR_LAUNCH;
  // the counter region is sized for the whole GPU so that calls with
  // different grids never see each other's partials in it
  int* counters = static_cast<int*>(ws);
  float* partials =
      reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kCounterBytes(d.sm_count));
  kern<<<grid, kThreads, Cfg::kSmemBytes, p.stream>>>(
      tA, tB, static_cast<__half*>(p.C), static_cast<int>(p.M), static_cast<int>(p.N),
      static_cast<int>(p.K), p.ldc, partials, counters, d.status, d.timeout_ns);
  return cudaGetLastError() == cudaSuccess ? 0 : GEMM_ERR_LAUNCH;
}

}  // namespace

int streamk_m_pad(int64_t M) {
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  return 0;
}

size_t streamk_workspace_bytes(int sm_count, int m_pad) {
  return kCounterBytes(sm_count) +
         static_cast<size_t>(sm_count) * 2 * kTN * static_cast<size_t>(m_pad) * sizeof(float);
}

int launch_streamk_gemm(const GemmProblem& p, const DeviceCtx& d, void* ws, size_t ws_bytes) {
  const int mp = streamk_m_pad(p.M);
  if (mp == 32)
    return p.relu ? launch_impl<32, 10, true>(p, d, ws, ws_bytes)
                  : launch_impl<32, 10, false>(p, d, ws, ws_bytes);
  if (mp == 64)
    return p.relu ? launch_impl<64, 8, true>(p, d, ws, ws_bytes)
                  : launch_impl<64, 8, false>(p, d, ws, ws_bytes);
  return GEMM_ERR_INVALID_ARG;
}

// ------------------------------------------------ allocation-free variant ---
// Scratch of gemm_relu_f16_noalloc: the same layout as the lazily allocated
// workspace (arrival counters, then two fp32 partial tiles per CTA), sized
// for M <= 32 (MMA N = 32) and at most kNoAllocMaxCtas CTAs.  It is part of
// the library image, so every GPU that loads the library holds it.
namespace {

constexpr int kNoAllocMP = 32;
constexpr int kNoAllocMaxCtas = 160;
constexpr size_t kNoAllocCounterBytes = kCounterBytes(kNoAllocMaxCtas);
constexpr size_t kNoAllocScratchBytes =
    kNoAllocCounterBytes +
    static_cast<size_t>(kNoAllocMaxCtas) * 2 * kTN * kNoAllocMP * sizeof(float);
static_assert(kNoAllocScratchBytes == 5243648, "documented scratch size");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_addr[64] = {};  // device address of g_noalloc_scratch, per device

// Host code cannot use the array's name as a device address (it names a host
// stand-in); look the real address up once per device, with it current.
int noalloc_scratch_address(int device, void** out) {
  if (device < 0 || device >= 64) return GEMM_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_addr[device] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return GEMM_ERR_LAUNCH;
    }
    g_noalloc_addr[device] = p;
  }
  *out = g_noalloc_addr[device];
  return GEMM_OK;
}

}  // namespace

int launch_streamk_gemm_noalloc(const GemmProblem& p, const DeviceCtx& d) {
  if (p.M > kNoAllocMP) return GEMM_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  int rc = noalloc_scratch_address(d.device, &scratch);
  if (rc != GEMM_OK) return rc;
  using Cfg = SkCfg<kNoAllocMP, 10>;
  static std::atomic<uint64_t> attr_done{0};
  const int64_t KB = (p.K + kBK - 1) / kBK;
  const int64_t T = (p.N + kTN - 1) / kTN;
  const int64_t total = KB * T;
  int64_t grid = total < d.sm_count ? total : d.sm_count;
  if (grid > kNoAllocMaxCtas) grid = kNoAllocMaxCtas;
  CUtensorMap tA, tB;
  rc = encode_tmap_f16_2d(&tA, p.A, p.K, p.M, p.lda, kBK, kNoAllocMP);
  if (rc == 0) rc = encode_tmap_f16_2d(&tB, p.B, p.N, p.K, p.ldb, 64, kBK);
  if (rc != 0) return rc;
  auto kern = streamk_gemm_kernel<kNoAllocMP, 10, true>;
  if (!ensure_smem_attr_sk(reinterpret_cast<const void*>(kern), Cfg::kSmemBytes, d.device,
                           attr_done))
    return GEMM_ERR_LAUNCH;
  // the array keeps the previous call's contents: the arrival counters must
  // start at zero (the partial tiles are always written before being read)
  if (cudaMemsetAsync(scratch, 0, kNoAllocCounterBytes, p.stream) != cudaSuccess)
    return GEMM_ERR_LAUNCH;
  int* counters = static_cast<int*>(scratch);
  float* partials =
      reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + kNoAllocCounterBytes);
  kern<<<static_cast<int>(grid), kThreads, Cfg::kSmemBytes, p.stream>>>(
      tA, tB, static_cast<__half*>(p.C), static_cast<int>(p.M), static_cast<int>(p.N),
      static_cast<int>(p.K), p.ldc, partials, counters, d.status, d.timeout_ns);
  return cudaGetLastError() == cudaSuccess ? GEMM_OK : GEMM_ERR_LAUNCH;
}

}  // namespace ttc
