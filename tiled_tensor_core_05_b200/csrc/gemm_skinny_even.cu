// Small-M (decode-shaped) path with an even share of B per SM, for sm_100a.
//
// The product is bound by streaming B from HBM once (see gemm_skinny.cu for
// the swap-AB formulation: C^T = B^T A^T, 128 columns of B per MMA as its M
// dimension, the few rows of A as its N dimension).  Cutting B's columns into
// equal tiles rarely matches the SM count: 28,672 columns in 256-column
// tiles keep 112 of 148 SMs busy, and 128-column tiles need one and a half
// waves.  This schedule gives each of the P CTAs (one per SM) the same bytes
// instead:
//   * the N columns are U = ceil(N / 64) units of 64; CTA c owns Q = U / P
//     whole units, columns [64 Q c, 64 Q (c + 1)), for the full K, streamed
//     in lock-step with every other CTA as the other small-M kernel does;
//   * the r = U - P Q leftover units are split along K: each gets s =
//     min(P / r, k-blocks) slices, one per CTA, so a CTA adds about K / s to
//     its Q K (for the decode shape: 3 units of 128 k-blocks plus 3 or 4
//     k-blocks of a leftover unit, against 4 units in the 256-column tiling);
//   * a leftover slice writes its fp32 partial (64 columns x MP) to the
//     workspace and bumps its unit's arrival counter; the slice that arrives
//     last sums the s partials in slice order (deterministic) and only then
//     adds the bias, applies the activation and stores fp16.  The leftover
//     slices run first, so that fix-up overlaps the CTA's own main stream.
// This is the split idea of "Writing high-performance kernels in TileLang"
// (atlascloud.ai blog), section "La parte buena: las optimizaciones son de
// una sola línea cada una" (split the reduction when the batch is small),
// used here only for the columns that whole units cannot spread evenly.
//
// MMA windows: the main units sit in ring slabs 0 .. Q-1 (64 columns each).
// The first MMA (M = 128) reads slabs 0-1; with Q = 3 a second one reads
// slabs 1-2 (its lanes 64-127 are columns 128-191), with Q = 4 slabs 2-3.
// With Q = 1, and for a leftover unit (one slab), lanes 64-127 of the
// accumulator read whatever the next slab holds and are never used: each
// accumulator lane depends only on its own row of the A operand.
#include <atomic>

#include "../../include/gemm_f16.h"
#include "internal.h"
#include "skinny_common.cuh"
#include "sm100.cuh"

namespace ttc {
namespace {

using namespace skinny;

constexpr int kSlab = kBK * 64 * 2;  // 64 columns of B by 64 k = 8 KiB

// Dynamic shared memory: 1 KiB of alignment slack, the ring (room for
// max(Q, 2) slabs of B and 8 KiB of A^T per stage), the mbarriers (full and
// empty per stage, leftover-full, accumulator-full, drain, one spare) and the
// TMEM address slot with two flags.
constexpr int even_smem_formula(int q, int stages) {
  return 1024 + stages * ((q < 2 ? 2 : q) * kSlab + 8192) + (2 * stages + 4) * 8 + 16;
}

template <int MP, int STAGES, int Q>
struct EvenCfg {
  static constexpr int kBBytes = (Q < 2 ? 2 : Q) * kSlab;
  static constexpr int kABytes = 8192;
  static constexpr int kStageBytes = kBBytes + kABytes;
  static constexpr int kNumBars = 2 * STAGES + 4;
  static constexpr int kSmemBytes = 1024 + STAGES * kStageBytes + kNumBars * 8 + 16;
  // accumulators: main window 0, main window 1, leftover (MP columns each)
  static constexpr uint32_t kTmemCols = 3 * MP <= 128 ? 128 : 256;
  static_assert(MP == 32 || MP == 64, "MP");
  static_assert(Q >= 1 && Q <= 4, "units per CTA");
  static_assert(kSmemBytes == even_smem_formula(Q, STAGES), "layout");
  static_assert(kSmemBytes <= kMaxDynamicSmem, "shared memory budget");
};

// Compiled: each Q with every ring depth from 4 to 6 that fits the budget.
struct EvenVariant {
  int q;
  int stages;
};
constexpr EvenVariant kEvenVariants[] = {{1, 4}, {1, 5}, {1, 6}, {2, 4}, {2, 5}, {2, 6},
                                         {3, 4}, {3, 5}, {3, 6}, {4, 4}, {4, 5}};
constexpr int kNumEvenVariants = sizeof(kEvenVariants) / sizeof(kEvenVariants[0]);

constexpr bool even_variants_complete() {
  for (int q = 1; q <= 4; ++q) {
    for (int st = 1; st <= 16; ++st) {
      bool built = false;
      for (const auto& v : kEvenVariants) built = built || (v.q == q && v.stages == st);
      const bool wanted = st >= 4 && st <= 6 && even_smem_formula(q, st) <= kMaxDynamicSmem;
      if (wanted != built) return false;
    }
  }
  return true;
}
static_assert(even_variants_complete(), "built even-schedule configurations != the rule");

// One CTA per SM.  blockIdx.x = c: main units [Q c, Q c + Q); leftover item c
// (unit P Q + c / s, slice c % s) when c < r s.
template <int MP, int STAGES, int Q, int ACT>
__global__ void __launch_bounds__(kThreads, 1)
    skinny_even_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, __half* __restrict__ C, int M,
                       int N, int K, int64_t ldc, const __half* __restrict__ bias, int layout,
                       int left_units, int left_slices, float* __restrict__ partials,
                       int* __restrict__ counters, int* status, uint64_t timeout_ns) {
  using Cfg = EvenCfg<MP, STAGES, Q>;
  const bool ta = (layout & kLayoutTransA) != 0;
  const bool tb = (layout & kLayoutTransB) != 0;
  const uint32_t a_bytes = ta ? 8192u : static_cast<uint32_t>(MP * kBK * 2);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* smB = smem;
  uint8_t* smA = smem + STAGES * Cfg::kBBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* left_full = bars + 2 * STAGES;
  uint64_t* acc_full = bars + 2 * STAGES + 1;
  uint64_t* drain = bars + 2 * STAGES + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int P = static_cast<int>(gridDim.x);
  const int cta = static_cast<int>(blockIdx.x);
  const int KB = (K + kBK - 1) / kBK;
  const int main_col = cta * 64 * Q;
  const bool has_left = left_units > 0 && cta < left_units * left_slices;
  int left_unit = 0, left_col = 0, lk0 = 0, lk1 = 0;
  if (has_left) {
    left_unit = cta / left_slices;
    const int slice = cta - left_unit * left_slices;
    lk0 = static_cast<int>(static_cast<int64_t>(slice) * KB / left_slices);
    lk1 = static_cast<int>(static_cast<int64_t>(slice + 1) * KB / left_slices);
    left_col = (P * Q + left_unit) * 64;
  }
  const int n_left = lk1 - lk0;  // >= 1 when has_left (the host keeps s <= KB)
  const int n_steps = n_left + KB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(left_full, 1);
    mbar_init(acc_full, 1);
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
  // the set-up above overlaps the previous kernel of the stream; inputs and
  // outputs are touched only after it has finished
  grid_dependency_trigger();
  grid_dependency_wait();

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer ---
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      bool ok = true;
      const uint64_t pol_b = l2_policy_evict_first();
      const uint64_t pol_a = l2_policy_evict_last();
      for (int i = 0; i < n_steps; ++i) {
        const bool left = i < n_left;
        const int kb = left ? lk0 + i : i - n_left;
        const int slabs = left ? 1 : Q;
        const int col = left ? left_col : main_col;
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, timeout_ns)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(slabs * kSlab) + a_bytes);
        uint8_t* bdst = smB + stage * Cfg::kBBytes;
#pragma unroll
        for (int j = 0; j < Q; ++j) {
          if (j >= slabs) break;
          if (!tb)  // row-major B: 64 columns by 64 k-rows
            tma_load_2d_hint(&tmB, &full[stage], bdst + j * kSlab, col + 64 * j, kb * kBK, pol_b);
          else  // B stored N x K: 64 rows of 64 k
            tma_load_2d_hint(&tmB, &full[stage], bdst + j * kSlab, kb * kBK, col + 64 * j, pol_b);
        }
        if (!ta)  // A stored M x K: MP rows of 64 k
          tma_load_2d_hint(&tmA, &full[stage], smA + stage * Cfg::kABytes, kb * kBK, 0, pol_a);
        else  // A stored K x M: 64 k-rows of 64 m
          tma_load_2d_hint(&tmA, &full[stage], smA + stage * Cfg::kABytes, 0, kb * kBK, pol_a);
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleProducer << 4) | 5);
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
      bool ok = true;
      const uint32_t idesc = idesc_f16_f32(kSub, MP, /*B^T MN-major*/ !tb, /*A^T MN-major*/ ta);
      for (int i = 0; i < n_steps; ++i) {
        const bool left = i < n_left;
        if (!mbar_wait(&full[stage], phase, abort_flag, timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t b_addr = smem_u32(smB + stage * Cfg::kBBytes);
        const uint32_t a_addr = smem_u32(smA + stage * Cfg::kABytes);
        const int step = left ? i : i - n_left;  // k-block index within its accumulator
#pragma unroll
        for (int k = 0; k < kBK / kUmmaK; ++k) {
          const uint32_t accumulate = (step > 0 || k > 0) ? 1u : 0u;
          const uint64_t bdesc = operand_desc(a_addr, k, ta, kSlab);
          const uint64_t w0 = operand_desc(b_addr, k, !tb, kSlab);
          if (left) {
            umma_f16(tmem_base + 2 * MP, w0, bdesc, idesc, accumulate);
          } else {
            umma_f16(tmem_base, w0, bdesc, idesc, accumulate);
            if constexpr (Q > 2) {
              const uint64_t w1 = operand_desc(b_addr + (Q - 2) * kSlab, k, !tb, kSlab);
              umma_f16(tmem_base + MP, w1, bdesc, idesc, accumulate);
            }
          }
        }
        umma_commit(&empty[stage]);
        if (left && i == n_left - 1) umma_commit(left_full);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) {
        umma_commit(acc_full);
      } else {
        raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleMma << 4) | 5);
        umma_commit(drain);
        (void)mbar_wait(drain, 0, nullptr, timeout_ns);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue ---
    const int q = warp & 3;
    const int row = q * 32 + lane;  // TMEM lane = column of B inside an MMA window
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int ok = 1;
    if (has_left) {
      if (lane == 0) ok = mbar_wait(left_full, 0, abort_flag, timeout_ns) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      // the four epilogue warps meet at named barriers below: all continue or
      // all stop
      ok = named_bar_and(1, kEpiWarps * 32, ok);
      if (ok) {
        tc_fence_after_sync();
        float v[MP];
        load_accumulator<MP>(t_lane + 2 * MP, v);
        // partial of this leftover item: [item][64 columns][MP]
        if (row < 64) {
          float* mine = partials + (static_cast<int64_t>(cta) * 64 + row) * MP;
#pragma unroll
          for (int m = 0; m < MP; m += 4)
            *reinterpret_cast<float4*>(mine + m) = make_float4(v[m], v[m + 1], v[m + 2], v[m + 3]);
        }
        __threadfence();
        named_bar_sync(1, kEpiWarps * 32);
        if (threadIdx.x == 64) {
          const int prev = atomicAdd(&counters[left_unit], 1);
          const int is_last = (prev == left_slices - 1) ? 1 : 0;
          if (is_last) atomicExch(&counters[left_unit], 0);  // ready for the next call
          *last_flag = is_last;
        }
        named_bar_sync(1, kEpiWarps * 32);
        if (*last_flag) {
          __threadfence();
          // Sum the unit's s partials in slice order: thread `row` takes
          // column row % 64 and half of the MP rows; the loads of four
          // slices are issued together before they are added (same sums in
          // the same order: same bits).
          constexpr int kHalf = MP / 2;
          const int col = row & 63;
          const int m0 = (row >> 6) * kHalf;
          const float* base = partials + (static_cast<int64_t>(left_unit) * left_slices * 64 + col) * MP + m0;
          float acc[kHalf];
#pragma unroll 1
          for (int s0 = 0; s0 < left_slices; s0 += 4) {
            float4 buf[4][kHalf / 4];
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              if (s0 + g < left_slices) {
                const float* src = base + static_cast<int64_t>(s0 + g) * 64 * MP;
#pragma unroll
                for (int j = 0; j < kHalf / 4; ++j) buf[g][j] = ld_cg_f4(src + 4 * j);
              }
            }
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              if (s0 + g < left_slices) {
#pragma unroll
                for (int j = 0; j < kHalf / 4; ++j) {
                  const float4 f = buf[g][j];
                  if (s0 + g == 0) {
                    acc[4 * j] = f.x;
                    acc[4 * j + 1] = f.y;
                    acc[4 * j + 2] = f.z;
                    acc[4 * j + 3] = f.w;
                  } else {
                    acc[4 * j] += f.x;
                    acc[4 * j + 1] += f.y;
                    acc[4 * j + 2] += f.z;
                    acc[4 * j + 3] += f.w;
                  }
                }
              }
            }
          }
          store_rows<kHalf, ACT>(acc, C, M, N, ldc, left_col + col, m0, bias);
        }
      } else if (lane == 0) {
        raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleEpilogue << 4) | 5);
      }
    }
    if (ok) {
      if (lane == 0) ok = mbar_wait(acc_full, 0, abort_flag, timeout_ns) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0)
          raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleEpilogue << 4) | 6);
      } else {
        tc_fence_after_sync();
        {
          float v[MP];
          load_accumulator<MP>(t_lane, v);  // window 0: columns 0 .. min(64 Q, 128) - 1
          if (row < 64 * Q) store_column<MP, ACT>(v, C, M, N, ldc, main_col + row, bias);
        }
        if constexpr (Q > 2) {
          float v[MP];
          load_accumulator<MP>(t_lane + MP, v);  // window 1: slabs Q-2, Q-1
          if (row >= 256 - 64 * Q)
            store_column<MP, ACT>(v, C, M, N, ldc, main_col + (Q - 2) * 64 + row, bias);
        }
      }
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

template <int MP, int STAGES, int Q, int ACT>
int launch_impl(const GemmProblem& p, const DeviceCtx& d, void* ws, size_t ws_bytes,
                const EvenPlan& plan) {
  using Cfg = EvenCfg<MP, STAGES, Q>;
  static std::atomic<uint64_t> attr_done{0};
  int* counters = nullptr;
  float* partials = nullptr;
  if (plan.left_units > 0) {
    const size_t need = counter_bytes(plan.ctas) + static_cast<size_t>(plan.left_units) *
                                                       plan.left_slices * 64 * MP * sizeof(float);
    if (ws == nullptr || ws_bytes < need) return GEMM_ERR_WORKSPACE;
    counters = static_cast<int*>(ws);
    partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + counter_bytes(plan.ctas));
  }
  CUtensorMap tA, tB;
  int rc;
  if (p.layout & kLayoutTransA)  // stored K x M: 64 k-rows of 64 m (rows >= M read as 0)
    rc = encode_tmap_f16_2d(&tA, p.A, p.M, p.K, p.lda, 64, kBK);
  else  // stored M x K: MP rows of 64 k
    rc = encode_tmap_f16_2d(&tA, p.A, p.K, p.M, p.lda, kBK, MP);
  if (rc != 0) return rc;
  if (p.layout & kLayoutTransB)  // stored N x K: 64 rows of 64 k
    rc = encode_tmap_f16_2d(&tB, p.B, p.K, p.N, p.ldb, kBK, 64);
  else  // row-major: 64 columns by 64 k-rows
    rc = encode_tmap_f16_2d(&tB, p.B, p.N, p.K, p.ldb, 64, kBK);
  if (rc != 0) return rc;
  auto kern = skinny_even_kernel<MP, STAGES, Q, ACT>;
  if (!ensure_smem_attr(reinterpret_cast<const void*>(kern), Cfg::kSmemBytes, d.device,
                        attr_done))
    return GEMM_ERR_LAUNCH;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(plan.ctas), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = p.stream;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_attribute(&attr[0]);
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, kern, tA, tB, static_cast<__half*>(p.C), static_cast<int>(p.M),
      static_cast<int>(p.N), static_cast<int>(p.K), p.ldc, static_cast<const __half*>(p.bias),
      p.layout, plan.left_units, plan.left_slices, partials, counters, d.status, d.timeout_ns);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? GEMM_OK : GEMM_ERR_LAUNCH;
}

template <int MP, int STAGES, int Q>
int launch_act(const GemmProblem& p, const DeviceCtx& d, void* ws, size_t ws_bytes,
               const EvenPlan& plan) {
  switch (p.act) {
    case kActRelu: return launch_impl<MP, STAGES, Q, kActRelu>(p, d, ws, ws_bytes, plan);
    case kActGelu: return launch_impl<MP, STAGES, Q, kActGelu>(p, d, ws, ws_bytes, plan);
    default: return launch_impl<MP, STAGES, Q, kActNone>(p, d, ws, ws_bytes, plan);
  }
}

template <int MP, int I = 0>
int dispatch_variant(const GemmProblem& p, const DeviceCtx& d, void* ws, size_t ws_bytes,
                     const EvenPlan& plan, int stages) {
  if constexpr (I == kNumEvenVariants) {
    return GEMM_ERR_CONFIG;
  } else {
    constexpr EvenVariant v = kEvenVariants[I];
    if (plan.q == v.q && stages == v.stages)
      return launch_act<MP, v.stages, v.q>(p, d, ws, ws_bytes, plan);
    return dispatch_variant<MP, I + 1>(p, d, ws, ws_bytes, plan, stages);
  }
}

}  // namespace

EvenPlan even_plan(int64_t N, int64_t K, int sm_count) {
  EvenPlan plan{};
  const int64_t U = (N + 63) / 64;
  const int64_t KB = (K + kBK - 1) / kBK;
  const int64_t q = sm_count > 0 ? U / sm_count : 0;
  if (q < 1 || q > 4 || KB < 1) return plan;  // q = 0: not valid
  const int64_t r = U - q * sm_count;
  int64_t s = 0;
  if (r > 0) {
    s = sm_count / r;
    if (s > KB) s = KB;
  }
  plan.q = static_cast<int>(q);
  plan.ctas = sm_count;
  plan.left_units = static_cast<int>(r);
  plan.left_slices = static_cast<int>(s);
  // k-blocks of 64 columns that the busiest CTA streams
  plan.work = q * KB + (r > 0 ? (KB + s - 1) / s : 0);
  return plan;
}

size_t even_workspace_bytes(const EvenPlan& plan, int m_pad) {
  if (plan.left_units == 0) return 0;
  return counter_bytes(plan.ctas) +
         static_cast<size_t>(plan.left_units) * plan.left_slices * 64 * m_pad * sizeof(float);
}

int launch_skinny_even(const GemmProblem& p, const DeviceCtx& d, void* ws, size_t ws_bytes,
                       const KernelConfig& c) {
  const EvenPlan plan = even_plan(p.N, p.K, d.sm_count);
  if (plan.q == 0 || 64 * plan.q != c.block_n || c.splits != 0) return GEMM_ERR_CONFIG;
  const int mp = skinny_m_pad(p.M);
  if (mp == 32) return dispatch_variant<32>(p, d, ws, ws_bytes, plan, c.stages);
  if (mp == 64) return dispatch_variant<64>(p, d, ws, ws_bytes, plan, c.stages);
  return GEMM_ERR_INVALID_ARG;
}

int even_config_smem_bytes(int block_n, int stages) {
  if (stages < 1 || stages > 64 || block_n % 64 != 0 || block_n < 64 || block_n > 256)
    return -1;
  return even_smem_formula(block_n / 64, stages);
}

int even_configs_built(KernelConfig* out, int cap) {
  for (int i = 0; i < kNumEvenVariants && i < cap; ++i)
    out[i] = KernelConfig{GEMM_PATH_SKINNY_EVEN, 64 * kEvenVariants[i].q,
                          kEvenVariants[i].stages, 0, 0};
  return kNumEvenVariants;
}

}  // namespace ttc
