// Small-M (decode-shaped) path of C = ReLU(A @ B) for sm_100a.
//
// With few rows in A the product is bound by reading B from HBM once; the
// tensor cores are nearly idle and what matters is how fast, and in which
// order, B streams in.
//
//   * swap-AB: the kernel computes C^T = B^T A^T, so a 128-wide slab of B's
//     columns is the MMA M dimension (B^T is MN-major in shared memory, read
//     straight from row-major B) and the few rows of A are the MMA N
//     dimension (MP = M rounded up to 32 or 64; A^T is K-major).  One CTA owns
//     a TW-column tile of C^T (TW = 256: two MMAs per 16-deep k step into two
//     TMEM accumulators; TW = 128, for problems with few column tiles: one).
//   * lock-step streaming: every CTA walks its k-range upward from the same
//     start at the same time, so at any moment the whole grid reads the same
//     band of rows of B across all N.  Row-major B then streams in long
//     contiguous runs, which HBM serves far better than the scattered k
//     offsets of a stream-K split (measured: 5.3 TB/s with stream-K over
//     148 SMs, 6.8+ TB/s in lock-step over 112 SMs for M=32, N=28672,
//     K=8192).
//   * split-K only when there are fewer tiles than SMs: the k range of each
//     tile is cut into S equal slices (one CTA each) -- the split-KV /
//     FlashDecoding idea of "Writing high-performance kernels in TileLang"
//     (atlascloud.ai blog), section "La parte buena: las optimizaciones son
//     de una sola línea cada una", applied to the K axis of the GEMM.  Each
//     slice writes its fp32 partial tile to a workspace and bumps the tile's
//     arrival counter; whichever slice arrives last sums the S partials in
//     slice order (deterministic), then applies the bias and activation --
//     only after the full K reduction -- and stores fp16.  No CTA ever waits
//     for another.
#include <atomic>
#include <mutex>

#include "../../include/gemm_f16.h"
#include "internal.h"
#include "skinny_common.cuh"
#include "sm100.cuh"

namespace ttc {
namespace {

using namespace skinny;
constexpr int kMaxTW = 256;    // widest tile: columns of B (rows of C^T) per CTA

// Dynamic shared memory of the small-M kernel with `tw` columns of B per CTA:
// 1 KiB of alignment slack, the ring (tw columns of B and room for A^T per
// stage), the mbarriers (full and empty per stage, accumulator-full, drain,
// one spare) and the TMEM address slot.  A^T takes 8 KiB per stage for
// either MP.
constexpr int skinny_smem_formula(int tw, int stages) {
  return 1024 + stages * (tw / 64 * kBK * 64 * 2 + 8192) + (2 * stages + 3) * 8 + 16;
}

// TW = 256 (two MMAs of M = 128 per 16-deep step) or 128 (one): narrower
// tiles give twice the CTAs where there are few column tiles.
template <int MP, int STAGES, int TW>
struct SkinnyCfg {
  static constexpr int kBChunk = kBK * 64 * 2;    // 64 columns x 64 k-rows = 8 KiB
  static constexpr int kBBytes = TW / 64 * kBChunk;  // TW columns
  // A^T: MP rows x 128 bytes (A stored M x K), or one 64-column slab of 64
  // k-rows (A stored K x M): room for the larger
  static constexpr int kABytesK = MP * kBK * 2;
  static constexpr int kABytes = kABytesK > 8192 ? kABytesK : 8192;
  static constexpr int kStageBytes = kBBytes + kABytes;
  static constexpr int kNumBars = 2 * STAGES + 3;
  static constexpr int kSmemBytes = 1024 + STAGES * kStageBytes + kNumBars * 8 + 16;
  static constexpr uint32_t kTmemCols = (TW / kSub * MP < 32) ? 32 : TW / kSub * MP;
  static_assert(MP == 32 || MP == 64, "MP");
  static_assert(TW == 128 || TW == 256, "tile width");
  static_assert(kABytes % 1024 == 0, "A tile alignment");
  static_assert(kSmemBytes == skinny_smem_formula(TW, STAGES), "layout");
  static_assert(kSmemBytes <= kMaxDynamicSmem, "shared memory budget");
};

// Configurations compiled (for MP 32 and 64 and every activation): each tile
// width with every ring depth from 3 up to what fits the shared-memory budget
// or 6, whichever is lower (a streaming ring gains nothing deeper: 6 stages of
// the narrow tile already keep 144 KiB in flight per SM).
struct SkinnyVariant {
  int tw;
  int stages;
};
constexpr SkinnyVariant kSkinnyVariants[] = {{256, 3}, {256, 4}, {256, 5}, {128, 3},
                                             {128, 4}, {128, 5}, {128, 6}};
constexpr int kNumSkinnyVariants = sizeof(kSkinnyVariants) / sizeof(kSkinnyVariants[0]);
constexpr int kMaxSkinnyStages = 6;

constexpr bool skinny_variants_complete() {
  for (int tw : {128, 256}) {
    for (int st = 3; st <= 16; ++st) {
      bool built = false;
      for (const auto& v : kSkinnyVariants) built = built || (v.tw == tw && v.stages == st);
      const bool wanted = skinny_smem_formula(tw, st) <= kMaxDynamicSmem && st <= kMaxSkinnyStages;
      if (wanted != built) return false;
    }
  }
  return true;
}
static_assert(skinny_variants_complete(),
              "built skinny configurations != those within the budget and depth cap");

// One CTA per (tile, k-slice); blockIdx.x = tile * S + slice.  B (streamed
// once) is loaded with an L2 evict-first policy and A (re-read by every CTA)
// with evict-last.
template <int MP, int STAGES, int TW, int ACT>
__global__ void __launch_bounds__(kThreads, 1)
    skinny_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, __half* __restrict__ C, int M,
                       int N, int K, int64_t ldc, const __half* __restrict__ bias, int S,
                       int layout, float* __restrict__ partials, int* __restrict__ counters,
                       const __half* __restrict__ Bg, int64_t ldb, int* status,
                       uint64_t timeout_ns) {
  using Cfg = SkinnyCfg<MP, STAGES, TW>;
  const bool ta = (layout & kLayoutTransA) != 0;
  const bool tb = (layout & kLayoutTransB) != 0;
  // bytes of one stage: TW columns of B, and A^T as stored
  const uint32_t stage_bytes = Cfg::kBBytes + (ta ? 8192u : static_cast<uint32_t>(Cfg::kABytesK));
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* smB = smem;
  uint8_t* smA = smem + STAGES * Cfg::kBBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* drain = bars + 2 * STAGES + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile = blockIdx.x / S;
  const int slice = blockIdx.x - tile * S;
  const int KB = (K + kBK - 1) / kBK;
  const int kb_begin = static_cast<int>(static_cast<int64_t>(slice) * KB / S);
  const int kb_end = static_cast<int>(static_cast<int64_t>(slice + 1) * KB / S);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
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
  {
    // Warm L2 with this CTA's first ring of B while the previous kernel of
    // the stream finishes (0.9-1.3 us of a 69 us decode launch): an L2
    // prefetch only moves lines into L2, the point of coherence that the
    // loads below read after the wait, so it cannot observe a value the
    // previous kernel has yet to write.
    const int kb_stop = min(kb_end, kb_begin + STAGES);
    if (!tb) {  // row-major B: TW columns (TW / 64 lines of 128 bytes) per k-row
      constexpr int kLines = TW / 64;
      const int total = (kb_stop - kb_begin) * kBK * kLines;
      for (int i = threadIdx.x; i < total; i += kThreads) {
        const int r = kb_begin * kBK + i / kLines;
        const int c = tile * TW + (i % kLines) * 64;
        if (r < K && c < N) prefetch_l2(Bg + static_cast<int64_t>(r) * ldb + c);
      }
    } else {  // B stored N x K: a run of the ring's k per row of the tile
      const int lines = ((kb_stop - kb_begin) * kBK * 2 + 127) / 128;
      const int total = TW * lines;
      for (int i = threadIdx.x; i < total; i += kThreads) {
        const int n = tile * TW + i / lines;
        const int k = kb_begin * kBK + (i % lines) * 64;
        if (n < N && k < K) prefetch_l2(Bg + static_cast<int64_t>(n) * ldb + k);
      }
    }
  }
  grid_dependency_wait();

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer ---
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      bool ok = true;
      const uint64_t pol_b = l2_policy_evict_first();
      const uint64_t pol_a = l2_policy_evict_last();
      for (int kb = kb_begin; kb < kb_end; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, timeout_ns)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], stage_bytes);
        uint8_t* bdst = smB + stage * Cfg::kBBytes;
        if (!tb) {  // row-major B: TW / 64 slabs of 64 columns by 64 k-rows
#pragma unroll
          for (int j = 0; j < TW / 64; ++j)
            tma_load_2d_hint(&tmB, &full[stage], bdst + j * Cfg::kBChunk, tile * TW + j * 64,
                             kb * kBK, pol_b);
        } else {  // B stored N x K: TW rows of 64 k
          tma_load_2d_hint(&tmB, &full[stage], bdst, kb * kBK, tile * TW, pol_b);
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
      bool ok = true;
      const uint32_t idesc = idesc_f16_f32(kSub, MP, /*B^T MN-major*/ !tb, /*A^T MN-major*/ ta);
      for (int kb = kb_begin; kb < kb_end; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag, timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t b_addr = smem_u32(smB + stage * Cfg::kBBytes);
        const uint32_t a_addr = smem_u32(smA + stage * Cfg::kABytes);
#pragma unroll
        for (int k = 0; k < kBK / kUmmaK; ++k) {
          // MMA B operand = A^T tile (K-major): 32 bytes per 16 k along the row
          // (A^T is K-major when A is stored M x K, MN-major when stored K x M)
          const uint64_t bdesc = operand_desc(a_addr, k, ta, Cfg::kBChunk);
#pragma unroll
          for (int h = 0; h < TW / kSub; ++h) {
            // MMA A operand = B^T sub-tile h (columns 128h..128h+127 of the
            // tile; 16 KiB into the stage in both layouts): N-major slabs of
            // row-major B, or K-major rows of B stored N x K
            const uint64_t adesc = operand_desc(b_addr + h * 2 * Cfg::kBChunk, k, !tb,
                                                Cfg::kBChunk);
            umma_f16(tmem_base + static_cast<uint32_t>(h * MP), adesc, bdesc, idesc,
                     (kb > kb_begin || k > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) {
        umma_commit(acc_full);
      } else {
        raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleMma << 4) | 4);
        umma_commit(drain);
        (void)mbar_wait(drain, 0, nullptr, timeout_ns);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue ---
    const int q = warp & 3;
    const int row = q * 32 + lane;  // TMEM lane = column of C inside each 128-wide half
    int ok = 1;
    if (lane == 0) ok = mbar_wait(acc_full, 0, abort_flag, timeout_ns) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    // the four epilogue warps meet at named barriers below: all continue or
    // all stop
    ok = named_bar_and(1, kEpiWarps * 32, ok);
    if (!ok) {
      if (lane == 0)
        raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleEpilogue << 4) | 2);
    } else {
      tc_fence_after_sync();
      const int n0 = tile * TW + row;
      const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      // one 128-column half at a time keeps only MP accumulators per thread live
      if (S == 1) {
        // The tile of C (MP rows x TW columns, fp16, row-major) is staged in
        // the ring's first B slot -- every stage has been read by the MMAs
        // once acc_full has completed -- and written out as 16-byte pieces of
        // whole rows; storing each thread's column element by element took
        // about 1.4 us of a 69 us decode launch.
        __half* tile_c = reinterpret_cast<__half*>(smB);
        static_assert(MP * TW * 2 <= Cfg::kBBytes, "staging fits one B slot");
#pragma unroll 1
        for (int h = 0; h < TW / kSub; ++h) {
          float v[MP];
          load_accumulator<MP>(t_lane + static_cast<uint32_t>(h * MP), v);
          stage_column<MP, ACT>(v, tile_c, TW, h * kSub + row, N, n0 + h * kSub, bias);
        }
        named_bar_sync(1, kEpiWarps * 32);
        store_staged_rows<MP, TW>(tile_c, C, M, N, ldc, tile * TW, threadIdx.x - 64,
                                  kEpiWarps * 32);
      } else {
        // partial tile of this slice: [item][TW columns][MP]
#pragma unroll 1
        for (int h = 0; h < TW / kSub; ++h) {
          float v[MP];
          load_accumulator<MP>(t_lane + static_cast<uint32_t>(h * MP), v);
          float* mine =
              partials + (static_cast<int64_t>(blockIdx.x) * TW + h * kSub + row) * MP;
#pragma unroll
          for (int m = 0; m < MP; m += 4)
            *reinterpret_cast<float4*>(mine + m) = make_float4(v[m], v[m + 1], v[m + 2], v[m + 3]);
        }
        __threadfence();
        named_bar_sync(1, kEpiWarps * 32);
        if (threadIdx.x == 64) {
          const int prev = atomicAdd(&counters[tile], 1);
          const int is_last = (prev == S - 1) ? 1 : 0;
          if (is_last) atomicExch(&counters[tile], 0);  // ready for the next call
          *last_flag = is_last;
        }
        named_bar_sync(1, kEpiWarps * 32);
        if (*last_flag) {
          __threadfence();
          // Sum the S partial tiles in slice order, 32 rows of C at a time;
          // the loads of four slices are issued together before they are
          // added, so the fix-up costs one L2 round trip per four slices
          // rather than per slice (same sums in the same order: same bits).
          // This slice's own partial is read back from TMEM at its turn.
          const int64_t slice_stride = static_cast<int64_t>(TW) * MP;
#pragma unroll 1
          for (int h = 0; h < TW / kSub; ++h) {
            const float* base =
                partials + ((static_cast<int64_t>(tile) * S) * TW + h * kSub + row) * MP;
#pragma unroll 1
            for (int mc = 0; mc < MP / 32; ++mc) {
              float acc[32];
#pragma unroll 1
              for (int s0 = 0; s0 < S; s0 += 4) {
                float4 buf[4][8];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                  const int sl = s0 + g;
                  if (sl < S && sl != slice) {
                    const float* src = base + sl * slice_stride + mc * 32;
#pragma unroll
                    for (int q = 0; q < 8; ++q) buf[g][q] = ld_cg_f4(src + 4 * q);
                  }
                }
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                  const int sl = s0 + g;
                  if (sl < S) {
                    float val[32];
                    if (sl == slice) {
                      uint32_t r[32];
                      tmem_load_32x32b_x32(t_lane + static_cast<uint32_t>(h * MP + mc * 32), r);
#pragma unroll
                      for (int i = 0; i < 32; ++i) val[i] = __uint_as_float(r[i]);
                    } else {
#pragma unroll
                      for (int q = 0; q < 8; ++q) {
                        val[4 * q] = buf[g][q].x;
                        val[4 * q + 1] = buf[g][q].y;
                        val[4 * q + 2] = buf[g][q].z;
                        val[4 * q + 3] = buf[g][q].w;
                      }
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) acc[i] = (sl == 0) ? val[i] : acc[i] + val[i];
                  }
                }
              }
              store_rows<32, ACT>(acc, C, M, N, ldc, n0 + h * kSub, mc * 32, bias);
            }
          }
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

// Number of k-slices per tile: 1 when the tiles already cover the SMs,
// otherwise as many as fit on the idle SMs, with at least 16 k-blocks of 64
// per slice, S * TW * MP <= 65536 (the last slice to arrive sums the S
// partial tiles of TW x MP fp32 alone, a cost that grows with S * TW * MP),
// and at most `max_items` (tile, slice) pairs.  Fitted to a sweep of small-M
// shapes (M 16-64, N 1024-28672, K 4096-16384): the best or tied-best slice
// count on each; the former rule (up to SMs / tiles slices of >= 4 k-blocks)
// was up to 1.85x slower where few column tiles allowed many slices.
int choose_slices(int64_t tiles, int64_t KB, int MP, int TW, int sm_count, int64_t max_items) {
  if (tiles >= sm_count) return 1;
  int64_t s = sm_count / tiles;
  const int64_t by_k = KB / 16;
  const int64_t by_fixup = 65536 / (static_cast<int64_t>(TW) * MP);
  if (s > by_k) s = by_k;
  if (s > by_fixup) s = by_fixup;
  if (s * tiles > max_items) s = max_items / tiles;
  return s < 1 ? 1 : static_cast<int>(s);
}

// `splits` = 0 chooses the k-slices from the shape; otherwise exactly that
// many (1 <= splits <= k-blocks, and splits * tiles <= max_items when > 1).
template <int MP, int STAGES, int TW, int ACT>
int launch_impl(const GemmProblem& p, const DeviceCtx& d, void* ws, size_t ws_bytes,
                int64_t max_items, int splits) {
  using Cfg = SkinnyCfg<MP, STAGES, TW>;
  static std::atomic<uint64_t> attr_done{0};
  const int64_t KB = (p.K + kBK - 1) / kBK;
  const int64_t tiles = (p.N + TW - 1) / TW;
  if (splits < 0 || splits > KB || (splits > 1 && splits * tiles > max_items))
    return GEMM_ERR_CONFIG;
  const int S = splits > 0 ? splits : choose_slices(tiles, KB, MP, TW, d.sm_count, max_items);
  int* counters = nullptr;
  float* partials = nullptr;
  if (S > 1) {
    // counters for the tiles, then one fp32 partial tile per (tile, slice)
    const size_t need = counter_bytes(static_cast<int>(max_items)) +
                        static_cast<size_t>(tiles) * S * TW * MP * sizeof(float);
    if (ws == nullptr || ws_bytes < need) return GEMM_ERR_WORKSPACE;
    counters = static_cast<int*>(ws);
    partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                        counter_bytes(static_cast<int>(max_items)));
  }
  CUtensorMap tA, tB;
  int rc;
  if (p.layout & kLayoutTransA)  // stored K x M: 64 k-rows of 64 m (rows >= M read as 0)
    rc = encode_tmap_f16_2d(&tA, p.A, p.M, p.K, p.lda, 64, kBK);
  else  // stored M x K: MP rows of 64 k
    rc = encode_tmap_f16_2d(&tA, p.A, p.K, p.M, p.lda, kBK, MP);
  if (rc != 0) return rc;
  if (p.layout & kLayoutTransB)  // stored N x K: TW rows of 64 k
    rc = encode_tmap_f16_2d(&tB, p.B, p.K, p.N, p.ldb, kBK, TW);
  else  // row-major: slabs of 64 columns by 64 k-rows
    rc = encode_tmap_f16_2d(&tB, p.B, p.N, p.K, p.ldb, 64, kBK);
  if (rc != 0) return rc;
  auto kern = skinny_gemm_kernel<MP, STAGES, TW, ACT>;
  if (!ensure_smem_attr(reinterpret_cast<const void*>(kern), Cfg::kSmemBytes, d.device,
                        attr_done))
    return GEMM_ERR_LAUNCH;
  const int64_t grid = tiles * S;
  if (grid > INT32_MAX) return GEMM_ERR_INVALID_ARG;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = p.stream;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_attribute(&attr[0]);
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, kern, tA, tB, static_cast<__half*>(p.C), static_cast<int>(p.M),
      static_cast<int>(p.N), static_cast<int>(p.K), p.ldc, static_cast<const __half*>(p.bias), S,
      p.layout, partials, counters, static_cast<const __half*>(p.B), p.ldb, d.status,
      d.timeout_ns);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? GEMM_OK : GEMM_ERR_LAUNCH;
}

}  // namespace

int skinny_m_pad(int64_t M) {
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  return 0;
}

size_t skinny_workspace_bytes(int sm_count, int m_pad) {
  // split-K happens only with fewer tiles than SMs, so at most sm_count
  // (tile, slice) items carry a partial tile
  return counter_bytes(sm_count) +
         static_cast<size_t>(sm_count) * kMaxTW * static_cast<size_t>(m_pad) * sizeof(float);
}

namespace {

template <int MP, int STAGES, int TW>
int launch_act(const GemmProblem& p, const DeviceCtx& d, void* ws, size_t ws_bytes, int splits) {
  switch (p.act) {
    case kActRelu:
      return launch_impl<MP, STAGES, TW, kActRelu>(p, d, ws, ws_bytes, d.sm_count, splits);
    case kActGelu:
      return launch_impl<MP, STAGES, TW, kActGelu>(p, d, ws, ws_bytes, d.sm_count, splits);
    default:
      return launch_impl<MP, STAGES, TW, kActNone>(p, d, ws, ws_bytes, d.sm_count, splits);
  }
}

template <int MP, int I = 0>
int dispatch_variant(const GemmProblem& p, const DeviceCtx& d, void* ws, size_t ws_bytes,
                     const KernelConfig& c) {
  if constexpr (I == kNumSkinnyVariants) {
    return GEMM_ERR_CONFIG;
  } else {
    constexpr SkinnyVariant v = kSkinnyVariants[I];
    if (c.block_n == v.tw && c.stages == v.stages)
      return launch_act<MP, v.stages, v.tw>(p, d, ws, ws_bytes, c.splits);
    return dispatch_variant<MP, I + 1>(p, d, ws, ws_bytes, c);
  }
}

}  // namespace

int launch_skinny_gemm(const GemmProblem& p, const DeviceCtx& d, void* ws, size_t ws_bytes,
                       const KernelConfig& c) {
  const int mp = skinny_m_pad(p.M);
  if (mp == 32) return dispatch_variant<32>(p, d, ws, ws_bytes, c);
  if (mp == 64) return dispatch_variant<64>(p, d, ws, ws_bytes, c);
  return GEMM_ERR_INVALID_ARG;
}

int skinny_config_smem_bytes(int block_n, int stages) {
  if (stages < 1 || stages > 64 || (block_n != 128 && block_n != 256)) return -1;
  return skinny_smem_formula(block_n, stages);
}

int skinny_configs_built(KernelConfig* out, int cap) {
  for (int i = 0; i < kNumSkinnyVariants && i < cap; ++i)
    out[i] = KernelConfig{GEMM_PATH_SKINNY, kSkinnyVariants[i].tw, kSkinnyVariants[i].stages, 0,
                          0};
  return kNumSkinnyVariants;
}

// ------------------------------------------------ allocation-free variant ---
// Scratch of gemm_relu_f16_noalloc: arrival counters for up to
// kNoAllocMaxItems tiles, then one fp32 partial tile (256 columns x 32) per
// (tile, slice) item, for at most kNoAllocMaxItems items.  It is part of the
// library image, so every GPU that loads the library holds it.
namespace {

constexpr int kNoAllocMP = 32;
constexpr int kNoAllocMaxItems = 160;
constexpr size_t kNoAllocCounterBytes = counter_bytes(kNoAllocMaxItems);
constexpr size_t kNoAllocScratchBytes =
    kNoAllocCounterBytes +
    static_cast<size_t>(kNoAllocMaxItems) * kMaxTW * kNoAllocMP * sizeof(float);
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

int launch_skinny_gemm_noalloc(const GemmProblem& p, const DeviceCtx& d) {
  if (p.M > kNoAllocMP) return GEMM_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  const int rc = noalloc_scratch_address(d.device, &scratch);
  if (rc != GEMM_OK) return rc;
  // the array keeps the previous call's contents: the arrival counters must
  // start at zero (partial tiles are always written before they are read)
  if (cudaMemsetAsync(scratch, 0, kNoAllocCounterBytes, p.stream) != cudaSuccess)
    return GEMM_ERR_LAUNCH;
  const int64_t items = d.sm_count < kNoAllocMaxItems ? d.sm_count : kNoAllocMaxItems;
  return launch_impl<kNoAllocMP, kDefaultStagesSkinny, kMaxTW, kActRelu>(p, d, scratch,
                                                             kNoAllocScratchBytes, items, 0);
}

}  // namespace ttc
