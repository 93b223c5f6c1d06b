// Large-shape path of C = ReLU(A @ B) (or A @ B) for sm_100a.
//
// The operation and its blocking follow "Writing high-performance kernels in
// TileLang" (atlascloud.ai blog), section "Escribamos un GEMM": one output
// tile of block_M x block_N per work item, A and B tiles of block_K staged in
// shared memory through a software pipeline, a tensor-core tile MMA into an
// fp32 accumulator, max(x, 0) on the accumulator, a cast to fp16 on the way
// out, and an L2-friendly ordering of the tiles (T.use_swizzle).
//
// Blackwell re-design:
//   * persistent grid (one CTA per SM) walking the output tiles in
//     grouped-panel order (group_m tile-rows per panel);
//   * warp 0: TMA producer filling a STAGES-deep ring of 128-byte-swizzled
//     A (128 x 64) and B (64 x BN) tiles, with mbarrier full/empty handshakes;
//   * warp 1: allocates TMEM and issues tcgen05.mma (128 x BN x 16) from one
//     thread into a double-buffered fp32 accumulator in TMEM;
//   * warps 2-5 (2-9 for the 512-row pair tile): epilogue.  tcgen05.ld ->
//     bias and activation in fp32 -> RNE to fp16 -> swizzled shared-memory
//     staging -> TMA store, which clips rows/columns beyond M/N (ragged
//     edges).  With a second accumulator the epilogue of tile i overlaps the
//     main loop of tile i+1.
// Out-of-range A/B elements (M, N or K not a multiple of the tile) are
// zero-filled by TMA and so contribute nothing to the sum.
#include <atomic>

#include "../../include/gemm_f16.h"
#include "internal.h"
#include "sm100.cuh"

namespace ttc {
namespace {

constexpr int kBM = 128;        // tile rows (MMA M)
constexpr int kBK = 64;         // k-block: 64 fp16 = one 128-byte swizzle row
constexpr int kUmmaK = 16;      // K of one tcgen05.mma kind::f16
// Epilogue warps: 4 (one per TMEM lane quarter) where the epilogue of a tile
// overlaps the next tile's main loop (double-buffered accumulators), 8 (two per
// quarter, each draining half of the tile's columns) where it cannot (the
// 512-row pair tile fills TMEM with one accumulator).  Either way eight 32 x 64
// staging boxes (32 KiB): two per warp or one.
constexpr int epi_threads(int epi_warps) { return 64 + 32 * epi_warps; }
constexpr int kEpiRows = 32;    // rows per epilogue warp
constexpr int kEpiCols = 64;    // columns per epilogue chunk (128 bytes of fp16)
constexpr int kEpiBuf = kEpiRows * kEpiCols * 2;

// Dynamic shared memory of a tile kernel: 1 KiB of alignment slack, the
// operand ring, eight 32 x 64 fp16 staging boxes for the epilogue warps, the
// mbarriers (full and empty per stage, two accumulator handshakes per
// buffer, one spare) and the TMEM address slot.
constexpr int kEpiStaging = 8 * kEpiBuf;  // all staging boxes of a CTA
constexpr int tile_smem_formula(int stage_bytes, int stages) {
  return 1024 + stages * stage_bytes + kEpiStaging + (2 * stages + 5) * 8 + 16;
}
// One ring stage: A (128 rows x 64 k) and B (64 k x bn columns) ...
constexpr int single_stage_bytes(int bn) { return kBM * kBK * 2 + kBK * bn * 2; }
// ... or, per CTA of a pair, `slabs` slabs of 128 rows of A and 128 columns of B.
constexpr int pair_stage_bytes(int slabs) { return slabs * kBM * kBK * 2 + kBK * 128 * 2; }

template <int BN, int STAGES>
struct TileCfg {
  static constexpr int kEpiWarps = 4;
  static constexpr int kThreads = epi_threads(kEpiWarps);
  static constexpr int kEpiBoxes = 8 / kEpiWarps;
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBChunk = kBK * 64 * 2;  // one 64-column slab of the B tile
  static constexpr int kBBytes = kBK * BN * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kEpiBytes = kEpiStaging;
  static constexpr int kNumBars = 2 * STAGES + 5;
  static constexpr int kSmemBytes = 1024 + STAGES * kStageBytes + kEpiBytes + kNumBars * 8 + 16;
  static constexpr uint32_t kTmemCols = 2 * BN;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
  static_assert(kTmemCols == 128 || kTmemCols == 256 || kTmemCols == 512, "TMEM columns");
  static_assert(kSmemBytes == tile_smem_formula(single_stage_bytes(BN), STAGES), "layout");
  static_assert(kSmemBytes <= kMaxDynamicSmem, "shared memory budget");
};

// The CTA-pair kernel: a (256 * SLABS) x 256 output tile per pair of SMs.
// Each CTA stages SLABS slabs of 128 rows of A and its own 128 columns of B
// per k-block; slab s of CTA r holds tile rows 256 s + 128 r .. + 127, and one
// pair MMA (M = 256) per slab and 16-deep k step covers tile rows
// 256 s .. 256 s + 255.  Each CTA keeps SLABS accumulators of 128 rows x 256
// columns in TMEM: two buffers of one slab (the epilogue of tile i overlaps
// the main loop of tile i+1), or the two slabs of one tile (25 % fewer bytes
// staged per MAC, the epilogue not overlapped).
template <int STAGES, int SLABS>
struct PairCfg {
  static constexpr int kEpiWarps = SLABS == 2 ? 8 : 4;
  static constexpr int kThreads = epi_threads(kEpiWarps);
  static constexpr int kEpiBoxes = 8 / kEpiWarps;
  static constexpr int kBN = 256;                         // pair tile columns
  static constexpr int kTileM = 2 * kBM * SLABS;          // pair tile rows
  static constexpr int kSlabBytes = kBM * kBK * 2;        // 128 rows of A, 64 k
  static constexpr int kABytes = SLABS * kSlabBytes;
  static constexpr int kBChunk = kBK * 64 * 2;
  static constexpr int kBBytes = kBK * 128 * 2;           // this CTA's 128 columns
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kEpiBytes = kEpiStaging;
  static constexpr int kNumBars = 2 * STAGES + 5;
  static constexpr int kSmemBytes = 1024 + STAGES * kStageBytes + kEpiBytes + kNumBars * 8 + 16;
  static constexpr int kNBuf = SLABS == 1 ? 2 : 1;        // accumulator buffers
  static constexpr uint32_t kTmemCols = 512;
  static_assert(SLABS == 1 || SLABS == 2, "SLABS");
  static_assert(kNBuf * SLABS * kBN == 512, "TMEM columns");
  static_assert(kSmemBytes == tile_smem_formula(pair_stage_bytes(SLABS), STAGES), "layout");
  static_assert(kSmemBytes <= kMaxDynamicSmem, "shared memory budget");
};

// Configurations compiled (for every activation): each tile shape with every
// ring depth from 3 up to what fits the shared-memory budget.  A ring of 2
// cannot keep a load in flight while the MMA reads the other stage and the
// next load waits, so it is not built.
struct TileVariant {
  int kernel;  // GEMM_PATH_TILE / _TILE_PAIR / _TILE_PAIR_TALL
  int block_n;
  int stages;
};
constexpr TileVariant kTileVariants[] = {
    {GEMM_PATH_TILE, 64, 3},       {GEMM_PATH_TILE, 64, 4},       {GEMM_PATH_TILE, 64, 5},
    {GEMM_PATH_TILE, 64, 6},       {GEMM_PATH_TILE, 64, 7},       {GEMM_PATH_TILE, 64, 8},
    {GEMM_PATH_TILE, 128, 3},      {GEMM_PATH_TILE, 128, 4},      {GEMM_PATH_TILE, 128, 5},
    {GEMM_PATH_TILE, 128, 6},      {GEMM_PATH_TILE, 256, 3},      {GEMM_PATH_TILE, 256, 4},
    {GEMM_PATH_TILE_PAIR, 256, 3}, {GEMM_PATH_TILE_PAIR, 256, 4}, {GEMM_PATH_TILE_PAIR, 256, 5},
    {GEMM_PATH_TILE_PAIR, 256, 6}, {GEMM_PATH_TILE_PAIR_TALL, 256, 3},
    {GEMM_PATH_TILE_PAIR_TALL, 256, 4}};
constexpr int kNumTileVariants = sizeof(kTileVariants) / sizeof(kTileVariants[0]);

constexpr int variant_smem_bytes(int kernel, int block_n, int stages) {
  return kernel == GEMM_PATH_TILE
             ? (block_n == 64 || block_n == 128 || block_n == 256
                    ? tile_smem_formula(single_stage_bytes(block_n), stages)
                    : -1)
         : block_n != 256                       ? -1
         : kernel == GEMM_PATH_TILE_PAIR        ? tile_smem_formula(pair_stage_bytes(1), stages)
         : kernel == GEMM_PATH_TILE_PAIR_TALL   ? tile_smem_formula(pair_stage_bytes(2), stages)
                                                : -1;
}

// The table holds exactly the depths from 3 to the budget's limit.
constexpr bool variants_complete() {
  const int kinds[5][2] = {{GEMM_PATH_TILE, 64}, {GEMM_PATH_TILE, 128}, {GEMM_PATH_TILE, 256},
                           {GEMM_PATH_TILE_PAIR, 256}, {GEMM_PATH_TILE_PAIR_TALL, 256}};
  for (const auto& k : kinds) {
    for (int st = 3; st <= 16; ++st) {
      const bool fits = variant_smem_bytes(k[0], k[1], st) <= kMaxDynamicSmem;
      bool built = false;
      for (const auto& v : kTileVariants)
        built = built || (v.kernel == k[0] && v.block_n == k[1] && v.stages == st);
      if (fits != built) return false;
    }
  }
  return true;
}
static_assert(variants_complete(), "built tile configurations != those within the budget");

// Grouped-panel rasterisation: consecutive tile indices sweep group_m
// tile-rows of one panel column by column, so the CTAs that run at the same
// time share A rows and B columns in L2.  Odd panels sweep their columns in
// reverse (a snake), so the first tiles of a panel reuse the B columns the
// previous panel read last.  A negative group_m gives panels of -group_m
// tile-columns swept row by row instead (the same with the roles of A and B
// exchanged).
__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int group_m,
                                            int& mb, int& nb) {
  if (group_m > 0) {
    const int per_group = group_m * num_n;
    const int g = tile / per_group;
    const int first_m = g * group_m;
    const int rows = min(num_m - first_m, group_m);
    const int r = tile - g * per_group;
    mb = first_m + r % rows;
    nb = r / rows;
    if (g & 1) nb = num_n - 1 - nb;
  } else {
    const int group_n = -group_m;
    const int per_group = group_n * num_m;
    const int g = tile / per_group;
    const int first_n = g * group_n;
    const int cols = min(num_n - first_n, group_n);
    const int r = tile - g * per_group;
    nb = first_n + r % cols;
    mb = r / cols;
    if (g & 1) mb = num_m - 1 - mb;
  }
}

// The 64 bias values of the chunk at column col0 as 32 packed pairs (0 past
// N): eight 16-byte loads (the same address in every lane) when the chunk
// lies inside N, else pair by pair.
__device__ __forceinline__ void load_bias_chunk(const __half* __restrict__ bias, int col0, int N,
                                                uint32_t (&bb)[32]) {
  if (col0 + kEpiCols <= N) {
    const uint4* src = reinterpret_cast<const uint4*>(bias + col0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 q = __ldg(src + i);
      bb[4 * i] = q.x;
      bb[4 * i + 1] = q.y;
      bb[4 * i + 2] = q.z;
      bb[4 * i + 3] = q.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int col = col0 + 2 * i;
      if (col + 1 < N) {
        bb[i] = __ldg(reinterpret_cast<const unsigned int*>(bias + col));
      } else {
        const unsigned short lo =
            col < N ? __ldg(reinterpret_cast<const unsigned short*>(bias + col)) : 0;
        bb[i] = lo;
      }
    }
  }
}

// Bias and activation in fp32, then RNE to fp16, of one 64-column chunk of a
// warp's 32 accumulator rows already in registers (`v`: 64 fp32 bit
// patterns of this thread's row) into 32 packed pairs `h`.
template <int ACT>
__device__ __forceinline__ void convert_chunk(const uint32_t* v, const __half* __restrict__ bias,
                                              int col0, int N, uint32_t* h) {
  uint32_t bb[32];
  if (bias != nullptr) load_bias_chunk(bias, col0, N, bb);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    // columns 2i, 2i + 1 and 32 + 2i, 32 + 2i + 1 of the chunk, in pairs
    float2 xv = make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
    float2 yv = make_float2(__uint_as_float(v[32 + 2 * i]), __uint_as_float(v[32 + 2 * i + 1]));
    if (bias != nullptr) {
      xv = __fadd2_rn(xv, __half22float2(*reinterpret_cast<const __half2*>(&bb[i])));
      yv = __fadd2_rn(yv, __half22float2(*reinterpret_cast<const __half2*>(&bb[16 + i])));
    }
    xv = activate2<ACT>(xv);
    yv = activate2<ACT>(yv);
    h[i] = pack_half2(xv.x, xv.y);
    h[16 + i] = pack_half2(yv.x, yv.y);
  }
}

// The converted chunk `h` (row `lane` of a 32 x 64 fp16 box) -> 128-byte
// swizzled staging row per thread -> TMA store of the box (BOXES boxes per
// warp in turn).  Columns at and beyond N rounded down to 8 (the TMA store
// writes whole 16-byte groups) are written with plain stores.
template <int BOXES>
__device__ __forceinline__ void stage_chunk(const uint32_t* h, uint8_t* bufs, uint32_t& chunk_no,
                                            const CUtensorMap* tmC, __half* C, int64_t ldc,
                                            int M, int N, int n8, int row0, int col0, int lane) {
  uint8_t* buf = bufs + (chunk_no % BOXES) * kEpiBuf;
  // the store that last used `buf` has read it
  if (lane == 0) bulk_wait_group_read<BOXES - 1>();
  __syncwarp();
  // row `lane`, 128 bytes = 8 chunks of 16 bytes, chunk j stored at j ^ (row & 7)
  const uint32_t row_addr = smem_u32(buf) + lane * 128;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    st_shared_v4(row_addr + ((j ^ (lane & 7)) << 4), h[4 * j], h[4 * j + 1], h[4 * j + 2],
                 h[4 * j + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    // C is written once and not read again here: evict-first keeps the
    // operand tiles that later tiles re-read in L2 (0.1-0.7 % faster)
    if (row0 < M && col0 < n8) tma_store_2d_hint(tmC, buf, col0, row0, l2_policy_evict_first());
    bulk_commit_group();
  }
  if (n8 < N && col0 + kEpiCols > n8 && col0 < N && row0 + lane < M) {
    // ragged tail columns [max(n8, col0), min(N, col0 + 64)) of this row,
    // read back from this thread's own (swizzled) staging row
    const int j_end = min(N, col0 + kEpiCols);
    __half* crow = C + static_cast<int64_t>(row0 + lane) * ldc;
    for (int j = max(n8, col0); j < j_end; ++j) {
      const int cc = j - col0;
      const uint32_t addr = row_addr + ((((cc >> 3) ^ (lane & 7)) << 4) | ((cc & 7) << 1));
      unsigned short bits;
      asm volatile("ld.shared.u16 %0, [%1];" : "=h"(bits) : "r"(addr) : "memory");
      crow[j] = __ushort_as_half(bits);
    }
  }
  ++chunk_no;
}

// Epilogue of one accumulator tile, run by one warp for its 32 TMEM lanes and
// COLS of the tile's columns, 64 at a time: tcgen05.ld -> convert_chunk ->
// stage_chunk, with each chunk staged only after the next chunk's TMEM load,
// so that `release()` runs as soon as the last TMEM load of the tile has
// completed (only the last chunk's conversion and two stagings follow it).
// `bias` (N fp16 values or null) is added per column before the activation.
template <int COLS, int BOXES, int ACT, class Release>
__device__ __forceinline__ void epilogue_tile(uint32_t t_row, uint8_t* bufs, uint32_t& chunk_no,
                                              const CUtensorMap* tmC, __half* C, int64_t ldc,
                                              const __half* __restrict__ bias, int M, int N,
                                              int n8, int row0, int col_base, int lane,
                                              Release release) {
  constexpr int kChunks = COLS / kEpiCols;
  uint32_t h[32];  // the previous chunk, converted, not yet staged
#pragma unroll 1
  for (int c = 0; c < kChunks; ++c) {
    uint32_t v[64];
    tmem_load_32x32b_x64(t_row + c * kEpiCols, v);
    if (c == kChunks - 1) {
      // the accumulator has been read: hand it back to the MMA issuer
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) release();
    }
    if (c > 0)
      stage_chunk<BOXES>(h, bufs, chunk_no, tmC, C, ldc, M, N, n8, row0,
                         col_base + (c - 1) * kEpiCols, lane);
    convert_chunk<ACT>(v, bias, col_base + c * kEpiCols, N, h);
  }
  stage_chunk<BOXES>(h, bufs, chunk_no, tmC, C, ldc, M, N, n8, row0,
                     col_base + (kChunks - 1) * kEpiCols, lane);
}

template <int BN, int STAGES, int ACT>
__global__ void __launch_bounds__(TileCfg<BN, STAGES>::kThreads, 1)
    tile_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, __half* __restrict__ C,
                     int64_t ldc, const __half* __restrict__ bias, int M, int N, int K,
                     int layout, int group_m, int* status, uint64_t timeout_ns) {
  using Cfg = TileCfg<BN, STAGES>;
  const bool ta = (layout & kLayoutTransA) != 0;
  const bool tb = (layout & kLayoutTransB) != 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* smA = smem;
  uint8_t* smB = smem + STAGES * Cfg::kABytes;
  uint8_t* smEpi = smem + STAGES * Cfg::kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smEpi + Cfg::kEpiBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = bars + 2 * STAGES + 2;
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_m = (M + kBM - 1) / kBM;
  const int num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = (K + kBK - 1) / kBK;
  // The TMA store writes whole 16-byte groups of columns, so it is given only
  // the first N rounded down to 8 columns; the (< 8) remaining columns of a
  // ragged edge are written with plain stores.
  const int n8 = N & ~7;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], Cfg::kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish_alloc_permit();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  // The coordinates of this CTA's first tile (three integer divisions, about
  // 0.3 us at the start of a small launch) are worked out before the wait, so
  // they overlap the previous kernel of the stream.
  int first_mb = 0, first_nb = 0;
  tile_coords(blockIdx.x, num_m, num_n, group_m, first_mb, first_nb);
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
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int mb = first_mb, nb = first_nb;
        if (tile != static_cast<int>(blockIdx.x)) tile_coords(tile, num_m, num_n, group_m, mb, nb);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], Cfg::kStageBytes);
          uint8_t* adst = smA + stage * Cfg::kABytes;
          if (!ta) {
            tma_load_2d(&tmA, &full[stage], adst, kb * kBK, mb * kBM);
          } else {  // two 64-row slabs of the M-contiguous storage
            tma_load_2d(&tmA, &full[stage], adst, mb * kBM, kb * kBK);
            tma_load_2d(&tmA, &full[stage], adst + Cfg::kBChunk, mb * kBM + 64, kb * kBK);
          }
          uint8_t* bdst = smB + stage * Cfg::kBBytes;
          if (!tb) {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_2d(&tmB, &full[stage], bdst + j * Cfg::kBChunk, nb * BN + j * 64,
                          kb * kBK);
          } else {  // BN rows of the K-contiguous storage
            tma_load_2d(&tmB, &full[stage], bdst, kb * kBK, nb * BN);
          }
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleProducer << 4) | 1);
        // let every load already issued land before shared memory is released
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s)) (void)mbar_wait(&full[s], (armed_parity >> s) & 1u, nullptr, timeout_ns);
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
      const uint32_t idesc = idesc_f16_f32(kBM, BN, ta, !tb);
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag, timeout_ns)) {
          ok = false;
          site = 1;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, timeout_ns)) {
            ok = false;
            site = 2;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(smA + stage * Cfg::kABytes);
          const uint32_t b_addr = smem_u32(smB + stage * Cfg::kBBytes);
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k) {
            // row-major A is K-major, row-major B is N-major (and the reverse
            // for the transposed storages)
            const uint64_t adesc = operand_desc(a_addr, k, ta, Cfg::kBChunk);
            const uint64_t bdesc = operand_desc(b_addr, k, !tb, Cfg::kBChunk);
            umma_f16(d_tmem, adesc, bdesc, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);  // frees the stage once these MMAs have read it
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);  // accumulator ready for the epilogue
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok) {
        raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleMma << 4) | site);
        umma_commit(drain);  // wait for MMAs in flight before TMEM is released
        (void)mbar_wait(drain, 0, nullptr, timeout_ns);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue ---
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int ew = warp - 2;
    constexpr int kCols = BN * 4 / Cfg::kEpiWarps;  // columns of the tile this warp drains
    const int g = ew >> 2;                  // its column group
    uint8_t* bufs = smEpi + ew * Cfg::kEpiBoxes * kEpiBuf;
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t chunk_no = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      int mb = first_mb, nb = first_nb;
      if (tile != static_cast<int>(blockIdx.x)) tile_coords(tile, num_m, num_n, group_m, mb, nb);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&acc_full[acc], acc_phase, abort_flag, timeout_ns) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0)
          raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleEpilogue << 4) | 1);
        break;
      }
      tc_fence_after_sync();
      const int row0 = mb * kBM + q * kEpiRows;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * BN + g * kCols);
      uint64_t* release_bar = &acc_empty[acc];
      epilogue_tile<kCols, Cfg::kEpiBoxes, ACT>(t_row, bufs, chunk_no, &tmC, C, ldc, bias, M, N,
                                                n8, row0, nb * BN + g * kCols, lane,
                                                [release_bar] { mbar_arrive(release_bar); });
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

// Busy-wait for about `ns` nanoseconds (bounded, used on the abort path only).
__device__ __forceinline__ void spin_ns(uint64_t ns) {
  const uint64_t t0 = globaltimer_ns();
  while (globaltimer_ns() - t0 < ns) {
  }
}

// CTA-pair kernel.  Launched with clusters of 2 CTAs; cluster rank 0 (the
// "leader") issues the tcgen05.mma.cta_group::2 for both SMs.
//   * both producers load their halves into their own shared memory and count
//     the bytes on the leader's full[stage] barrier (armed by the leader for
//     both halves);
//   * the leader's commit frees stage s in both CTAs and tells both epilogues
//     that an accumulator is ready (multicast arrive);
//   * each CTA's epilogue warps (4, or 8 for the 512-row tile) drain its own
//     TMEM rows and arrive on the leader's acc_empty barrier (one arrival per
//     warp of both CTAs per accumulator use).
template <int STAGES, int SLABS, int ACT>
__global__ void __launch_bounds__(PairCfg<STAGES, SLABS>::kThreads, 1)
    tile_pair_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                          const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmC, __half* __restrict__ C,
                          int64_t ldc, const __half* __restrict__ bias, int M, int N, int K,
                          int layout, int group_m, int split_from, int* status,
                          uint64_t timeout_ns) {
  using Cfg = PairCfg<STAGES, SLABS>;
  const bool ta = (layout & kLayoutTransA) != 0;
  const bool tb = (layout & kLayoutTransB) != 0;
  constexpr int BN = Cfg::kBN;
  constexpr int NBUF = Cfg::kNBuf;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* smA = smem;
  uint8_t* smB = smem + STAGES * Cfg::kABytes;
  uint8_t* smEpi = smem + STAGES * Cfg::kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smEpi + Cfg::kEpiBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = bars + 2 * STAGES + 2;
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int pair = static_cast<int>(cluster_id_x());
  const int npairs = static_cast<int>(num_clusters_x());
  const int num_m = (M + Cfg::kTileM - 1) / Cfg::kTileM;
  const int num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = (K + kBK - 1) / kBK;
  const int n8 = N & ~7;
  // Work units: tiles [0, split_from) whole, then each tile from split_from
  // on as two units of one 256-row slab (the host splits the tiles of a last
  // wave that holds at most half as many tiles as there are pairs, so that
  // wave takes about half a tile's time; split_from == num_tiles otherwise).
  const int num_units = 2 * num_tiles - split_from;
  // unit -> tile coordinates, first row of the unit and its slab count
  auto unit_coords = [&](int u, int& mb, int& nb, int& row_base, int& slabs) {
    const bool half = u >= split_from;
    tile_coords(half ? split_from + (u - split_from) / 2 : u, num_m, num_n, group_m, mb, nb);
    row_base = mb * Cfg::kTileM + (half ? ((u - split_from) & 1) * 2 * kBM : 0);
    slabs = half ? 1 : SLABS;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * Cfg::kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish_alloc_permit_pair();
  }
  tc_fence_before_sync();
  cluster_sync();  // barriers of both CTAs initialised, TMEM of both SMs allocated
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  grid_dependency_trigger();
  grid_dependency_wait();
  // the leader's barriers, as addresses this CTA can signal
  const uint32_t full_leader = map_to_cta(smem_u32(full), 0);
  const uint32_t acc_empty_leader = map_to_cta(smem_u32(acc_empty), 0);

  if (warp == 0) {
    // --------------------------------------------- TMA producer (both CTAs) ---
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      bool ok = true;
      // The pairs run their j-th units at about the same time (a wave); odd
      // waves sweep K from the top down, so a wave starts on the k-blocks the
      // previous wave read last -- still in L2 -- instead of the ones it read
      // first, which it evicted long ago.  The MMA issuer consumes the stages
      // in ring order either way; only its first k-block (not k-block 0)
      // starts the accumulation.
      uint32_t down = 0;
      for (int unit = pair; unit < num_units && ok; unit += npairs, down ^= 1u) {
        int mb, nb, row_base, slabs;
        unit_coords(unit, mb, nb, row_base, slabs);
        const int a_row = row_base + static_cast<int>(rank) * kBM;  // slab 0
        const int b_col = nb * BN + static_cast<int>(rank) * 128;
        const uint32_t tx = 2u * static_cast<uint32_t>(slabs * Cfg::kSlabBytes + Cfg::kBBytes);
        for (int i = 0; i < num_kb; ++i) {
          const int kb = down ? num_kb - 1 - i : i;  // the k-block this stage holds
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, timeout_ns)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], tx);
          const uint32_t bar = full_leader + stage * 8;
#pragma unroll
          for (int s = 0; s < SLABS; ++s) {
            if (s >= slabs) break;
            uint8_t* adst = smA + stage * Cfg::kABytes + s * Cfg::kSlabBytes;
            const int row = a_row + s * 2 * kBM;
            if (!ta) {
              tma_load_2d_pair(&tmA, bar, adst, kb * kBK, row);
            } else {
              tma_load_2d_pair(&tmA, bar, adst, row, kb * kBK);
              tma_load_2d_pair(&tmA, bar, adst + Cfg::kBChunk, row + 64, kb * kBK);
            }
          }
          uint8_t* bdst = smB + stage * Cfg::kBBytes;
          if (!tb) {
            tma_load_2d_pair(&tmB, bar, bdst, b_col, kb * kBK);
            tma_load_2d_pair(&tmB, bar, bdst + Cfg::kBChunk, b_col + 64, kb * kBK);
          } else {
            tma_load_2d_pair(&tmB, bar, bdst, kb * kBK, b_col);
          }
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleProducer << 4) | 3);
        if (leader) {
          for (int s = 0; s < STAGES; ++s)
            if (armed & (1u << s))
              (void)mbar_wait(&full[s], (armed_parity >> s) & 1u, nullptr, timeout_ns);
        } else {
          // this CTA's loads complete on the leader's barriers, which it cannot
          // poll; give loads already issued ample time to land
          spin_ns(2000000);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer (leader) ---
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;  // also the phase of acc_empty[0] with two slabs
      uint32_t slab1_phase = 0;
      bool ok = true;
      int site = 0;
      const uint32_t idesc = idesc_f16_f32(2 * kBM, BN, ta, !tb);
      // The MMAs of the unit's kb-th k-block in load order (held in ring
      // stage `st`; the first one starts the accumulation) for slabs
      // [s_begin, s_end) into the accumulator at `d_tmem`.
      auto issue = [&](uint32_t d_tmem, int st, int kb, int s_begin, int s_end) {
        const uint32_t a_addr = smem_u32(smA + st * Cfg::kABytes);
        const uint32_t b_addr = smem_u32(smB + st * Cfg::kBBytes);
#pragma unroll
        for (int k = 0; k < kBK / kUmmaK; ++k) {
          const uint64_t bdesc = operand_desc(b_addr, k, !tb, Cfg::kBChunk);
#pragma unroll
          for (int s = 0; s < SLABS; ++s) {
            if (s < s_begin || s >= s_end) continue;
            const uint64_t adesc = operand_desc(a_addr + s * Cfg::kSlabBytes, k, ta, Cfg::kBChunk);
            umma_f16_pair(d_tmem + static_cast<uint32_t>(s * BN), adesc, bdesc, idesc,
                          (kb | k) != 0 ? 1u : 0u);
          }
        }
      };
      for (int unit = pair; unit < num_units && ok; unit += npairs) {
        if constexpr (SLABS == 2) {
          // One accumulator of two slabs; the epilogue hands each slab back on
          // its own barrier (acc_empty[s]) as soon as it has read it.  The
          // next tile's slab-0 MMAs start on the k-blocks already in the ring
          // while slab 1 is still being drained; those stages are freed once
          // their slab-1 MMAs have been issued too.
          if (!mbar_wait(&acc_empty[0], acc_phase ^ 1u, abort_flag, timeout_ns)) {
            ok = false;
            site = 5;
            break;
          }
          tc_fence_after_sync();
          // a half tile (a unit from split_from on) has slab 0 only: no early
          // start, every k-block in the loop below
          const bool whole = unit < split_from;
          const int early = !whole ? 0 : (num_kb < STAGES ? num_kb : STAGES);
          const int stage0 = stage;
          for (int kb = 0; kb < early; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort_flag, timeout_ns)) {
              ok = false;
              site = 6;
              break;
            }
            tc_fence_after_sync();
            issue(tmem_base, stage, kb, 0, 1);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          if (whole) {
            if (!mbar_wait(&acc_empty[1], slab1_phase ^ 1u, abort_flag, timeout_ns)) {
              ok = false;
              site = 7;
              break;
            }
            slab1_phase ^= 1u;
            tc_fence_after_sync();
          }
          for (int kb = 0, st = stage0; kb < early; ++kb) {
            issue(tmem_base, st, kb, 1, 2);
            umma_commit_pair(&empty[st], 0x3);  // stage free in both CTAs
            if (++st == STAGES) st = 0;
          }
          const int slab_end = whole ? 2 : 1;
          for (int kb = early; kb < num_kb; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort_flag, timeout_ns)) {
              ok = false;
              site = 6;
              break;
            }
            tc_fence_after_sync();
            issue(tmem_base, stage, kb, 0, slab_end);
            umma_commit_pair(&empty[stage], 0x3);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          umma_commit_pair(&acc_full[0], 0x3);  // both epilogues may read
          acc_phase ^= 1u;
        } else {
          if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag, timeout_ns)) {
            ok = false;
            site = 5;
            break;
          }
          tc_fence_after_sync();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * SLABS * BN);
          for (int kb = 0; kb < num_kb; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort_flag, timeout_ns)) {
              ok = false;
              site = 6;
              break;
            }
            tc_fence_after_sync();
            issue(d_tmem, stage, kb, 0, SLABS);
            umma_commit_pair(&empty[stage], 0x3);  // stage s free in both CTAs
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          umma_commit_pair(&acc_full[acc], 0x3);  // both epilogues may read
          if (++acc == NBUF) {
            acc = 0;
            acc_phase ^= 1u;
          }
        }
      }
      if (!ok) {
        raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleMma << 4) | site);
        umma_commit_pair(drain, 0x1);
        (void)mbar_wait(drain, 0, nullptr, timeout_ns);
      }
    }
  } else {
    // ------------------------------------------------ epilogue (both CTAs) ---
    const int q = warp & 3;
    const int ew = warp - 2;
    constexpr int kCols = BN * 4 / Cfg::kEpiWarps;
    const int g = ew >> 2;
    uint8_t* bufs = smEpi + ew * Cfg::kEpiBoxes * kEpiBuf;
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t chunk_no = 0;
    for (int unit = pair; unit < num_units; unit += npairs) {
      int mb, nb, row_base, slabs;
      unit_coords(unit, mb, nb, row_base, slabs);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&acc_full[acc], acc_phase, abort_flag, timeout_ns) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0)
          raise_abort(status, abort_flag, kStatusTimeoutBase | (kRoleEpilogue << 4) | 3);
        break;
      }
      tc_fence_after_sync();
#pragma unroll 1
      for (int s = 0; s < slabs; ++s) {
        // two slabs (single accumulator): each slab has its own barrier and is
        // handed back as soon as it has been read; one slab (two accumulator
        // buffers): the buffer's barrier
        const uint32_t release_bar = acc_empty_leader + (SLABS == 2 ? s : acc) * 8;
        const int row0 = row_base + s * 2 * kBM + static_cast<int>(rank) * kBM + q * kEpiRows;
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>((acc * SLABS + s) * BN + g * kCols);
        epilogue_tile<kCols, Cfg::kEpiBoxes, ACT>(
            t_row, bufs, chunk_no, &tmC, C, ldc, bias, M, N, n8, row0, nb * BN + g * kCols, lane,
            [release_bar] { mbar_arrive_cluster_relaxed(release_bar); });
      }
      if (++acc == NBUF) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  tc_fence_before_sync();
  // no CTA of the pair leaves (or frees TMEM) while the other may still signal
  // its barriers or use its TMEM
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
  }
}

// Sets the dynamic shared-memory limit of a kernel once per device.
bool ensure_smem_attr(const void* func, int bytes, int device, std::atomic<uint64_t>& done) {
  const uint64_t bit = 1ull << (device & 63);
  if (done.load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  done.fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

// TMA maps of A (tile of `a_rows` rows of op(A) by 64 k) and B (64 k by
// `b_cols` columns of op(B)) for the operand layouts of `p`.
int encode_operand_maps(const GemmProblem& p, int a_rows, int b_cols, CUtensorMap* tA,
                        CUtensorMap* tB) {
  int rc;
  if (p.layout & kLayoutTransA)  // stored K x M: boxes of 64 m by 64 k
    rc = encode_tmap_f16_2d(tA, p.A, p.M, p.K, p.lda, 64, kBK);
  else  // stored M x K: boxes of 64 k by a_rows m
    rc = encode_tmap_f16_2d(tA, p.A, p.K, p.M, p.lda, kBK, a_rows);
  if (rc != 0) return rc;
  if (p.layout & kLayoutTransB)  // stored N x K: boxes of 64 k by b_cols n
    return encode_tmap_f16_2d(tB, p.B, p.K, p.N, p.ldb, kBK, b_cols);
  return encode_tmap_f16_2d(tB, p.B, p.N, p.K, p.ldb, 64, kBK);  // 64 n by 64 k
}

// Raster panel of the tile kernels in tiles: `group` > 0 rows of A per row
// panel -> that many tile-rows (at least 1); `group` < 0 columns of B per
// column panel -> minus that many tile-columns.
int group_tiles(int group, int tile_rows, int tile_cols) {
  if (group < 0) {
    const int g = -group / tile_cols;
    return g > 0 ? -g : -1;
  }
  const int g = group / tile_rows;
  return g > 0 ? g : 1;
}

template <int BN, int STAGES, int ACT>
int launch_impl(const GemmProblem& p, const DeviceCtx& d, int group_rows) {
  using Cfg = TileCfg<BN, STAGES>;
  static std::atomic<uint64_t> attr_done{0};
  CUtensorMap tA, tB, tC;
  int rc = encode_operand_maps(p, kBM, BN, &tA, &tB);
  // inner extent N rounded down to 8 columns (see the kernel's ragged tail);
  // the map is never used when that is 0
  const uint64_t n8 = static_cast<uint64_t>(p.N) & ~7ull;
  if (rc == 0) rc = encode_tmap_f16_2d(&tC, p.C, n8 > 0 ? n8 : 8, p.M, p.ldc, kEpiCols, kEpiRows);
  if (rc != 0) return rc;
  auto kern = tile_gemm_kernel<BN, STAGES, ACT>;
  if (!ensure_smem_attr(reinterpret_cast<const void*>(kern), Cfg::kSmemBytes, d.device,
                        attr_done))
    return GEMM_ERR_LAUNCH;
  const int64_t num_tiles = ((p.M + kBM - 1) / kBM) * ((p.N + BN - 1) / BN);
  const int grid = static_cast<int>(num_tiles < d.sm_count ? num_tiles : d.sm_count);
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = p.stream;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_attribute(&attr[0]);
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, kern, tA, tB, tC, static_cast<__half*>(p.C), p.ldc,
      static_cast<const __half*>(p.bias), static_cast<int>(p.M), static_cast<int>(p.N),
      static_cast<int>(p.K), p.layout, group_tiles(group_rows, kBM, BN), d.status,
      d.timeout_ns);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? 0 : GEMM_ERR_LAUNCH;
}

template <int STAGES, int SLABS, int ACT>
int launch_pair_impl(const GemmProblem& p, const DeviceCtx& d, int group_rows) {
  using Cfg = PairCfg<STAGES, SLABS>;
  static std::atomic<uint64_t> attr_done{0};
  // pairs that can be resident at once, per device (0 = not asked yet; racing
  // first calls store the same value)
  static std::atomic<int> max_pairs[64] = {};
  CUtensorMap tA, tB, tC;
  int rc = encode_operand_maps(p, kBM, 128, &tA, &tB);  // this CTA's half: 128 columns
  const uint64_t n8 = static_cast<uint64_t>(p.N) & ~7ull;
  if (rc == 0) rc = encode_tmap_f16_2d(&tC, p.C, n8 > 0 ? n8 : 8, p.M, p.ldc, kEpiCols, kEpiRows);
  if (rc != 0) return rc;
  auto kern = tile_pair_gemm_kernel<STAGES, SLABS, ACT>;
  if (!ensure_smem_attr(reinterpret_cast<const void*>(kern), Cfg::kSmemBytes, d.device,
                        attr_done))
    return GEMM_ERR_LAUNCH;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = p.stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // pairs that can be resident at once (GPC layout may leave an SM unpaired)
  int resident = max_pairs[d.device & 63].load(std::memory_order_relaxed);
  if (resident == 0) {
    cfg.gridDim = dim3(2 * (d.sm_count / 2), 1, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = d.sm_count / 2;
    }
    resident = n;
    max_pairs[d.device & 63].store(n, std::memory_order_relaxed);
  }
  const int64_t num_tiles = ((p.M + Cfg::kTileM - 1) / Cfg::kTileM) * ((p.N + 255) / 256);
  // with the 512-row tile, a last wave of at most resident / 2 tiles runs as
  // twice as many 256-row halves
  int64_t split_from = num_tiles;
  if constexpr (SLABS == 2) {
    const int64_t rem = num_tiles % resident;
    if (rem != 0 && 2 * rem <= resident) split_from = num_tiles - rem;
  }
  const int64_t units = 2 * num_tiles - split_from;
  const int pairs = static_cast<int>(units < resident ? units : resident);
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.numAttrs = 1 + pdl_attribute(&attr[1]);
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, kern, tA, tB, tC, static_cast<__half*>(p.C), p.ldc,
      static_cast<const __half*>(p.bias), static_cast<int>(p.M), static_cast<int>(p.N),
      static_cast<int>(p.K), p.layout, group_tiles(group_rows, Cfg::kTileM, Cfg::kBN),
      static_cast<int>(split_from), d.status, d.timeout_ns);
  return (e == cudaSuccess && cudaGetLastError() == cudaSuccess) ? 0 : GEMM_ERR_LAUNCH;
}

template <int KERNEL, int BN, int STAGES, int ACT>
int launch_variant(const GemmProblem& p, const DeviceCtx& d, int group_rows) {
  if constexpr (KERNEL == GEMM_PATH_TILE)
    return launch_impl<BN, STAGES, ACT>(p, d, group_rows);
  else
    return launch_pair_impl<STAGES, KERNEL == GEMM_PATH_TILE_PAIR_TALL ? 2 : 1, ACT>(p, d,
                                                                                  group_rows);
}

// Finds the table entry of `c` at compile-time-unrolled depth I and launches
// its kernel for the problem's activation.
template <int I = 0>
int dispatch_variant(const GemmProblem& p, const DeviceCtx& d, const KernelConfig& c) {
  if constexpr (I == kNumTileVariants) {
    return GEMM_ERR_CONFIG;
  } else {
    constexpr TileVariant v = kTileVariants[I];
    if (c.kernel != v.kernel || c.block_n != v.block_n || c.stages != v.stages)
      return dispatch_variant<I + 1>(p, d, c);
    switch (p.act) {
      case kActRelu: return launch_variant<v.kernel, v.block_n, v.stages, kActRelu>(p, d, c.group_rows);
      case kActGelu: return launch_variant<v.kernel, v.block_n, v.stages, kActGelu>(p, d, c.group_rows);
      default: return launch_variant<v.kernel, v.block_n, v.stages, kActNone>(p, d, c.group_rows);
    }
  }
}

}  // namespace

int launch_tile_gemm(const GemmProblem& p, const DeviceCtx& d, const KernelConfig& c) {
  return dispatch_variant(p, d, c);
}

int tile_config_smem_bytes(int kernel, int block_n, int stages) {
  if (stages < 1 || stages > 64) return -1;
  return variant_smem_bytes(kernel, block_n, stages);
}

int tile_configs_built(KernelConfig* out, int cap) {
  for (int i = 0; i < kNumTileVariants && i < cap; ++i)
    out[i] = KernelConfig{kTileVariants[i].kernel, kTileVariants[i].block_n,
                          kTileVariants[i].stages, 0, 0};
  return kNumTileVariants;
}

}  // namespace ttc
