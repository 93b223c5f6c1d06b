// Host-side declarations shared by the translation units of libttc05.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ttc {

struct GemmProblem {
  const void* A;
  const void* B;
  void* C;
  int64_t M, N, K;
  int64_t lda, ldb, ldc;
  int act;             // kActNone / kActRelu / kActGelu (sm100.cuh), = gemm_activation
  const void* bias;    // N fp16 values added per column before the activation, or null
  int layout;          // kLayoutTransA | kLayoutTransB (sm100.cuh): transposed storages
  cudaStream_t stream;
};

// One kernel configuration, resolved (no zero "default" fields left): the
// validated form of the public gemm_config.
struct KernelConfig {
  int kernel;      // GEMM_PATH_TILE / _TILE_PAIR / _TILE_PAIR_TALL / _SKINNY / _SKINNY_EVEN
  int block_n;     // output columns per CTA (TILE: 128 or 256) or per pair / tile (256)
  int stages;      // depth of the shared-memory operand ring
  int group_rows;  // tile kernels: rows of A per raster panel
  int splits;      // SKINNY: k-slices per tile, 0 = chosen from the shape
};

// Largest dynamic shared memory a CTA may opt into on sm_100.
constexpr int kMaxDynamicSmem = 232448;

// Defaults used by GEMM_PATH_AUTO and by a gemm_config field left at 0.
constexpr int kDefaultGroupRows = 2048;
// The pair tiles: 4096-row panels read 21 % fewer DRAM bytes than 2048-row
// ones with the 256 x 256 tile on the MLP up-projection shape (1-2 % faster,
// bias + GELU too), and with the 512 x 256 tile, whose waves alternate their
// direction along K, 653 MB instead of 711 MB per 8192^3 launch.
constexpr int kDefaultGroupRowsPair = 4096;
constexpr int kDefaultStagesTile64 = 4;
constexpr int kDefaultStagesTile128 = 6;
constexpr int kDefaultStagesTile256 = 4;
constexpr int kDefaultStagesPair = 6;
constexpr int kDefaultStagesTall = 4;
// 4 ties 5 on the decode shape (one k-slice) and is up to 1.95x faster than 5
// at the same count of several k-slices (offline sweep of small-M shapes)
constexpr int kDefaultStagesSkinny = 4;
// The small-M kernel takes 128-column tiles (twice the CTAs of 256-column
// ones) when they fit on the SMs in one wave, ceil(N / 128) <= SMs, with a
// 6-stage ring.  Measured (M 16-64, N 1024-14336, K 4096-16384): 1.1-1.5x
// faster than 256-column tiles there; on N = 28672 (224 narrow tiles) the
// wide ones are 1.3x faster.
constexpr int kDefaultStagesSkinnyNarrow = 6;
// The even small-M schedule: 6 stages (5 with four units per CTA, the
// deepest ring that fits), about 144-200 KiB in flight per SM.
constexpr int kDefaultStagesEven = 6;
constexpr int kDefaultStagesEven4 = 5;

struct DeviceCtx {
  int device;
  int sm_count;
  int* status;          // device address of the status word of this device
  uint64_t timeout_ns;  // limit for every device-side wait
};

// Whether kernels are launched with programmatic stream serialisation, so
// their set-up overlaps the previous kernel of the stream (TTC_PDL=0 turns it
// off for comparisons).
bool pdl_enabled();

// Fills `attr` with the programmatic-serialisation attribute when enabled;
// returns the number of attributes written (0 or 1).
int pdl_attribute(cudaLaunchAttribute* attr);

// Encode a 2-D row-major fp16 tensor map with 128-byte swizzle.
//   inner/outer: extents in elements (inner is contiguous)
//   ld: row stride in elements; box_inner/box_outer: box extents in elements
// Returns 0 or a GEMM_ERR_* code.
int encode_tmap_f16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                       uint64_t ld, uint32_t box_inner, uint32_t box_outer);

// Large-shape path: persistent warp-specialised tcgen05 kernel, one SM per
// 128 x block_n tile (GEMM_PATH_TILE), or a pair of SMs per 256 x 256
// (GEMM_PATH_TILE_PAIR) or 512 x 256 (GEMM_PATH_TILE_PAIR_TALL) tile
// (tcgen05.mma.cta_group::2).  Returns GEMM_ERR_CONFIG when no kernel was
// compiled for (kernel, block_n, stages).
int launch_tile_gemm(const GemmProblem& p, const DeviceCtx& d, const KernelConfig& c);
// Dynamic shared memory per CTA of a tile-kernel configuration (built or
// not), or -1 when (kernel, block_n) names no tile kernel.
int tile_config_smem_bytes(int kernel, int block_n, int stages);
// Tile-kernel configurations with a compiled kernel: writes up to `cap` of
// them to `out` (group_rows and splits 0) and returns how many there are.
int tile_configs_built(KernelConfig* out, int cap);

// Small-M path: swap-AB, lock-step split-K kernel.  `workspace` holds
// per-tile arrival counters and split-K partial tiles (counters must be zero
// on entry; the kernel leaves them zero).
size_t skinny_workspace_bytes(int sm_count, int m_pad);
int launch_skinny_gemm(const GemmProblem& p, const DeviceCtx& d, void* workspace,
                       size_t workspace_bytes, const KernelConfig& c);
int skinny_m_pad(int64_t M);  // MMA N used for M rows (0 if M is too large)
int skinny_config_smem_bytes(int block_n, int stages);  // -1 when block_n is not 128 / 256
int skinny_configs_built(KernelConfig* out, int cap);

// Even small-M schedule (gemm_skinny_even.cu): one CTA per SM, each with q
// whole 64-column units of B for the full K, the left_units leftover units
// split along K into left_slices slices each.  q == 0 when the shape does not
// suit it (fewer units than SMs, or more than four per SM).  `work` is the
// busiest CTA's k-blocks of 64 columns.
struct EvenPlan {
  int q;
  int ctas;
  int left_units;
  int left_slices;
  int64_t work;
};
EvenPlan even_plan(int64_t N, int64_t K, int sm_count);
size_t even_workspace_bytes(const EvenPlan& plan, int m_pad);
int launch_skinny_even(const GemmProblem& p, const DeviceCtx& d, void* workspace,
                       size_t workspace_bytes, const KernelConfig& c);
int even_config_smem_bytes(int block_n, int stages);  // -1 when block_n is not 64 q, q in 1..4
int even_configs_built(KernelConfig* out, int cap);

// The small-M kernel with its scratch in a fixed device array of the library
// (no allocation); M <= 32.  Returns GEMM_ERR_SCRATCH_LIMIT beyond.
int launch_skinny_gemm_noalloc(const GemmProblem& p, const DeviceCtx& d);

// Writes C = 0 (used when K == 0: the empty sum, and ReLU of it, is +0).
int launch_zero_fill(const GemmProblem& p);
// Writes C[i, j] = act(bias[j]) (K == 0 with a bias).
int launch_bias_act_fill(const GemmProblem& p);

}  // namespace ttc
