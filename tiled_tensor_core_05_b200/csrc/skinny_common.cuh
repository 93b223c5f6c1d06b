// Device and host helpers shared by the small-M (swap-AB) kernels of
// gemm_skinny.cu and gemm_skinny_even.cu: the epilogue's column stores, the
// TMEM read of an accumulator column, and host-side launch helpers.
#pragma once

#include <atomic>

#include "internal.h"
#include "sm100.cuh"

namespace ttc {
namespace skinny {

constexpr int kBK = 64;        // k-depth of a stage: one 128-byte swizzle row of A
constexpr int kUmmaK = 16;     // K of one tcgen05.mma kind::f16
constexpr int kSub = 128;      // columns of B per MMA (MMA M)
constexpr int kThreads = 192;  // producer, MMA, 4 epilogue warps
constexpr int kEpiWarps = 4;

__device__ __forceinline__ float4 ld_cg_f4(const float* p) {
  return __ldcg(reinterpret_cast<const float4*>(p));
}

// Column n of C (rows m < M): activation of the fp32 sums plus the column's
// bias, rounded to fp16.
template <int MP, int ACT>
__device__ __forceinline__ void store_column(const float (&v)[MP], __half* C, int M, int N,
                                             int64_t ldc, int n, const __half* bias) {
  if (n >= N) return;
  const float b = bias != nullptr ? __half2float(bias[n]) : 0.0f;
#pragma unroll
  for (int m = 0; m < MP; m += 2) {
    const float2 x = activate2<ACT>(__fadd2_rn(make_float2(v[m], v[m + 1]), splat2(b)));
    if (m < M) C[static_cast<int64_t>(m) * ldc + n] = __float2half_rn(x.x);
    if (m + 1 < M) C[static_cast<int64_t>(m + 1) * ldc + n] = __float2half_rn(x.y);
  }
}

// Column `col` of a staged MP x TW fp16 tile of C (row-major, TW columns per
// row) from this thread's MP fp32 sums: bias of column n, activation, RNE.
// Columns at or past N are left unwritten (never copied out).
template <int MP, int ACT>
__device__ __forceinline__ void stage_column(const float (&v)[MP], __half* tile, int tw, int col,
                                             int N, int n, const __half* bias) {
  if (n >= N) return;
  const float b = bias != nullptr ? __half2float(bias[n]) : 0.0f;
#pragma unroll
  for (int m = 0; m < MP; m += 2) {
    const float2 x = activate2<ACT>(__fadd2_rn(make_float2(v[m], v[m + 1]), splat2(b)));
    tile[m * tw + col] = __float2half_rn(x.x);
    tile[(m + 1) * tw + col] = __float2half_rn(x.y);
  }
}

// Copies the staged tile's rows m < M, columns n0 .. min(N, n0 + TW) - 1, to
// C with 16-byte stores (`nthreads` threads, this one `tid`); a piece that
// crosses N is stored element by element.
template <int MP, int TW>
__device__ __forceinline__ void store_staged_rows(const __half* tile, __half* C, int M, int N,
                                                  int64_t ldc, int n0, int tid, int nthreads) {
  constexpr int kPieces = TW / 8;  // 16-byte pieces per row
  const int rows = M < MP ? M : MP;
  for (int i = tid; i < rows * kPieces; i += nthreads) {
    const int m = i / kPieces;
    const int j = i - m * kPieces;
    const int n = n0 + 8 * j;
    if (n >= N) continue;
    const __half* src = tile + m * TW + 8 * j;
    __half* dst = C + static_cast<int64_t>(m) * ldc + n;
    if (n + 8 <= N) {
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    } else {
      for (int e = 0; n + e < N; ++e) dst[e] = src[e];
    }
  }
}

// Rows m0 .. m0 + R - 1 (those < M) of column n of C from R fp32 sums, as
// store_column does for all MP rows.
template <int R, int ACT>
__device__ __forceinline__ void store_rows(const float (&v)[R], __half* C, int M, int N,
                                           int64_t ldc, int n, int m0, const __half* bias) {
  if (n >= N) return;
  const float b = bias != nullptr ? __half2float(bias[n]) : 0.0f;
#pragma unroll
  for (int i = 0; i < R; i += 2) {
    const float2 x = activate2<ACT>(__fadd2_rn(make_float2(v[i], v[i + 1]), splat2(b)));
    const int m = m0 + i;
    if (m < M) C[static_cast<int64_t>(m) * ldc + n] = __float2half_rn(x.x);
    if (m + 1 < M) C[static_cast<int64_t>(m + 1) * ldc + n] = __float2half_rn(x.y);
  }
}

// MP fp32 accumulator columns of this thread's TMEM lane (executed by the
// whole warp: tcgen05.ld is warp-collective).
template <int MP>
__device__ __forceinline__ void load_accumulator(uint32_t taddr, float (&v)[MP]) {
#pragma unroll
  for (int j = 0; j < MP / 32; ++j) {
    uint32_t r[32];
    tmem_load_32x32b_x32(taddr + j * 32, r);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[j * 32 + i] = __uint_as_float(r[i]);
  }
}

// Bytes of `n` int32 arrival counters, padded to 256 bytes.
constexpr size_t counter_bytes(int n) {
  return (static_cast<size_t>(n) * sizeof(int) + 255) & ~static_cast<size_t>(255);
}

// Sets the dynamic shared-memory limit of a kernel once per device.
inline bool ensure_smem_attr(const void* func, int bytes, int device,
                             std::atomic<uint64_t>& done) {
  const uint64_t bit = 1ull << (device & 63);
  if (done.load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  done.fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

}  // namespace skinny
}  // namespace ttc
