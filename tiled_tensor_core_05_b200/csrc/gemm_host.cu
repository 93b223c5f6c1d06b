// Host-buffer entry points of libttc05 (gemm_f16_host, gemm_relu_f16_host):
// the fused GEMM + activation of "Writing high-performance kernels in
// TileLang" (atlascloud.ai blog), section "Escribamos un GEMM", for operands
// and result in host memory.  The pages only run the kernel on device
// tensors; moving the data in and out is an interface addition.
//
// The copies over the host link (tens of GB/s) take several times longer than
// the product itself on a B200, so they are pipelined rather than run one
// after the other:
//   1. the operand that every panel needs is copied whole (B when the output
//      is cut into row panels, A when it is cut into column panels);
//   2. the other operand is copied panel by panel on a host-to-device stream;
//   3. as each panel lands, the caller's stream runs the library's kernel on
//      it (the same AUTO path as gemm_f16_general, on the panel's shape);
//   4. a device-to-host stream copies each finished panel of C back while the
//      next panels are still coming in (the link carries both directions at
//      once).
// The split (rows or columns) and the panel count come from a plan that
// minimises an estimate of the copy time (gemm_host_plan_for).  Every step is
// ordered after earlier work on the caller's stream and the caller's stream
// waits for the last copy, so the entry points keep stream order.
#include <cuda_runtime.h>
#include <stdint.h>

#include <memory>
#include <mutex>
#include <vector>

#include "../../include/gemm_f16.h"

namespace ttc {
namespace {

constexpr int kMaxPanels = 16;
constexpr int64_t kRowUnit = 512;  // rows of the 512-row pair tile
constexpr int64_t kColUnit = 256;  // columns of the widest tile
// Column panels are copied as strided runs, one per row of the panel; runs
// of 2048 columns (4 KiB) or more keep the copy near the contiguous rate on
// a B200's host link, narrower ones fall well below it (measured: the MLP
// up-projection 8192 x 14336 x 4096 end to end in 6.9 ms with 1024-column
// panels, 6.2 ms with 2048).
constexpr int64_t kMinColPanel = 2048;
constexpr double kPanelTargetBytes = 32.0 * 1024 * 1024;  // streamed bytes per panel

int64_t round8(int64_t x) { return (x + 7) / 8 * 8; }

// One candidate split: `first` bytes go in whole, `streamed` bytes and the
// `out` bytes of C in `panels` pieces.  Copy time in units of bytes over the
// link, one direction each way: the host-to-device stream carries first +
// streamed, the device-to-host stream starts after the first panel is in and
// cannot end before the last panel's product.
double copy_estimate(double first, double streamed, double out, int panels) {
  const double p = panels;
  const double in_done = first + streamed + out / p;   // last panel in, then its C out
  const double out_done = first + streamed / p + out;  // C copies back-to-back after panel 1
  return in_done > out_done ? in_done : out_done;
}

void plan_split(int64_t dim, int64_t unit, int64_t min_extent, double first, double streamed,
                double out, gemm_host_plan* p) {
  int panels = static_cast<int>((streamed + out) / kPanelTargetBytes);
  if (panels < 1) panels = 1;
  if (panels > kMaxPanels) panels = kMaxPanels;
  const int64_t units = (dim + unit - 1) / unit;
  if (panels > units) panels = static_cast<int>(units);
  int64_t extent = ((dim + panels - 1) / panels + unit - 1) / unit * unit;
  if (extent < min_extent) extent = min_extent;
  if (extent > dim) extent = dim;
  p->panels = static_cast<int32_t>((dim + extent - 1) / extent);
  p->panel_extent = extent;
  p->estimate_bytes = copy_estimate(first, streamed, out, p->panels);
}

int make_plan(int64_t M, int64_t N, int64_t K, gemm_host_plan* out) {
  const double a = 2.0 * M * K, b = 2.0 * K * N, c = 2.0 * M * N;
  gemm_host_plan rows{}, cols{};
  rows.split = GEMM_HOST_SPLIT_ROWS;
  plan_split(M, kRowUnit, kRowUnit, b, a, c, &rows);
  cols.split = GEMM_HOST_SPLIT_COLS;
  plan_split(N, kColUnit, kMinColPanel, a, b, c, &cols);
  // rows on a tie: their copies are contiguous runs of memory
  *out = cols.estimate_bytes < rows.estimate_bytes ? cols : rows;
  return GEMM_OK;
}

// Host memory only: pageable (unregistered) or page-locked.  Device and
// managed memory are refused.
bool is_host_memory(const void* p) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return attr.type == cudaMemoryTypeHost || attr.type == cudaMemoryTypeUnregistered;
}

// Staging of one (device, caller stream): device copies of A, B, C and the
// bias (grow-only), two copy streams and the events that order them.  Every
// call ends with its device-to-host stream waiting for its last kernel, so
// `join` (recorded there last) completes only once nothing of the call uses
// the buffers any more; the next call's copies wait for it, and growing or
// freeing the buffers waits for it, without touching the caller's stream
// (whose handle may be gone by then).
struct Staging {
  int device = -1;
  cudaStream_t user = nullptr;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t fork = nullptr, tail = nullptr, join = nullptr;
  cudaEvent_t in[kMaxPanels] = {}, out[kMaxPanels] = {};
  void* buf[4] = {};  // A, B, C, bias
  size_t cap[4] = {};
  std::mutex m;

  bool init() {
    if (cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&tail, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess)
      return false;
    for (int i = 0; i < kMaxPanels; ++i)
      if (cudaEventCreateWithFlags(&in[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&out[i], cudaEventDisableTiming) != cudaSuccess)
        return false;
    return true;
  }

  // Frees everything, once the last call's work is done.
  void release() {
    if (join != nullptr) cudaEventSynchronize(join);
    if (h2d != nullptr) cudaStreamSynchronize(h2d);
    if (d2h != nullptr) cudaStreamSynchronize(d2h);
    for (int i = 0; i < 4; ++i) {
      if (buf[i] != nullptr) cudaFree(buf[i]);
      buf[i] = nullptr;
      cap[i] = 0;
    }
    for (int i = 0; i < kMaxPanels; ++i) {
      if (in[i] != nullptr) cudaEventDestroy(in[i]);
      if (out[i] != nullptr) cudaEventDestroy(out[i]);
      in[i] = out[i] = nullptr;
    }
    if (fork != nullptr) cudaEventDestroy(fork);
    if (tail != nullptr) cudaEventDestroy(tail);
    if (join != nullptr) cudaEventDestroy(join);
    if (h2d != nullptr) cudaStreamDestroy(h2d);
    if (d2h != nullptr) cudaStreamDestroy(d2h);
    fork = tail = join = nullptr;
    h2d = d2h = nullptr;
  }

  // Buffer `i` of at least `bytes`.  Growing waits for the earlier calls'
  // work (their `join`) before freeing the old one.
  int reserve(int i, size_t bytes) {
    if (bytes == 0 || cap[i] >= bytes) return GEMM_OK;
    if (buf[i] != nullptr) {
      if (cudaEventSynchronize(join) != cudaSuccess) return GEMM_ERR_LAUNCH;
      cudaFree(buf[i]);
      buf[i] = nullptr;
      cap[i] = 0;
    }
    if (cudaMalloc(&buf[i], bytes) != cudaSuccess) {
      cudaGetLastError();
      buf[i] = nullptr;
      return GEMM_ERR_WORKSPACE;
    }
    cap[i] = bytes;
    return GEMM_OK;
  }
};

std::mutex g_staging_mutex;
std::vector<std::unique_ptr<Staging>> g_staging;

int get_staging(int device, cudaStream_t user, Staging** out) {
  std::lock_guard<std::mutex> lock(g_staging_mutex);
  for (auto& s : g_staging)
    if (s->device == device && s->user == user) {
      *out = s.get();
      return GEMM_OK;
    }
  auto s = std::make_unique<Staging>();
  s->device = device;
  s->user = user;
  if (!s->init()) {
    cudaGetLastError();
    s->release();
    return GEMM_ERR_LAUNCH;
  }
  *out = s.get();
  g_staging.push_back(std::move(s));
  return GEMM_OK;
}

// 2-D copy of `rows` runs of `width` bytes; nothing for an empty one.
cudaError_t copy2d(void* dst, int64_t dpitch, const void* src, int64_t spitch, int64_t width,
                   int64_t rows, cudaMemcpyKind kind, cudaStream_t s) {
  if (width <= 0 || rows <= 0) return cudaSuccess;
  return cudaMemcpy2DAsync(dst, static_cast<size_t>(dpitch), src, static_cast<size_t>(spitch),
                           static_cast<size_t>(width), static_cast<size_t>(rows), kind, s);
}

// A caller's plan: a split, and panels of whole 8-element column groups
// (16-byte device addresses) when the split is by columns; at most
// kMaxPanels of them.
int check_plan(const gemm_host_plan& p, int64_t M, int64_t N) {
  if (p.split != GEMM_HOST_SPLIT_ROWS && p.split != GEMM_HOST_SPLIT_COLS) return GEMM_ERR_CONFIG;
  const int64_t dim = p.split == GEMM_HOST_SPLIT_ROWS ? M : N;
  if (p.panel_extent < 1) return GEMM_ERR_CONFIG;
  if (p.split == GEMM_HOST_SPLIT_COLS && p.panel_extent < N && p.panel_extent % 8 != 0)
    return GEMM_ERR_CONFIG;
  if ((dim + p.panel_extent - 1) / p.panel_extent > kMaxPanels) return GEMM_ERR_CONFIG;
  return GEMM_OK;
}

int run_host(const void* A, const void* B, const void* bias, void* C, int64_t M, int64_t N,
             int64_t K, int64_t lda, int64_t ldb, int64_t ldc, int activation,
             const gemm_host_plan* given, gemm_stream_t stream_handle) {
  if (M < 0 || N < 0 || K < 0) return GEMM_ERR_INVALID_ARG;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return GEMM_ERR_INVALID_ARG;
  if (activation != GEMM_ACT_NONE && activation != GEMM_ACT_RELU &&
      activation != GEMM_ACT_GELU)
    return GEMM_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return GEMM_OK;
  if (given != nullptr && check_plan(*given, M, N) != GEMM_OK) return GEMM_ERR_CONFIG;
  if (C == nullptr || ldc < N) return GEMM_ERR_INVALID_ARG;
  if (K > 0 && (A == nullptr || B == nullptr || lda < K || ldb < N)) return GEMM_ERR_INVALID_ARG;
  if (!is_host_memory(C) || (bias != nullptr && !is_host_memory(bias)) ||
      (K > 0 && (!is_host_memory(A) || !is_host_memory(B))))
    return GEMM_ERR_INVALID_ARG;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return GEMM_ERR_LAUNCH;
  cudaStream_t user = reinterpret_cast<cudaStream_t>(stream_handle);
  Staging* st = nullptr;
  int rc = get_staging(device, user, &st);
  if (rc != GEMM_OK) return rc;
  std::lock_guard<std::mutex> lock(st->m);

  // device layout: packed rows, each ld rounded up to 8 elements (16 bytes)
  const int64_t lda_d = round8(K), ldb_d = round8(N), ldc_d = round8(N);
  rc = st->reserve(0, static_cast<size_t>(M * lda_d * 2));
  if (rc == GEMM_OK) rc = st->reserve(1, static_cast<size_t>(K * ldb_d * 2));
  if (rc == GEMM_OK) rc = st->reserve(2, static_cast<size_t>(M * ldc_d * 2));
  if (rc == GEMM_OK && bias != nullptr) rc = st->reserve(3, static_cast<size_t>(round8(N) * 2));
  if (rc != GEMM_OK) return rc;
  uint16_t* dA = static_cast<uint16_t*>(st->buf[0]);
  uint16_t* dB = static_cast<uint16_t*>(st->buf[1]);
  uint16_t* dC = static_cast<uint16_t*>(st->buf[2]);
  uint16_t* dbias = bias != nullptr ? static_cast<uint16_t*>(st->buf[3]) : nullptr;
  const char* hA = static_cast<const char*>(A);
  const char* hB = static_cast<const char*>(B);
  char* hC = static_cast<char*>(C);

  gemm_host_plan plan;
  if (given != nullptr) {
    plan = *given;
    const int64_t d = plan.split == GEMM_HOST_SPLIT_ROWS ? M : N;
    if (plan.panel_extent > d) plan.panel_extent = d;
    plan.panels = static_cast<int32_t>((d + plan.panel_extent - 1) / plan.panel_extent);
  } else {
    make_plan(M, N, K, &plan);
  }
  const bool by_rows = plan.split == GEMM_HOST_SPLIT_ROWS;
  const int64_t dim = by_rows ? M : N;

  // fork: both copy streams start after the caller's earlier work, and the
  // copies into the buffers after the previous call's last use of them
  bool ok = cudaEventRecord(st->fork, user) == cudaSuccess &&
            cudaStreamWaitEvent(st->h2d, st->fork, 0) == cudaSuccess &&
            cudaStreamWaitEvent(st->h2d, st->join, 0) == cudaSuccess &&
            cudaStreamWaitEvent(st->d2h, st->fork, 0) == cudaSuccess;
  int gemm_rc = GEMM_OK;
  if (ok && bias != nullptr)
    ok = cudaMemcpyAsync(dbias, bias, static_cast<size_t>(N * 2), cudaMemcpyHostToDevice,
                         st->h2d) == cudaSuccess;
  // the operand every panel needs, whole
  if (ok)
    ok = by_rows ? copy2d(dB, ldb_d * 2, hB, ldb * 2, N * 2, K, cudaMemcpyHostToDevice,
                          st->h2d) == cudaSuccess
                 : copy2d(dA, lda_d * 2, hA, lda * 2, K * 2, M, cudaMemcpyHostToDevice,
                          st->h2d) == cudaSuccess;
  for (int i = 0; ok && i < plan.panels; ++i) {
    const int64_t lo = i * plan.panel_extent;
    const int64_t hi = lo + plan.panel_extent < dim ? lo + plan.panel_extent : dim;
    const int64_t ext = hi - lo;
    if (by_rows) {
      ok = copy2d(dA + lo * lda_d, lda_d * 2, hA + lo * lda * 2, lda * 2, K * 2, ext,
                  cudaMemcpyHostToDevice, st->h2d) == cudaSuccess;
    } else {
      ok = copy2d(dB + lo, ldb_d * 2, hB + lo * 2, ldb * 2, ext * 2, K, cudaMemcpyHostToDevice,
                  st->h2d) == cudaSuccess;
    }
    ok = ok && cudaEventRecord(st->in[i], st->h2d) == cudaSuccess &&
         cudaStreamWaitEvent(user, st->in[i], 0) == cudaSuccess;
    if (!ok) break;
    gemm_rc = by_rows ? gemm_f16_general(dA + lo * lda_d, dB, dbias, dC + lo * ldc_d, ext, N, K,
                                         lda_d, ldb_d, ldc_d, 0, 0, activation, GEMM_PATH_AUTO,
                                         stream_handle)
                      : gemm_f16_general(dA, dB + lo, dbias != nullptr ? dbias + lo : nullptr,
                                         dC + lo, M, ext, K, lda_d, ldb_d, ldc_d, 0, 0,
                                         activation, GEMM_PATH_AUTO, stream_handle);
    ok = gemm_rc == GEMM_OK && cudaEventRecord(st->out[i], user) == cudaSuccess &&
         cudaStreamWaitEvent(st->d2h, st->out[i], 0) == cudaSuccess;
    if (!ok) break;
    ok = by_rows ? copy2d(hC + lo * ldc * 2, ldc * 2, dC + lo * ldc_d, ldc_d * 2, N * 2, ext,
                          cudaMemcpyDeviceToHost, st->d2h) == cudaSuccess
                 : copy2d(hC + lo * 2, ldc * 2, dC + lo, ldc_d * 2, ext * 2, M,
                          cudaMemcpyDeviceToHost, st->d2h) == cudaSuccess;
  }
  // join, also after a failure: the device-to-host stream waits for the
  // last kernel enqueued on the caller's stream, `join` marks the end of
  // everything, and later work on the caller's stream waits for it
  const bool joined = cudaEventRecord(st->tail, user) == cudaSuccess &&
                      cudaStreamWaitEvent(st->d2h, st->tail, 0) == cudaSuccess &&
                      cudaEventRecord(st->join, st->d2h) == cudaSuccess &&
                      cudaStreamWaitEvent(user, st->join, 0) == cudaSuccess;
  if (gemm_rc != GEMM_OK) return gemm_rc;
  if (!ok || !joined) {
    cudaGetLastError();
    return GEMM_ERR_LAUNCH;
  }
  return GEMM_OK;
}

}  // namespace
}  // namespace ttc

extern "C" {

int gemm_host_plan_for(int64_t M, int64_t N, int64_t K, gemm_host_plan* out) {
  if (out == nullptr || M < 1 || N < 1 || K < 0) return GEMM_ERR_INVALID_ARG;
  return ttc::make_plan(M, N, K, out);
}

int gemm_f16_host(const void* A, const void* B, const void* bias, void* C, int64_t M, int64_t N,
                  int64_t K, int64_t lda, int64_t ldb, int64_t ldc, int activation,
                  gemm_stream_t stream) {
  return ttc::run_host(A, B, bias, C, M, N, K, lda, ldb, ldc, activation, nullptr, stream);
}

int gemm_f16_host_planned(const void* A, const void* B, const void* bias, void* C, int64_t M,
                          int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc,
                          int activation, const gemm_host_plan* plan, gemm_stream_t stream) {
  if (plan == nullptr) return GEMM_ERR_INVALID_ARG;
  return ttc::run_host(A, B, bias, C, M, N, K, lda, ldb, ldc, activation, plan, stream);
}

int gemm_relu_f16_host(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K,
                       int64_t lda, int64_t ldb, int64_t ldc, gemm_stream_t stream) {
  return ttc::run_host(A, B, nullptr, C, M, N, K, lda, ldb, ldc, GEMM_ACT_RELU, nullptr,
                       stream);
}

int gemm_host_release(void) {
  std::lock_guard<std::mutex> lock(ttc::g_staging_mutex);
  int prev = 0;
  if (cudaGetDevice(&prev) != cudaSuccess) return GEMM_ERR_LAUNCH;
  for (auto& s : ttc::g_staging) {
    std::lock_guard<std::mutex> l(s->m);
    cudaSetDevice(s->device);
    s->release();
  }
  ttc::g_staging.clear();
  cudaSetDevice(prev);
  return GEMM_OK;
}

}  // extern "C"
