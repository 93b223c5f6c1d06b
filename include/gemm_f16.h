/*
 * gemm_f16.h -- C ABI of libttc05: fp16 GEMM with a fused ReLU epilogue on
 * NVIDIA B200 (sm_100a).
 *
 * The operation is the one of "Writing high-performance kernels in TileLang"
 * (atlascloud.ai blog), section "Escribamos un GEMM": A (M x K) and B (K x N)
 * are row-major fp16 matrices, the products are accumulated in fp32, the
 * accumulator is clamped with max(x, 0), and the result is written to the
 * row-major fp16 matrix C (M x N), rounding to nearest-even.  The page checks
 * the kernel against relu(a @ b) with rtol = atol = 1e-2, and so do the tests
 * of this library.
 *
 * Conventions shared by every entry point
 *   - A, B, C are DEVICE pointers (cudaMalloc / torch CUDA memory) to IEEE
 *     binary16 storage on the current CUDA device.  Host pointers are rejected
 *     with GEMM_ERR_INVALID_ARG.  (The host-buffer entry points, gemm_f16_host
 *     and its companions, take host pointers instead and state their own
 *     rules.)
 *   - lda, ldb, ldc are row strides in ELEMENTS (lda >= K, ldb >= N, ldc >= N).
 *     Columns are contiguous.
 *   - Pointers must be 16-byte aligned and every ld a multiple of 8 elements
 *     (16 bytes): the tiles are moved by the Tensor Memory Accelerator, whose
 *     global strides must be multiples of 16 bytes.  Otherwise
 *     GEMM_ERR_ALIGNMENT.
 *   - M, N, K are in [0, 2^31 - 1].  M == 0 or N == 0 is a no-op that returns
 *     GEMM_OK.  K == 0 writes C = +0 (the empty sum; ReLU of it is +0 too).
 *   - The caller owns A, B and C; the library keeps no reference to them after
 *     the call.  C must not overlap A or B (undefined result).
 *   - Calls are asynchronous and stream-ordered on `stream` (0 = legacy default
 *     stream): the return value only reports argument and launch errors.
 *     Errors found on the device (a bounded wait that ran out) are recorded in
 *     a per-device status word, read with gemm_get_device_status().
 *   - Results are deterministic: the same inputs give the same bits on every
 *     run, whatever the scheduling.
 *   - Small-M problems (M <= 64) use a split-K path whose fp32 partial tiles
 *     and arrival counters live in a workspace the library allocates once per
 *     (device, stream) on first use (cudaMalloc of SMs x 256 x 64 x 4 bytes
 *     plus the counters: 9.7 MB on a 148-SM GPU) and keeps until
 *     gemm_release() or process exit, so a caller that cycles through many
 *     streams holds 9.7 MB per stream it used.  Make that first call outside
 *     CUDA-graph capture.  Two calls on different streams never share a
 *     workspace.
 *   - The device-pointer entry points can be captured in CUDA graphs once a
 *     first call on the same device and stream has run outside the capture
 *     (it creates the workspace and caches kernel attributes); replays read
 *     the buffers' current contents.
 *   - No entry point throws; errors are negative return codes.
 */
#ifndef TTC05_GEMM_F16_H
#define TTC05_GEMM_F16_H

#include <stdint.h>

#if defined(__GNUC__)
#define GEMM_API __attribute__((visibility("default")))
#else
#define GEMM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without including the CUDA headers */
typedef struct CUstream_st* gemm_stream_t;

enum gemm_status {
  GEMM_OK = 0,
  GEMM_ERR_INVALID_ARG = -1,        /* negative size, ld < cols, null or host pointer, size too large */
  GEMM_ERR_ALIGNMENT = -2,          /* pointer not 16-byte aligned or ld % 8 != 0 */
  GEMM_ERR_UNSUPPORTED_DEVICE = -3, /* current device is not compute capability 10.0 */
  GEMM_ERR_LAUNCH = -4,             /* a CUDA runtime call or kernel launch failed */
  GEMM_ERR_WORKSPACE = -5,          /* small-M workspace allocation failed */
  GEMM_ERR_DEVICE_TIMEOUT = -6,     /* reported by gemm_get_device_status */
  GEMM_ERR_SCRATCH_LIMIT = -7,      /* problem too large for gemm_relu_f16_noalloc's fixed scratch */
  GEMM_ERR_CONFIG = -8              /* gemm_f16_config: configuration not built or not valid
                                       for this problem */
};

enum gemm_path {
  GEMM_PATH_AUTO = 0,      /* choose by shape: M <= 64 -> SKINNY; fewer than 64 tiles of
                              256 x 256 -> TILE; K < 4096 (K < 6144 with GELU) ->
                              TILE_PAIR; otherwise TILE_PAIR_TALL, or TILE_PAIR when
                              the 512-row tiles leave a much emptier last wave
                              (SKINNY_EVEN only when asked for) */
  GEMM_PATH_TILE = 1,      /* persistent kernel, one SM per 128 x BN tile, BN = 64, 128 or
                              256 by the tile count (any shape) */
  GEMM_PATH_SKINNY = 2,    /* small-M kernel: swap-AB, 128 columns of B per CTA when
                              ceil(N / 128) <= SMs, else 256, streamed in lock-step,
                              split-K only when tiles < SMs (M <= 64 only) */
  GEMM_PATH_TILE_PAIR = 3, /* persistent kernel, two SMs (a CTA pair) per 256 x 256 tile
                              (any shape) */
  GEMM_PATH_TILE_PAIR_TALL = 4, /* persistent kernel, a CTA pair per 512 x 256 tile: fewer
                                   bytes staged per MAC; a single accumulator, so a tile's
                                   epilogue overlaps only the start of the next tile */
  GEMM_PATH_SKINNY_EVEN = 5 /* small-M kernel with the same bytes of B on every SM: one
                               CTA per SM with q = floor(ceil(N / 64) / SMs) whole
                               64-column units for the full K, the leftover units split
                               along K over the CTAs with a deterministic fix-up (M <= 64
                               and 1 <= q <= 4 only; GEMM_ERR_INVALID_ARG otherwise) */
};

enum gemm_activation {
  GEMM_ACT_NONE = 0,  /* identity */
  GEMM_ACT_RELU = 1,  /* max(x, 0); -0 and NaN give +0 */
  GEMM_ACT_GELU = 2   /* x * Phi(x), Phi the standard normal CDF (exact "erf" GELU) */
};

/* C = ReLU(A @ B).  "Escribamos un GEMM": the tiled fp16 matmul with the
 * max(x, 0) epilogue fused before the fp16 store.  Returns GEMM_OK or a
 * negative gemm_status. */
GEMM_API int gemm_relu_f16(const void* A, const void* B, void* C, int64_t M, int64_t N,
                           int64_t K, int64_t lda, int64_t ldb, int64_t ldc, gemm_stream_t stream);

/* C = A @ B, the same kernels without the activation (no bias). */
GEMM_API int gemm_f16(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K,
             int64_t lda, int64_t ldb, int64_t ldc, gemm_stream_t stream);

/* Either of the above with an explicit kernel choice.  relu: 0 or 1.  path:
 * a gemm_path value; GEMM_PATH_SKINNY with M > 64 returns
 * GEMM_ERR_INVALID_ARG. */
GEMM_API int gemm_f16_ex(const void* A, const void* B, void* C, int64_t M, int64_t N, int64_t K,
                int64_t lda, int64_t ldb, int64_t ldc, int relu, int path,
                gemm_stream_t stream);

/* C = act(A @ B + bias): the fused epilogue of "TileLang simplifica la
 * creación de kernels GPU de alto rendimiento" (posicionamiento-web.ar),
 * section "Fusionar operaciones para reducir viajes a memoria" -- the bias is
 * added and the activation applied to the fp32 accumulator on chip, and C is
 * written once.
 *   bias: device pointer to N fp16 values (one per column of C), 16-byte
 *         aligned, or NULL for no bias.
 *   activation: a gemm_activation value.
 *   path: a gemm_path value (as in gemm_f16_ex).
 * With K == 0 the result is C = act(bias) (act(0) = +0 without a bias).
 * Returns GEMM_OK or a negative gemm_status. */
GEMM_API int gemm_bias_act_f16(const void* A, const void* B, const void* bias, void* C,
                               int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb,
                               int64_t ldc, int activation, int path, gemm_stream_t stream);

/* C = act(op(A) @ op(B) + bias) with T.gemm's transpose_A / transpose_B
 * options ("Writing high-performance kernels in TileLang", atlascloud.ai
 * blog, section "Escribamos un GEMM"):
 *   trans_a = 0: A stored M x K row-major, lda >= K;
 *   trans_a = 1: A stored K x M row-major (M contiguous), lda >= M, op(A) = A^T;
 *   trans_b = 0: B stored K x N row-major, ldb >= N;
 *   trans_b = 1: B stored N x K row-major (K contiguous, the layout of a
 *                linear layer's weight), ldb >= K, op(B) = B^T.
 * Everything else as in gemm_bias_act_f16 (which is trans_a = trans_b = 0). */
GEMM_API int gemm_f16_general(const void* A, const void* B, const void* bias, void* C,
                              int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb,
                              int64_t ldc, int trans_a, int trans_b, int activation, int path,
                              gemm_stream_t stream);

/* One kernel configuration, for choosing configurations offline: the tuning
 * workflow of "TileLang simplifica la creación de kernels GPU de alto
 * rendimiento" (posicionamiento-web.ar) and "TileLang explicado: kernels de IA
 * escritos por mosaicos" (easyairoute.com), sections on tuning tile sizes,
 * pipeline stages and L2 ordering per GPU, done as a sweep outside the library
 * (the library itself never times or chooses among these at run time).
 * A field left at 0 takes the value GEMM_PATH_AUTO would use. */
typedef struct gemm_config {
  int32_t kernel;     /* GEMM_PATH_TILE, _TILE_PAIR, _TILE_PAIR_TALL, _SKINNY or
                         _SKINNY_EVEN (not AUTO) */
  int32_t block_n;    /* output columns per tile: 64, 128 or 256 for GEMM_PATH_TILE; 128
                         or 256 for GEMM_PATH_SKINNY; 256 (the only width) for the pair
                         kernels; for GEMM_PATH_SKINNY_EVEN the main columns per CTA,
                         64 q (fixed by the shape: 0 takes it, another value is
                         GEMM_ERR_CONFIG) */
  int32_t stages;     /* depth of the shared-memory operand ring (k-blocks of 64 in flight) */
  int32_t group_rows; /* tile kernels: the L2 grouping of the tile order.  > 0: rows of
                         op(A) per row panel (tiles walked column by column inside
                         it); < 0: minus the columns of op(B) per column panel (tiles
                         walked row by row inside it); odd panels are walked in
                         reverse; 0 = the default (4096 for the pair kernels, 2048
                         for GEMM_PATH_TILE).  Must be 0 for the small-M kernels */
  int32_t splits;     /* GEMM_PATH_SKINNY: k-slices per column tile, 1 <= splits <=
                         ceil(K / 64) and splits * ceil(N / block_n) <= the SM count when
                         > 1; 0 = chosen from the shape.  Must be 0 for the tile kernels
                         and GEMM_PATH_SKINNY_EVEN */
} gemm_config;

/* gemm_f16_general with the kernel configuration `cfg` instead of a path.
 * Results are the same operation: every configuration meets the same
 * accuracy, though fp32 sums in another order may differ in the last bits.
 * Returns GEMM_ERR_CONFIG (and launches nothing) when `cfg` names no compiled
 * kernel (see gemm_config_list) or does not fit the problem (GEMM_PATH_SKINNY
 * with M > 64, a splits value out of range), GEMM_ERR_INVALID_ARG for a null
 * `cfg`; otherwise as gemm_f16_general. */
GEMM_API int gemm_f16_config(const void* A, const void* B, const void* bias, void* C, int64_t M,
                             int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc,
                             int trans_a, int trans_b, int activation, const gemm_config* cfg,
                             gemm_stream_t stream);

/* Dynamic shared memory per CTA (bytes) that the kernel, block_n and stages of
 * `cfg` need, whether or not that configuration is compiled (stages 0 = the
 * default).  A configuration fits a B200 when this is <= 232448.  Returns
 * GEMM_ERR_CONFIG when kernel / block_n name no kernel (block_n must be given
 * for GEMM_PATH_TILE and GEMM_PATH_SKINNY).  Pure host function. */
GEMM_API int gemm_config_smem_bytes(const gemm_config* cfg);

/* The compiled configurations (kernel, block_n, stages; group_rows and
 * splits 0, free at call time): every stage count from 3 up to the shared
 * memory budget of each tile shape (up to 6 for the small-M kernel's
 * streaming ring).  Writes up to `capacity` of them to `out`
 * (may be null when capacity is 0) and returns how many there are.  Pure host
 * function. */
GEMM_API int gemm_config_list(gemm_config* out, int capacity);

/* The configuration GEMM_PATH_AUTO takes for this problem on the current
 * device (all fields resolved).  Returns GEMM_OK, or a negative gemm_status
 * (invalid sizes or activation, no sm_100 device). */
GEMM_API int gemm_auto_config(int64_t M, int64_t N, int64_t K, int activation, gemm_config* out);

/* The path GEMM_PATH_AUTO takes for this shape with ReLU (or no activation)
 * on a 148-SM B200 (pure host function; GEMM_PATH_AUTO itself uses the SM
 * count of the current device, and with GELU keeps the 256-row pair tile up
 * to K < 6144, where ReLU switches to the 512-row tile from K = 4096). */
GEMM_API int gemm_select_path(int64_t M, int64_t N, int64_t K);

/* Human-readable text for a gemm_status value (static storage). */
GEMM_API const char* gemm_status_string(int status);

/* Synchronises `stream`, then reports and clears the status word of the
 * current device: *device_status = 0 if every kernel finished normally, else
 * the code of the first bounded wait that gave up (non-zero; the kernel that
 * gave up returned without completing its output).  After a non-zero status
 * the small-M workspaces of the device are re-zeroed.  Returns GEMM_OK, or
 * GEMM_ERR_LAUNCH if a CUDA call failed. */
GEMM_API int gemm_get_device_status(gemm_stream_t stream, int* device_status);

/* Failure-detection self test: launches one CTA that waits, with the same
 * bounded wait as the GEMM kernels and a limit of `timeout_ns`, on an mbarrier
 * nothing will ever arrive on.  The wait runs out, the kernel records a
 * timeout in the status word and returns normally; the context stays usable.
 * Synchronises `stream` and stores the status word (then clears it) in
 * *device_status.  Returns GEMM_OK or a negative gemm_status. */
GEMM_API int gemm_selftest_wait_timeout(int64_t timeout_ns, gemm_stream_t stream, int* device_status);

/* C = ReLU(A @ B) for callers that must not allocate device memory.
 *
 * No counterpart in the pages: this is an interface addition, not part of the
 * method.  gemm_relu_f16 lazily cudaMalloc's a workspace for its small-M
 * (split-K) kernel on the first call per (device, stream).  Some callers
 * cannot allow that: plugins whose enqueue step is forbidden to allocate,
 * processes whose device memory is owned and accounted for by a pool
 * allocator, and latency-critical loops where cudaMalloc's implicit device
 * synchronisation would stall other work.  This entry point runs the same
 * small-M kernel, but keeps its scratch (fp32 partial tiles and per-tile
 * arrival counters) in a fixed array that is part of the library image: every
 * GPU that loads the library holds those 5,243,648 bytes (5 MiB) until the
 * process exits.  It calls no cudaMalloc, cudaFree or other allocating routine.
 *
 *   - Arguments, layout and ownership are those of gemm_relu_f16: device
 *     pointers, row-major fp16, ld in elements (multiples of 8), 16-byte
 *     aligned pointers; the caller still provides A, B and C.
 *   - Limit: M <= 32 (any N and K up to 2^31 - 1).  Larger M returns
 *     GEMM_ERR_SCRATCH_LIMIT and launches nothing.  M == 0 or N == 0 is a
 *     no-op; K == 0 writes C = +0.
 *   - The first call on each device looks up the device address of the array
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.
 *   - Every call on a device shares the one array and it keeps the last
 *     call's contents; each call clears the arrival counters on `stream`
 *     before its kernel.  Calls whose kernels overlap on the GPU (other
 *     streams, other host threads) race on the array and give wrong results:
 *     serialise them.
 * Returns GEMM_OK or a negative gemm_status. */
GEMM_API int gemm_relu_f16_noalloc(const void* A, const void* B, void* C, int64_t M, int64_t N,
                                   int64_t K, int64_t lda, int64_t ldb, int64_t ldc,
                                   gemm_stream_t stream);

/* ---------------------------------------------------------------------------
 * Host-buffer entry points.  C = act(A @ B + bias), the operation of
 * gemm_bias_act_f16 ("Writing high-performance kernels in TileLang",
 * atlascloud.ai blog, section "Escribamos un GEMM"; the bias + activation
 * epilogue of "TileLang simplifica la creación de kernels GPU de alto
 * rendimiento", posicionamiento-web.ar, section "Fusionar operaciones para
 * reducir viajes a memoria"), with A, B, bias and C in HOST memory.  The pages
 * run the kernel on device tensors only; moving the data is an interface
 * addition.
 *
 *   - A (M x K, lda >= K), B (K x N, ldb >= N) and C (M x N, ldc >= N) are
 *     row-major fp16 host arrays, ld in elements; bias is N fp16 values or
 *     NULL.  Host pointers have no alignment or ld rule (the library copies
 *     them into 16-byte-aligned device rows).  Device or managed pointers are
 *     refused with GEMM_ERR_INVALID_ARG.
 *   - Page-locked host memory (cudaHostAlloc, cudaHostRegister, torch's
 *     pin_memory) lets the copies run asynchronously and overlap one another
 *     and the kernels.  Pageable memory gives the same result, but the driver
 *     stages it and the call blocks for its copies.
 *   - The library copies one operand whole and streams the other, and C, in
 *     panels (the plan of gemm_host_plan_for): panel i's kernel runs on
 *     `stream` as soon as its rows (or columns) are on the device, and its
 *     part of C is copied back while later panels are still coming in.  The
 *     kernel of each panel is the one GEMM_PATH_AUTO takes for the panel's
 *     shape, so the bits may differ in the last place from one
 *     gemm_bias_act_f16 over the whole problem (the same accuracy).
 *   - Stream-ordered and asynchronous: the work starts after earlier work on
 *     `stream`, later work on `stream` starts after C is in host memory, and
 *     the call returns once everything is enqueued.  Read C, and reuse A, B
 *     and bias, only after synchronising `stream`.
 *   - Device memory: per (device, stream) the library keeps device copies of
 *     A, B, C and bias (16-byte rows), two copy streams and their events,
 *     allocated on first use and grown when a larger problem comes
 *     (cudaMalloc; growing waits for the earlier calls' work first), until
 *     gemm_host_release() or process exit.  A call's copies into them start
 *     after the previous call on the same staging has finished with them.  Not for use inside CUDA-graph
 *     capture.  Calls on one stream from several host threads at once are
 *     not supported.
 *   - M == 0 or N == 0 is a no-op; K == 0 writes C = act(bias) (+0 without a
 *     bias), and A and B are not read.
 * Returns GEMM_OK or a negative gemm_status (GEMM_ERR_WORKSPACE when the
 * device copies cannot be allocated). */
GEMM_API int gemm_f16_host(const void* A, const void* B, const void* bias, void* C, int64_t M,
                           int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc,
                           int activation, gemm_stream_t stream);

/* C = ReLU(A @ B) with host buffers: gemm_f16_host with no bias and
 * GEMM_ACT_RELU, the signature of gemm_relu_f16. */
GEMM_API int gemm_relu_f16_host(const void* A, const void* B, void* C, int64_t M, int64_t N,
                                int64_t K, int64_t lda, int64_t ldb, int64_t ldc,
                                gemm_stream_t stream);

enum gemm_host_split {
  GEMM_HOST_SPLIT_ROWS = 0, /* B copied whole; A and C in panels of rows */
  GEMM_HOST_SPLIT_COLS = 1  /* A copied whole; B and C in panels of columns */
};

/* How gemm_f16_host splits an M x N x K problem. */
typedef struct gemm_host_plan {
  int32_t split;         /* a gemm_host_split value */
  int32_t panels;        /* number of panels, 1..16 */
  int64_t panel_extent;  /* rows (multiple of 512) or columns (multiple of 256, at least
                            2048) per panel, or all of M or N; the last panel possibly
                            fewer */
  double estimate_bytes; /* the plan's copy-time estimate, as bytes over one direction of
                            the host link: max(first + streamed + C / panels,
                            first + streamed / panels + C) */
} gemm_host_plan;

/* The plan gemm_f16_host takes: of the two splits, the one with the smaller
 * estimate (rows on a tie); panels of about 32 MiB of streamed bytes (operand
 * + C), at most 16, whole 512-row or 256-column tiles each, and column panels
 * at least 2048 columns wide (narrower strided copies are slow).  Pure host
 * function.  Returns GEMM_OK, or GEMM_ERR_INVALID_ARG for a null `out`,
 * M < 1, N < 1 or K < 0. */
GEMM_API int gemm_host_plan_for(int64_t M, int64_t N, int64_t K, gemm_host_plan* out);

/* gemm_f16_host with the caller's plan instead of gemm_host_plan_for's, for
 * choosing plans offline (as gemm_f16_config does for kernels).  Only
 * plan->split and plan->panel_extent are read: the split, and the rows or
 * columns per panel (clamped to M or N).  GEMM_ERR_CONFIG when the split is
 * not a gemm_host_split value, panel_extent < 1, a column panel is not a
 * multiple of 8 columns (unless it covers all N), or there would be more
 * than 16 panels; GEMM_ERR_INVALID_ARG for a null plan; otherwise as
 * gemm_f16_host. */
GEMM_API int gemm_f16_host_planned(const void* A, const void* B, const void* bias, void* C,
                                   int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb,
                                   int64_t ldc, int activation, const gemm_host_plan* plan,
                                   gemm_stream_t stream);

/* Frees the device copies, copy streams and events of every (device, stream)
 * gemm_f16_host has used, after waiting for the work of each one's last call
 * (on the library's own copy stream and event: the callers' streams need not
 * exist any more).  Not to be called while another thread is inside
 * gemm_f16_host.  Returns GEMM_OK or GEMM_ERR_LAUNCH. */
GEMM_API int gemm_host_release(void);

/* Frees every device buffer the library holds: the small-M workspaces of all
 * (device, stream) pairs and the host-buffer staging (gemm_host_release).  It
 * first waits for all work on each device that holds a workspace
 * (cudaDeviceSynchronize), since a workspace may still be in use by a kernel
 * in flight on a stream the caller no longer has.  The next small-M call
 * allocates a fresh workspace.  Not to be called while another thread is
 * inside an entry point of the library, nor during CUDA-graph capture, nor
 * while a captured graph that uses a workspace may still be launched.
 * Returns GEMM_OK or GEMM_ERR_LAUNCH. */
GEMM_API int gemm_release(void);

/* y[i] = act(x[i]) for n fp32 values in device memory, with the exact code
 * the GEMM epilogues use (GELU: x * Phi(x), Phi from Abramowitz & Stegun
 * 7.1.26, |Phi error| <= 1e-6).  For checking the activations on their own.
 * Asynchronous on `stream`. */
GEMM_API int gemm_activation_f32(const void* x, void* y, int64_t n, int activation,
                                 gemm_stream_t stream);

/* Measurement tool, not part of the GEMM: reads n_bytes of device memory at
 * `src` once, with 16-byte streaming loads spread over the whole GPU, and
 * stores the XOR of all its 32-bit words in *sink (a device pointer to 4
 * bytes, zeroed first on `stream`).  Timed over a buffer larger than L2 it
 * gives the streaming-read bandwidth that bounds the small-M kernel, which
 * reads B once.  It is the bandwidth-bound environment check of "TileLang
 * simplifica la creación de kernels GPU de alto rendimiento"
 * (posicionamiento-web.ar), section "Del entorno CUDA a la primera medición
 * reproducible" (a vector sum there), reduced to its reads.
 *   - src 16-byte aligned, n_bytes a multiple of 16 (0 stores 0); sink
 *     4-byte aligned; both device memory of the current device.
 *   - Asynchronous on `stream`.  Returns GEMM_OK or a negative gemm_status. */
GEMM_API int gemm_read_probe(const void* src, int64_t n_bytes, void* sink, gemm_stream_t stream);

/* Version of this ABI (major * 10000 + minor * 100 + patch). */
GEMM_API int gemm_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TTC05_GEMM_F16_H */
