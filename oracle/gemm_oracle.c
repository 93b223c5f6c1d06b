/*
 * CPU oracle for the fused fp16 GEMM + ReLU,  C = ReLU(A @ B).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker, not the product: only
 * the test suite, the smoke check and the benchmark's CPU-baseline leg load it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes follows "Writing high-performance kernels in TileLang"
 * (atlascloud.ai blog), section "Escribamos un GEMM": A is M x K, B is K x N,
 * both row-major fp16; the product is accumulated at (at least) fp32; the
 * accumulator is clamped with max(x, 0); the result is written to the fp16
 * matrix C.  The page checks the kernel against relu(a @ b) with
 * rtol = atol = 1e-2.
 *
 * Readings taken where the page is silent (each one is listed in the design
 * notes):
 *   - The sum is carried in fp64 in ascending k.  Every fp16 x fp16 product is
 *     exact in fp64 (11-bit x 11-bit significands), so the only rounding
 *     before the final one is the fp64 addition, far below the fp16 ulp.
 *   - ReLU is applied to the unrounded fp64 sum, then the value is rounded
 *     once, directly from fp64 to fp16, round-to-nearest-even (no double
 *     rounding through fp32).  Rounding is monotone and odd, so ReLU before or
 *     after the rounding gives the same fp16 value.
 *   - ReLU maps every x that is not > 0 (negative values, -0 and NaN) to +0.
 *   - Overflow rounds to +-Inf, as IEEE round-to-nearest prescribes.
 *   - Out-of-range elements do not exist here: the oracle only reads A[i,k]
 *     for i < M, k < K and B[k,j] for k < K, j < N, with row strides lda/ldb
 *     and writes C[i,j] for i < M, j < N with row stride ldc.
 *
 * Loop order: the full-matrix routine walks i, then k, then j with an fp64 row
 * accumulator.  Each element C[i,j] still receives exactly the sequence
 * 0 + a[i,0]b[0,j] + a[i,1]b[1,j] + ... in ascending k, the same arithmetic as
 * the one-element routine below; only the order in which different elements
 * are visited differs.  No blocking, no reassociation.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- IEEE binary16 <-> binary64, written from the format definition ---- */

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * exponent 0: subnormal, value = fraction * 2^-24
 * exponent 31: Inf (fraction 0) or NaN
 * otherwise: value = (1024 + fraction) * 2^(exponent - 25)               */
double oracle_f16_to_f64(uint16_t h)
{
    const unsigned sign = (h >> 15) & 1u;
    const unsigned expo = (h >> 10) & 0x1fu;
    const unsigned frac = h & 0x3ffu;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -24);
    else if (expo == 31)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(1024u + frac), (int)expo - 25);
    return sign ? -v : v;
}

/* Round-half-to-even of a non-negative double that is < 2^52, by hand. */
static double round_half_even(double s)
{
    double fl = floor(s);
    double diff = s - fl; /* exact: s and fl share the exponent range */
    if (diff > 0.5) return fl + 1.0;
    if (diff < 0.5) return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* binary64 -> binary16, round to nearest, ties to even. */
uint16_t oracle_f64_to_f16(double x)
{
    if (isnan(x)) return (uint16_t)0x7e00u;
    const uint16_t sign = signbit(x) ? (uint16_t)0x8000u : (uint16_t)0u;
    const double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7c00u);
    int e2;
    (void)frexp(a, &e2);           /* a = f * 2^e2 with f in [0.5, 1)      */
    const int E = e2 - 1;          /* a in [2^E, 2^(E+1))                   */
    if (E > 15) return (uint16_t)(sign | 0x7c00u);
    /* spacing of binary16 numbers around a: 2^(E-10) for normals, 2^-24 below */
    const int qexp = (E < -14) ? -24 : E - 10;
    const double m = round_half_even(ldexp(a, -qexp)); /* a / spacing, rounded */
    if (qexp == -24) {
        /* subnormal range; m == 1024 lands exactly on the smallest normal,
         * whose bit pattern is also 1024 */
        return (uint16_t)(sign | (uint16_t)m);
    }
    unsigned mi = (unsigned)m;     /* in [1024, 2048] */
    int biased = E + 15;
    if (mi == 2048u) { mi = 1024u; biased += 1; }
    if (biased >= 31) return (uint16_t)(sign | 0x7c00u);
    return (uint16_t)(sign | (unsigned)(biased << 10) | (mi - 1024u));
}

void oracle_decode_f16(const uint16_t* in, double* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f16_to_f64(in[i]);
}

void oracle_encode_f16(const double* in, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f64_to_f16(in[i]);
}

/* ReLU as read from the page: max(x, 0), with everything that is not > 0
 * (including -0 and NaN) sent to +0. */
static double relu64(double x) { return (x > 0.0) ? x : 0.0; }

static double* decode_table(void)
{
    double* t = (double*)malloc(sizeof(double) * 65536);
    if (!t) return NULL;
    for (unsigned h = 0; h < 65536u; ++h) t[h] = oracle_f16_to_f64((uint16_t)h);
    return t;
}

static int resolve_threads(int nthreads)
{
#ifdef _OPENMP
    return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/* Full matrix: C[i,j] = fp16( relu?( sum_{k<K} A[i,k] * B[k,j] ) ).
 * Returns 0, or -1 on allocation failure / bad arguments. */
int oracle_gemm_f16(const uint16_t* A, const uint16_t* B, uint16_t* C,
                    int64_t M, int64_t N, int64_t K,
                    int64_t lda, int64_t ldb, int64_t ldc,
                    int relu, int nthreads)
{
    if (M < 0 || N < 0 || K < 0) return -1;
    if (M == 0 || N == 0) return 0;
    if (lda < K || ldb < N || ldc < N) return -1;
    double* tab = decode_table();
    if (!tab) return -1;
    int failed = 0;
    const int nt = resolve_threads(nthreads);
#pragma omp parallel num_threads(nt)
    {
        double* acc = (double*)malloc(sizeof(double) * (size_t)N);
        if (!acc) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < M; ++i) {
            if (!acc) continue;
            for (int64_t j = 0; j < N; ++j) acc[j] = 0.0;
            const uint16_t* arow = A + i * lda;
            for (int64_t k = 0; k < K; ++k) {
                const double a = tab[arow[k]];
                const uint16_t* brow = B + k * ldb;
                for (int64_t j = 0; j < N; ++j) acc[j] += a * tab[brow[j]];
            }
            uint16_t* crow = C + i * ldc;
            for (int64_t j = 0; j < N; ++j)
                crow[j] = oracle_f64_to_f16(relu ? relu64(acc[j]) : acc[j]);
        }
        free(acc);
    }
    free(tab);
    return failed ? -1 : 0;
}

/* Selected elements only: out[s] = C[rows[s], cols[s]], each one a plain dot
 * product over ascending k.  For checking full-size problems at sample
 * points. */
int oracle_gemm_f16_at(const uint16_t* A, const uint16_t* B,
                       int64_t K, int64_t lda, int64_t ldb, int relu,
                       int64_t nsamples, const int64_t* rows, const int64_t* cols,
                       uint16_t* out, int nthreads)
{
    if (K < 0 || nsamples < 0) return -1;
    double* tab = decode_table();
    if (!tab) return -1;
    const int nt = resolve_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 16) num_threads(nt)
    for (int64_t s = 0; s < nsamples; ++s) {
        const uint16_t* arow = A + rows[s] * lda;
        const uint16_t* bcol = B + cols[s];
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) acc += tab[arow[k]] * tab[bcol[k * ldb]];
        out[s] = oracle_f64_to_f16(relu ? relu64(acc) : acc);
    }
    free(tab);
    return 0;
}

/* The unrounded fp64 sums at selected elements (before ReLU and rounding),
 * used by tests to measure how far a result is from the exact value. */
int oracle_gemm_f64_at(const uint16_t* A, const uint16_t* B,
                       int64_t K, int64_t lda, int64_t ldb,
                       int64_t nsamples, const int64_t* rows, const int64_t* cols,
                       double* out, int nthreads)
{
    if (K < 0 || nsamples < 0) return -1;
    double* tab = decode_table();
    if (!tab) return -1;
    const int nt = resolve_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 16) num_threads(nt)
    for (int64_t s = 0; s < nsamples; ++s) {
        const uint16_t* arow = A + rows[s] * lda;
        const uint16_t* bcol = B + cols[s];
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) acc += tab[arow[k]] * tab[bcol[k * ldb]];
        out[s] = acc;
    }
    free(tab);
    return 0;
}

/* ---- fused bias + activation epilogue --------------------------------- */
/* "TileLang simplifica la creación de kernels GPU de alto rendimiento"
 * (posicionamiento-web.ar), section "Fusionar operaciones para reducir viajes
 * a memoria": the bias is added and GELU applied while the accumulator is
 * still on chip, and the result is written once.  Read here as
 *   C[i,j] = fp16_RNE( act( sum_k A[i,k] B[k,j] + bias[j] ) )
 * with bias an fp16 vector over the output columns (absent = 0), the sum
 * exact as above, and act one of
 *   0: identity, 1: max(x, 0) (-0 and NaN -> +0),
 *   2: GELU(x) = x * Phi(x) with Phi the standard normal CDF (the plain
 *      definition), Phi(x) = 0.5 * erfc(-x / sqrt(2)): the same function as
 *      0.5 * (1 + erf(x / sqrt(2))) without its cancellation for negative x
 *      (libm's erfc in fp64). */
enum { ORACLE_ACT_NONE = 0, ORACLE_ACT_RELU = 1, ORACLE_ACT_GELU = 2 };

static double act64(double x, int act)
{
    if (act == ORACLE_ACT_RELU) return relu64(x);
    if (act == ORACLE_ACT_GELU) return x * (0.5 * erfc(-x / sqrt(2.0)));
    return x;
}

int oracle_gemm_bias_act_f16(const uint16_t* A, const uint16_t* B, const uint16_t* bias,
                             uint16_t* C, int64_t M, int64_t N, int64_t K,
                             int64_t lda, int64_t ldb, int64_t ldc, int act, int nthreads)
{
    if (M < 0 || N < 0 || K < 0 || act < 0 || act > 2) return -1;
    if (M == 0 || N == 0) return 0;
    if (lda < K || ldb < N || ldc < N) return -1;
    double* tab = decode_table();
    if (!tab) return -1;
    int failed = 0;
    const int nt = resolve_threads(nthreads);
#pragma omp parallel num_threads(nt)
    {
        double* acc = (double*)malloc(sizeof(double) * (size_t)N);
        if (!acc) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < M; ++i) {
            if (!acc) continue;
            for (int64_t j = 0; j < N; ++j) acc[j] = 0.0;
            const uint16_t* arow = A + i * lda;
            for (int64_t k = 0; k < K; ++k) {
                const double a = tab[arow[k]];
                const uint16_t* brow = B + k * ldb;
                for (int64_t j = 0; j < N; ++j) acc[j] += a * tab[brow[j]];
            }
            uint16_t* crow = C + i * ldc;
            for (int64_t j = 0; j < N; ++j) {
                const double x = acc[j] + (bias ? tab[bias[j]] : 0.0);
                crow[j] = oracle_f64_to_f16(act64(x, act));
            }
        }
        free(acc);
    }
    free(tab);
    return failed ? -1 : 0;
}

/* ---- operand layouts ----------------------------------------------------- */
/* T.gemm's transpose_A / transpose_B options ("Writing high-performance
 * kernels in TileLang", atlascloud.ai blog, section "Escribamos un GEMM"):
 * op(A) is M x K and op(B) is K x N, with
 *   trans_a = 0: A stored M x K row-major (A[i,k] at A + i*lda + k)
 *   trans_a = 1: A stored K x M row-major (op(A)[i,k] at A + k*lda + i)
 *   trans_b = 0: B stored K x N row-major (B[k,j] at B + k*ldb + j)
 *   trans_b = 1: B stored N x K row-major (op(B)[k,j] at B + j*ldb + k)
 * C = fp16_RNE(act(sum_k op(A)[i,k] op(B)[k,j] + bias[j])), ascending k in
 * fp64, one element at a time. */
int oracle_gemm_general_f16(const uint16_t* A, const uint16_t* B, const uint16_t* bias,
                            uint16_t* C, int64_t M, int64_t N, int64_t K,
                            int64_t lda, int64_t ldb, int64_t ldc,
                            int trans_a, int trans_b, int act, int nthreads)
{
    if (M < 0 || N < 0 || K < 0 || act < 0 || act > 2) return -1;
    if (M == 0 || N == 0) return 0;
    if (lda < (trans_a ? M : K) || ldb < (trans_b ? K : N) || ldc < N) return -1;
    double* tab = decode_table();
    if (!tab) return -1;
    const int64_t sa_i = trans_a ? 1 : lda, sa_k = trans_a ? lda : 1;
    const int64_t sb_k = trans_b ? 1 : ldb, sb_j = trans_b ? ldb : 1;
    const int nt = resolve_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int64_t i = 0; i < M; ++i) {
        for (int64_t j = 0; j < N; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += tab[A[i * sa_i + k * sa_k]] * tab[B[k * sb_k + j * sb_j]];
            const double x = acc + (bias ? tab[bias[j]] : 0.0);
            C[i * ldc + j] = oracle_f64_to_f16(act64(x, act));
        }
    }
    free(tab);
    return 0;
}

/* The activations alone on fp64 inputs (unrounded), for pinning act64. */
void oracle_activation_f64(const double* in, double* out, int64_t n, int act)
{
    for (int64_t i = 0; i < n; ++i) out[i] = act64(in[i], act);
}

int oracle_max_threads(void) { return resolve_threads(0); }
