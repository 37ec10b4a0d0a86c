/*
 * oracle.c -- plain, slow, obviously-correct CPU reference for the ternary
 * linear layer and its two lossless packings.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product (the libternary C ABI,
 * its kernels or its Python binding) may include, link or call this file.
 * Only the test suite, the package smoke check and the benchmark's CPU
 * baseline leg load it.  It shares no code, header, table or constant
 * generator with the CUDA path.
 *
 * Sources (all from "Pith review of Spectra 1.1: Scaling Laws and Efficient
 * Inference for Ternary Language Models", pith.science, unless noted):
 *   - "What carries the argument": the ternary linear layer is a linear layer
 *     whose weights are restricted to {-1,0,1} times one shared
 *     floating-point scale; k ternary digits fit in p bits when 2^p > 3^k,
 *     so k = 5 trits fit p = 8 bits (1.6 bits per weight).
 *   - "Core claim": ternary weights pack losslessly at 2 bits with a base-4
 *     encoding and at 1.6 bits with a base-3 encoding.
 *   - Referee report, minor comment 5 (paper section 3.2): the 1.6-bit decode
 *     is written with running quotients b'_i and digits x_i; the handling of
 *     a partial final block is left unspecified.
 *   - "Circularity Check": the packing map P and unpacking map U satisfy a
 *     correctness theorem proved from their definitions (paper appendix E).
 *
 * Readings taken where the pages are silent (each also listed in the
 * design notes):
 *   R1  trit t maps to digit d = t + 1 (-1 -> 0, 0 -> 1, +1 -> 2).
 *   R2  digit i of a byte has weight base^i (least-significant digit first),
 *       trit k of a row goes to byte k / g, digit k % g (g = 4 or 5).
 *   R3  trits are packed along the reduction dimension K, row n of T in
 *       row n of the packed matrix, row stride ldp bytes.
 *   R4  a partial final byte is completed with 0-trits (digit 1); bytes in
 *       [row_bytes, ldp) are written as 0 by pack and ignored by unpack.
 *   R5  a byte is a valid code iff every base-b digit is <= 2 and nothing is
 *       left after g digits (2-bit: no field equals 3; 1.6-bit: byte < 243).
 *       Pad digits inside the last byte may hold any valid digit.
 *   R6  y[m][n] = alpha * sum_k T[n][k] * x[m][k], computed here in double
 *       (fp16 inputs are exact in double).
 *
 * Build: gcc -O2 -shared -fPIC -pthread oracle.c -o liboracle.so
 * A -DORACLE_MUTANT=<n> build plants one deliberate mistake (see the MUTANT
 * blocks); the tests use those builds to show the pins catch each mistake.
 */
#include <stdint.h>
#include <stddef.h>
#include <math.h>
#include <pthread.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

enum { OR_OK = 0, OR_INVALID_ARG = 1, OR_BAD_TRIT = 2, OR_BAD_CODE = 3 };
enum { OR_FMT_2BIT = 2, OR_FMT_1P6BIT = 16 };

/* Digits per byte g and digit base b of each format ("Core claim"). */
static int fmt_group(int fmt) { return fmt == OR_FMT_2BIT ? 4 : (fmt == OR_FMT_1P6BIT ? 5 : 0); }
static int fmt_base(int fmt) { return fmt == OR_FMT_2BIT ? 4 : (fmt == OR_FMT_1P6BIT ? 3 : 0); }

int or_digits_per_byte(int fmt) { return fmt_group(fmt); }
int or_digit_base(int fmt) { return fmt_base(fmt); }

/* Lossless-packing condition ("What carries the argument"): k trits fit in p
 * bits iff the 3^k distinct tuples can have distinct p-bit codes, i.e.
 * 3^k <= 2^p.  For p >= 1, 3^k is odd and 2^p even, so this is the pages'
 * 2^p > 3^k; the two differ only at the trivial k = p = 0. */
int or_fits(int k, int p)
{
    if (k < 0 || p < 0 || p > 62) return 0;
    uint64_t three_k = 1, two_p = (uint64_t)1 << p;
    for (int i = 0; i < k; ++i) {
        three_k *= 3;
        if (three_k > two_p) return 0;
    }
    return three_k <= two_p;
}

/* Bytes per packed row: ceil(K / g). */
int64_t or_row_bytes(int fmt, int64_t K)
{
    int g = fmt_group(fmt);
    if (g == 0 || K < 0) return -1;
    return (K + g - 1) / g;
}

/* Digit of a trit (reading R1). */
static int trit_to_digit(int t)
{
#if ORACLE_MUTANT == 2
    return (t + 3) % 3;           /* mistake: t mod 3 instead of t + 1 */
#else
    return t + 1;
#endif
}

/* Packing map P (reading R2-R4): byte = sum_{i<g} d_i * b^i, evaluated by
 * Horner's rule from the most significant digit down. */
int or_pack(int fmt, const int8_t *T, int64_t N, int64_t K, int64_t ldt,
            uint8_t *P, int64_t ldp)
{
    int g = fmt_group(fmt), b = fmt_base(fmt);
    int64_t rb = or_row_bytes(fmt, K);
    if (g == 0 || N < 0 || K < 0 || ldt < K || ldp < rb) return OR_INVALID_ARG;
    if ((N > 0 && K > 0) && (T == NULL || P == NULL)) return OR_INVALID_ARG;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            int t = T[n * ldt + k];
            if (t < -1 || t > 1) return OR_BAD_TRIT;
        }
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < rb; ++j) {
            int value = 0;
            for (int i = g - 1; i >= 0; --i) {
                int64_t k = j * g + i;
#if ORACLE_MUTANT == 1
                k = j * g + (g - 1 - i);  /* mistake: most-significant digit first */
#endif
#if ORACLE_MUTANT == 3
                int d = (k < K) ? trit_to_digit(T[n * ldt + k]) : 0; /* mistake: pad digit 0 */
#else
                int d = (k < K) ? trit_to_digit(T[n * ldt + k]) : trit_to_digit(0);
#endif
                value = value * b + d;
            }
            P[n * ldp + j] = (uint8_t)value;
        }
        for (int64_t j = rb; j < ldp; ++j) P[n * ldp + j] = 0;
    }
    return OR_OK;
}

/* Unpacking map U: b'_0 = byte, digit x_i = b'_i mod b, b'_{i+1} =
 * floor(b'_i / b), trit = x_i - 1 (referee minor comment 5 notation; reading
 * R5 for validity).  Pad trits (k >= K) are dropped.  On an invalid byte the
 * offset n*ldp + j of the first one (row-major scan) goes to *bad. */
int or_unpack(int fmt, const uint8_t *P, int64_t N, int64_t K, int64_t ldp,
              int8_t *T, int64_t ldt, int64_t *bad)
{
    int g = fmt_group(fmt), b = fmt_base(fmt);
    int64_t rb = or_row_bytes(fmt, K);
    if (g == 0 || N < 0 || K < 0 || ldt < K || ldp < rb) return OR_INVALID_ARG;
    if ((N > 0 && K > 0) && (T == NULL || P == NULL)) return OR_INVALID_ARG;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < rb; ++j) {
            int q = P[n * ldp + j];
            int valid = 1;
            for (int i = 0; i < g; ++i) {
                int x = q % b;
                q = q / b;
#if ORACLE_MUTANT == 4
                (void)0;              /* mistake: a digit of 3 is not rejected */
#else
                if (x > 2) valid = 0;
#endif
                int64_t k = j * g + i;
                if (k < K) T[n * ldt + k] = (int8_t)(x - 1);
            }
#if ORACLE_MUTANT == 5
            (void)q;                  /* mistake: leftover quotient not checked */
#else
            if (q != 0) valid = 0;
#endif
            if (!valid) {
                if (bad) *bad = n * ldp + j;
                return OR_BAD_CODE;
            }
        }
    }
    return OR_OK;
}

/* IEEE 754 binary16 -> double from the bit fields: sign s, exponent e
 * (bias 15), fraction f.  e = 0: subnormal f * 2^-24; e = 31: inf / NaN. */
double or_half_to_double(uint16_t h)
{
    int s = (h >> 15) & 1, e = (h >> 10) & 31, f = h & 1023;
    double v;
    if (e == 0) {
#if ORACLE_MUTANT == 6
        v = ldexp(1024.0 + f, -25); /* mistake: implicit bit kept for subnormals */
#else
        v = ldexp((double)f, -24);
#endif
    } else if (e == 31) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp(1024.0 + f, e - 25);
    }
    return s ? -v : v;
}

/* One output element of the layer (reading R6). */
static double linear_one(const int8_t *T, int64_t ldt, const uint16_t *X, int64_t ldx,
                         double alpha, int64_t m, int64_t n, int64_t K)
{
    double acc = 0.0;
    int64_t kend = K;
#if ORACLE_MUTANT == 7
    kend = K > 0 ? K - 1 : 0;         /* mistake: last term dropped */
#endif
    for (int64_t k = 0; k < kend; ++k) {
#if ORACLE_MUTANT == 8
        double t = -(double)T[n * ldt + k];  /* mistake: sign flipped */
#elif ORACLE_MUTANT == 9
        double t = (double)T[n * ldt + (K - 1 - k)]; /* mistake: k index reversed */
#else
        double t = (double)T[n * ldt + k];
#endif
        acc += t * or_half_to_double(X[m * ldx + k]);
    }
    return alpha * acc;
}

typedef struct {
    const int8_t *T; int64_t ldt; const uint16_t *X; int64_t ldx; double alpha;
    int64_t M, N, K; double *Y; int64_t ldy; int64_t n0, n1;
} linear_job;

static void *linear_worker(void *arg)
{
    linear_job *j = (linear_job *)arg;
    for (int64_t n = j->n0; n < j->n1; ++n)
        for (int64_t m = 0; m < j->M; ++m)
            j->Y[m * j->ldy + n] = linear_one(j->T, j->ldt, j->X, j->ldx, j->alpha, m, n, j->K);
    return NULL;
}

/* Y[m][n] = alpha * sum_k T[n][k] * X[m][k] for all m < M, n < N.
 * T: int8 [N][ldt]; X: binary16 bits [M][ldx]; Y: double [M][ldy].
 * nthreads > 1 splits the rows n across POSIX threads. */
int or_linear(const int8_t *T, int64_t ldt, const uint16_t *X, int64_t ldx, double alpha,
              int64_t M, int64_t N, int64_t K, double *Y, int64_t ldy, int nthreads)
{
    if (M < 0 || N < 0 || K < 0 || ldt < K || ldx < K || ldy < N) return OR_INVALID_ARG;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nthreads > N) nthreads = (int)(N > 0 ? N : 1);
    pthread_t tid[256];
    linear_job job[256];
    for (int i = 0; i < nthreads; ++i) {
        job[i] = (linear_job){T, ldt, X, ldx, alpha, M, N, K, Y, ldy,
                              N * i / nthreads, N * (i + 1) / nthreads};
    }
    if (nthreads == 1) {
        linear_worker(&job[0]);
        return OR_OK;
    }
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&tid[i], NULL, linear_worker, &job[i]) != 0) {
            linear_worker(&job[i]);
            tid[i] = 0;
        } else {
            ++started;
        }
    }
    for (int i = 0; i < nthreads; ++i)
        if (tid[i]) pthread_join(tid[i], NULL);
    (void)started;
    return OR_OK;
}

/* The same definition evaluated only at the listed (m, n) pairs, for spot
 * checks of outputs too large to compute in full.  out[i] = Y[ms[i]][ns[i]]. */
int or_linear_at(const int8_t *T, int64_t ldt, const uint16_t *X, int64_t ldx, double alpha,
                 int64_t K, const int64_t *ms, const int64_t *ns, int64_t count, double *out)
{
    if (K < 0 || ldt < K || ldx < K || count < 0) return OR_INVALID_ARG;
    for (int64_t i = 0; i < count; ++i)
        out[i] = linear_one(T, ldt, X, ldx, alpha, ms[i], ns[i], K);
    return OR_OK;
}
