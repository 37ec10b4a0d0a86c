/*
 * synth.c -- seeded synthetic inputs shared by the oracle side and the CUDA
 * side of every test and benchmark.
 *
 * This module holds random-number generation only: none of the ternary
 * layer's arithmetic, packing or decoding lives here.
 *
 * Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014).  Its state advances by the
 * odd "golden gamma" 0x9E3779B97F4A7C15 and each output is the state passed
 * through the published 64-bit finaliser (xor-shift 30 / multiply / xor-shift
 * 27 / multiply / xor-shift 31).  Because the state after j steps is
 * seed + j * gamma, element j of a stream is computed directly from its
 * index, so large arrays are filled in parallel with identical results.
 *
 * Derived variates:
 *   uniform  u = (z >> 11) * 2^-53 in [0, 1)
 *   normal   Box-Muller on consecutive pairs (u1, u2):
 *            r = sqrt(-2 ln(1 - u1)), z0 = r cos(2 pi u2), z1 = r sin(2 pi u2)
 *   trit     0 if u < p0, -1 if u < p0 + (1 - p0) / 2, else +1
 *
 * Build: gcc -O2 -shared -fPIC -pthread synth.c -o libsynth.so -lm
 */
#include <stdint.h>
#include <math.h>
#include <pthread.h>

#define SY_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t sy_mix(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Plain sequential SplitMix64: advance *state by gamma, return the mix. */
uint64_t sy_next(uint64_t *state)
{
    *state += SY_GAMMA;
    return sy_mix(*state);
}

/* Element j of the stream that starts from state `key` (j counts from 0,
 * i.e. the value sy_next would return on its (j+1)-th call). */
static inline uint64_t sy_at(uint64_t key, uint64_t j)
{
    return sy_mix(key + (j + 1) * SY_GAMMA);
}

static inline double sy_unit(uint64_t z) { return (double)(z >> 11) * 0x1.0p-53; }

/* Key of an independent stream: the seed and a small stream tag mixed. */
uint64_t sy_key(uint64_t seed, uint64_t stream)
{
    return sy_mix(sy_mix(seed) + stream * SY_GAMMA + 0x5EEDULL);
}

void sy_u64(uint64_t key, int64_t n, uint64_t *out)
{
    for (int64_t j = 0; j < n; ++j) out[j] = sy_at(key, (uint64_t)j);
}

void sy_uniform(uint64_t key, int64_t n, double lo, double hi, double *out)
{
    for (int64_t j = 0; j < n; ++j) out[j] = lo + (hi - lo) * sy_unit(sy_at(key, (uint64_t)j));
}

typedef struct {
    int kind;               /* 0: trits, 1: normals */
    uint64_t key;
    int64_t rows, cols, ld;
    double p0;
    int8_t *trits;
    double *normals;
    int64_t r0, r1;
} sy_job;

static void sy_fill_rows(const sy_job *j)
{
    if (j->kind == 0) {
        double lo = j->p0, mid = j->p0 + 0.5 * (1.0 - j->p0);
        for (int64_t r = j->r0; r < j->r1; ++r) {
            int8_t *row = j->trits + r * j->ld;
            uint64_t base = (uint64_t)r * (uint64_t)j->cols;
            for (int64_t c = 0; c < j->cols; ++c) {
                double u = sy_unit(sy_at(j->key, base + (uint64_t)c));
                row[c] = (int8_t)(u < lo ? 0 : (u < mid ? -1 : 1));
            }
        }
    } else {
        /* normals are generated over the flat index so that a row split does
         * not change the values; rows*cols values, pairs (2i, 2i+1). */
        int64_t total = j->rows * j->cols;
        int64_t p0 = (j->r0 * j->cols) / 2, p1 = (j->r1 * j->cols + 1) / 2;
        for (int64_t p = p0; p < p1; ++p) {
            double u1 = sy_unit(sy_at(j->key, 2 * (uint64_t)p));
            double u2 = sy_unit(sy_at(j->key, 2 * (uint64_t)p + 1));
            double r = sqrt(-2.0 * log(1.0 - u1));
            double a = 6.283185307179586476925286766559 * u2;
            int64_t i0 = 2 * p, i1 = 2 * p + 1;
            if (i0 >= j->r0 * j->cols && i0 < j->r1 * j->cols && i0 < total)
                j->normals[(i0 / j->cols) * j->ld + i0 % j->cols] = r * cos(a);
            if (i1 >= j->r0 * j->cols && i1 < j->r1 * j->cols && i1 < total)
                j->normals[(i1 / j->cols) * j->ld + i1 % j->cols] = r * sin(a);
        }
    }
}

static void *sy_worker(void *arg)
{
    sy_fill_rows((const sy_job *)arg);
    return NULL;
}

static void sy_run(sy_job proto, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 128) nthreads = 128;
    if (nthreads > proto.rows) nthreads = proto.rows > 0 ? (int)proto.rows : 1;
    sy_job jobs[128];
    pthread_t tid[128];
    int ok[128];
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = proto;
        jobs[i].r0 = proto.rows * i / nthreads;
        jobs[i].r1 = proto.rows * (i + 1) / nthreads;
    }
    for (int i = 1; i < nthreads; ++i) ok[i] = pthread_create(&tid[i], NULL, sy_worker, &jobs[i]) == 0;
    sy_fill_rows(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) {
        if (ok[i]) pthread_join(tid[i], NULL);
        else sy_fill_rows(&jobs[i]);
    }
}

/* T[r][c] (r < rows, c < cols, row stride ld) = trit of stream element
 * r*cols + c with P(0) = p0 and P(-1) = P(+1) = (1 - p0) / 2. */
void sy_trits(uint64_t key, int64_t rows, int64_t cols, int64_t ld, double p0, int8_t *T,
              int nthreads)
{
    sy_job j = {0, key, rows, cols, ld, p0, T, 0, 0, rows};
    sy_run(j, nthreads);
}

/* Standard normals in double, flat index r*cols + c, row stride ld. */
void sy_normals(uint64_t key, int64_t rows, int64_t cols, int64_t ld, double *out, int nthreads)
{
    sy_job j = {1, key, rows, cols, ld, 0.0, 0, out, 0, rows};
    sy_run(j, nthreads);
}
