/*
 * synth.c -- seeded synthetic inputs shared by the tests, the benchmark and
 * the oracle checks.  It holds none of the method's arithmetic: it only makes
 * BF16 activation tensors of the shapes and value distribution the workloads
 * call for (N(0,1) with 1% of the channels scaled x8 as outliers).
 *
 * Generator: counter-based.  Element i of a stream with key K draws
 *   u1 = (splitmix64(K + 2i)     >> 11 + 1) * 2^-53   in (0, 1]
 *   u2 = (splitmix64(K + 2i + 1) >> 11)     * 2^-53   in [0, 1)
 *   z  = sqrt(-2 ln u1) * cos(2 pi u2)                 (Box-Muller, fp64)
 * splitmix64 is Steele, Lea and Flood's SplitMix finaliser (OOPSLA 2014) with
 * the 64-bit constants published with Vigna's splitmix64.  The outlier
 * columns are chosen per tensor by a partial Fisher-Yates shuffle on a
 * second stream; their values are multiplied by 8 in fp64 before the single
 * round-to-nearest-even step to bfloat16.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static inline uint64_t splitmix64(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t synth_splitmix64(uint64_t x) { return splitmix64(x); }

/* Stream key for (seed, slot, tensor): three chained finaliser rounds. */
uint64_t synth_key(uint64_t seed, uint64_t slot, uint64_t tensor) {
    uint64_t k = splitmix64(seed);
    k = splitmix64(k ^ (slot * 0xD1B54A32D192ED03ULL));
    k = splitmix64(k ^ (tensor * 0x8CB92BA72F3D8DD7ULL));
    return k;
}

/* One N(0,1) draw for element i of stream key. */
double synth_normal(uint64_t key, uint64_t i) {
    uint64_t a = splitmix64(key + 2 * i);
    uint64_t b = splitmix64(key + 2 * i + 1);
    double u1 = (double)((a >> 11) + 1) * 0x1.0p-53;
    double u2 = (double)(b >> 11) * 0x1.0p-53;
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

/* Round a double to bfloat16 bits, nearest-even, in one step (no detour
 * through fp32, so no double rounding).  Inputs here are finite and far from
 * the bf16 overflow and subnormal ranges. */
uint16_t synth_double_to_bf16(double d) {
    if (d == 0.0) return signbit(d) ? 0x8000 : 0x0000;
    int e2;
    double fr = frexp(fabs(d), &e2);
    double r = ldexp(rint(ldexp(fr, 8)), e2 - 8);
    float f = (float)r;
    if (signbit(d)) f = -f;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* The n_out distinct outlier columns of [0, ncols) for stream key, written in
 * draw order (partial Fisher-Yates on a stream derived from key). */
int synth_outlier_columns(uint64_t key, int32_t ncols, int32_t n_out, int32_t* cols) {
    if (n_out < 0 || n_out > ncols) return -1;
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)(ncols > 0 ? ncols : 1));
    if (!perm) return -2;
    for (int32_t i = 0; i < ncols; ++i) perm[i] = i;
    uint64_t k2 = splitmix64(key ^ 0x5EEDC0DE0FF1CE55ULL);
    for (int32_t i = 0; i < n_out; ++i) {
        uint64_t r = splitmix64(k2 + (uint64_t)i);
        int32_t j = i + (int32_t)(r % (uint64_t)(ncols - i));
        int32_t t = perm[i];
        perm[i] = perm[j];
        perm[j] = t;
        cols[i] = perm[i];
    }
    free(perm);
    return 0;
}

typedef struct {
    uint64_t key;
    int64_t row0, row1, ncols;
    double factor;
    const uint8_t* is_outlier;
    uint16_t* out;
} synth_job;

static void* synth_worker(void* arg) {
    synth_job* j = (synth_job*)arg;
    for (int64_t r = j->row0; r < j->row1; ++r) {
        for (int64_t c = 0; c < j->ncols; ++c) {
            uint64_t i = (uint64_t)(r * j->ncols + c);
            double z = synth_normal(j->key, i);
            if (j->is_outlier[c]) z *= j->factor;
            j->out[i] = synth_double_to_bf16(z);
        }
    }
    return NULL;
}

/* Fill out[rows, ncols] (bf16 bits) for stream key.  n_out columns (drawn by
 * synth_outlier_columns) are scaled by `factor`.  Deterministic for any
 * thread count.  Returns 0 on success. */
int synth_fill_bf16(uint64_t key, int64_t rows, int64_t ncols, int32_t n_out, double factor,
                    int32_t n_threads, uint16_t* out) {
    if (rows < 0 || ncols <= 0 || ncols > 0x7FFFFFFF) return -1;
    uint8_t* mask = (uint8_t*)calloc((size_t)ncols, 1);
    int32_t* cols = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n_out > 0 ? n_out : 1));
    if (!mask || !cols) {
        free(mask);
        free(cols);
        return -2;
    }
    if (synth_outlier_columns(key, (int32_t)ncols, n_out, cols) != 0) {
        free(mask);
        free(cols);
        return -1;
    }
    for (int32_t i = 0; i < n_out; ++i) mask[cols[i]] = 1;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 256) n_threads = 256;
    if ((int64_t)n_threads > rows) n_threads = rows > 0 ? (int32_t)rows : 1;
    pthread_t th[256];
    int joinable[256];
    synth_job jobs[256];
    int64_t per = (rows + n_threads - 1) / n_threads;
    for (int32_t t = 0; t < n_threads; ++t) {
        jobs[t].key = key;
        jobs[t].row0 = t * per < rows ? t * per : rows;
        jobs[t].row1 = (t + 1) * per < rows ? (t + 1) * per : rows;
        jobs[t].ncols = ncols;
        jobs[t].factor = factor;
        jobs[t].is_outlier = mask;
        jobs[t].out = out;
        joinable[t] = 0;
        if (t == 0) continue;
        if (pthread_create(&th[t], NULL, synth_worker, &jobs[t]) == 0)
            joinable[t] = 1;
        else
            synth_worker(&jobs[t]); /* could not start a thread: run it here */
    }
    synth_worker(&jobs[0]);
    for (int32_t t = 1; t < n_threads; ++t)
        if (joinable[t]) pthread_join(th[t], NULL);
    free(mask);
    free(cols);
    return 0;
}
