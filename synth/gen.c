/*
 * Seeded BF16 normal draws for the synthetic workloads (no attention,
 * RoPE or quantisation arithmetic here). Shared by the CPU oracle's tests
 * and the CUDA library's tests and benchmark through synth/__init__.py.
 *
 * Element i of a stream `key`:
 *   r_j = mix(key + (j + 1) * 0x9E3779B97F4A7C15) for j = 2i, 2i+1
 *   mix = the SplitMix64 finaliser (Steele, Lea, Flood, OOPSLA 2014)
 *   u1 = ((r_2i >> 11) + 1) * 2^-53, u2 = (r_2i+1 >> 11) * 2^-53
 *   z  = sqrt(-2 ln u1) cos(2 pi u2)                    (Box-Muller, 1958)
 *   out = bf16_rne(float(z * std))
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

static uint64_t mix64(uint64_t z) {
    z ^= z >> 30;
    z *= 0xBF58476D1CE4E5B9ull;
    z ^= z >> 27;
    z *= 0x94D049BB133111EBull;
    z ^= z >> 31;
    return z;
}

static uint16_t bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

typedef struct {
    uint64_t key;
    int64_t lo, hi;
    double std;
    uint16_t *out;
} job;

static void *work(void *p) {
    job *j = (job *)p;
    const uint64_t g = 0x9E3779B97F4A7C15ull;
    const double two_pi = 6.283185307179586476925286766559;
    for (int64_t i = j->lo; i < j->hi; ++i) {
        uint64_t r1 = mix64(j->key + (uint64_t)(2 * i + 1) * g);
        uint64_t r2 = mix64(j->key + (uint64_t)(2 * i + 2) * g);
        double u1 = ((double)(r1 >> 11) + 1.0) * 0x1.0p-53;
        double u2 = (double)(r2 >> 11) * 0x1.0p-53;
        double z = sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
        j->out[i] = bf16_rne((float)(z * j->std));
    }
    return NULL;
}

void synth_bf16_normal(uint64_t key, int64_t n, double std, uint16_t *out, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 128) nthreads = 128;
    if (n < 65536) nthreads = 1;
    pthread_t th[128];
    job jobs[128];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].key = key;
        jobs[t].lo = n * t / nthreads;
        jobs[t].hi = n * (t + 1) / nthreads;
        jobs[t].std = std;
        jobs[t].out = out;
        if (nthreads == 1)
            work(&jobs[t]);
        else
            pthread_create(&th[t], NULL, work, &jobs[t]);
    }
    if (nthreads > 1)
        for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
}
