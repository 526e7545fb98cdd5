/*
 * Seeded synthetic inputs shared by the tests, the benchmark and the oracle's
 * callers.  This file holds random-number generation only, none of the
 * attention arithmetic, and is built into its own library (libta23_synth.so).
 *
 * Generator: the splitmix64 output function (Steele, Lea and Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014), used in counter
 * mode.  A tensor is identified by (seed, stream); its key is
 *     key = mix(seed + G * (stream + 1))
 * and word c of the tensor is the c-th splitmix64 output from state key:
 *     word(c) = mix(key + G * (c + 1)),   G = 0x9E3779B97F4A7C15.
 *
 * Normal values: Box-Muller on word pairs.  Pair p gives
 *     u1 = ((word(2p) >> 11) + 1) * 2^-53   in (0, 1]
 *     u2 =  (word(2p+1) >> 11)    * 2^-53   in [0, 1)
 *     x[2p] = r cos(2 pi u2),  x[2p+1] = r sin(2 pi u2),  r = sqrt(-2 ln u1)
 * in fp64, then rounded to fp32 (nearest-even) and to bf16 (nearest-even),
 * then multiplied by 2^pow2 (exact in bf16 for these magnitudes).
 *
 * Uniform integers in [lo, hi]: lo + word(c) mod (hi - lo + 1).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define SM_G 0x9E3779B97F4A7C15ULL

static uint64_t sm_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0; /* NaN */
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static float bf16_to_f32(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

typedef struct {
    uint16_t* out;
    int64_t n, p0, p1;  /* pair range */
    uint64_t key;
    float mult;
} normal_job;

static void* normal_worker(void* a_) {
    normal_job* a = (normal_job*)a_;
    const double two_pi = 6.283185307179586476925286766559;
    const double inv53 = 1.0 / 9007199254740992.0; /* 2^-53 */
    for (int64_t p = a->p0; p < a->p1; ++p) {
        uint64_t w0 = sm_mix(a->key + SM_G * (uint64_t)(2 * p + 1));
        uint64_t w1 = sm_mix(a->key + SM_G * (uint64_t)(2 * p + 2));
        double u1 = (double)((w0 >> 11) + 1) * inv53;
        double u2 = (double)(w1 >> 11) * inv53;
        double r = sqrt(-2.0 * log(u1));
        double x0 = r * cos(two_pi * u2), x1 = r * sin(two_pi * u2);
        int64_t e = 2 * p;
        uint16_t b0 = f32_to_bf16_rne((float)x0);
        uint16_t b1 = f32_to_bf16_rne((float)x1);
        if (a->mult != 1.0f) {
            b0 = f32_to_bf16_rne(bf16_to_f32(b0) * a->mult);
            b1 = f32_to_bf16_rne(bf16_to_f32(b1) * a->mult);
        }
        a->out[e] = b0;
        if (e + 1 < a->n) a->out[e + 1] = b1;
    }
    return NULL;
}

uint64_t ta23_synth_key(uint64_t seed, uint64_t stream) { return sm_mix(seed + SM_G * (stream + 1)); }

uint64_t ta23_synth_word(uint64_t seed, uint64_t stream, uint64_t c) {
    return sm_mix(ta23_synth_key(seed, stream) + SM_G * (c + 1));
}

/* Fill out[0..n) with bf16 N(0,1) * 2^pow2 bit patterns.  Returns 0 on success. */
int ta23_synth_normal_bf16(uint16_t* out, int64_t n, uint64_t seed, uint64_t stream, int pow2,
                           int nthreads) {
    if (n < 0 || !out || pow2 < -20 || pow2 > 20) return 1;
    if (n == 0) return 0;
    int64_t pairs = (n + 1) / 2;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (pairs < 65536) nthreads = 1;
    normal_job jobs[256];
    pthread_t th[256];
    uint64_t key = ta23_synth_key(seed, stream);
    float mult = ldexpf(1.0f, pow2);
    int64_t chunk = (pairs + nthreads - 1) / nthreads;
    int started = 0;
    for (int t = 0; t < nthreads; ++t) {
        int64_t p0 = (int64_t)t * chunk, p1 = p0 + chunk;
        if (p0 > pairs) p0 = pairs;
        if (p1 > pairs) p1 = pairs;
        jobs[t] = (normal_job){out, n, p0, p1, key, mult};
    }
    if (nthreads == 1) {
        normal_worker(&jobs[0]);
        return 0;
    }
    for (int t = 0; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, normal_worker, &jobs[t]) != 0) {
            normal_worker(&jobs[t]);  /* run it here instead */
            continue;
        }
        th[started++] = th[t];
    }
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    return 0;
}

/* Fill out[0..n) with integers uniform in [lo, hi].  Returns 0 on success. */
int ta23_synth_uniform_int(int32_t* out, int64_t n, uint64_t seed, uint64_t stream, int32_t lo,
                           int32_t hi) {
    if (n < 0 || !out || hi < lo) return 1;
    uint64_t key = ta23_synth_key(seed, stream);
    uint64_t span = (uint64_t)((int64_t)hi - (int64_t)lo + 1);
    for (int64_t c = 0; c < n; ++c)
        out[c] = (int32_t)((int64_t)lo + (int64_t)(sm_mix(key + SM_G * (uint64_t)(c + 1)) % span));
    return 0;
}
