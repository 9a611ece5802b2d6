/*
 * Seeded synthetic BF16 weight generators.
 *
 * This file holds random-number generation only: no part of the compression
 * method lives here. Both the CPU oracle's tests and the GPU path's tests and
 * benchmark draw their inputs from it, so the two sides always see identical
 * bits.
 *
 * Generator: counter-based SplitMix64 (Steele, Lea and Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014). Output k of stream `seed` is
 * the SplitMix64 finaliser applied to seed + (k+1) * 0x9E3779B97F4A7C15, so any
 * element can be generated independently and the work splits across threads
 * without changing a single bit.
 *
 * Uniforms in (0,1): ((x >> 11) + 0.5) * 2^-53.
 * Normals: Box-Muller on one pair of uniforms per pair of normals
 *   (even index takes r*cos(theta), odd index r*sin(theta)).
 * Rounding to BF16: the double is narrowed to float32 by the C cast (IEEE
 * round-to-nearest-even), then to BF16 by round-to-nearest-even on the bit
 * pattern (the compressr page's "dtype cast ... round-to-nearest-even" row
 * names this rounding). The generators never produce NaN before rounding.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

uint64_t synth_splitmix64(uint64_t seed, uint64_t k) {
    uint64_t z = seed + (k + 1) * GOLDEN_GAMMA;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

double synth_uniform(uint64_t seed, uint64_t k) {
    return ((double)(synth_splitmix64(seed, k) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

/* Normal number k of stream `seed` (Box-Muller, pair k/2). */
static double normal_at(uint64_t seed, uint64_t k) {
    uint64_t pair = k >> 1;
    double u1 = synth_uniform(seed, 2 * pair);
    double u2 = synth_uniform(seed, 2 * pair + 1);
    double r = sqrt(-2.0 * log(u1));
    double th = 6.283185307179586476925286766559 * u2;
    return (k & 1) ? r * sin(th) : r * cos(th);
}

double synth_normal(uint64_t seed, uint64_t k) { return normal_at(seed, k); }

uint16_t synth_f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

static uint16_t to_bf16(double x) { return synth_f32_to_bf16_rne((float)x); }

/* ---- kinds of tensor --------------------------------------------------- */
enum {
    SYNTH_NORMAL = 0,      /* mean + std * N(0,1)                             */
    SYNTH_STUDENT_T3 = 1,  /* heavy tails: std * t(3), outliers, exact zeros  */
    SYNTH_CONST_EXP = 2,   /* exponent 127 (values in [1,2)), random s and m  */
    SYNTH_ALL_EXP = 3      /* exponent = i mod 256, random s and m            */
};

typedef struct {
    int kind;
    uint64_t seed;
    double mean, std;
    double outlier_p, outlier_mul, zero_p; /* SYNTH_STUDENT_T3 only */
    uint16_t* out;
    uint64_t lo, hi;
} job_t;

static void gen_range(const job_t* j) {
    uint64_t i;
    switch (j->kind) {
    case SYNTH_NORMAL:
        for (i = j->lo; i < j->hi; ++i) j->out[i] = to_bf16(j->mean + j->std * normal_at(j->seed, i));
        break;
    case SYNTH_STUDENT_T3: {
        /* independent streams for the decisions */
        uint64_t s_out = synth_splitmix64(j->seed, 0x07u) ^ 0x6F75746C69657273ULL;
        uint64_t s_zero = synth_splitmix64(j->seed, 0x2u) ^ 0x7A65726F73ULL;
        for (i = j->lo; i < j->hi; ++i) {
            double z0 = normal_at(j->seed, 4 * i);
            double z1 = normal_at(j->seed, 4 * i + 1);
            double z2 = normal_at(j->seed, 4 * i + 2);
            double z3 = normal_at(j->seed, 4 * i + 3);
            double chi2 = z1 * z1 + z2 * z2 + z3 * z3;
            double t = z0 / sqrt(chi2 / 3.0);
            double x = j->std * t;
            if (synth_uniform(s_out, i) < j->outlier_p) x *= j->outlier_mul;
            uint64_t zr = synth_splitmix64(s_zero, i);
            if (((double)(zr >> 11) + 0.5) * (1.0 / 9007199254740992.0) < j->zero_p) {
                j->out[i] = (uint16_t)((zr & 1u) ? 0x8000u : 0x0000u);
                continue;
            }
            j->out[i] = to_bf16(x);
        }
        break;
    }
    case SYNTH_CONST_EXP:
        for (i = j->lo; i < j->hi; ++i) {
            uint64_t r = synth_splitmix64(j->seed, i);
            j->out[i] = (uint16_t)(((r & 1u) << 15) | (127u << 7) | ((r >> 1) & 0x7Fu));
        }
        break;
    case SYNTH_ALL_EXP:
        for (i = j->lo; i < j->hi; ++i) {
            uint64_t r = synth_splitmix64(j->seed, i);
            j->out[i] = (uint16_t)(((r & 1u) << 15) | ((uint32_t)(i & 0xFFu) << 7) | ((r >> 1) & 0x7Fu));
        }
        break;
    default:
        break;
    }
}

static void* worker(void* arg) {
    gen_range((const job_t*)arg);
    return 0;
}

/* Fill out[0..n) with tensor `kind`; returns 0, or -1 for an unknown kind. */
int synth_fill(int kind, uint64_t seed, double mean, double std, double outlier_p, double outlier_mul,
               double zero_p, uint16_t* out, uint64_t n, int threads) {
    if (kind < 0 || kind > 3) return -1;
    if (threads < 1) threads = 1;
    if (threads > 256) threads = 256;
    if ((uint64_t)threads > n / 65536 + 1) threads = (int)(n / 65536 + 1);
    job_t jobs[256];
    pthread_t tids[256];
    uint64_t per = (n + (uint64_t)threads - 1) / (uint64_t)threads;
    per = (per + 1) & ~1ULL; /* even split points keep Box-Muller pairs whole */
    int t;
    for (t = 0; t < threads; ++t) {
        job_t* j = &jobs[t];
        j->kind = kind;
        j->seed = seed;
        j->mean = mean;
        j->std = std;
        j->outlier_p = outlier_p;
        j->outlier_mul = outlier_mul;
        j->zero_p = zero_p;
        j->out = out;
        j->lo = per * (uint64_t)t;
        j->hi = per * (uint64_t)(t + 1);
        if (j->lo > n) j->lo = n;
        if (j->hi > n) j->hi = n;
    }
    if (threads == 1) {
        gen_range(&jobs[0]);
        return 0;
    }
    int started = 0;
    for (t = 0; t < threads; ++t) {
        if (pthread_create(&tids[t], 0, worker, &jobs[t]) != 0) break;
        started++;
    }
    for (t = started; t < threads; ++t) gen_range(&jobs[t]);
    for (t = 0; t < started; ++t) pthread_join(tids[t], 0);
    return 0;
}
