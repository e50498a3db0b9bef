/*
 * Seeded synthetic inputs: weights, gains, prompts, KV fills.
 *
 * This file holds no layer arithmetic. It defines one counter-based
 * generator, used by both the CPU oracle and the CUDA path:
 *
 *   SplitMix64 finaliser (Steele, Lea & Flood, "Fast splittable pseudorandom
 *   number generators", OOPSLA 2014): mix(z) = three xor-shift-multiply rounds
 *   with the published constants 0xBF58476D1CE4E5B9 and 0x94D049BB133111EB.
 *
 *   stream key   K(seed, id) = mix(mix(seed + G) ^ (id * G + 1))
 *   raw word n   R(K, n)     = mix(K + (n + 1) * G)        G = 0x9E3779B97F4A7C15
 *
 * Normals come in pairs (Box & Muller 1958): for pair j take two raw words
 * a = R(K, 2j), b = R(K, 2j+1); u1 = ((a >> 11) + 1) / 2^53 in (0, 1],
 * u2 = (b >> 11) / 2^53 in [0, 1); r = sqrt(-2 ln u1), t = 2 pi u2;
 * element 2j = r cos t, element 2j+1 = r sin t. All in fp64.
 * A value mean + std * z is rounded once from fp64 to bf16, nearest-even.
 *
 * Uniform integers in [0, V): R(K, n) mod V.
 *
 * int8 values (synthetic q8_row weight rows): nearbyint(std * z) clamped to
 * [-127, 127], z a normal of the same stream definition.
 *
 * The device twin of these functions lives in synth_fill.cu and follows the
 * same definitions; tests compare the two.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYN_G 0x9E3779B97F4A7C15ULL

static inline uint64_t syn_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t syn_stream_key(uint64_t seed, uint64_t id) {
    return syn_mix(syn_mix(seed + SYN_G) ^ (id * SYN_G + 1ULL));
}

uint64_t syn_raw(uint64_t key, uint64_t n) { return syn_mix(key + (n + 1ULL) * SYN_G); }

/* fp64 -> bf16 bits, round to nearest, ties to even (finite inputs). */
uint16_t syn_round_bf16(double v) {
    if (v == 0.0) return signbit(v) ? 0x8000u : 0u;
    int e;
    double m = frexp(fabs(v), &e);          /* |v| = m * 2^e, m in [0.5, 1) */
    /* bf16 keeps 8 significant bits for normals; below 2^-126 the quantum is 2^-133. */
    int q = e - 8;
    if (q < -133) q = -133;
    double scaled = ldexp(fabs(v), -q);     /* exact */
    double r = nearbyint(scaled);           /* default rounding mode: nearest-even */
    double a = ldexp(r, q);
    float f = (float)a;                     /* exact: a has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t h = (uint16_t)(u >> 16);
    if (v < 0) h |= 0x8000u;
    return h;
}

double syn_normal(uint64_t key, uint64_t i) {
    uint64_t j = i >> 1;
    uint64_t a = syn_raw(key, 2 * j), b = syn_raw(key, 2 * j + 1);
    double u1 = (double)((a >> 11) + 1ULL) * 0x1.0p-53;
    double u2 = (double)(b >> 11) * 0x1.0p-53;
    double r = sqrt(-2.0 * log(u1));
    double t = 6.283185307179586476925286766559 * u2;
    return (i & 1ULL) ? r * sin(t) : r * cos(t);
}

/* out[i] = bf16(mean + std * z_i), i in [0, n); z from stream (seed, id). */
void syn_fill_bf16(uint16_t* out, int64_t n, uint64_t seed, uint64_t id, double mean, double std) {
    uint64_t key = syn_stream_key(seed, id);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = syn_round_bf16(mean + std * syn_normal(key, (uint64_t)i));
}

/* Same values as syn_fill_bf16, widened to fp32 (1-D parameters). */
void syn_fill_bf16_as_f32(float* out, int64_t n, uint64_t seed, uint64_t id, double mean, double std) {
    uint64_t key = syn_stream_key(seed, id);
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u = (uint32_t)syn_round_bf16(mean + std * syn_normal(key, (uint64_t)i)) << 16;
        memcpy(&out[i], &u, 4);
    }
}

/* out[i] = R(K, i) mod V. */
void syn_fill_tokens(int32_t* out, int64_t n, uint64_t seed, uint64_t id, int32_t vocab) {
    uint64_t key = syn_stream_key(seed, id);
    for (int64_t i = 0; i < n; ++i) out[i] = (int32_t)(syn_raw(key, (uint64_t)i) % (uint64_t)vocab);
}

/* Raw fp64 normals (no rounding), for generators that post-process them. */
void syn_fill_normal_f64(double* out, int64_t n, uint64_t seed, uint64_t id) {
    uint64_t key = syn_stream_key(seed, id);
    for (int64_t i = 0; i < n; ++i) out[i] = syn_normal(key, (uint64_t)i);
}

/* Uniform fp64 in [0, 1) from raw word i. */
void syn_fill_uniform_f64(double* out, int64_t n, uint64_t seed, uint64_t id) {
    uint64_t key = syn_stream_key(seed, id);
    for (int64_t i = 0; i < n; ++i) out[i] = (double)(syn_raw(key, (uint64_t)i) >> 11) * 0x1.0p-53;
}

/* out[i] = clamp(nearbyint(std * z_i), -127, 127) as int8; z from stream (seed, id). */
void syn_fill_i8(int8_t* out, int64_t n, uint64_t seed, uint64_t id, double std) {
    uint64_t key = syn_stream_key(seed, id);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double v = nearbyint(std * syn_normal(key, (uint64_t)i));
        if (v > 127.0) v = 127.0;
        if (v < -127.0) v = -127.0;
        out[i] = (int8_t)v;
    }
}
