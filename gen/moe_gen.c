/*
 * Seeded synthetic inputs for the MoE expert layer.
 *
 * This module is shared by the CPU oracle and the CUDA path: it only draws
 * random bits and lays them out as bytes.  It holds none of the layer's
 * arithmetic (no dequantisation, no routing, no matmul).
 *
 * Random source: SplitMix64 (Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014).  Its i-th output from state
 * s is mix64(s + (i+1) * golden), so every element of a tensor is a pure
 * function of (key, index) and the generator parallelises without changing a
 * single bit.
 *
 * Streams: key(seed, tensor, layer) = out(out(seed, tensor), layer), where
 * out(s, i) is the i-th SplitMix64 output from state s.
 *
 * Normals: Box-Muller on two 53-bit uniforms (draws 2i and 2i+1 of the
 * stream give element i), computed in double, rounded to fp32 and then to
 * bf16 round-to-nearest-even.
 *
 * Codes: draw j of a code stream fills u32 words 2j (low half) and 2j+1 (high
 * half), so every nibble is uniform on 0..15.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* i-th (0-based) SplitMix64 output from state s. */
uint64_t gen_draw(uint64_t s, uint64_t i) { return mix64(s + (i + 1) * GOLDEN); }

uint64_t gen_key(uint64_t seed, uint64_t tensor, uint64_t layer) {
    return gen_draw(gen_draw(seed, tensor), layer);
}

/* fp32 -> bf16 bits, round to nearest even (inputs are finite). */
static inline uint16_t f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

static inline double normal_at(uint64_t key, int64_t i) {
    const double two_pi = 6.283185307179586476925286766559;
    uint64_t a = gen_draw(key, (uint64_t)(2 * i));
    uint64_t b = gen_draw(key, (uint64_t)(2 * i + 1));
    double u1 = ((double)(a >> 11) + 1.0) * 0x1.0p-53; /* (0, 1] */
    double u2 = (double)(b >> 11) * 0x1.0p-53;         /* [0, 1) */
    return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

/* out[i] = bf16(std * N(0,1)), or its absolute value when absval != 0. */
void gen_normal_bf16(uint64_t key, double std, int absval, uint16_t* out, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double z = std * normal_at(key, i);
        if (absval) z = fabs(z);
        out[i] = f32_to_bf16((float)z);
    }
}

/* nwords u32 words of uniform nibbles; nwords must be even. */
void gen_codes(uint64_t key, uint32_t* out, int64_t nwords) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nwords / 2; ++j) {
        uint64_t d = gen_draw(key, (uint64_t)j);
        out[2 * j] = (uint32_t)d;
        out[2 * j + 1] = (uint32_t)(d >> 32);
    }
}

/* ngroups (scale, bias) bf16 pairs: scale = bf16(|N(0, std)|), bias = -8*scale.
 * Multiplying a bf16 by 8 only moves its exponent, so the bias is exact. */
void gen_scale_bias(uint64_t key, double std, uint16_t* sb, int64_t ngroups) {
#pragma omp parallel for schedule(static)
    for (int64_t g = 0; g < ngroups; ++g) {
        float s = fabsf((float)(std * normal_at(key, g)));
        uint16_t sbits = f32_to_bf16(s);
        uint32_t u = (uint32_t)sbits << 16;
        float sr;
        memcpy(&sr, &u, 4);
        sb[2 * g] = sbits;
        sb[2 * g + 1] = f32_to_bf16(-8.0f * sr);
    }
}

/* First m entries of a Fisher-Yates shuffle of 0..n-1; swap j takes draw j
 * modulo (n - j). */
void gen_partial_shuffle(uint64_t key, int32_t n, int32_t m, int32_t* out_first_m, int32_t* scratch_n) {
    for (int32_t i = 0; i < n; ++i) scratch_n[i] = i;
    for (int32_t j = 0; j < m; ++j) {
        uint64_t d = gen_draw(key, (uint64_t)j);
        int32_t r = j + (int32_t)(d % (uint64_t)(n - j));
        int32_t t = scratch_n[j];
        scratch_n[j] = scratch_n[r];
        scratch_n[r] = t;
        out_first_m[j] = scratch_n[j];
    }
}

/* ---- inputs of the recurrent-state scan (a second workload of the pages) */

/* out[i] = float(lo + (hi - lo) * u), u = the top 24 bits of draw i / 2^24 in [0, 1). */
void gen_uniform_f32(uint64_t key, double lo, double hi, float* out, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double u = (double)(gen_draw(key, (uint64_t)i) >> 40) * 0x1.0p-24;
        out[i] = (float)(lo + (hi - lo) * u);
    }
}

/* out[i] = float(std * N(0,1)). */
void gen_normal_f32(uint64_t key, double std, float* out, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (float)(std * normal_at(key, i));
}

/* nvec vectors of dim elements drawn uniformly on the unit sphere: N(0,1)
 * elements (element j of vector v is normal j + v*dim of the stream) divided
 * by their Euclidean norm in double, then rounded to fp32 and to bf16. */
void gen_unit_bf16(uint64_t key, int64_t nvec, int64_t dim, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t v = 0; v < nvec; ++v) {
        double ss = 0.0;
        for (int64_t j = 0; j < dim; ++j) {
            double z = normal_at(key, v * dim + j);
            ss += z * z;
        }
        double inv = ss > 0.0 ? 1.0 / sqrt(ss) : 0.0;
        for (int64_t j = 0; j < dim; ++j) out[v * dim + j] = f32_to_bf16((float)(normal_at(key, v * dim + j) * inv));
    }
}
