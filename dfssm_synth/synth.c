/*
 * Seeded synthetic inputs for the DF-SSM scaffold linear.
 *
 * This file only DRAWS inputs: activations x, packed sign bits, per-row scales,
 * int8 LoRA factors. It computes nothing of the layer itself (no quantizer,
 * no contraction, no dequantisation), so both the CPU oracle and the CUDA path
 * can read the same bytes without sharing any of the method's arithmetic.
 *
 * Random numbers: SplitMix64 (Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014) used in counter mode:
 *   key     = mix(seed + mix(stream_id))
 *   draw(i) = mix(key + (i + 1) * 0x9E3779B97F4A7C15)
 * where mix() is the SplitMix64 output function. Every element is a pure
 * function of (seed, stream_id, index), so generation order and thread count
 * do not change the bytes.
 *
 * Distributions (the Mamba-2-1.3B-shaped workload of the scaffold linear):
 *   x      bf16, z ~ N(0,1) by Box-Muller in f64; round(0.01*d_in) seeded
 *          "outlier" input channels are scaled by 20; one RNE rounding f64->bf16
 *   sign   Bernoulli(0.5) bits written straight into the packed bytes
 *   alpha  fp32 ~ U(0.005, 0.05)
 *   wa, wb int8 ~ U{-127..127}
 *   sa, sb fp32 ~ U(1e-4, 1e-3)
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t dfssm_synth_key(uint64_t seed, uint64_t stream_id) {
    return mix64(seed + mix64(stream_id + GOLDEN));
}

static inline uint64_t draw(uint64_t key, uint64_t i) {
    return mix64(key + (i + 1) * GOLDEN);
}

/* uniform in [0, 1) with 53 random bits */
static inline double u01(uint64_t r) { return (double)(r >> 11) * 0x1.0p-53; }

/* f64 -> bf16 bit pattern, round to nearest, ties to even, one rounding. */
static uint16_t f64_to_bf16_rne(double v) {
    if (v == 0.0) return signbit(v) ? 0x8000 : 0x0000;
    int e;
    double f = frexp(fabs(v), &e);           /* |v| = f * 2^e, f in [0.5, 1) */
    double s = nearbyint(ldexp(f, 8));       /* 8 significant bits, RNE      */
    float r = (float)ldexp(s, e - 8);        /* exact in fp32 for our range  */
    uint32_t b;
    memcpy(&b, &r, 4);
    if (v < 0) b |= 0x80000000u;
    return (uint16_t)(b >> 16);
}

/* Raw 64-bit draws (exposed so tests can pin the generator itself). */
void dfssm_synth_raw(uint64_t key, uint64_t start, int64_t n, uint64_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = draw(key, start + (uint64_t)i);
}

/* Seeded set of n_out distinct column indices in [0, d_in): partial Fisher-Yates. */
void dfssm_synth_outlier_cols(uint64_t key, int d_in, int n_out, int32_t* cols) {
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)d_in);
    for (int j = 0; j < d_in; ++j) perm[j] = j;
    for (int i = 0; i < n_out; ++i) {
        uint64_t r = draw(key, (uint64_t)i);
        int span = d_in - i;
        int pick = i + (int)(((r >> 32) * (uint64_t)span) >> 32);
        int32_t t = perm[i]; perm[i] = perm[pick]; perm[pick] = t;
        cols[i] = perm[i];
    }
    free(perm);
}

/* x: m x d_in bf16 bits, row-major. scale[j] = 20 for outlier channels else 1. */
void dfssm_synth_x(uint64_t key_x, uint64_t key_cols, int m, int d_in, uint16_t* x) {
    int n_out = (int)floor(0.01 * d_in + 0.5);
    float* scale = (float*)malloc(sizeof(float) * (size_t)d_in);
    for (int j = 0; j < d_in; ++j) scale[j] = 1.0f;
    if (n_out > 0) {
        int32_t* cols = (int32_t*)malloc(sizeof(int32_t) * (size_t)n_out);
        dfssm_synth_outlier_cols(key_cols, d_in, n_out, cols);
        for (int i = 0; i < n_out; ++i) scale[cols[i]] = 20.0f;
        free(cols);
    }
    int64_t total = (int64_t)m * d_in;
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < total; ++i) {
        double u1 = ((double)(draw(key_x, 2 * (uint64_t)i) >> 11) + 1.0) * 0x1.0p-53; /* (0,1] */
        double u2 = u01(draw(key_x, 2 * (uint64_t)i + 1));
        double z = sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
        x[i] = f64_to_bf16_rne((double)scale[i % d_in] * z);
    }
    free(scale);
}

/* n_bytes of Bernoulli(0.5) bits, 8 bytes per draw. */
void dfssm_synth_bits(uint64_t key, int64_t n_bytes, uint8_t* out) {
    int64_t words = n_bytes / 8;
    #pragma omp parallel for schedule(static)
    for (int64_t w = 0; w < words; ++w) {
        uint64_t r = draw(key, (uint64_t)w);
        memcpy(out + 8 * w, &r, 8);
    }
    if (n_bytes % 8) {
        uint64_t r = draw(key, (uint64_t)words);
        memcpy(out + 8 * words, &r, (size_t)(n_bytes % 8));
    }
}

/* fp32 ~ U(lo, hi), computed in f64 then rounded once to fp32. */
void dfssm_synth_uniform_f32(uint64_t key, int64_t n, double lo, double hi, float* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (float)(lo + (hi - lo) * u01(draw(key, (uint64_t)i)));
}

/* int8 ~ U{-127..127} by multiply-shift of the high 32 bits (bias < 2^-24). */
void dfssm_synth_int8_sym127(uint64_t key, int64_t n, int8_t* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint64_t r = draw(key, (uint64_t)i);
        out[i] = (int8_t)((int)(((r >> 32) * 255ULL) >> 32) - 127);
    }
}

/* n normals z ~ N(0,1) (Box-Muller in f64, two draws each) times `scale`, rounded once to fp32
   (bf16 = 0) or to bf16 bits (bf16 = 1). */
void dfssm_synth_normal(uint64_t key, int64_t n, double scale, int bf16, void* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double u1 = ((double)(draw(key, 2 * (uint64_t)i) >> 11) + 1.0) * 0x1.0p-53; /* (0,1] */
        double u2 = u01(draw(key, 2 * (uint64_t)i + 1));
        double z = scale * sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
        if (bf16) ((uint16_t*)out)[i] = f64_to_bf16_rne(z);
        else ((float*)out)[i] = (float)z;
    }
}

/* Exposed for the generator's own tests (bf16 rounding of the x draws). */
uint16_t dfssm_synth_f64_to_bf16(double v) { return f64_to_bf16_rne(v); }
