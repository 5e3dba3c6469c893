/*
 * Seeded synthetic inputs, host side.
 *
 * This file holds the input generator only: no step of the CSA2 method is
 * computed here.  The same generator is implemented for the device in
 * synth_dev.cu from the same definition, so both produce identical values:
 *
 *   mix(z)        SplitMix64 output function (Steele, Lea & Flood, "Fast
 *                 splittable pseudorandom number generators", OOPSLA 2014):
 *                 z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27;
 *                 z *= 0x94D049BB133111EB; z ^= z>>31   (mod 2^64)
 *   key(seed, tensor, sub)
 *                 = mix(mix(mix(seed + G) + tensor*G) + sub*G),
 *                   G = 0x9E3779B97F4A7C15 (the SplitMix64 increment)
 *   u64(key, i)   = mix(key + (i+1)*G)     -- counter based: element i
 *                   of a tensor never depends on any other element
 *   normal(key,i) = Irwin-Hall sum of twelve 16-bit uniforms taken from
 *                   u64(key,3i), u64(key,3i+1), u64(key,3i+2):
 *                   S = sum of the twelve chunks, value = (2S - 786420)/131072.
 *                   Mean 0, variance 1 - 2^-32, support [-6, 6]; the value is
 *                   an integer over 2^17, so it is exact in fp32.
 *   uniform(key,i)= (u64(key,i) >> 40) * 2^-24, exact fp32 in [0, 1).
 *   bf16 values   = round-to-nearest-even of the fp32 product
 *                   normal * chan_scale[channel] (fp32 multiply, RNE).
 *
 * Only integer arithmetic and single IEEE fp32 operations are used, so the
 * host and device generators agree bit for bit by construction.
 */
#include <stdint.h>
#include <string.h>

#define SYNTH_G 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t synth_key(uint64_t seed, uint64_t tensor, uint64_t sub) {
    return mix64(mix64(mix64(seed + SYNTH_G) + tensor * SYNTH_G) + sub * SYNTH_G);
}

uint64_t synth_u64(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * SYNTH_G); }

static inline int32_t ih12(uint64_t key, uint64_t i) {
    int64_t s = 0;
    for (int k = 0; k < 3; ++k) {
        uint64_t u = synth_u64(key, 3 * i + (uint64_t)k);
        s += (int64_t)(u & 0xFFFF) + (int64_t)((u >> 16) & 0xFFFF) +
             (int64_t)((u >> 32) & 0xFFFF) + (int64_t)(u >> 48);
    }
    return (int32_t)(2 * s - 786420);
}

static inline float normal_f32(uint64_t key, uint64_t i) {
    return (float)ih12(key, i) * (1.0f / 131072.0f); /* exact: |num| < 2^20 */
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

void synth_normal_f32(uint64_t key, uint64_t start, int64_t n, float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) out[j] = normal_f32(key, start + (uint64_t)j);
}

/* out[j] = bf16(normal(start+j) * scale[(start+j) % nchan]); scale may be NULL (=1). */
void synth_normal_bf16(uint64_t key, uint64_t start, int64_t n, const float* scale,
                       int64_t nchan, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        uint64_t i = start + (uint64_t)j;
        float v = normal_f32(key, i);
        if (scale) v = v * scale[i % (uint64_t)nchan];
        out[j] = f32_to_bf16_rne(v);
    }
}

/* out[j] = normal(start+j) * scale (one fp32 multiply). */
void synth_normal_scaled_f32(uint64_t key, uint64_t start, int64_t n, float scale, float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) out[j] = normal_f32(key, start + (uint64_t)j) * scale;
}

/* 2-D form: out[r][j] = element start + r * row_stride + j, j < row_len. */
void synth_normal_bf16_rows(uint64_t key, uint64_t start, uint64_t row_stride, int64_t rows,
                            int64_t row_len, const float* scale, int64_t nchan, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < row_len; ++j) {
            uint64_t i = start + (uint64_t)r * row_stride + (uint64_t)j;
            float v = normal_f32(key, i);
            if (scale) v = v * scale[i % (uint64_t)nchan];
            out[r * row_len + j] = f32_to_bf16_rne(v);
        }
}

void synth_normal_f32_rows(uint64_t key, uint64_t start, uint64_t row_stride, int64_t rows,
                           int64_t row_len, float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < row_len; ++j)
            out[r * row_len + j] = normal_f32(key, start + (uint64_t)r * row_stride + (uint64_t)j);
}

void synth_uniform_f32(uint64_t key, uint64_t start, int64_t n, float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        out[j] = (float)(synth_u64(key, start + (uint64_t)j) >> 40) * (1.0f / 16777216.0f);
}

void synth_u64_array(uint64_t key, uint64_t start, int64_t n, uint64_t* out) {
    for (int64_t j = 0; j < n; ++j) out[j] = synth_u64(key, start + (uint64_t)j);
}
