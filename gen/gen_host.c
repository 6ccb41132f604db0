/*
 * Seeded synthetic inputs, host side.
 *
 * This file is shared test/bench infrastructure: it produces the raw K, V
 * and q tensors (and small host-side draws such as lengths and residual
 * weights) that both the CUDA path and the fp64 oracle consume.  It holds
 * none of the method's arithmetic.
 *
 * Generator (one counter-based definition, implemented identically here and
 * in gen_device.cu so that host and device produce the same bits):
 *   mix64 is the SplitMix64 output function of Steele, Lea and Flood,
 *   "Fast splittable pseudorandom number generators" (OOPSLA 2014):
 *       z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
 *       z ^= z >> 27; z *= 0x94D049BB133111EB;  z ^= z >> 31.
 *   key(seed, stream)   = mix64(seed + GAMMA * (stream + 1)) ^ stream
 *   draw(key, counter)  = mix64(key + GAMMA * (counter + 1))
 *   with GAMMA = 0x9E3779B97F4A7C15 (the SplitMix64 increment).
 *   normal(key, i): the twelve 16-bit fields u_0..u_11 of draw(key, 3i),
 *   draw(key, 3i+1), draw(key, 3i+2) (low field first) give
 *       S = sum u_j,  x = (2 S - 12 * 65535) * 2^-17,
 *   an Irwin-Hall(12) approximation of N(0,1) (mean 0, variance ~1).
 *   The numerator is an integer below 2^20 in magnitude, so x is exact in
 *   fp32 on both sides.  bf16 values are x rounded to nearest-even.
 */
#include <stdint.h>
#include <string.h>
#include <omp.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z ^= z >> 30; z *= 0xBF58476D1CE4E5B9ULL;
    z ^= z >> 27; z *= 0x94D049BB133111EBULL;
    z ^= z >> 31;
    return z;
}

uint64_t gen_key(uint64_t seed, uint64_t stream) {
    return mix64(seed + GAMMA * (stream + 1)) ^ stream;
}

static inline uint64_t draw(uint64_t key, uint64_t counter) {
    return mix64(key + GAMMA * (counter + 1));
}

static inline float normal_at(uint64_t key, uint64_t i) {
    int32_t s = 0;
    for (int w = 0; w < 3; ++w) {
        uint64_t r = draw(key, 3 * i + (uint64_t)w);
        s += (int32_t)(r & 0xFFFF) + (int32_t)((r >> 16) & 0xFFFF)
           + (int32_t)((r >> 32) & 0xFFFF) + (int32_t)(r >> 48);
    }
    return (float)(2 * s - 12 * 65535) * (1.0f / 131072.0f);
}

static inline uint16_t f32_to_bf16_rne(float x) {
    uint32_t u;
    memcpy(&u, &x, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* Raw 64-bit draws for counters [offset, offset + n). */
void gen_u64(uint64_t key, uint64_t offset, int64_t n, uint64_t* out) {
    for (int64_t j = 0; j < n; ++j) out[j] = draw(key, offset + (uint64_t)j);
}

/* Elements [offset, offset + n) of the normal tensor with this key. */
void gen_normal_f32(uint64_t key, uint64_t offset, int64_t n, float* out, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    #pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t j = 0; j < n; ++j) out[j] = normal_at(key, offset + (uint64_t)j);
}

void gen_normal_bf16(uint64_t key, uint64_t offset, int64_t n, uint16_t* out, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    #pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t j = 0; j < n; ++j) out[j] = f32_to_bf16_rne(normal_at(key, offset + (uint64_t)j));
}

/* Round fp32 values to bf16 (nearest-even); used to store host-built rows
 * (the planted key) in the same way as generated ones. */
void gen_round_bf16(const float* in, int64_t n, uint16_t* out) {
    for (int64_t j = 0; j < n; ++j) out[j] = f32_to_bf16_rne(in[j]);
}
