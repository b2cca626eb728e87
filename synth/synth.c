/*
 * Seeded synthetic input generator shared by the tests, the bench and the
 * oracle's callers.  It holds none of the attention method's arithmetic: it
 * only turns (seed, stream, index) into numbers.
 *
 * Generator (counter based, so any element can be produced independently and
 * in parallel):
 *   - mixing function: the SplitMix64 output function (Steele, Lea & Flood,
 *     "Fast splittable pseudorandom number generators", OOPSLA 2014: add the
 *     golden-ratio increment, then Stafford's "Mix13" 64-bit finaliser);
 *   - a stream key  K = mix(seed) ^ mix(stream + 0x5bd1e995);
 *   - element i draws two 64-bit words  w1 = mix(K + 2i), w2 = mix(K + 2i + 1);
 *   - uniforms  u1 = ((w1 >> 11) + 1) * 2^-53  in (0, 1],
 *               u2 =  (w2 >> 11)      * 2^-53  in [0, 1);
 *   - standard normal by the Box–Muller transform (cosine branch):
 *               z = sqrt(-2 ln u1) * cos(2 pi u2), evaluated in fp64.
 * Narrower outputs are rounded from the fp64 value: fp32 by C's
 * round-to-nearest-even conversion, bf16 from that fp32 by round-to-nearest-
 * even on the upper 16 bits.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t mix64(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
    return mix64(seed) ^ mix64(stream + 0x5bd1e995ull);
}

static inline double normal_at(uint64_t key, uint64_t i) {
    const double two_pow_m53 = 1.0 / 9007199254740992.0;
    uint64_t w1 = mix64(key + 2 * i);
    uint64_t w2 = mix64(key + 2 * i + 1);
    double u1 = (double)((w1 >> 11) + 1) * two_pow_m53;
    double u2 = (double)(w2 >> 11) * two_pow_m53;
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* Raw 64-bit draw number i of (seed, stream). */
uint64_t synth_u64(uint64_t seed, uint64_t stream, uint64_t i) {
    return mix64(stream_key(seed, stream) + i);
}

void synth_normal_f64(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double* out) {
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = normal_at(key, offset + (uint64_t)i);
}

void synth_normal_f32(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, float* out) {
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (float)normal_at(key, offset + (uint64_t)i);
}

void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, uint16_t* out) {
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne((float)normal_at(key, offset + (uint64_t)i));
}

/* Round fp64 values to the storage types (same rounding as above). */
void synth_round_f32(const double* in, int64_t n, float* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = (float)in[i];
}

void synth_round_bf16(const double* in, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne((float)in[i]);
}
