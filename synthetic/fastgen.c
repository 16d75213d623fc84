/* fastgen.c -- host implementation of the synthetic weight generator
 * (same definition as synthetic/weights.py, written again for speed):
 *   h1 = lowbias32(lowbias32(i) ^ key), h2 = lowbias32(h1 ^ 0x9E3779B9)
 *   S  = sum of the 16-bit halves of h1 and h2 - 131070
 *   w  = fp32(S) * scale (+ offset), rounded to the storage type (bf16: nearest-even)
 * lowbias32: C. Wellons, "Prospecting for hash functions" (2018).
 * Holds no arithmetic of the decoding method. */
#include <stdint.h>
#include <string.h>

static inline uint32_t lowbias32(uint32_t x) {
    x ^= x >> 16;
    x *= 0x7feb352du;
    x ^= x >> 15;
    x *= 0x846ca68bu;
    x ^= x >> 16;
    return x;
}

static inline float value(uint64_t i, uint32_t key, float scale, float offset, int add_offset) {
    uint32_t h1 = lowbias32(lowbias32((uint32_t)i) ^ key);
    uint32_t h2 = lowbias32(h1 ^ 0x9E3779B9u);
    int32_t s = (int32_t)(h1 & 0xFFFFu) + (int32_t)(h1 >> 16) + (int32_t)(h2 & 0xFFFFu) + (int32_t)(h2 >> 16) - 131070;
    float v = (float)s * scale;
    if (add_offset) v = v + offset;
    return v;
}

void fastgen_f32(float *out, uint64_t n, uint32_t key, float scale, float offset, int add_offset) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = value((uint64_t)i, key, scale, offset, add_offset);
}

void fastgen_bf16(uint16_t *out, uint64_t n, uint32_t key, float scale) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) {
        float v = value((uint64_t)i, key, scale, 0.0f, 0);
        uint32_t b;
        memcpy(&b, &v, 4);
        b += 0x7FFFu + ((b >> 16) & 1u);   /* round to nearest even (finite values) */
        out[i] = (uint16_t)(b >> 16);
    }
}
