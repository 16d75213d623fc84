// philox.cuh -- the counter-based generator of temperature sampling.
//
// Philox4x32 with 10 rounds (J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel
// random numbers: as easy as 1, 2, 3", SC 2011): each round multiplies counter
// words 0 and 2 by the two Philox multipliers, and the high halves, XORed with
// the other two words and the round key, become the new words 0 and 2; the key
// grows by the two Weyl constants between rounds.
//
// Draws of temperature sampling: key = the 64-bit seed (low word first),
// counter = (j / 4, position, sequence slot, purpose) and word j % 4 give draw
// j of a vocabulary-wide vector; scalar draws take j = 0.  A word w becomes
// u = (floor(w / 512) + 1/2) * 2^-23: 23 random bits, exact in fp32.  Tokens are
// drawn by Gumbel-max, argmax_v (s_v - log(-log(u_v))).
//
// Host and device share this code (a host build is checked against the
// generator's published known-answer vectors).
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define DFL_HD __host__ __device__ __forceinline__
#else
#define DFL_HD inline
#endif

namespace dfl {

enum SamplePurpose : uint32_t { SP_DRAFT = 1, SP_ACCEPT = 2, SP_RESIDUAL = 3, SP_TARGET = 4 };

DFL_HD void philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0, uint32_t k1,
                          uint32_t out[4]) {
#if defined(__CUDA_ARCH__)
#pragma unroll
#endif
    for (int r = 0; r < 10; ++r) {
        if (r) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        c1 = (uint32_t)p1;
        c3 = (uint32_t)p0;
        c0 = n0;
        c2 = n2;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

DFL_HD float word_to_uniform(uint32_t w) { return ((float)(w >> 9) + 0.5f) * (1.0f / 8388608.0f); }

struct SampleKey {
    uint32_t k0, k1;  // seed, low word first
};

DFL_HD SampleKey sample_key(uint64_t seed) { return SampleKey{(uint32_t)seed, (uint32_t)(seed >> 32)}; }

// draws 4q .. 4q+3 of (position, slot, purpose)
DFL_HD void uniforms4(SampleKey key, uint32_t q, uint32_t pos, uint32_t slot, uint32_t purpose, float u[4]) {
    uint32_t w[4];
    philox4x32_10(q, pos, slot, purpose, key.k0, key.k1, w);
    for (int i = 0; i < 4; ++i) u[i] = word_to_uniform(w[i]);
}

// draw 0 of (position, slot, purpose)
DFL_HD float uniform1(SampleKey key, uint32_t pos, uint32_t slot, uint32_t purpose) {
    uint32_t w[4];
    philox4x32_10(0, pos, slot, purpose, key.k0, key.k1, w);
    return word_to_uniform(w[0]);
}

}  // namespace dfl
