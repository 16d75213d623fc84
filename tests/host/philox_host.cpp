// Host build of the library's sampling generator (csrc/philox.cuh) for the CPU
// tests.  Reads lines "c0 c1 c2 c3 k0 k1" (hex) or "u seed pos slot purpose n"
// from stdin; prints the four output words, or n uniforms as exact hex floats.
#include <cstdio>
#include <cstring>

#include "philox.cuh"

int main() {
    char kind[8];
    while (std::scanf("%7s", kind) == 1) {
        if (!std::strcmp(kind, "p")) {
            unsigned c[4], k[2];
            if (std::scanf("%x %x %x %x %x %x", &c[0], &c[1], &c[2], &c[3], &k[0], &k[1]) != 6) return 2;
            uint32_t out[4];
            dfl::philox4x32_10(c[0], c[1], c[2], c[3], k[0], k[1], out);
            std::printf("%08x %08x %08x %08x\n", out[0], out[1], out[2], out[3]);
        } else if (!std::strcmp(kind, "u")) {
            unsigned long long seed;
            unsigned pos, slot, purpose, n;
            if (std::scanf("%llu %u %u %u %u", &seed, &pos, &slot, &purpose, &n) != 5) return 2;
            const dfl::SampleKey key = dfl::sample_key(seed);
            for (unsigned q = 0; 4 * q < n; ++q) {
                float u[4];
                dfl::uniforms4(key, q, pos, slot, purpose, u);
                for (unsigned i = 0; i < 4 && 4 * q + i < n; ++i) std::printf("%a\n", (double)u[i]);
            }
            std::printf("s %a\n", (double)dfl::uniform1(key, pos, slot, purpose));
        } else {
            return 2;
        }
    }
    return 0;
}
