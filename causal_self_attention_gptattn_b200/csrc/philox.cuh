// philox.cuh -- the counter-based generator behind the attention-dropout mask.
//
// Philox4x32-10 (J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3", SC 2011): ten rounds over a 128-bit counter
// under a 64-bit key.  Each round forms the 64-bit products of the first and
// third counter words with the two round multipliers and rebuilds the counter
// from their halves, the other two words and the key; the key then advances by
// the two Weyl constants.
//
// Mask convention (shared with the rest of the library): the weight of query t
// for key s in batch-head pair bh is kept iff word s % 4 of the generator at
// counter (s / 4, t, bh, 0), key (seed low word, seed high word), is at least
// floor(p * 2^32); kept weights are scaled by 1 / (1 - p).
#pragma once
#include <stdint.h>

namespace gptattn {

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint32_t lo0 = c.x * 0xD2511F53u, hi0 = __umulhi(c.x, 0xD2511F53u);
        const uint32_t lo1 = c.z * 0xCD9E8D57u, hi1 = __umulhi(c.z, 0xCD9E8D57u);
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c;
}

// Keep bits of the 4 keys s0 .. s0+3 (s0 a multiple of 4) for query t: bit i <-> key s0 + i.
__device__ __forceinline__ uint32_t dropout_keep4(uint64_t seed, uint32_t threshold, uint32_t bh, uint32_t t,
                                                  uint32_t s0) {
    const uint4 r = philox4x32_10(make_uint4(s0 >> 2, t, bh, 0u), (uint32_t)seed, (uint32_t)(seed >> 32));
    return (r.x >= threshold ? 1u : 0u) | (r.y >= threshold ? 2u : 0u) | (r.z >= threshold ? 4u : 0u) |
           (r.w >= threshold ? 8u : 0u);
}

// Dropout parameters as the kernels take them: threshold 0 means no dropout.
struct DropoutParams {
    uint64_t seed;
    uint32_t threshold;  // floor(p * 2^32)
    float scale;         // 1 / (1 - p)
};

}  // namespace gptattn
