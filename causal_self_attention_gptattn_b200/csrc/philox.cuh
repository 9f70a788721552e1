// philox.cuh -- the counter-based generator behind the attention-dropout mask.
//
// Philox4x32-10 (J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3", SC 2011): ten rounds over a 128-bit counter
// under a 64-bit key.  Each round forms the 64-bit products of the first and
// third counter words with the two round multipliers and rebuilds the counter
// from their halves, the other two words and the key; the key then advances by
// the two Weyl constants.
//
// Mask convention (shared with the rest of the library): one generator call
// covers a 4 x 4 block of (query t, key s) pairs of batch-head pair bh: counter
// (s / 4, t / 4, bh, 0), key (seed low word, seed high word); the pair's 8 bits
// are byte s % 4 (least significant first) of output word t % 4, and the weight
// is kept iff that byte is at least theta = round(256 p) (at most 255); kept
// weights are scaled by 1 / (1 - theta / 256).
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

// Keep bits of the four bytes of w against theta: bit i <-> byte i.
__device__ __forceinline__ uint32_t keep_bits4(uint32_t w, uint32_t theta) {
    return ((w & 0xFFu) >= theta ? 1u : 0u) | (((w >> 8) & 0xFFu) >= theta ? 2u : 0u) |
           (((w >> 16) & 0xFFu) >= theta ? 4u : 0u) | ((w >> 24) >= theta ? 8u : 0u);
}

// Keep bits of the 4 keys s0 .. s0+3 (s0 a multiple of 4) for query t: bit i <-> key s0 + i.
__device__ __forceinline__ uint32_t dropout_keep4(uint64_t seed, uint32_t theta, uint32_t bh, uint32_t t,
                                                  uint32_t s0) {
    const uint4 r = philox4x32_10(make_uint4(s0 >> 2, t >> 2, bh, 0u), (uint32_t)seed, (uint32_t)(seed >> 32));
    const uint32_t q = t & 3u;
    return keep_bits4(q == 0u ? r.x : q == 1u ? r.y : q == 2u ? r.z : r.w, theta);
}

// Keep bits of the 4 queries t0 .. t0+3 (t0 a multiple of 4) for key s: bit i <-> query t0 + i.
__device__ __forceinline__ uint32_t dropout_keep4_keys(uint64_t seed, uint32_t theta, uint32_t bh, uint32_t t0,
                                                       uint32_t s) {
    const uint4 r = philox4x32_10(make_uint4(s >> 2, t0 >> 2, bh, 0u), (uint32_t)seed, (uint32_t)(seed >> 32));
    const uint32_t sh = 8u * (s & 3u);
    return (((r.x >> sh) & 0xFFu) >= theta ? 1u : 0u) | (((r.y >> sh) & 0xFFu) >= theta ? 2u : 0u) |
           (((r.z >> sh) & 0xFFu) >= theta ? 4u : 0u) | (((r.w >> sh) & 0xFFu) >= theta ? 8u : 0u);
}

// The same decisions with the generator calls shared by the four lanes that hold
// four consecutive query rows (forward) or key rows (backward) of one 4 x 4 block
// row: lanes 4k..4k+3 of a warp, the row's lane at position row % 4.  Each lane
// draws a quarter of the blocks and the four exchange what the others need in
// four shuffle rounds (in round k, lane r reads from lane (r + k) % 4, which sends
// the part meant for lane (its own position - k) % 4).  Every lane of the warp
// must call these together.

// Keep bits of keys s_base .. s_base+31 (s_base a multiple of 32) for query t:
// bit i <-> key s_base + i.  Requires lane % 4 == t % 4.
__device__ __forceinline__ uint32_t dropout_keep32_rows(uint64_t seed, uint32_t theta, uint32_t bh, uint32_t t,
                                                        uint32_t s_base, int lane) {
    const int r = lane & 3;
    uint32_t acc = 0u;
#pragma unroll
    for (int hb = 0; hb < 2; ++hb) {  // key groups 4*hb .. 4*hb+3 of 4 keys; this lane draws group 4*hb + r
        const uint4 blk = philox4x32_10(make_uint4((s_base >> 2) + 4u * hb + r, t >> 2, bh, 0u), (uint32_t)seed,
                                        (uint32_t)(seed >> 32));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int w = (r - k) & 3;  // the row (word) wanted by the lane reading this one
            const uint32_t send = w == 0 ? blk.x : w == 1 ? blk.y : w == 2 ? blk.z : blk.w;
            const int src = (r + k) & 3;
            const uint32_t got = __shfl_sync(0xFFFFFFFFu, send, (lane & ~3) | src);
            acc |= keep_bits4(got, theta) << (4 * (4 * hb + src));
        }
    }
    return acc;
}

// Keep bits of queries t_base .. t_base+15 (t_base a multiple of 16) for key s:
// bit i <-> query t_base + i.  Requires lane % 4 == s % 4.
__device__ __forceinline__ uint32_t dropout_keep16_keys(uint64_t seed, uint32_t theta, uint32_t bh, uint32_t t_base,
                                                        uint32_t s, int lane) {
    const int r = lane & 3;
    // this lane draws the block of queries t_base + 4r .. t_base + 4r + 3
    const uint4 blk = philox4x32_10(make_uint4(s >> 2, (t_base >> 2) + r, bh, 0u), (uint32_t)seed,
                                    (uint32_t)(seed >> 32));
    uint32_t acc = 0u;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t d = (uint32_t)((r - k) & 3);  // key position (byte) wanted by the reading lane
        const uint32_t sel = d | ((4u + d) << 4);
        const uint32_t send = __byte_perm(__byte_perm(blk.x, blk.y, sel), __byte_perm(blk.z, blk.w, sel), 0x5410);
        const int src = (r + k) & 3;
        const uint32_t got = __shfl_sync(0xFFFFFFFFu, send, (lane & ~3) | src);
        acc |= keep_bits4(got, theta) << (4 * src);
    }
    return acc;
}

// Dropout parameters as the kernels take them: threshold 0 means no dropout.
struct DropoutParams {
    uint64_t seed;
    uint32_t threshold;  // theta = round(256 p), at most 255
    float scale;         // 1 / (1 - theta / 256)
};

}  // namespace gptattn
