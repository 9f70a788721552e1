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

// Keep flags of the four bytes of w against theta, each in its byte's top bit:
// bit 8i+7 <-> byte i >= theta, every other bit 0.  t7 holds theta mod 128 in
// every byte; kHigh = (theta >= 128).  Setting each byte's top bit and
// subtracting t7 never borrows across bytes, and leaves the top bit set exactly
// when the byte's low seven bits reach theta's; the byte's own top bit then
// decides: with theta < 128 a set top bit is enough, with theta >= 128 it is
// required.
template <bool kHigh>
__device__ __forceinline__ uint32_t keep_msb4(uint32_t w, uint32_t t7) {
    const uint32_t d = (w | 0x80808080u) - t7;
    return kHigh ? (w & d & 0x80808080u) : ((w | d) & 0x80808080u);
}
__device__ __forceinline__ uint32_t theta_low7(uint32_t theta) { return (theta & 0x7Fu) * 0x01010101u; }

// Packed keep words.  A word holds the flags of 32 consecutive columns; column
// 4j + k (j = 0..7, k = 0..3) is bit 8k + 7 - j, so that (word << j) carries
// columns 4j .. 4j+3 in the top bits of its four bytes, where one byte permute
// with sign replication turns them into masks (keep_pair_mask, keep_word_mask).

// Keep words of keys s0 .. s0+31 (s0 a multiple of 32) for the four queries
// t0 .. t0+3 (t0 a multiple of 4): out[r] for query t0 + r, column i = key
// s0 + i.  Eight generator calls, one per 4 x 4 block.
template <bool kHigh>
__device__ __forceinline__ void dropout_keep32x4(uint64_t seed, uint32_t t7, uint32_t bh, uint32_t t0, uint32_t s0,
                                                 uint32_t (&out)[4]) {
    out[0] = out[1] = out[2] = out[3] = 0u;
#pragma unroll 2
    for (int blk = 0; blk < 8; ++blk) {
        const uint4 r = philox4x32_10(make_uint4((s0 >> 2) + (uint32_t)blk, t0 >> 2, bh, 0u), (uint32_t)seed,
                                      (uint32_t)(seed >> 32));
        out[0] |= keep_msb4<kHigh>(r.x, t7) >> blk;
        out[1] |= keep_msb4<kHigh>(r.y, t7) >> blk;
        out[2] |= keep_msb4<kHigh>(r.z, t7) >> blk;
        out[3] |= keep_msb4<kHigh>(r.w, t7) >> blk;
    }
}

// Keep words of queries t0 .. t0+31 (t0 a multiple of 32) for the four keys
// s0 .. s0+3 (s0 a multiple of 4): out[c] for key s0 + c, column i = query
// t0 + i.  Eight generator calls, one per 4 x 4 block; each call's flags
// (word q = query, byte c = key) are transposed to (word c, byte q).
template <bool kHigh>
__device__ __forceinline__ void dropout_keep32x4_keys(uint64_t seed, uint32_t t7, uint32_t bh, uint32_t s0,
                                                      uint32_t t0, uint32_t (&out)[4]) {
    out[0] = out[1] = out[2] = out[3] = 0u;
#pragma unroll 2
    for (int blk = 0; blk < 8; ++blk) {
        const uint4 r = philox4x32_10(make_uint4(s0 >> 2, (t0 >> 2) + (uint32_t)blk, bh, 0u), (uint32_t)seed,
                                      (uint32_t)(seed >> 32));
        const uint32_t m0 = keep_msb4<kHigh>(r.x, t7), m1 = keep_msb4<kHigh>(r.y, t7);
        const uint32_t m2 = keep_msb4<kHigh>(r.z, t7), m3 = keep_msb4<kHigh>(r.w, t7);
        // 4 x 4 byte transpose: interleave bytes of (m0, m1) and of (m2, m3), then halves
        const uint32_t a = __byte_perm(m0, m1, 0x5140), b = __byte_perm(m0, m1, 0x7362);
        const uint32_t c = __byte_perm(m2, m3, 0x5140), d = __byte_perm(m2, m3, 0x7362);
        out[0] |= __byte_perm(a, c, 0x5410) >> blk;
        out[1] |= __byte_perm(a, c, 0x7632) >> blk;
        out[2] |= __byte_perm(b, d, 0x5410) >> blk;
        out[3] |= __byte_perm(b, d, 0x7632) >> blk;
    }
}

__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
// Mask of the bf16 pair of columns 4j + 2h, 4j + 2h + 1 (0xFFFF per kept
// column), from ws = word << j.
__device__ __forceinline__ uint32_t keep_pair_mask(uint32_t ws, int h) {
    return prmt_b32(ws, 0u, h ? 0xBBAAu : 0x9988u);
}
// Mask of the 32-bit value of column 4j + k (all ones if kept), from ws = word << j.
__device__ __forceinline__ uint32_t keep_word_mask(uint32_t ws, int k) {
    return prmt_b32(ws, 0u, 0x8888u | (0x1111u * (uint32_t)k));
}

// Dropout parameters as the kernels take them: threshold 0 means no dropout.
struct DropoutParams {
    uint64_t seed;
    uint32_t threshold;  // theta = round(256 p), at most 255
    float scale;         // 1 / (1 - theta / 256)
};

}  // namespace gptattn
