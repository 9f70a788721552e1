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

// Keep flags of the four bytes of w against theta (1..255), each in its byte's
// top bit: bit 8i+7 <-> byte i >= theta, every other bit 0.  Even and odd
// bytes are compared in two 16-bit lanes: byte + 256 - theta reaches bit 8 of
// its lane exactly when byte >= theta, and no lane carries into the next.
__device__ __forceinline__ uint32_t keep_msb4(uint32_t w, uint32_t theta) {
    const uint32_t k = (256u - theta) * 0x00010001u;
    const uint32_t e = (w & 0x00FF00FFu) + k;         // bits 8, 24: bytes 0, 2
    const uint32_t o = ((w >> 8) & 0x00FF00FFu) + k;  // bits 8, 24: bytes 1, 3
    return ((e >> 1) & 0x00800080u) | ((o << 7) & 0x80008000u);
}

// Packed keep words.  A word holds the flags of 32 consecutive columns; column
// 4j + k (j = 0..7, k = 0..3) is bit 8k + 7 - j, so that (word << j) carries
// columns 4j .. 4j+3 in the top bits of its four bytes, where one byte permute
// with sign replication turns them into masks (keep_pair_mask, keep_word_mask).

// Keep words of keys s0 .. s0+31 (s0 a multiple of 32) for the four queries
// t0 .. t0+3 (t0 a multiple of 4): out[r] for query t0 + r, column i = key
// s0 + i.  Eight generator calls, one per 4 x 4 block.
__device__ __forceinline__ void dropout_keep32x4(uint64_t seed, uint32_t theta, uint32_t bh, uint32_t t0, uint32_t s0,
                                                 uint32_t (&out)[4]) {
    out[0] = out[1] = out[2] = out[3] = 0u;
#pragma unroll 2
    for (int blk = 0; blk < 8; ++blk) {
        const uint4 r = philox4x32_10(make_uint4((s0 >> 2) + (uint32_t)blk, t0 >> 2, bh, 0u), (uint32_t)seed,
                                      (uint32_t)(seed >> 32));
        out[0] |= keep_msb4(r.x, theta) >> blk;
        out[1] |= keep_msb4(r.y, theta) >> blk;
        out[2] |= keep_msb4(r.z, theta) >> blk;
        out[3] |= keep_msb4(r.w, theta) >> blk;
    }
}

// Keep words of queries t0 .. t0+31 (t0 a multiple of 32) for the four keys
// s0 .. s0+3 (s0 a multiple of 4): out[c] for key s0 + c, column i = query
// t0 + i.  Eight generator calls, one per 4 x 4 block.
__device__ __forceinline__ void dropout_keep32x4_keys(uint64_t seed, uint32_t theta, uint32_t bh, uint32_t s0,
                                                      uint32_t t0, uint32_t (&out)[4]) {
    out[0] = out[1] = out[2] = out[3] = 0u;
#pragma unroll 2
    for (int blk = 0; blk < 8; ++blk) {
        const uint4 r = philox4x32_10(make_uint4(s0 >> 2, (t0 >> 2) + (uint32_t)blk, bh, 0u), (uint32_t)seed,
                                      (uint32_t)(seed >> 32));
        // byte c of word q: (query 4*blk + q, key s0 + c); gather byte c of the four words
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint32_t sel = (uint32_t)c | ((4u + (uint32_t)c) << 4);
            out[c] |= keep_msb4(__byte_perm(__byte_perm(r.x, r.y, sel), __byte_perm(r.z, r.w, sel), 0x5410), theta) >>
                      blk;
        }
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
