// fwd_common.cuh -- pieces shared by the two persistent bf16 forward kernels
// (fwd_h64_sm100.cu for head size 64, fwd_sm100.cu for head size 128): the walk
// over work items, bounded warp-wide waits, and the warpgroup that draws the
// dropout keep words ahead of the softmax warpgroups.
//
// Work item = a pair of consecutive query tiles (A = 2m, B = 2m+1) of one
// (batch, head); items with the most key tiles come first, and CTA c of a grid
// of G takes items c, 2G-1-c, 2G+c, ... (a snake order that evens out the
// causal triangle's work).
#pragma once
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace gptattn {
namespace fwdc {

// Warp-uniform bounded wait (all 32 lanes call it; all get the same answer).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const WaitGuard &g) {
    bool ok = mbar_wait(bar, parity, g);
    return __all_sync(0xffffffffu, ok);
}

// Wait used only while draining after an abort: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t budget_ns) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > budget_ns) break;
    }
}

// Item k of this CTA in the snake walk.
__device__ __forceinline__ int item_index(int k, int cta, int grid) {
    return (k & 1) ? (k * grid + (grid - 1 - cta)) : (k * grid + cta);
}

// Item w -> (pair m, batch*head pair bh); pairs with the most key tiles first.
__device__ __forceinline__ void decode_item(int w, int n_pairs, int BH, int &m, int &bh) {
    m = n_pairs - 1 - w / BH;
    bh = w % BH;
}

// First key tile that query tile qt's band reaches (query t sees keys t-window < s <= t).
__device__ __forceinline__ int band_lo_tile(int qt, int window) {
    const int s = qt * kTile - window + 1;
    return s > 0 ? s / kTile : 0;
}

// ---------------------------------------------------------------------------
// Dropout keep words.  For every (query tile, key tile) that a softmax
// warpgroup processes, the mask warpgroup writes 128 rows x 16 bytes: row r
// holds the keep words (philox.cuh layout) of query row r for the tile's 128
// keys, word q for keys 32q .. 32q+31.  Each query-tile stream (A, B) has its
// own ring of kMStages tiles, filled in the order the stream uses them.
constexpr int kMStages = 4;
constexpr uint32_t kMaskTileBytes = 128u * 16u;
constexpr uint32_t kMaskRingBytes = 2u * kMStages * kMaskTileBytes;

// Body of the mask warpgroup (128 threads, warps 4k .. 4k+3).  ring: shared
// address of the two rings (stream t's stage st at (t * kMStages + st) tiles);
// full0 / empty0: shared addresses of the barriers of stream 0 stage 0
// (8 bytes apart, stream-major); each full barrier counts the 128 producer
// threads, each empty barrier the 128 threads of the consuming warpgroup.
// Thread -> rows 4*rg .. 4*rg+3 and keys 32*kq .. 32*kq+31 of every tile.
__device__ __forceinline__ void mask_producer(const DropoutParams &dp, uint32_t ring, uint32_t full0, uint32_t empty0,
                                              int n_items, int n_pairs, int BH, int n_qt, int window, int cta,
                                              int grid, const WaitGuard &g) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rg = (warp & 3) * 8 + (lane >> 2), kq = lane & 3;
    const uint32_t t7 = theta_low7(dp.threshold);
    bool ok = true;
    int mc[2] = {0, 0};
    for (int k = 0; ok; ++k) {
        const int w = item_index(k, cta, grid);
        if (w >= n_items) break;
        int m, bh;
        decode_item(w, n_pairs, BH, m, bh);
        const bool hasB = 2 * m + 1 < n_qt;
        const int lo[2] = {band_lo_tile(2 * m, window), hasB ? band_lo_tile(2 * m + 1, window) : 1};
        const int hi[2] = {2 * m, hasB ? 2 * m + 1 : 0};
        // key tile by key tile, stream A before stream B: the order the MMA issuer serves them
        for (int j = lo[0]; j <= hi[1] || j <= hi[0]; ++j) {
            for (int t = 0; t < 2; ++t) {
                if (j < lo[t] || j > hi[t]) continue;
                const int slot = t * kMStages + mc[t] % kMStages;
                if (mc[t] >= kMStages &&
                    !(ok = warp_wait(empty0 + 8u * (uint32_t)slot, (uint32_t)((mc[t] / kMStages) & 1) ^ 1u, g)))
                    break;
                uint32_t bits[4];
                const uint32_t t0 = (uint32_t)((2 * m + t) * kTile + 4 * rg), s0 = (uint32_t)(j * kTile + 32 * kq);
                if (dp.threshold >= 128u)
                    dropout_keep32x4<true>(dp.seed, t7, (uint32_t)bh, t0, s0, bits);
                else
                    dropout_keep32x4<false>(dp.seed, t7, (uint32_t)bh, t0, s0, bits);
                const uint32_t dst = ring + (uint32_t)slot * kMaskTileBytes + (uint32_t)(4 * rg) * 16u + (uint32_t)kq * 4u;
#pragma unroll
                for (int r = 0; r < 4; ++r) st_shared_u32(dst + (uint32_t)r * 16u, bits[r]);
                mbar_arrive(full0 + 8u * (uint32_t)slot);
                ++mc[t];
            }
            if (!ok) break;
        }
    }
}

// Consumer side: the keep words of query row `row` for the stream's tile number
// `it` (counted over all its tiles), then the slot released.  Returns false if
// the wait gave up.
__device__ __forceinline__ bool mask_take(uint32_t ring, uint32_t full0, uint32_t empty0, int t, int it, int row,
                                          const WaitGuard &g, uint32_t (&kb)[4]) {
    const int slot = t * kMStages + it % kMStages;
    if (!warp_wait(full0 + 8u * (uint32_t)slot, (uint32_t)(it / kMStages) & 1u, g)) return false;
    const uint4 v = ld_shared_v4(ring + (uint32_t)slot * kMaskTileBytes + (uint32_t)row * 16u);
    kb[0] = v.x;
    kb[1] = v.y;
    kb[2] = v.z;
    kb[3] = v.w;
    mbar_arrive(empty0 + 8u * (uint32_t)slot);
    return true;
}

}  // namespace fwdc
}  // namespace gptattn
