// fwd_h64_sm100.cu -- persistent bf16 causal self-attention forward, head size 64.
//
// Same function as fwd_sm100.cu (lecture page "Let's build GPT: from scratch,
// in code, spelled out", chapters "version 3: adding softmax" and "version 4:
// self-attention"; note 6 / correction 01:20:05 for the 1/sqrt(head_size)
// scale; correction 00:57:00 for the causal mask), organised for head size 64,
// where all six TMEM buffers fit at once:
//   TMEM (512 columns): S_A [0,128)  S_B [128,256)  P_A [256,320)  P_B [320,384)
//                       O_A [384,448)  O_B [448,512)
// Work item = query tiles A = 2m and B = 2m+1 of one (batch, head), sharing the
// key/value tiles; one persistent CTA per SM walks the items longest first in
// a snake order.  Warpgroup 0: warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer (warps 2, 3 idle); warpgroup 1: softmax of tile A, warpgroup 2:
// softmax of tile B (one query row per thread).  setmaxnreg moves registers
// from warpgroup 0 to the softmax warpgroups.
// Because P has its own buffer, a softmax warpgroup copies S_j to registers
// in one pass and releases it immediately; the MMA warp then computes S_{j+1}
// while the warpgroup exponentiates tile j, and P V of tile j runs while the
// warpgroup starts tile j+1.  MMA order per key tile j:
//     S_A(j+1)  S_B(j+1)  PV_A(j)  PV_B(j)
// Lazy rescaling (O is rescaled only when a row max grows by more than 2^8)
// and y normalised by the sum of the bf16-rounded weights, as in fwd_sm100.cu.
// Local window (minGPT README page, reference notes on GPT-3: locally banded
// attention): query t sees keys t-window < s <= t; key tiles below a query
// tile's band are skipped, and the band's lower edge is masked element-wise
// like the diagonal.  window >= T is the causal case.
// Dropout (lecture chapter "adding dropout", read as inverted dropout on the
// weights): P goes into TMEM with dropped weights zeroed (Philox mask, see
// philox.cuh); l and the rounded-weight sum stay those of the undropped weights,
// and the epilogue scales y by 1/(1-p).
// Every barrier wait is bounded; on a timeout all roles stop, drain and exit.
#include <type_traits>

#include "fwd_common.cuh"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace gptattn {
namespace {

using fwdc::band_lo_tile;
using fwdc::drain_wait;
using fwdc::item_index;
using fwdc::kMaskRingBytes;
using fwdc::kMStages;
using fwdc::warp_wait;

// Threads and register budgets per thread.  The plain kernel has three
// warpgroups (control, two softmax); with dropout a fourth draws the keep bits
// into shared memory.  The budgets add up to (warpgroups x kLaunchRegs), what
// the CTA is launched with.
template <bool kDropout>
struct FwdCfg {
    static constexpr int kThreads = kDropout ? 512 : 384;
    static constexpr int kLaunchRegs = kDropout ? 128 : 168;
    static constexpr uint32_t kRegsCtl = kDropout ? 80 : 88;
    static constexpr uint32_t kRegsSoftmax = kDropout ? 192 : 208;
    static constexpr uint32_t kRegsMask = kDropout ? 48 : 0;
    static constexpr uint32_t kMaskBytes = kDropout ? kMaskRingBytes : 0u;
    static_assert(kRegsCtl + 2 * kRegsSoftmax + kRegsMask == (kThreads / 128) * kLaunchRegs, "register split");
};
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlabBytes = 128 * 128;
constexpr int HS = 64;
constexpr uint32_t kTileBytes = 128u * 64u * 2u;
constexpr int kQStages = 2;   // pairs of Q tiles
constexpr int kKVStages = 4;
constexpr uint32_t kOffQ = 0;                                   // kQStages x 2 tiles
constexpr uint32_t kOffK = kOffQ + kQStages * 2 * kTileBytes;    // kKVStages tiles
constexpr uint32_t kOffV = kOffK + kKVStages * kTileBytes;       // kKVStages tiles
constexpr uint32_t kOffBar = kOffV + kKVStages * kTileBytes;
constexpr uint32_t kBarArea = 512;
constexpr uint32_t kOffM = kOffBar + kBarArea;                   // 2 streams x kMStages mask tiles
template <bool kDropout>
constexpr uint32_t smem_bytes() { return kOffM + FwdCfg<kDropout>::kMaskBytes + 1024; }
static_assert(smem_bytes<true>() <= 227 * 1024, "shared memory");
constexpr uint32_t kColS = 0, kColP = 256, kColO = 384;  // + 128 t, + 64 t, + 64 t

constexpr int kBarQFull = 0;
constexpr int kBarQEmpty = kBarQFull + kQStages;
constexpr int kBarKFull = kBarQEmpty + kQStages;
constexpr int kBarVFull = kBarKFull + kKVStages;
constexpr int kBarKVEmpty = kBarVFull + kKVStages;
constexpr int kBarSFull = kBarKVEmpty + kKVStages;  // 2
constexpr int kBarSEmpty = kBarSFull + 2;           // 2
constexpr int kBarPFull = kBarSEmpty + 2;           // 2
constexpr int kBarPVDone = kBarPFull + 2;           // 2
constexpr int kBarOFree = kBarPVDone + 2;           // 2
constexpr int kBarDone = kBarOFree + 2;
constexpr int kBarMFull = kBarDone + 1;              // 2 x kMStages
constexpr int kBarMEmpty = kBarMFull + 2 * kMStages;  // 2 x kMStages
constexpr int kNumBars = kBarMEmpty + 2 * kMStages;
static_assert(kNumBars * 8 + 16 <= kBarArea, "barrier area");


template <bool kDropout>
__global__ void __launch_bounds__(FwdCfg<kDropout>::kThreads, 1)
    fwd_h64_kernel(const __grid_constant__ CUtensorMap map_qkv, const __grid_constant__ CUtensorMap map_y,
                   float *__restrict__ lse, int B, int T, int C, int n_head, int n_qt, int window, DropoutParams dp,
                   int *status, unsigned long long budget_ns) {
    using Cfg = FwdCfg<kDropout>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_base & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int wg = warp >> 2;
    const int BH = B * n_head;
    const int n_pairs = (n_qt + 1) >> 1;
    const int n_items = n_pairs * BH;
    const int grid = gridDim.x, cta = blockIdx.x;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    auto bar = [&](int idx) -> uint32_t { return smem_u32(&bars[idx]); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffBar + kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffBar + kNumBars * 8 + 4);
    const WaitGuard g{abort_flag, status, budget_ns};

    auto sQ = [&](int qs, int t) -> uint32_t { return sbase + kOffQ + (uint32_t)(2 * qs + t) * kTileBytes; };
    auto sK = [&](int st) -> uint32_t { return sbase + kOffK + (uint32_t)st * kTileBytes; };
    auto sV = [&](int st) -> uint32_t { return sbase + kOffV + (uint32_t)st * kTileBytes; };
    auto decode = [&](int w, int &m, int &bh) { fwdc::decode_item(w, n_pairs, BH, m, bh); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(bar(kBarQFull + s), 1);
            mbar_init(bar(kBarQEmpty + s), 2);
        }
        for (int s = 0; s < kKVStages; ++s) {
            mbar_init(bar(kBarKFull + s), 1);
            mbar_init(bar(kBarVFull + s), 1);
            mbar_init(bar(kBarKVEmpty + s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(kBarSFull + t), 1);
            mbar_init(bar(kBarSEmpty + t), 128);
            mbar_init(bar(kBarPFull + t), 128);
            mbar_init(bar(kBarPVDone + t), 1);
            mbar_init(bar(kBarOFree + t), 128);
            for (int st = 0; st < kMStages; ++st) {
                mbar_init(bar(kBarMFull + t * kMStages + st), 128);
                mbar_init(bar(kBarMEmpty + t * kMStages + st), 128);
            }
        }
        mbar_init(bar(kBarDone), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    griddep_launch_dependents();
    griddep_wait();  // the previous kernel's outputs (qkv, y, lse, dy, workspace) are complete

    if (wg == 0) {
        regs_dec<Cfg::kRegsCtl>();
        if (warp == 0) {
            // ================================================================ producer
            if (lane == 0) {
                tma_prefetch_map(&map_qkv);
                tma_prefetch_map(&map_y);
                bool ok = true;
                int nq = 0, gkv = 0;
                for (int k = 0; ok; ++k) {
                    const int w = item_index(k, cta, grid);
                    if (w >= n_items) break;
                    int m, bh;
                    decode(w, m, bh);
                    const int b = bh / n_head, h = bh % n_head;
                    const bool hasB = 2 * m + 1 < n_qt;
                    const int jlo = band_lo_tile(2 * m, window);
                    const int nkv = (hasB ? 2 * m + 2 : 2 * m + 1) - jlo;
                    const int qs = nq % kQStages;
                    if (nq >= kQStages && !(ok = mbar_wait(bar(kBarQEmpty + qs), (uint32_t)((nq / kQStages) & 1) ^ 1u, g)))
                        break;
                    const uint32_t qb = bar(kBarQFull + qs);
                    mbar_arrive_expect_tx(qb, (hasB ? 2u : 1u) * kTileBytes);
                    for (int t = 0; t < (hasB ? 2 : 1); ++t)
                        tma_load_3d(sQ(qs, t), &map_qkv, qb, h * HS, (2 * m + t) * kTile, b);
                    // Without a tile B the stage's release counts one arrival for it, made here: the
                    // wait above has just seen the stage's previous phase complete, so the arrival
                    // falls into this item's phase.  (Made by tile B's idle warpgroup instead, it could
                    // run several such items ahead and arrive into a phase still open for tile A.)
                    if (!hasB) mbar_arrive(bar(kBarQEmpty + qs));
                    ++nq;
                    for (int j = 0; j < nkv; ++j) {
                        const int st = gkv % kKVStages;
                        const uint32_t ph = (uint32_t)(gkv / kKVStages) & 1u;
                        if (gkv >= kKVStages && !(ok = mbar_wait(bar(kBarKVEmpty + st), ph ^ 1u, g))) break;
                        mbar_arrive_expect_tx(bar(kBarKFull + st), kTileBytes);
                        tma_load_3d(sK(st), &map_qkv, bar(kBarKFull + st), C + h * HS, (jlo + j) * kTile, b);
                        mbar_arrive_expect_tx(bar(kBarVFull + st), kTileBytes);
                        tma_load_3d(sV(st), &map_qkv, bar(kBarVFull + st), 2 * C + h * HS, (jlo + j) * kTile, b);
                        ++gkv;
                    }
                }
                if (!ok || *abort_flag) {
                    for (int q = (nq > kQStages ? nq - kQStages : 0); q < nq; ++q)
                        drain_wait(bar(kBarQFull + q % kQStages), (uint32_t)(q / kQStages) & 1u, budget_ns);
                    for (int q = (gkv > kKVStages ? gkv - kKVStages : 0); q < gkv; ++q) {
                        drain_wait(bar(kBarKFull + q % kKVStages), (uint32_t)(q / kKVStages) & 1u, budget_ns);
                        drain_wait(bar(kBarVFull + q % kKVStages), (uint32_t)(q / kKVStages) & 1u, budget_ns);
                    }
                }
            }
        } else if (warp == 1) {
            // ================================================================ MMA issuer
            if (lane == 0) {
                constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
                constexpr uint32_t idPV = idesc_bf16_f32(128, HS, false, true);
                const uint64_t dQ0 = sdesc_sw128(sQ(0, 0), 16, 1024);
                const uint64_t dK0 = sdesc_sw128(sK(0), 16, 1024);
                const uint64_t dV0 = sdesc_sw128(sV(0), kSlabBytes, 1024);
                auto at = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
                bool ok = true, any = false;
                int n = 0, gkv = 0;
                int sc[2] = {0, 0};     // S issued per stream
                int pc[2] = {0, 0};     // P V issued per stream
                int items[2] = {0, 0};  // items that used each stream
                auto issue_S = [&](int qs, int t, int st) {
                    const uint64_t a = at(dQ0, (uint32_t)(2 * qs + t) * kTileBytes);
                    const uint64_t bk = at(dK0, (uint32_t)st * kTileBytes);
    #pragma unroll
                    for (int kk = 0; kk < HS / 16; ++kk)
                        umma_ss(tmem + kColS + 128u * t, at(a, kk * 32u), at(bk, kk * 32u), idS, kk > 0 ? 1u : 0u);
                    umma_commit(bar(kBarSFull + t));
                    ++sc[t];
                };
                auto issue_PV = [&](int t, int st, bool first) {
                    const uint64_t bv = at(dV0, (uint32_t)st * kTileBytes);
    #pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_ts(tmem + kColO + 64u * t, tmem + kColP + 64u * t + 8u * kk, at(bv, kk * 2048u), idPV,
                                (!first || kk > 0) ? 1u : 0u);
                    umma_commit(bar(kBarPVDone + t));
                    ++pc[t];
                };
                for (int k = 0; ok; ++k, ++n) {
                    const int w = item_index(k, cta, grid);
                    if (w >= n_items) break;
                    int m, bh;
                    decode(w, m, bh);
                    const bool hasB = 2 * m + 1 < n_qt;
                    // key tiles of each stream: [lo, hi]; the item walks their union [jlo, jlo + nkv)
                    const int lo[2] = {band_lo_tile(2 * m, window), hasB ? band_lo_tile(2 * m + 1, window) : 1};
                    const int hi[2] = {2 * m, hasB ? 2 * m + 1 : 0};
                    const int jlo = lo[0];
                    const int nkv = (hasB ? 2 * m + 2 : 2 * m + 1) - jlo;
                    auto part = [&](int t, int j) { return j >= lo[t] && j <= hi[t]; };
                    const int qs = n % kQStages;
                    if (!(ok = mbar_wait(bar(kBarQFull + qs), (uint32_t)(n / kQStages) & 1u, g))) break;
                    if (!(ok = mbar_wait(bar(kBarKFull + gkv % kKVStages), (uint32_t)(gkv / kKVStages) & 1u, g))) break;
                    for (int t = 0; t < 2 && ok; ++t) {
                        if (!part(t, jlo)) continue;
                        if (sc[t] > 0 && !(ok = mbar_wait(bar(kBarSEmpty + t), (uint32_t)(sc[t] - 1) & 1u, g))) break;
                        tc_fence_after();
                        issue_S(qs, t, gkv % kKVStages);
                        any = true;
                    }
                    for (int j = 0; j < nkv && ok; ++j) {
                        const int st = (gkv + j) % kKVStages;
                        // S of the next key tile for each stream, as soon as its S buffer is free
                        if (j + 1 < nkv) {
                            const int st1 = (gkv + j + 1) % kKVStages;
                            if (!(ok = mbar_wait(bar(kBarKFull + st1), (uint32_t)((gkv + j + 1) / kKVStages) & 1u, g))) break;
                            for (int t = 0; t < 2 && ok; ++t) {
                                if (!part(t, jlo + j + 1)) continue;
                                if (!(ok = mbar_wait(bar(kBarSEmpty + t), (uint32_t)(sc[t] - 1) & 1u, g))) break;
                                tc_fence_after();
                                issue_S(qs, t, st1);
                            }
                            if (!ok) break;
                        }
                        // P V of key tile j for each stream
                        if (!(ok = mbar_wait(bar(kBarVFull + st), (uint32_t)((gkv + j) / kKVStages) & 1u, g))) break;
                        for (int t = 0; t < 2 && ok; ++t) {
                            if (!part(t, jlo + j)) continue;
                            if (!(ok = mbar_wait(bar(kBarPFull + t), (uint32_t)pc[t] & 1u, g))) break;
                            if (jlo + j == lo[t] && items[t] > 0 &&
                                !(ok = mbar_wait(bar(kBarOFree + t), (uint32_t)(items[t] - 1) & 1u, g)))
                                break;
                            tc_fence_after();
                            issue_PV(t, st, jlo + j == lo[t]);
                        }
                        if (ok) umma_commit(bar(kBarKVEmpty + st));
                    }
                    gkv += nkv;
                    items[0] += 1;
                    items[1] += hasB ? 1 : 0;
                }
                if (any) {
                    umma_commit(bar(kBarDone));
                    drain_wait(bar(kBarDone), 0, budget_ns);
                }
            }
        }
    } else if (wg <= 2) {
        // ================================================================ softmax warpgroups
        regs_inc<Cfg::kRegsSoftmax>();
        const int t = wg - 1;
        const int sp = warp & 3;
        const int row = sp * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(sp * 32) << 16);
        const uint32_t tS = trow + kColS + 128u * t;
        const uint32_t tP = trow + kColP + 64u * t;
        const uint32_t tO = trow + kColO + 64u * t;
        const float scale_log2 = 0.125f * 1.4426950408889634f;
        const uint64_t c2 = f32x2_pack(scale_log2, scale_log2);
        const bool leader = (sp == 0 && lane == 0);
        bool ok = true;
        int it = 0, n = 0;
        for (int k = 0;; ++k, ++n) {
            const int w = item_index(k, cta, grid);
            if (w >= n_items) break;
            int m, bh;
            decode(w, m, bh);
            const int b = bh / n_head, h = bh % n_head;
            const int qt = 2 * m + t;
            const int qs = n % kQStages;
            if (qt >= n_qt) continue;  // no tile B in this item (the producer released its share of the stage)
            const int jlo_t = band_lo_tile(qt, window);
            // key tiles at or below this one need the band's lower edge masked
            const int j_edge = (qt * kTile + kTile - 1 - window) / kTile;
            float mrow = -INFINITY, l = 0.f, l_r = 0.f;
            for (int j = jlo_t; j <= qt; ++j, ++it) {
                // dropout keep bits of this row's 128 keys of tile j (bit c%32 of kb[c/32] <-> key
                // j*128 + c), drawn ahead by the mask warpgroup; tile number `it` of this stream
                uint32_t kb[4] = {0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu};
                if constexpr (kDropout) {
                    if (ok) ok = fwdc::mask_take(sbase + kOffM, bar(kBarMFull), bar(kBarMEmpty), t, it, row, g, kb);
                    if (!ok) continue;
                }
                if (ok) ok = warp_wait(bar(kBarSFull + t), (uint32_t)it & 1u, g);
                if (!ok) continue;
                tc_fence_after();
                uint32_t sr[128];
                // four loads in flight, one wait (the waits name every destination register)
                tmem_ld_x32_nowait(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                tmem_ld_x32_nowait(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                tmem_ld_x32_nowait(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
                tmem_ld_x32_nowait(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
                tmem_ld_wait_32(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                tmem_ld_wait_32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                tmem_ld_wait_32(*reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
                tmem_ld_wait_32(*reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
                tc_fence_before();
                mbar_arrive(bar(kBarSEmpty + t));  // S buffer may take the next tile
                if (j == qt) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c > row) sr[c] = __float_as_uint(-INFINITY);
                }
                if (j <= j_edge && qt * kTile + kTile - 1 - window >= 0) {  // key s visible only if s > t - window
                    const int cut = (qt - j) * kTile + row - window;       // columns c <= cut are masked
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c <= cut) sr[c] = __float_as_uint(-INFINITY);
                }
                // row max: eight independent chains of 16 columns, then a short tree
                float mp[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) mp[q] = __uint_as_float(sr[16 * q]);
#pragma unroll
                for (int c = 1; c < 15; c += 2)
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        mp[q] = fmax3(mp[q], __uint_as_float(sr[16 * q + c]), __uint_as_float(sr[16 * q + c + 1]));
#pragma unroll
                for (int q = 0; q < 8; ++q) mp[q] = fmaxf(mp[q], __uint_as_float(sr[16 * q + 15]));
                const float mx = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
                const float m_cand = mx * scale_log2;
                const bool grow = m_cand > mrow + 8.f;
                const float m_new = grow ? m_cand : mrow;
                const float alpha = grow ? ex2_approx(mrow - m_new) : 1.f;
                // a row with no visible key yet (band edge) keeps weight 0, not NaN
                const float m_use = m_new == -INFINITY ? 0.f : m_new;
                const uint64_t negm2 = f32x2_pack(-m_use, -m_use);
                // four independent partial sums each, so the adds do not form one long chain
                uint64_t sum2[4], sumr2[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) sum2[a] = sumr2[a] = f32x2_pack(0.f, 0.f);
                uint32_t pk[64];
                // the exponentials; with dropout the stored weights are masked, the sums are not
                auto exps = [&](auto drop_tag) {
                    constexpr bool kDrop = decltype(drop_tag)::value;
#pragma unroll
                    for (int c = 0; c < 128; c += 2) {
                        const uint64_t x = ffma2(f32x2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), c2, negm2);
                        float x0, x1;
                        f32x2_unpack(x, x0, x1);
                        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                        const uint32_t wv = pack_bf16x2(p0, p1);
                        if constexpr (kDrop) {
                            const int cc = c & 31;
                            pk[c >> 1] = wv & keep_pair_mask(kb[c >> 5] << (cc >> 2), (cc >> 1) & 1);
                        } else {
                            pk[c >> 1] = wv;
                        }
                        const int a = (c >> 1) & 3;
                        sum2[a] = fadd2(sum2[a], f32x2_pack(p0, p1));
                        sumr2[a] = fadd2(sumr2[a], f32x2_pack(bf16lo_to_f32(wv), bf16hi_to_f32(wv)));
                    }
                };
                exps(std::integral_constant<bool, kDropout>{});
                float s0, s1, r0, r1;
                f32x2_unpack(fadd2(fadd2(sum2[0], sum2[1]), fadd2(sum2[2], sum2[3])), s0, s1);
                f32x2_unpack(fadd2(fadd2(sumr2[0], sumr2[1]), fadd2(sumr2[2], sumr2[3])), r0, r1);
                l = l * alpha + (s0 + s1);
                l_r = l_r * alpha + (r0 + r1);
                mrow = m_new;
                // P buffer and O are free once the previous P V of this stream retired
                if (j > jlo_t) {
                    ok = warp_wait(bar(kBarPVDone + t), (uint32_t)(it - 1) & 1u, g);
                    if (!ok) continue;
                    tc_fence_after();
                }
                tmem_st_x32(tP + 0, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
                tmem_st_x32(tP + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
                if (j > jlo_t && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                    for (int c0 = 0; c0 < HS; c0 += 32) {
                        uint32_t o[32];
                        tmem_ld_x32(tO + c0, o);
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                        tmem_st_x32(tO + c0, o);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(bar(kBarPFull + t));
            }
            // ------------------------------------------------------------ epilogue of this tile
            const uint32_t stg = sQ(qs, t);
            if (ok) ok = warp_wait(bar(kBarPVDone + t), (uint32_t)(it - 1) & 1u, g);
            if (ok) {
                tc_fence_after();
                uint32_t o[64];
                tmem_ld_x32(tO + 0, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
                tmem_ld_x32(tO + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
                tc_fence_before();
                mbar_arrive(bar(kBarOFree + t));
                const float inv_l = (kDropout ? dp.scale : 1.f) / l_r;  // 1/(1-p) with dropout
                const uint32_t rbase = stg + (uint32_t)row * 128u;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint32_t wv[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        wv[e] = pack_bf16x2(__uint_as_float(o[8 * q + 2 * e]) * inv_l,
                                            __uint_as_float(o[8 * q + 2 * e + 1]) * inv_l);
                    st_shared_v4(rbase + (((uint32_t)q ^ (uint32_t)(row & 7)) << 4), wv[0], wv[1], wv[2], wv[3]);
                }
                fence_proxy_async_smem();
                const int tq = qt * kTile + row;
                if (tq < T && lse) lse[(size_t)bh * (size_t)T + (size_t)tq] = (mrow + __log2f(l)) * 0.6931471805599453f;
            }
            named_bar_sync(1 + t, 128);
            if (leader) {
                if (ok && !*abort_flag) {
                    tma_store_3d(&map_y, stg, h * HS, qt * kTile, b);
                    bulk_commit_group();
                    bulk_wait_group_read_0();
                }
                mbar_arrive(bar(kBarQEmpty + qs));
            }
        }
        if (leader) bulk_wait_group_0();
    } else {
        // ================================================================ dropout mask warpgroup
        if constexpr (kDropout) {
            regs_dec<Cfg::kRegsMask>();
            fwdc::mask_producer(dp, sbase + kOffM, bar(kBarMFull), bar(kBarMEmpty), n_items, n_pairs, BH, n_qt, window,
                                cta, grid, g);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

cudaError_t launch_fwd_h64(const CUtensorMap &map_qkv, const CUtensorMap &map_y, float *lse, int B, int T, int C,
                           int n_head, int window, DropoutParams dp, DevCtx ctx, cudaStream_t s) {
    const bool drop = dp.threshold != 0u;
    auto kern = drop ? fwd_h64_kernel<true> : fwd_h64_kernel<false>;
    const uint32_t smem = drop ? smem_bytes<true>() : smem_bytes<false>();
    const int threads = drop ? FwdCfg<true>::kThreads : FwdCfg<false>::kThreads;
    const int launch_regs = drop ? FwdCfg<true>::kLaunchRegs : FwdCfg<false>::kLaunchRegs;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // the warpgroups' register budgets add up to the launch allocation only at kLaunchRegs per
    // thread; otherwise a setmaxnreg.inc could never be satisfied, so refuse to launch
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != launch_regs) return cudaErrorInvalidConfiguration;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int n_qt = ceil_div(T, kTile);
    const long long items = (long long)((n_qt + 1) / 2) * B * n_head;
    const int grid = (int)(items < sms ? items : sms);
    return launch_pdl(kern, dim3((unsigned)grid), dim3((unsigned)threads), smem, s, map_qkv, map_y, lse, B, T, C,
                      n_head, n_qt, window, dp, ctx.status, ctx.budget_ns);
}

}  // namespace gptattn
