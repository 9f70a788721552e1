// fwd_sm100.cu -- persistent bf16 causal self-attention forward for sm_100a.
//
// Computes, for every (batch b, head h) and 128-row query tile (lecture page
// "Let's build GPT: from scratch, in code, spelled out", chapters "version 3:
// adding softmax" and "version 4: self-attention"; note 6 / correction 01:20:05
// for the 1/sqrt(head_size) scale; correction 00:57:00 for the causal mask):
//     S_j = Q K_j^T                   (tcgen05 MMA, fp32 accumulators in TMEM)
//     online softmax of S_j * scale   (fp32, one TMEM lane = one query row per thread)
//     O  += P_j V_j                   (tcgen05 MMA, P read straight from TMEM)
// over the key tiles j at or below the diagonal (tiles above it are skipped,
// the diagonal tile is masked element-wise), then y = O / l and lse = m + ln l.
// Local window (minGPT README page, reference notes on GPT-3: locally banded
// attention): query t sees keys t-window < s <= t; key tiles below a query
// tile's band are skipped and the band's lower edge is masked element-wise like
// the diagonal.  window >= T is the causal case.
//
// Work item = a pair of consecutive query tiles (A = 2m, B = 2m+1) of one
// (b, h); both share the K_j / V_j tiles.  One persistent CTA per SM walks
// the items longest first, in a snake order over the CTAs.  Ten warps:
//   warp 0      TMA producer: Q_A, Q_B per item, K_j / V_j through a ring
//   warp 1      TMEM owner + MMA issuer (one elected lane)
//   warps 2..5  softmax, O rescale and epilogue of tile A (one query row per thread)
//   warps 6..9  the same for tile B
// The two softmax warpgroups ping-pong: the MMA order
//     S_A0 S_B0 | PV_A0 S_A1 | PV_B0 S_B1 | PV_A1 S_A2 | ...
// lets one tile's exponentials run while the other tile's P V and next S run.
// TMEM (512 columns): S_A [0,128), S_B [128,256) (P written back over the
// first 64 columns of its S), O_A [256, 256+hs), O_B [256+hs, 256+2hs).
// The softmax keeps the running max lazily (rescaling O only when the max
// grows by more than 2^8) and normalises y by the sum of the bf16-rounded
// weights that the P V product used; lse uses the sum of the fp32 weights.
// Dropout (lecture chapter "adding dropout", read as inverted dropout on the
// weights): P goes into TMEM with dropped weights zeroed, l and the rounded-
// weight sum stay those of the undropped weights, and the epilogue scales y by
// 1/(1-p).  The keep words come from a fourth warpgroup that draws them a few
// tiles ahead (fwd_common.cuh); the dropout instantiation therefore places the
// roles in whole warpgroups (warps 0-3: producer, MMA issuer, two idle; 4-11:
// softmax; 12-15: mask) and moves registers to the softmax warps with setmaxnreg.
// Every barrier wait is bounded (sm100_ptx.cuh); on a timeout all roles stop
// issuing work, drain and exit.
#include "fwd_common.cuh"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace gptattn {
namespace {

using fwdc::band_lo_tile;
using fwdc::drain_wait;
using fwdc::item_index;
using fwdc::warp_wait;

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlabBytes = 128 * 128;  // 128 rows x 128 bytes (64 bf16 columns), one swizzle slab

template <int HS, bool kDropout>
struct FwdCfg {
    // warp 0 producer, warp 1 MMA issuer, eight softmax warps from kSoftBase on; with
    // dropout, warps 12-15 draw the mask and registers move by setmaxnreg (launch: 128)
    static constexpr int kThreads = kDropout ? 512 : 384;
    static constexpr int kSoftBase = 4;
    static constexpr int kLaunchRegs = kDropout ? 128 : 168;
    static constexpr uint32_t kRegsCtl = kDropout ? 96 : 104, kRegsSoftmax = kDropout ? 192 : 200,
                              kRegsMask = kDropout ? 32 : 0;
    static_assert(kRegsCtl + 2 * kRegsSoftmax + kRegsMask == (kThreads / 128) * kLaunchRegs, "register split");
    static constexpr int kSlabs = HS / 64;
    static constexpr uint32_t kTileBytes = 128u * HS * 2u;
    static constexpr int kQStages = (HS == 64) ? 2 : 1;   // pairs of Q tiles
    static constexpr int kKVStages = (HS == 64) ? 4 : 2;
    static constexpr uint32_t kOffQ = 0;                                      // kQStages x 2 tiles
    static constexpr uint32_t kOffK = kOffQ + kQStages * 2 * kTileBytes;     // kKVStages tiles
    static constexpr uint32_t kOffV = kOffK + kKVStages * kTileBytes;        // kKVStages tiles
    static constexpr uint32_t kOffBar = kOffV + kKVStages * kTileBytes;
    static constexpr uint32_t kBarArea = 512;
    static constexpr uint32_t kOffM = kOffBar + kBarArea;                     // dropout keep-word rings
    static constexpr uint32_t kSmemBytes =
        kOffM + (kDropout ? fwdc::kMaskRingBytes : 0u) + 1024;                // + slack for 1024-byte alignment
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
    static constexpr uint32_t kColS = 0;    // + 128 * tile
    static constexpr uint32_t kColO = 256;  // + HS * tile
    // barrier slots (8 bytes each)
    static constexpr int kBarQFull = 0;
    static constexpr int kBarQEmpty = kBarQFull + kQStages;
    static constexpr int kBarKFull = kBarQEmpty + kQStages;
    static constexpr int kBarVFull = kBarKFull + kKVStages;
    static constexpr int kBarKVEmpty = kBarVFull + kKVStages;
    static constexpr int kBarSFull = kBarKVEmpty + kKVStages;  // 2 (per tile)
    static constexpr int kBarPFull = kBarSFull + 2;            // 2
    static constexpr int kBarODone = kBarPFull + 2;            // 2
    static constexpr int kBarOFree = kBarODone + 2;            // 2
    static constexpr int kBarDone = kBarOFree + 2;
    static constexpr int kBarMFull = kBarDone + 1;                     // 2 x fwdc::kMStages
    static constexpr int kBarMEmpty = kBarMFull + 2 * fwdc::kMStages;  // 2 x fwdc::kMStages
    static constexpr int kNumBars = kBarMEmpty + 2 * fwdc::kMStages;
    static_assert(kNumBars * 8 + 16 <= kBarArea, "barrier area");
};

// kBand: a local window narrower than T (key-tile ranges and edge masks); the causal
// instantiation compiles none of it.
template <int HS, bool kBand, bool kDropout>
__global__ void __launch_bounds__(FwdCfg<HS, kDropout>::kThreads, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap map_qkv, const __grid_constant__ CUtensorMap map_y,
                    float *__restrict__ lse, int B, int T, int C, int n_head, int n_qt, int window, DropoutParams dp,
                    int *status, unsigned long long budget_ns) {
    using K = FwdCfg<HS, kDropout>;
    if constexpr (!kBand) window = 1 << 30;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_base & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int BH = B * n_head;
    const int n_pairs = (n_qt + 1) >> 1;
    const int n_items = n_pairs * BH;
    const int grid = gridDim.x, cta = blockIdx.x;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + K::kOffBar);
    auto bar = [&](int idx) -> uint32_t { return smem_u32(&bars[idx]); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + K::kOffBar + K::kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + K::kOffBar + K::kNumBars * 8 + 4);
    const WaitGuard g{abort_flag, status, budget_ns};

    auto sQ = [&](int qs, int t) -> uint32_t { return sbase + K::kOffQ + (uint32_t)(2 * qs + t) * K::kTileBytes; };
    auto sK = [&](int st) -> uint32_t { return sbase + K::kOffK + (uint32_t)st * K::kTileBytes; };
    auto sV = [&](int st) -> uint32_t { return sbase + K::kOffV + (uint32_t)st * K::kTileBytes; };

    // item -> (pair m, batch*head); pairs with the most key tiles first
    auto decode = [&](int w, int &m, int &bh) { fwdc::decode_item(w, n_pairs, BH, m, bh); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < K::kQStages; ++s) {
            mbar_init(bar(K::kBarQFull + s), 1);
            mbar_init(bar(K::kBarQEmpty + s), 2);  // one arrival per softmax warpgroup
        }
        for (int s = 0; s < K::kKVStages; ++s) {
            mbar_init(bar(K::kBarKFull + s), 1);
            mbar_init(bar(K::kBarVFull + s), 1);
            mbar_init(bar(K::kBarKVEmpty + s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(K::kBarSFull + t), 1);
            mbar_init(bar(K::kBarPFull + t), 128);
            mbar_init(bar(K::kBarODone + t), 1);
            mbar_init(bar(K::kBarOFree + t), 128);
            for (int st = 0; st < fwdc::kMStages; ++st) {
                mbar_init(bar(K::kBarMFull + t * fwdc::kMStages + st), 128);
                mbar_init(bar(K::kBarMEmpty + t * fwdc::kMStages + st), 128);
            }
        }
        mbar_init(bar(K::kBarDone), 1);
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

    if (warp < K::kSoftBase) {
        regs_dec<K::kRegsCtl>();
    if (warp == 0) {
        // ================================================================ producer
        if (lane == 0) {
            tma_prefetch_map(&map_qkv);
            tma_prefetch_map(&map_y);
            bool ok = true;
            int nq = 0, gkv = 0;  // Q stages and K/V stages filled so far
            for (int k = 0; ok; ++k) {
                const int w = item_index(k, cta, grid);
                if (w >= n_items) break;
                int m, bh;
                decode(w, m, bh);
                const int b = bh / n_head, h = bh % n_head;
                const bool hasB = 2 * m + 1 < n_qt;
                const int jlo = kBand ? band_lo_tile(2 * m, window) : 0;
                const int nkv = (hasB ? 2 * m + 2 : 2 * m + 1) - jlo;
                const int qs = nq % K::kQStages;
                if (nq >= K::kQStages &&
                    !(ok = mbar_wait(bar(K::kBarQEmpty + qs), (uint32_t)((nq / K::kQStages) & 1) ^ 1u, g)))
                    break;
                const uint32_t qb = bar(K::kBarQFull + qs);
                mbar_arrive_expect_tx(qb, (hasB ? 2u : 1u) * K::kTileBytes);
                for (int t = 0; t < (hasB ? 2 : 1); ++t)
                    for (int s = 0; s < K::kSlabs; ++s)
                        tma_load_3d(sQ(qs, t) + s * kSlabBytes, &map_qkv, qb, h * HS + 64 * s, (2 * m + t) * kTile, b);
                // Without a tile B the stage's release counts one arrival for it, made here: the
                // wait above has just seen the stage's previous phase complete, so the arrival falls
                // into this item's phase.  (Made by tile B's idle warpgroup instead, it could run
                // several such items ahead and arrive into a phase still open for tile A.)
                if (!hasB) mbar_arrive(bar(K::kBarQEmpty + qs));
                ++nq;
                for (int j = 0; j < nkv; ++j) {
                    const int st = gkv % K::kKVStages;
                    const uint32_t ph = (uint32_t)(gkv / K::kKVStages) & 1u;
                    if (gkv >= K::kKVStages && !(ok = mbar_wait(bar(K::kBarKVEmpty + st), ph ^ 1u, g))) break;
                    mbar_arrive_expect_tx(bar(K::kBarKFull + st), K::kTileBytes);
                    for (int s = 0; s < K::kSlabs; ++s)
                        tma_load_3d(sK(st) + s * kSlabBytes, &map_qkv, bar(K::kBarKFull + st), C + h * HS + 64 * s,
                                    (jlo + j) * kTile, b);
                    mbar_arrive_expect_tx(bar(K::kBarVFull + st), K::kTileBytes);
                    for (int s = 0; s < K::kSlabs; ++s)
                        tma_load_3d(sV(st) + s * kSlabBytes, &map_qkv, bar(K::kBarVFull + st), 2 * C + h * HS + 64 * s,
                                    (jlo + j) * kTile, b);
                    ++gkv;
                }
            }
            if (!ok || *abort_flag) {
                // let this CTA's last copies land before shared memory is released
                for (int q = (nq > K::kQStages ? nq - K::kQStages : 0); q < nq; ++q)
                    drain_wait(bar(K::kBarQFull + q % K::kQStages), (uint32_t)(q / K::kQStages) & 1u, budget_ns);
                for (int q = (gkv > K::kKVStages ? gkv - K::kKVStages : 0); q < gkv; ++q) {
                    drain_wait(bar(K::kBarKFull + q % K::kKVStages), (uint32_t)(q / K::kKVStages) & 1u, budget_ns);
                    drain_wait(bar(K::kBarVFull + q % K::kKVStages), (uint32_t)(q / K::kKVStages) & 1u, budget_ns);
                }
            }
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);  // Q, K both K-major
            constexpr uint32_t idPV = idesc_bf16_f32(128, HS, false, true);   // P from TMEM, V N-major
            const uint64_t dQ0 = sdesc_sw128(sQ(0, 0), 16, 1024);
            const uint64_t dK0 = sdesc_sw128(sK(0), 16, 1024);
            const uint64_t dV0 = sdesc_sw128(sV(0), kSlabBytes, 1024);
            auto at = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
            bool ok = true, any = false;
            int n = 0, gkv = 0;
            int it[2] = {0, 0};     // S / P V iterations issued per tile stream
            int items[2] = {0, 0};  // items that used each tile stream
            auto issue_S = [&](int qs, int t, int st) {
                const uint64_t a = at(dQ0, (uint32_t)(2 * qs + t) * K::kTileBytes);
                const uint64_t bk = at(dK0, (uint32_t)st * K::kTileBytes);
#pragma unroll
                for (int kk = 0; kk < HS / 16; ++kk) {
                    const uint32_t koff = (uint32_t)(kk >> 2) * kSlabBytes + (uint32_t)(kk & 3) * 32u;
                    umma_ss(tmem + K::kColS + 128u * t, at(a, koff), at(bk, koff), idS, kk > 0 ? 1u : 0u);
                }
                umma_commit(bar(K::kBarSFull + t));
            };
            auto issue_PV = [&](int t, int st, bool first) {
                const uint64_t bv = at(dV0, (uint32_t)st * K::kTileBytes);
                const uint32_t p = tmem + K::kColS + 128u * t;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    umma_ts(tmem + K::kColO + HS * t, p + 8u * kk, at(bv, kk * 2048u), idPV,
                            (!first || kk > 0) ? 1u : 0u);
                umma_commit(bar(K::kBarODone + t));
            };
            for (int k = 0; ok; ++k, ++n) {
                const int w = item_index(k, cta, grid);
                if (w >= n_items) break;
                int m, bh;
                decode(w, m, bh);
                const bool hasB = 2 * m + 1 < n_qt;
                // key tiles of each stream: [lo, hi] (a band narrower than T starts later); the
                // item walks their union [jlo, jlo + nkv)
                const int lo[2] = {kBand ? band_lo_tile(2 * m, window) : 0,
                                   hasB ? (kBand ? band_lo_tile(2 * m + 1, window) : 0) : 1};
                const int hi[2] = {2 * m, hasB ? 2 * m + 1 : 0};
                const int jlo = lo[0];
                const int nkv = (hasB ? 2 * m + 2 : 2 * m + 1) - jlo;
                auto part = [&](int t, int jj) { return jj >= lo[t] && jj <= hi[t]; };
                const int qs = n % K::kQStages;
                if (!(ok = mbar_wait(bar(K::kBarQFull + qs), (uint32_t)(n / K::kQStages) & 1u, g))) break;
                if (!(ok = mbar_wait(bar(K::kBarKFull + gkv % K::kKVStages), (uint32_t)(gkv / K::kKVStages) & 1u, g)))
                    break;
                tc_fence_after();
                for (int t = 0; t < 2; ++t)
                    if (part(t, jlo)) issue_S(qs, t, gkv % K::kKVStages);
                any = true;
                for (int j = 0; j < nkv && ok; ++j) {
                    const int jj = jlo + j;  // key tile
                    const int st = (gkv + j) % K::kKVStages;
                    const uint32_t ph = (uint32_t)((gkv + j) / K::kKVStages) & 1u;
                    const int st1 = (gkv + j + 1) % K::kKVStages;
                    const uint32_t ph1 = (uint32_t)((gkv + j + 1) / K::kKVStages) & 1u;
                    if (!(ok = mbar_wait(bar(K::kBarVFull + st), ph, g))) break;
                    for (int t = 0; t < 2 && ok; ++t) {
                        if (!part(t, jj)) continue;
                        if (jj == lo[t] && jj > jlo) {  // this stream's band starts after the item's
                            if (!(ok = mbar_wait(bar(K::kBarKFull + st), ph, g))) break;
                            tc_fence_after();
                            issue_S(qs, t, st);
                        }
                        if (!(ok = mbar_wait(bar(K::kBarPFull + t), (uint32_t)it[t] & 1u, g))) break;
                        if (jj == lo[t] && items[t] > 0 &&
                            !(ok = mbar_wait(bar(K::kBarOFree + t), (uint32_t)(items[t] - 1) & 1u, g)))
                            break;
                        tc_fence_after();
                        issue_PV(t, st, jj == lo[t]);
                        ++it[t];
                        if (jj + 1 <= hi[t]) {
                            if (!(ok = mbar_wait(bar(K::kBarKFull + st1), ph1, g))) break;
                            tc_fence_after();
                            issue_S(qs, t, st1);
                        }
                    }
                    if (ok) umma_commit(bar(K::kBarKVEmpty + st));
                }
                gkv += nkv;
                items[0] += 1;
                items[1] += hasB ? 1 : 0;
            }
            if (any) {
                // all MMAs of this CTA retired before TMEM can be released
                umma_commit(bar(K::kBarDone));
                drain_wait(bar(K::kBarDone), 0, budget_ns);
            }
        }
    }
    } else if (warp < K::kSoftBase + 8) {
        // ================================================================ softmax warpgroups
        regs_inc<K::kRegsSoftmax>();
        const int t = (warp - K::kSoftBase) >> 2;  // tile stream: 0 = A, 1 = B
        const int sp = warp & 3;                 // TMEM sub-partition this warp may access
        const int row = sp * 32 + lane;          // query row within the tile
        const uint32_t trow = tmem + ((uint32_t)(sp * 32) << 16);
        const uint32_t tS = trow + K::kColS + 128u * t;
        const uint32_t tO = trow + K::kColO + (uint32_t)HS * t;
        const float scale_log2 = (HS == 64 ? 0.125f : 0.08838834764831845f) * 1.4426950408889634f;
        const uint64_t c2 = f32x2_pack(scale_log2, scale_log2);
        const bool leader = (sp == 0 && lane == 0);  // one thread of this warpgroup
        bool ok = true;
        int it = 0, n = 0;
        for (int k = 0;; ++k, ++n) {
            const int w = item_index(k, cta, grid);
            if (w >= n_items) break;
            int m, bh;
            decode(w, m, bh);
            const int b = bh / n_head, h = bh % n_head;
            const int qt = 2 * m + t;
            const int qs = n % K::kQStages;
            if (qt >= n_qt) continue;  // no work for this stream in this item (the producer released its share)
            const int jlo_t = kBand ? band_lo_tile(qt, window) : 0;
            // key tiles at or below j_edge need the band's lower edge masked (a band narrower
            // than T: query t sees keys t-window < s <= t)
            const bool banded = kBand && qt * kTile + kTile - 1 - window >= 0;
            const int j_edge = banded ? (qt * kTile + kTile - 1 - window) / kTile : -1;
            float mrow = -INFINITY;  // reference max of scaled scores (log2 units), lazily updated
            float l = 0.f;           // running normaliser of the fp32 weights
            float l_r = 0.f;         // running normaliser of the bf16-rounded weights
            for (int j = jlo_t; j <= qt; ++j, ++it) {
                // dropout keep words of this row's 128 keys of tile j (bit layout of philox.cuh)
                uint32_t kb[4] = {0u, 0u, 0u, 0u};
                if constexpr (kDropout) {
                    if (ok) ok = fwdc::mask_take(sbase + K::kOffM, bar(K::kBarMFull), bar(K::kBarMEmpty), t, it, row, g, kb);
                    if (!ok) continue;
                }
                if (ok) ok = warp_wait(bar(K::kBarSFull + t), (uint32_t)it & 1u, g);
                if (!ok) continue;
                tc_fence_after();
                const bool diag = (j == qt);
                const bool edge = j <= j_edge;
                const int cut = (qt - j) * kTile + row - window;  // on an edge tile, columns <= cut are masked
                uint64_t sum2 = f32x2_pack(0.f, 0.f), sumr2 = f32x2_pack(0.f, 0.f);
                float m_new, alpha;
                if constexpr (!kDropout) {
                    // one pass: the whole S row into registers (four loads in flight, one wait),
                    // masked, its max, then the weights written back over its first 64 columns
                    uint32_t sr[128];
                    tmem_ld_x32_nowait(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                    tmem_ld_x32_nowait(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                    tmem_ld_x32_nowait(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
                    tmem_ld_x32_nowait(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
                    tmem_ld_wait_32(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                    tmem_ld_wait_32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                    tmem_ld_wait_32(*reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
                    tmem_ld_wait_32(*reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
                    if (diag) {
#pragma unroll
                        for (int c = 0; c < 128; ++c)
                            if (c > row) sr[c] = __float_as_uint(-INFINITY);
                    }
                    if (kBand && edge) {
#pragma unroll
                        for (int c = 0; c < 128; ++c)
                            if (c <= cut) sr[c] = __float_as_uint(-INFINITY);
                    }
                    float mp[8];  // eight independent max chains of 16 columns
#pragma unroll
                    for (int q = 0; q < 8; ++q) mp[q] = __uint_as_float(sr[16 * q]);
#pragma unroll
                    for (int c = 1; c < 15; c += 2)
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            mp[q] = fmax3(mp[q], __uint_as_float(sr[16 * q + c]), __uint_as_float(sr[16 * q + c + 1]));
#pragma unroll
                    for (int q = 0; q < 8; ++q) mp[q] = fmaxf(mp[q], __uint_as_float(sr[16 * q + 15]));
                    const float mx =
                        fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
                    const float m_cand = mx * scale_log2;
                    const bool grow = m_cand > mrow + 8.f;
                    m_new = grow ? m_cand : mrow;
                    alpha = grow ? ex2_approx(mrow - m_new) : 1.f;
                    // a row with no visible key yet (band edge) keeps weight 0, not NaN
                    const float m_use = (kBand && m_new == -INFINITY) ? 0.f : m_new;
                    const uint64_t negm2 = f32x2_pack(-m_use, -m_use);
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t pk[16];
#pragma unroll
                        for (int c = 0; c < 32; c += 2) {
                            const uint64_t x = ffma2(
                                f32x2_pack(__uint_as_float(sr[32 * ch + c]), __uint_as_float(sr[32 * ch + c + 1])), c2,
                                negm2);
                            float x0, x1;
                            f32x2_unpack(x, x0, x1);
                            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                            const uint32_t wv = pack_bf16x2(p0, p1);
                            pk[c >> 1] = wv;
                            sum2 = fadd2(sum2, f32x2_pack(p0, p1));
                            sumr2 = fadd2(sumr2, f32x2_pack(bf16lo_to_f32(wv), bf16hi_to_f32(wv)));
                        }
                        tmem_st_x16(tS + 16 * ch, pk);
                    }
                } else {
                    // pass 1: row maximum
                    float mx = -INFINITY;
    #pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t sr[32];
                        tmem_ld_x32(tS + 32 * ch, sr);
                        if (diag) {
    #pragma unroll
                            for (int c = 0; c < 32; ++c)
                                if (32 * ch + c > row) sr[c] = __float_as_uint(-INFINITY);
                        }
                        if (kBand && edge) {
    #pragma unroll
                            for (int c = 0; c < 32; ++c)
                                if (32 * ch + c <= cut) sr[c] = __float_as_uint(-INFINITY);
                        }
                        float a = __uint_as_float(sr[0]), bb = __uint_as_float(sr[1]);
    #pragma unroll
                        for (int c = 2; c < 32; c += 2) a = fmax3(a, __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
                        mx = fmax3(mx, a, bb);
                    }
                    // lazy max: keep the reference unless it grows by more than 8 (log2 units)
                    const float m_cand = mx * scale_log2;
                    const bool grow = m_cand > mrow + 8.f;
                    m_new = grow ? m_cand : mrow;
                    alpha = grow ? ex2_approx(mrow - m_new) : 1.f;
                    // a row with no visible key yet (band edge) keeps weight 0, not NaN
                    const float m_use = (kBand && m_new == -INFINITY) ? 0.f : m_new;
                    const uint64_t negm2 = f32x2_pack(-m_use, -m_use);
                    // pass 2: weights, sums, P back into TMEM (bf16 pairs over columns already read)
    #pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t sr[32];
                        tmem_ld_x32(tS + 32 * ch, sr);
                        if (diag) {
    #pragma unroll
                            for (int c = 0; c < 32; ++c)
                                if (32 * ch + c > row) sr[c] = __float_as_uint(-INFINITY);
                        }
                        if (kBand && edge) {
    #pragma unroll
                            for (int c = 0; c < 32; ++c)
                                if (32 * ch + c <= cut) sr[c] = __float_as_uint(-INFINITY);
                        }
                        uint32_t pk[16];
    #pragma unroll
                        for (int c = 0; c < 32; c += 2) {
                            const uint64_t x = ffma2(f32x2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), c2, negm2);
                            float x0, x1;
                            f32x2_unpack(x, x0, x1);
                            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                            const uint32_t wv = pack_bf16x2(p0, p1);
                            // with dropout the stored weights are masked, the sums are not
                            if constexpr (kDropout)
                                pk[c >> 1] = wv & keep_pair_mask(kb[ch] << (c >> 2), (c >> 1) & 1);
                            else
                                pk[c >> 1] = wv;
                            sum2 = fadd2(sum2, f32x2_pack(p0, p1));
                            sumr2 = fadd2(sumr2, f32x2_pack(bf16lo_to_f32(wv), bf16hi_to_f32(wv)));
                        }
                        tmem_st_x16(tS + 16 * ch, pk);
                    }
                }
                float s0, s1, r0, r1;
                f32x2_unpack(sum2, s0, s1);
                f32x2_unpack(sumr2, r0, r1);
                l = l * alpha + (s0 + s1);
                l_r = l_r * alpha + (r0 + r1);
                mrow = m_new;
                if (j > jlo_t && __any_sync(0xffffffffu, alpha != 1.f)) {
                    // rescale O once the previous P V product of this tile has landed
                    ok = warp_wait(bar(K::kBarODone + t), (uint32_t)(it - 1) & 1u, g);
                    if (ok) {
                        tc_fence_after();
#pragma unroll
                        for (int c0 = 0; c0 < HS; c0 += 32) {
                            uint32_t o[32];
                            tmem_ld_x32(tO + c0, o);
#pragma unroll
                            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                            tmem_st_x32(tO + c0, o);
                        }
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(bar(K::kBarPFull + t));
            }
            // ------------------------------------------------------------ epilogue of this tile
            // staging: this tile's Q buffer (its last S MMA retired before the last P V)
            const uint32_t stg = sQ(qs, t);
            if (ok) ok = warp_wait(bar(K::kBarODone + t), (uint32_t)(it - 1) & 1u, g);
            if (ok) {
                tc_fence_after();
                const float inv_l = (kDropout ? dp.scale : 1.f) / l_r;  // 1/(1-p) with dropout
#pragma unroll
                for (int c0 = 0; c0 < HS; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld_x32(tO + c0, o);
                    if (c0 + 32 == HS) {
                        tc_fence_before();
                        mbar_arrive(bar(K::kBarOFree + t));  // O may be overwritten by the next item
                    }
                    uint32_t wv[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        wv[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
                    const uint32_t slab = stg + (uint32_t)(c0 >> 6) * kSlabBytes + (uint32_t)row * 128u;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t chunk = (uint32_t)(((c0 & 63) >> 3) + q);
                        st_shared_v4(slab + ((chunk ^ (uint32_t)(row & 7)) << 4), wv[4 * q], wv[4 * q + 1],
                                     wv[4 * q + 2], wv[4 * q + 3]);
                    }
                }
                fence_proxy_async_smem();
                const int tq = qt * kTile + row;
                if (tq < T && lse) lse[(size_t)bh * (size_t)T + (size_t)tq] = (mrow + __log2f(l)) * 0.6931471805599453f;
            }
            named_bar_sync(1 + t, 128);
            if (leader) {
                if (ok && !*abort_flag) {
                    for (int s = 0; s < K::kSlabs; ++s)
                        tma_store_3d(&map_y, stg + s * kSlabBytes, h * HS + 64 * s, qt * kTile, b);
                    bulk_commit_group();
                    bulk_wait_group_read_0();  // staging (this Q buffer) may now be refilled
                }
                mbar_arrive(bar(K::kBarQEmpty + qs));
            }
        }
        if (leader) bulk_wait_group_0();
    } else {
        // ================================================================ dropout mask warpgroup
        if constexpr (kDropout) {
            regs_dec<K::kRegsMask>();
            fwdc::mask_producer(dp, sbase + K::kOffM, bar(K::kBarMFull), bar(K::kBarMEmpty), n_items, n_pairs, BH, n_qt,
                                window, cta, grid, g);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int HS, bool kBand, bool kDropout>
cudaError_t launch_fwd_variant(const CUtensorMap &map_qkv, const CUtensorMap &map_y, float *lse, int B, int T, int C,
                               int n_head, int window, DropoutParams dp, DevCtx ctx, cudaStream_t s) {
    using K = FwdCfg<HS, kDropout>;
    auto kern = fwd_bf16_kernel<HS, kBand, kDropout>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)K::kSmemBytes);
    if (e != cudaSuccess) return e;
    {
        // the warpgroups' register budgets add up to the launch allocation only at kLaunchRegs
        // per thread; otherwise a setmaxnreg.inc could never be satisfied, so refuse to launch
        cudaFuncAttributes fa{};
        e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != K::kLaunchRegs) return cudaErrorInvalidConfiguration;
    }
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int n_qt = ceil_div(T, kTile);
    const long long items = (long long)((n_qt + 1) / 2) * B * n_head;
    const int grid = (int)(items < sms ? items : sms);
    return launch_pdl(kern, dim3((unsigned)grid), dim3(K::kThreads), K::kSmemBytes, s, map_qkv, map_y, lse, B, T, C,
                      n_head, n_qt, window, dp, ctx.status, ctx.budget_ns);
}

template <int HS>
cudaError_t launch_fwd_impl(const CUtensorMap &map_qkv, const CUtensorMap &map_y, float *lse, int B, int T, int C,
                            int n_head, int window, DropoutParams dp, DevCtx ctx, cudaStream_t s) {
    const bool band = window < T, drop = dp.threshold != 0u;
    if (band)
        return drop ? launch_fwd_variant<HS, true, true>(map_qkv, map_y, lse, B, T, C, n_head, window, dp, ctx, s)
                    : launch_fwd_variant<HS, true, false>(map_qkv, map_y, lse, B, T, C, n_head, window, dp, ctx, s);
    return drop ? launch_fwd_variant<HS, false, true>(map_qkv, map_y, lse, B, T, C, n_head, window, dp, ctx, s)
                : launch_fwd_variant<HS, false, false>(map_qkv, map_y, lse, B, T, C, n_head, window, dp, ctx, s);
}

}  // namespace

cudaError_t launch_fwd_bf16(int hs, const CUtensorMap &map_qkv, const CUtensorMap &map_y, float *lse, int B, int T,
                            int C, int n_head, int window, DropoutParams dp, DevCtx ctx, cudaStream_t s) {
    if (hs == 64) return launch_fwd_h64(map_qkv, map_y, lse, B, T, C, n_head, window, dp, ctx, s);
    if (hs == 128) return launch_fwd_impl<128>(map_qkv, map_y, lse, B, T, C, n_head, window, dp, ctx, s);
    return cudaErrorInvalidValue;
}

}  // namespace gptattn
