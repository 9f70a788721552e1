// bwd_sm100.cu -- bf16 causal self-attention backward for sm_100a.
//
// Chain rule through the forward (lecture page "Let's build GPT: from scratch,
// in code, spelled out", chapters "version 3: adding softmax" and "version 4:
// self-attention"), with P recomputed from the saved logsumexp instead of
// stored:
//     P   = exp(S * scale - lse)           S = Q K^T, masked causally
//     dV  = P^T dY,  dP = dY V^T
//     dS  = P o (dP - D),  D = rowsum(dY o y)   (= rowsum(P o dP))
//     dQ  = dS K * scale,  dK = dS^T Q * scale
//
// Three kernels:
//   pre   D and lse*log2(e) per query row into the workspace; zero dQ accumulator
//   main  one CTA per (key tile j, b, h); loops over query tiles i >= j (for a
//         local window only those its band reaches; the band's far edge is
//         masked element-wise like the diagonal):
//           S^T = K Q_i^T, dP^T = V dO_i^T          (tcgen05, TMEM)
//           P^T (bf16) back into TMEM; dS^T (bf16) into shared memory
//           dV += P^T dO_i (P from TMEM), dK += dS^T Q_i   (TMEM accumulators)
//           dQ_i = dS K -> TMEM -> smem (32 columns at a time) -> TMA reduce-add
//           into the fp32 accumulator
//         epilogue: dK * scale and dV -> bf16 -> TMA store into dqkv
//   post  dQ accumulator * scale -> bf16 into dqkv[..., 0:C]
// Deterministic mode (n_slots > 0): each (query tile, key tile) partial of dQ is
// stored in a slot of its own and the postprocess sums a query tile's slots in
// a fixed order, so the result does not depend on the order CTAs finish in.
//
// Main kernel (head size 128; head size 64 has the persistent bwd_h64_sm100.cu).
// Four warpgroups, registers moved among them by setmaxnreg:
//   warp 0      TMA producer (K, V once; Q_i with lse_i and D_i through a two-stage
//               ring, dO_i through one buffer refilled once dV_i has read it)
//   warp 1      TMEM owner + MMA issuer
//   warps 2,3   with dropout: the keep words of each (key tile, query tile),
//               drawn a few tiles ahead into a shared-memory ring
//   warps 4..11 "softmax" warps, one key row and 64 query columns each (two
//               warpgroups, one per half of the query tile): P, dS, dK/dV epilogue
//   warps 12..15 dQ drain, one query row each: TMEM -> smem -> TMA reduce
// Dropout (inverted, Philox mask of philox.cuh): the preprocess folds the
// scale 1/(1-p) into lse and D, so the recomputed weights are P * scale; P^T
// goes to the dV product with dropped weights zeroed, and
// dS = (P scale) o (dP o keep - D / scale).
// TMEM columns: S^T [0,128) (P^T packed into [0,64)), dP^T [128,256), dV
// [256,384), dK [384,512); dQ_i in the dP^T columns once the softmax warps have
// read dP_i^T.  MMA order per query tile i: dV_i, S_{i+1} | dK_i, dQ_i, dP_{i+1}:
// the next scores are computed while the softmax warps form dS_i, and dP_{i+1}
// waits only for dQ_i to be drained out of its columns.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace gptattn {
namespace {

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlabBytes = 128 * 128;
// dropout keep words: kMStages tiles of 128 key rows x 128 query columns (16 bytes a row)
constexpr int kMStages = 4;
constexpr uint32_t kMaskTileBytes = 128u * 16u;
constexpr int kMaskThreads = 64;

// Head size 128 only (head size 64 has its own persistent kernel).  Q_i travels with
// -lse_i*log2(e) and -D_i through a two-stage ring; dO_i has a single buffer, refilled
// once dV_i has read it; the dQ staging is one 16 KB slab (32 fp32 columns).
template <int HS, bool kDropout = false>
struct BwdCfg {
    static_assert(HS == 128, "head size 128");
    // four warpgroups: control (producer, MMA issuer; with dropout two mask warps), two softmax
    // warpgroups (64 query columns each), the dQ drain; registers moved by setmaxnreg
    static constexpr int kThreads = 512;
    static constexpr int kLaunchRegs = 128;
    static constexpr uint32_t kRegsCtl = 64, kRegsSoftmax = 136, kRegsDrain = 176;
    static_assert(kRegsCtl + 2 * kRegsSoftmax + kRegsDrain == 4 * kLaunchRegs, "register split");
    static constexpr int kSlabs = HS / 64;
    static constexpr uint32_t kTileBytes = 128u * HS * 2u;
    static constexpr int kQStages = 2;
    static constexpr uint32_t kOffK = 0;
    static constexpr uint32_t kOffV = kOffK + kTileBytes;
    static constexpr uint32_t kOffQ = kOffV + kTileBytes;                // kQStages tiles
    static constexpr uint32_t kOffdO = kOffQ + kQStages * kTileBytes;    // one tile
    static constexpr uint32_t kOffdS = kOffdO + kTileBytes;              // 128 x 128 bf16, two slabs
    static constexpr uint32_t kOffdQ = kOffdS + 2 * kSlabBytes;          // 128 x 32 fp32 staging, one slab
    static constexpr uint32_t kOffLse = kOffdQ + kSlabBytes;             // kQStages x 128 fp32
    static constexpr uint32_t kOffD = kOffLse + kQStages * 512;
    static constexpr uint32_t kOffBar = kOffD + kQStages * 512;
    static constexpr uint32_t kOffM = kOffBar + 256;
    static constexpr uint32_t kSmemBytes = kOffM + (kDropout ? kMStages * kMaskTileBytes : 0u) + 1024;
    // TMEM: S^T (P^T packed into its first 64 columns), dP^T, dV, dK; dQ_i in the dP^T
    // columns once the softmax warps have read dP_i^T, in two 64-column halves
    static constexpr uint32_t kColS = 0, kColdP = 128, kColdV = 256, kColdK = 256 + HS;
    static constexpr uint32_t kColdQ0 = 128, kColdQ1 = 192;
    // barriers
    static constexpr int kBarKV = 0;
    static constexpr int kBarQFull = 1;                    // kQStages: Q_i, lse_i, D_i landed
    static constexpr int kBarQEmpty = kBarQFull + kQStages;  // kQStages: dK_i has read Q_i
    static constexpr int kBardOFull = kBarQEmpty + kQStages;
    static constexpr int kBardOEmpty = kBardOFull + 1;     // dV_i has read dO_i
    static constexpr int kBarS = kBardOEmpty + 1;
    static constexpr int kBardP = kBarS + 1;
    static constexpr int kBarP = kBardP + 1;
    static constexpr int kBardS = kBarP + 1;
    static constexpr int kBardQFull = kBardS + 1;
    static constexpr int kBardQEmpty = kBardQFull + 1;
    static constexpr int kBarKdV = kBardQEmpty + 1;
    static constexpr int kBarDone = kBarKdV + 1;
    static constexpr int kBarMFull = kBarDone + 1;          // kMStages
    static constexpr int kBarMEmpty = kBarMFull + kMStages;  // kMStages
    static constexpr int kNumBars = kBarMEmpty + kMStages;
    static_assert(kNumBars * 8 + 16 <= 256, "barrier area");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const WaitGuard &g) {
    bool ok = mbar_wait(bar, parity, g);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t budget_ns) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > budget_ns) break;
    }
}

// kBand: a local window narrower than T (shorter query range, far-edge mask); the
// causal instantiation compiles none of it.
template <int HS, bool kBand, bool kDropout>
__global__ void __launch_bounds__(BwdCfg<HS, kDropout>::kThreads, 1)
    bwd_bf16_kernel(const __grid_constant__ CUtensorMap map_qkv, const __grid_constant__ CUtensorMap map_dy,
                    const __grid_constant__ CUtensorMap map_dqkv, const __grid_constant__ CUtensorMap map_dq,
                    const float *__restrict__ lse2, const float *__restrict__ Dvec, int B, int T, int C, int n_head,
                    int T_pad, int n_t, int window, int n_slots, DropoutParams dp, int *status,
                    unsigned long long budget_ns) {
    using K = BwdCfg<HS, kDropout>;
    if constexpr (!kBand) window = 1 << 30;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_base & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int BH = B * n_head;
    const int bh = blockIdx.x % BH;
    const int kt = blockIdx.x / BH;   // key tile; small kt = most query tiles = scheduled first
    const int b = bh / n_head;
    const int h = bh % n_head;
    // query tiles kt..: up to the last one the key tile's band reaches (all of them when causal)
    const long long last_t = (long long)kt * kTile + kTile - 2 + window;  // largest key + window - 1
    const int niter = (last_t / kTile < n_t ? (int)(last_t / kTile) : n_t - 1) - kt + 1;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + K::kOffBar);
    auto bar = [&](int idx) -> uint32_t { return smem_u32(&bars[idx]); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + K::kOffBar + K::kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + K::kOffBar + K::kNumBars * 8 + 4);
    const WaitGuard g{abort_flag, status, budget_ns};

    const uint32_t sK = sbase + K::kOffK, sV = sbase + K::kOffV;
    auto sQ = [&](int st) -> uint32_t { return sbase + K::kOffQ + st * K::kTileBytes; };
    const uint32_t sdO = sbase + K::kOffdO;
    const uint32_t sdS = sbase + K::kOffdS, sdQ = sbase + K::kOffdQ;
    const float *sLse = reinterpret_cast<const float *>(smem + K::kOffLse);
    const float *sD = reinterpret_cast<const float *>(smem + K::kOffD);
    const uint32_t sM = sbase + K::kOffM;

    if (threadIdx.x == 0) {
        mbar_init(bar(K::kBarKV), 1);
        for (int s = 0; s < kMStages; ++s) {
            mbar_init(bar(K::kBarMFull + s), kMaskThreads);
            mbar_init(bar(K::kBarMEmpty + s), 256);
        }
        for (int s = 0; s < K::kQStages; ++s) {
            mbar_init(bar(K::kBarQFull + s), 1);
            mbar_init(bar(K::kBarQEmpty + s), 1);
        }
        mbar_init(bar(K::kBardOFull), 1);
        mbar_init(bar(K::kBardOEmpty), 1);
        mbar_init(bar(K::kBarS), 1);
        mbar_init(bar(K::kBardP), 1);
        mbar_init(bar(K::kBarP), 256);
        mbar_init(bar(K::kBardS), 256);
        mbar_init(bar(K::kBardQFull), 1);
        mbar_init(bar(K::kBardQEmpty), 128);
        mbar_init(bar(K::kBarKdV), 1);
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

    if (warp < 4) {
        regs_dec<K::kRegsCtl>();
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_map(&map_qkv);
            tma_prefetch_map(&map_dy);
            const int col_q = h * HS, col_k = C + h * HS, col_v = 2 * C + h * HS;
            mbar_arrive_expect_tx(bar(K::kBarKV), 2 * K::kTileBytes);
            for (int s = 0; s < K::kSlabs; ++s) {
                tma_load_3d(sK + s * kSlabBytes, &map_qkv, bar(K::kBarKV), col_k + 64 * s, kt * kTile, b);
                tma_load_3d(sV + s * kSlabBytes, &map_qkv, bar(K::kBarKV), col_v + 64 * s, kt * kTile, b);
            }
            int q_issued = 0, do_issued = 0;
            bool ok = true;
            for (int it = 0; it < niter && ok; ++it) {
                const int qt = kt + it;
                const int st = it % K::kQStages;
                // Q_i, -lse_i*log2(e), -D_i into stage st once dK of tile i-2 has read it
                if (it >= K::kQStages &&
                    !(ok = mbar_wait(bar(K::kBarQEmpty + st), (uint32_t)((it / K::kQStages) & 1) ^ 1u, g)))
                    break;
                const uint32_t fb = bar(K::kBarQFull + st);
                mbar_arrive_expect_tx(fb, K::kTileBytes + 1024);
                for (int s = 0; s < K::kSlabs; ++s)
                    tma_load_3d(sQ(st) + s * kSlabBytes, &map_qkv, fb, col_q + 64 * s, qt * kTile, b);
                const size_t rowoff = (size_t)bh * (size_t)T_pad + (size_t)qt * kTile;
                bulk_load(sbase + K::kOffLse + st * 512, lse2 + rowoff, 512, fb);
                bulk_load(sbase + K::kOffD + st * 512, Dvec + rowoff, 512, fb);
                q_issued = it + 1;
                // dO_i into its single buffer once dV of tile i-1 has read it
                if (it >= 1 && !(ok = mbar_wait(bar(K::kBardOEmpty), (uint32_t)((it - 1) & 1), g))) break;
                mbar_arrive_expect_tx(bar(K::kBardOFull), K::kTileBytes);
                for (int s = 0; s < K::kSlabs; ++s)
                    tma_load_3d(sdO + s * kSlabBytes, &map_dy, bar(K::kBardOFull), h * HS + 64 * s, qt * kTile, b);
                do_issued = it + 1;
            }
            if (!ok || *abort_flag) {
                // let this CTA's last copies land before shared memory is released
                drain_wait(bar(K::kBarKV), 0, budget_ns);
                for (int q = (q_issued > K::kQStages ? q_issued - K::kQStages : 0); q < q_issued; ++q)
                    drain_wait(bar(K::kBarQFull + q % K::kQStages), (uint32_t)(q / K::kQStages) & 1u, budget_ns);
                if (do_issued > 0) drain_wait(bar(K::kBardOFull), (uint32_t)((do_issued - 1) & 1), budget_ns);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idSS = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T
            constexpr uint32_t idAcc = idesc_bf16_f32(128, HS, false, true);   // dV, dK (B = dO / Q, N-major)
            constexpr uint32_t idQ = idesc_bf16_f32(128, 64, true, true);      // dQ half (A = dS, M-major)
            bool ok = mbar_wait(bar(K::kBarKV), 0, g);
            bool any = false;
            // S^T = K Q^T and dP^T = V dO^T (both operands K-major)
            auto issue_S = [&](int st) {
#pragma unroll
                for (int kk = 0; kk < HS / 16; ++kk) {
                    const uint32_t koff = (uint32_t)(kk >> 2) * kSlabBytes + (uint32_t)(kk & 3) * 32u;
                    umma_ss(tmem + K::kColS, sdesc_sw128(sK + koff, 16, 1024), sdesc_sw128(sQ(st) + koff, 16, 1024),
                            idSS, kk > 0 ? 1u : 0u);
                }
                umma_commit(bar(K::kBarS));
            };
            auto issue_dP = [&]() {
#pragma unroll
                for (int kk = 0; kk < HS / 16; ++kk) {
                    const uint32_t koff = (uint32_t)(kk >> 2) * kSlabBytes + (uint32_t)(kk & 3) * 32u;
                    umma_ss(tmem + K::kColdP, sdesc_sw128(sV + koff, 16, 1024), sdesc_sw128(sdO + koff, 16, 1024),
                            idSS, kk > 0 ? 1u : 0u);
                }
                umma_commit(bar(K::kBardP));
            };
            // Order per tile i: dV_i, S_{i+1} | dK_i, dQ_i, dP_{i+1}.  S_{i+1} goes right after dV_i
            // (which has read P_i^T out of the S^T columns), so the softmax warps find the next
            // scores ready when they finish dS_i; dP_{i+1} waits for dQ_i, which shares its
            // columns, to be drained.
            if (ok && (ok = mbar_wait(bar(K::kBarQFull), 0, g)) && (ok = mbar_wait(bar(K::kBardOFull), 0, g))) {
                tc_fence_after();
                issue_S(0);
                issue_dP();
                any = true;
            }
            for (int it = 0; it < niter && ok; ++it) {
                const int st = it % K::kQStages;
                // dV += P^T dO   (A = P^T in TMEM, K = query rows)
                if (!(ok = mbar_wait(bar(K::kBarP), (uint32_t)it & 1u, g))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    // A = P^T: query columns 16kk.. sit packed in half kk/4's S^T columns
                    umma_ts(tmem + K::kColdV, tmem + K::kColS + 64u * (uint32_t)(kk >> 2) + 8u * (uint32_t)(kk & 3),
                            sdesc_sw128(sdO + kk * 2048u, kSlabBytes, 1024), idAcc, (it > 0 || kk > 0) ? 1u : 0u);
                umma_commit(bar(K::kBardOEmpty));  // dO_i read by dP_i and dV_i
                if (it + 1 < niter) {
                    const int st1 = (it + 1) % K::kQStages;
                    if (!(ok = mbar_wait(bar(K::kBarQFull + st1), (uint32_t)(((it + 1) / K::kQStages) & 1), g))) break;
                    tc_fence_after();
                    issue_S(st1);
                }
                // dK += dS^T Q   (A = dS^T in smem, key rows x query cols, K-major)
                if (!(ok = mbar_wait(bar(K::kBardS), (uint32_t)it & 1u, g))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t koff = (uint32_t)(kk >> 2) * kSlabBytes + (uint32_t)(kk & 3) * 32u;
                    umma_ss(tmem + K::kColdK, sdesc_sw128(sdS + koff, 16, 1024),
                            sdesc_sw128(sQ(st) + kk * 2048u, kSlabBytes, 1024), idAcc, (it > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(bar(K::kBarQEmpty + st));  // Q_i, lse_i, D_i no longer needed
                // dQ_i = dS K   (A = dS, M-major view of the same smem; B = K, N-major), into the
                // dP^T columns, which the softmax warps read out before they stored dS_i
#pragma unroll
                for (int half = 0; half < HS / 64; ++half) {
                    const uint32_t dcol = half == 0 ? K::kColdQ0 : K::kColdQ1;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_ss(tmem + dcol, sdesc_sw128(sdS + kk * 2048u, kSlabBytes, 1024),
                                sdesc_sw128(sK + half * kSlabBytes + kk * 2048u, kSlabBytes, 1024), idQ,
                                kk > 0 ? 1u : 0u);
                }
                umma_commit(bar(K::kBardQFull));
                if (it + 1 < niter) {
                    if (!(ok = mbar_wait(bar(K::kBardOFull), (uint32_t)((it + 1) & 1), g))) break;
                    if (!(ok = mbar_wait(bar(K::kBardQEmpty), (uint32_t)it & 1u, g))) break;
                    tc_fence_after();
                    issue_dP();
                }
            }
            if (ok) umma_commit(bar(K::kBarKdV));
            if (any || ok) {
                umma_commit(bar(K::kBarDone));
                drain_wait(bar(K::kBarDone), 0, budget_ns);
            }
        }
    } else {
        // ------------------------------------------------------------ dropout keep words (warps 2, 3)
        if constexpr (kDropout) {
            // thread -> key rows 4*kg .. 4*kg+3 and query columns 64*qh .. 64*qh+63 of every tile
            const int u = threadIdx.x - 64, kg = u >> 1, qh = u & 1;
            const uint32_t t7 = theta_low7(dp.threshold);
            const uint32_t s0 = (uint32_t)(kt * kTile + 4 * kg);
            for (int it = 0; it < niter; ++it) {
                const int ms = it % kMStages;
                if (it >= kMStages && !warp_wait(bar(K::kBarMEmpty + ms), (uint32_t)((it / kMStages) & 1) ^ 1u, g))
                    break;
                const uint32_t t0 = (uint32_t)((kt + it) * kTile + 64 * qh);
                uint32_t lo[4], hi[4];
                if (dp.threshold >= 128u) {
                    dropout_keep32x4_keys<true>(dp.seed, t7, (uint32_t)bh, s0, t0, lo);
                    dropout_keep32x4_keys<true>(dp.seed, t7, (uint32_t)bh, s0, t0 + 32u, hi);
                } else {
                    dropout_keep32x4_keys<false>(dp.seed, t7, (uint32_t)bh, s0, t0, lo);
                    dropout_keep32x4_keys<false>(dp.seed, t7, (uint32_t)bh, s0, t0 + 32u, hi);
                }
                const uint32_t dst = sM + (uint32_t)ms * kMaskTileBytes + (uint32_t)(4 * kg) * 16u + (uint32_t)qh * 8u;
#pragma unroll
                for (int c = 0; c < 4; ++c) st_shared_v2(dst + (uint32_t)c * 16u, lo[c], hi[c]);
                mbar_arrive(bar(K::kBarMFull + ms));
            }
        }
    }
    } else if (warp < 12) {
        // ------------------------------------------------------------ softmax warpgroups (key rows)
        regs_inc<K::kRegsSoftmax>();
        const int half = (warp >> 2) - 1;  // query columns 64*half .. 64*half+63 of each tile
        const int sp = warp & 3;
        const int row = sp * 32 + lane;  // key row within the tile
        const uint32_t trow = tmem + ((uint32_t)(sp * 32) << 16);
        const float scale_log2 = 0.08838834764831845f * 1.4426950408889634f;
        bool ok = true;
        for (int it = 0; it < niter; ++it) {
            const int st = it % K::kQStages;
            const uint32_t ph = (uint32_t)(it / K::kQStages) & 1u;
            // dropout keep words of this key row's 64 query columns (bit layout of philox.cuh)
            uint32_t kb[2] = {0u, 0u};
            if constexpr (kDropout) {
                const int ms = it % kMStages;
                if (!(ok = warp_wait(bar(K::kBarMFull + ms), (uint32_t)(it / kMStages) & 1u, g))) break;
                const uint2 v = ld_shared_v2(sM + (uint32_t)ms * kMaskTileBytes + (uint32_t)row * 16u + (uint32_t)half * 8u);
                kb[0] = v.x;
                kb[1] = v.y;
                mbar_arrive(bar(K::kBarMEmpty + ms));
            }
            ok = warp_wait(bar(K::kBarQFull + st), ph, g) && warp_wait(bar(K::kBarS), (uint32_t)it & 1u, g);
            if (!ok) break;
            tc_fence_after();
            const float *lse_i = sLse + st * 128 + 64 * half;
            const float *D_i = sD + st * 128 + 64 * half;
            uint32_t pk[32];  // P^T row segment, bf16 pairs
            // this half's S^T columns in, P^T packed back over the first 32 of them
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t sr[32];
                tmem_ld_x32(trow + K::kColS + 64 * half + 32 * ch, sr);
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int cl = 32 * ch + e;      // column within the half
                    const int c = 64 * half + cl;    // query column within the tile
                    float p0 = ex2_approx(fmaf(__uint_as_float(sr[e]), scale_log2, lse_i[cl]));
                    float p1 = ex2_approx(fmaf(__uint_as_float(sr[e + 1]), scale_log2, lse_i[cl + 1]));
                    if (it == 0) {  // diagonal tile: query c sees key row only if row <= c
                        if (c < row) p0 = 0.f;
                        if (c + 1 < row) p1 = 0.f;
                    }
                    if (kBand && it * kTile + kTile - 1 >= window) {  // band's far edge: t - s < window
                        const int cut = window + row - it * kTile;  // query columns >= cut are masked
                        if (c >= cut) p0 = 0.f;
                        if (c + 1 >= cut) p1 = 0.f;
                    }
                    pk[cl >> 1] = pack_bf16x2(p0, p1);
                }
                // packed columns [16ch, 16ch+16) of this half were read in an earlier (or this) chunk;
                // with dropout the dV product gets the dropped weights zeroed, dS below the undropped ones
                if constexpr (kDropout) {
                    uint32_t pm[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) pm[q] = pk[16 * ch + q] & keep_pair_mask(kb[ch] << (q >> 1), q & 1);
                    tmem_st_x16(trow + K::kColS + 64 * half + 16 * ch, pm);
                } else {
                    tmem_st_x16(trow + K::kColS + 64 * half + 16 * ch,
                                *reinterpret_cast<const uint32_t(*)[16]>(&pk[16 * ch]));
                }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bar(K::kBarP));

            ok = warp_wait(bar(K::kBardP), (uint32_t)it & 1u, g);
            if (ok && it > 0) ok = warp_wait(bar(K::kBardQFull), (uint32_t)(it - 1) & 1u, g);  // dS buffer free
            if (!ok) break;
            tc_fence_after();
            // dS^T row `row`, this half's query columns = slab `half`, 16-byte chunks 4*ch .. 4*ch+3
            const uint32_t rbase = sdS + (uint32_t)half * kSlabBytes + (uint32_t)row * 128u;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t dr[32];
                tmem_ld_x32(trow + K::kColdP + 64 * half + 32 * ch, dr);
                if constexpr (kDropout) {  // dropped columns: dP^T o keep = 0
#pragma unroll
                    for (int e = 0; e < 32; ++e) dr[e] &= keep_word_mask(kb[ch] << (e >> 2), e & 3);
                }
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int cl = 32 * ch + e;
                    const uint32_t pp = pk[cl >> 1];
                    const float ds0 = bf16lo_to_f32(pp) * (__uint_as_float(dr[e]) + D_i[cl]);
                    const float ds1 = bf16hi_to_f32(pp) * (__uint_as_float(dr[e + 1]) + D_i[cl + 1]);
                    w[e >> 1] = pack_bf16x2(ds0, ds1);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t chunk = (uint32_t)(4 * ch + q);
                    st_shared_v4(rbase + ((chunk ^ (uint32_t)(row & 7)) << 4), w[4 * q], w[4 * q + 1], w[4 * q + 2],
                                 w[4 * q + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar(K::kBardS));
        }
        // -------------------------------------------------------- dK / dV epilogue
        // this half's 64 columns of dV and dK (scaled) -> bf16 -> slab `half` of the staging
        // tiles (dV in the stage-0 Q buffer, dK in the dO buffer, both free once the last MMAs ran)
        if (ok) ok = warp_wait(bar(K::kBarKdV), 0, g);
        if (ok) {
            tc_fence_after();
            const float scale = 0.08838834764831845f;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint32_t col = (which == 0 ? K::kColdV : K::kColdK) + 64u * (uint32_t)half;
                const float mul = which == 0 ? 1.f : scale;
                const uint32_t rbase0 = (which == 0 ? sQ(0) : sdO) + (uint32_t)half * kSlabBytes + (uint32_t)row * 128u;
#pragma unroll
                for (int c0 = 0; c0 < 64; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld_x32(trow + col + c0, o);
                    uint32_t w[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        w[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * mul, __uint_as_float(o[2 * c + 1]) * mul);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t chunk = (uint32_t)((c0 >> 3) + q);
                        st_shared_v4(rbase0 + ((chunk ^ (uint32_t)(row & 7)) << 4), w[4 * q], w[4 * q + 1],
                                     w[4 * q + 2], w[4 * q + 3]);
                    }
                }
            }
            fence_proxy_async_smem();
        }
        named_bar_sync(1, 256);
        if (warp == 4 && lane == 0 && !*abort_flag) {
            for (int s = 0; s < K::kSlabs; ++s) {
                tma_store_3d(&map_dqkv, sQ(0) + s * kSlabBytes, 2 * C + h * HS + 64 * s, kt * kTile, b);
                tma_store_3d(&map_dqkv, sdO + s * kSlabBytes, C + h * HS + 64 * s, kt * kTile, b);
            }
            bulk_commit_group();
            bulk_wait_group_0();
        }
    } else {
        // ------------------------------------------------------------ dQ drain warpgroup (query rows)
        regs_inc<K::kRegsDrain>();
        const int sp = warp & 3;
        const int row = sp * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(sp * 32) << 16);
        const bool leader = (warp == 12 && lane == 0);
        // Every thread of this role executes the same sequence of named
        // barriers whatever happens; after a failed wait the work is skipped.
        bool ok = true;
        for (int it = 0; it < niter; ++it) {
            const int qt = kt + it;
            if (ok) ok = warp_wait(bar(K::kBardQFull), (uint32_t)it & 1u, g);
            // both 64-column halves out of TMEM first, so that dP_{i+1} may take the columns
            uint32_t v[HS];
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < HS; c += 32)
                    tmem_ld_x32(trow + (c < 64 ? K::kColdQ0 + c : K::kColdQ1 + (c - 64)),
                                *reinterpret_cast<uint32_t(*)[32]>(&v[c]));
                tc_fence_before();
                mbar_arrive(bar(K::kBardQEmpty));
            }
            // then 32 columns at a time through the staging slab
#pragma unroll
            for (int u = 0; u < HS / 32; ++u) {
                if (leader) bulk_wait_group_read_0();  // the slab's previous copy-out has read it
                named_bar_sync(2, 128);
                if (ok) {
                    const uint32_t rbase = sdQ + (uint32_t)row * 128u;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        st_shared_v4(rbase + (((uint32_t)q ^ (uint32_t)(row & 7)) << 4), v[32 * u + 4 * q],
                                     v[32 * u + 4 * q + 1], v[32 * u + 4 * q + 2], v[32 * u + 4 * q + 3]);
                    fence_proxy_async_smem();
                }
                named_bar_sync(2, 128);
                if (leader && ok && !*abort_flag) {
                    if (n_slots == 0)  // add into the (b, h, query tile) rows of the accumulator
                        tma_reduce_add_2d(&map_dq, sdQ, 32 * u, bh * T_pad + qt * kTile);
                    else  // deterministic: a slot of its own per (query tile, key tile)
                        tma_store_2d(&map_dq, sdQ, 32 * u, (bh * n_slots + qt * (qt + 1) / 2 + kt) * kTile);
                    bulk_commit_group();
                }
            }
        }
        if (leader) bulk_wait_group_0();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// preprocess: per (b, h, t) store -D = -rowsum(dy o y) and -lse * log2(e)
// (negated so the main kernels add them); rows t >= T of each (b, h) get
// 0 and -inf (so the recomputed P there is 0); dQ accumulator zeroed.
// With dropout (kept weights scaled by s = 1/(1-p)) the caller passes
// lse_bias = log2(s) and d_mul = 1/s: the main kernel's recomputed weights are
// then P * s, what the dV product needs, and dS = (P s) o (dP o keep - D / s).
// ---------------------------------------------------------------------------
// 128-thread blocks, so that a whole (B * n_head, T_pad / 128) grid is resident at once
// for the usual sizes (16 blocks per SM).
constexpr int kPPThreads = 128;

// Grid (B * n_head, T_pad / 128): a block takes one 128-row tile of one (b, h).
// HS/8 lanes share a row (16 bytes of y and of dy each), so every warp load is a
// set of whole 128-byte rows; the dot product is finished with shuffles.  The
// block also zeroes its tile of the dQ accumulator.
template <int HS>
__global__ void __launch_bounds__(kPPThreads) bwd_pre_kernel(const __nv_bfloat16 *__restrict__ y,
                                                      const __nv_bfloat16 *__restrict__ dy,
                                                      const float *__restrict__ lse, float *__restrict__ D,
                                                      float *__restrict__ lse2, float4 *__restrict__ dqacc, int T,
                                                      int C, int n_head, int T_pad, int zero_acc, float lse_bias,
                                                      float d_mul) {
    constexpr int kLanesPerRow = HS / 8;
    constexpr int kRowsPerPass = kPPThreads / kLanesPerRow;
    const int bh = blockIdx.x, b = bh / n_head, h = bh % n_head;
    const int sub = threadIdx.x / kLanesPerRow, part = threadIdx.x % kLanesPerRow;
    const size_t row0 = (size_t)bh * T_pad + (size_t)blockIdx.y * kTile;
    griddep_launch_dependents();
    // The accumulator tile is zeroed before the wait for the previous kernel: no kernel of
    // this library that may still run reads it (the postprocess kernels, its only readers,
    // let their dependents start only after their reads), so the zeroing overlaps the
    // previous kernel's tail.
    if (zero_acc) {
        float4 *acc = dqacc + row0 * (HS / 4);
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int i = threadIdx.x; i < kTile * HS / 4; i += kPPThreads) acc[i] = z;
    }
    griddep_wait();
#pragma unroll
    for (int r = 0; r < kTile; r += kRowsPerPass) {
        const int t = blockIdx.y * kTile + r + sub;
        float d = 0.f;
        if (t < T) {
            const size_t off = ((size_t)b * T + t) * (size_t)C + (size_t)h * HS + (size_t)part * 8;
            const uint4 a = *reinterpret_cast<const uint4 *>(y + off);
            const uint4 c = *reinterpret_cast<const uint4 *>(dy + off);
            const uint32_t av[4] = {a.x, a.y, a.z, a.w}, cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                d = fmaf(bf16lo_to_f32(av[q]), bf16lo_to_f32(cv[q]), d);
                d = fmaf(bf16hi_to_f32(av[q]), bf16hi_to_f32(cv[q]), d);
            }
        }
#pragma unroll
        for (int o = kLanesPerRow / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        if (part == 0) {  // stored negated: -D and -lse*log2(e); padded rows 0 and -inf
            D[row0 + r + sub] = -d * d_mul;
            lse2[row0 + r + sub] = t < T ? -lse[(size_t)bh * T + t] * 1.4426950408889634f + lse_bias : -INFINITY;
        }
    }
}

// postprocess: dq = bf16(dqacc * scale) into dqkv[..., 0:C].  Grid (B * n_head,
// T_pad / 128): a block converts one 128-row tile of one (b, h), which is 32 KB
// contiguous in the accumulator; a thread moves 8 elements at a time.
template <int HS>
__global__ void __launch_bounds__(kPPThreads) bwd_post_kernel(const float *__restrict__ dqacc, __nv_bfloat16 *__restrict__ dqkv,
                                                       int T, int C, int n_head, int T_pad) {
    constexpr int kPerRow = HS / 8;
    const float scale = (HS == 64 ? 0.125f : 0.08838834764831845f);
    griddep_wait();
    const int bh = blockIdx.x, b = bh / n_head, h = bh % n_head;
    const int t0 = blockIdx.y * kTile;
    const float4 *src = reinterpret_cast<const float4 *>(dqacc + ((size_t)bh * T_pad + t0) * HS);
    __nv_bfloat16 *dst = dqkv + ((size_t)b * T + t0) * (size_t)(3 * C) + (size_t)h * HS;
#pragma unroll
    for (int i = threadIdx.x; i < kTile * kPerRow; i += kPPThreads) {
        const int r = i / kPerRow, k = i % kPerRow;
        if (t0 + r < T) {
            const float4 a = src[2 * i], c = src[2 * i + 1];
            uint4 o;
            o.x = pack_bf16x2(a.x * scale, a.y * scale);
            o.y = pack_bf16x2(a.z * scale, a.w * scale);
            o.z = pack_bf16x2(c.x * scale, c.y * scale);
            o.w = pack_bf16x2(c.z * scale, c.w * scale);
            *reinterpret_cast<uint4 *>(dst + (size_t)r * (size_t)(3 * C) + (size_t)k * 8) = o;
        }
    }
    // dependents may start only now: the next call's preprocess zeroes this accumulator
    // before it waits for this kernel
    griddep_launch_dependents();
}

// deterministic postprocess: dq = bf16(scale * sum over key tiles j of partial(i, j)),
// the partials of query tile i summed in increasing j, so the result does not
// depend on the order in which CTAs produced them.  Same grid as above; slots
// of key tiles outside the band (window) were never written and are not read.
template <int HS>
__global__ void __launch_bounds__(kPPThreads) bwd_post_det_kernel(const float *__restrict__ part,
                                                           __nv_bfloat16 *__restrict__ dqkv, int T, int C, int n_head,
                                                           int n_slots, int window) {
    griddep_wait();
    constexpr int kPerRow = HS / 8;
    const float scale = (HS == 64 ? 0.125f : 0.08838834764831845f);
    const int bh = blockIdx.x, b = bh / n_head, h = bh % n_head;
    const int qt = blockIdx.y, t0 = qt * kTile;
    const int s_first = qt * kTile - window + 1;
    const int jlo = s_first > 0 ? s_first / kTile : 0;
    __nv_bfloat16 *dst = dqkv + ((size_t)b * T + t0) * (size_t)(3 * C) + (size_t)h * HS;
#pragma unroll
    for (int i = threadIdx.x; i < kTile * kPerRow; i += kPPThreads) {
        const int r = i / kPerRow, k = i % kPerRow;
        if (t0 + r >= T) continue;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j = jlo; j <= qt; ++j) {
            const float4 *src = reinterpret_cast<const float4 *>(
                part + ((size_t)bh * n_slots + (size_t)(qt * (qt + 1) / 2 + j)) * kTile * HS);
            const float4 a = src[2 * i], c = src[2 * i + 1];
            acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
            acc[4] += c.x; acc[5] += c.y; acc[6] += c.z; acc[7] += c.w;
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0] * scale, acc[1] * scale);
        o.y = pack_bf16x2(acc[2] * scale, acc[3] * scale);
        o.z = pack_bf16x2(acc[4] * scale, acc[5] * scale);
        o.w = pack_bf16x2(acc[6] * scale, acc[7] * scale);
        *reinterpret_cast<uint4 *>(dst + (size_t)r * (size_t)(3 * C) + (size_t)k * 8) = o;
    }
    griddep_launch_dependents();  // after the reads of the workspace, as in bwd_post_kernel
}

template <int HS, bool kBand, bool kDropout>
cudaError_t launch_main_variant(const CUtensorMap &map_qkv, const CUtensorMap &map_dy, const CUtensorMap &map_dqkv,
                                const CUtensorMap &map_dq, const float *lse2, const float *D, int B, int T, int C,
                                int n_head, int T_pad, int window, int n_slots, DropoutParams dp, DevCtx ctx,
                                cudaStream_t s) {
    using K = BwdCfg<HS, kDropout>;
    auto kern = bwd_bf16_kernel<HS, kBand, kDropout>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)K::kSmemBytes);
    if (e != cudaSuccess) return e;
    // the warpgroups' register budgets add up to the launch allocation only at kLaunchRegs per
    // thread; otherwise a setmaxnreg.inc could never be satisfied, so refuse to launch
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != K::kLaunchRegs) return cudaErrorInvalidConfiguration;
    const int n_t = ceil_div(T, kTile);
    const long long blocks = (long long)n_t * B * n_head;
    return launch_pdl(kern, dim3((unsigned)blocks), dim3(K::kThreads), K::kSmemBytes, s, map_qkv, map_dy, map_dqkv,
                      map_dq, lse2, D, B, T, C, n_head, T_pad, n_t, window, n_slots, dp, ctx.status, ctx.budget_ns);
}

template <int HS>
cudaError_t launch_main_impl(const CUtensorMap &map_qkv, const CUtensorMap &map_dy, const CUtensorMap &map_dqkv,
                             const CUtensorMap &map_dq, const float *lse2, const float *D, int B, int T, int C,
                             int n_head, int T_pad, int window, int n_slots, DropoutParams dp, DevCtx ctx,
                             cudaStream_t s) {
    const bool band = window < T, drop = dp.threshold != 0u;
    auto run = [&](auto kern_launch) {
        return kern_launch(map_qkv, map_dy, map_dqkv, map_dq, lse2, D, B, T, C, n_head, T_pad, window, n_slots, dp, ctx,
                           s);
    };
    if (band) return drop ? run(launch_main_variant<HS, true, true>) : run(launch_main_variant<HS, true, false>);
    return drop ? run(launch_main_variant<HS, false, true>) : run(launch_main_variant<HS, false, false>);
}

}  // namespace

cudaError_t launch_bwd_pre_bf16(int hs, const void *y, const void *dy, const float *lse, float *D, float *lse2,
                                float *dqacc, int B, int T, int C, int n_head, int T_pad, bool zero_acc, float lse_bias,
                                float d_mul, cudaStream_t s) {
    const dim3 grid((unsigned)(B * n_head), (unsigned)(T_pad / kTile));
    auto yy = static_cast<const __nv_bfloat16 *>(y);
    auto gg = static_cast<const __nv_bfloat16 *>(dy);
    auto zz = reinterpret_cast<float4 *>(dqacc);
    const int za = zero_acc ? 1 : 0;
    if (hs == 64)
        return launch_pdl(bwd_pre_kernel<64>, grid, dim3(kPPThreads), 0, s, yy, gg, lse, D, lse2, zz, T, C, n_head, T_pad,
                          za, lse_bias, d_mul);
    if (hs == 128)
        return launch_pdl(bwd_pre_kernel<128>, grid, dim3(kPPThreads), 0, s, yy, gg, lse, D, lse2, zz, T, C, n_head, T_pad,
                          za, lse_bias, d_mul);
    return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_main_bf16(int hs, const CUtensorMap &map_qkv, const CUtensorMap &map_dy,
                                 const CUtensorMap &map_dqkv, const CUtensorMap &map_dq, const float *lse2,
                                 const float *D, int B, int T, int C, int n_head, int T_pad, int window, int n_slots,
                                 DropoutParams dp, DevCtx ctx, cudaStream_t s) {
    if (hs == 64)
        return launch_bwd_main_h64(map_qkv, map_dy, map_dqkv, map_dq, lse2, D, B, T, C, n_head, T_pad, window, n_slots,
                                   dp, ctx, s);
    if (hs == 128)
        return launch_main_impl<128>(map_qkv, map_dy, map_dqkv, map_dq, lse2, D, B, T, C, n_head, T_pad, window, n_slots,
                                     dp, ctx, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_post_bf16(int hs, const float *dqacc, void *dqkv, int B, int T, int C, int n_head, int T_pad,
                                 cudaStream_t s) {
    const dim3 grid((unsigned)(B * n_head), (unsigned)(T_pad / kTile));
    auto out = static_cast<__nv_bfloat16 *>(dqkv);
    if (hs == 64) return launch_pdl(bwd_post_kernel<64>, grid, dim3(kPPThreads), 0, s, dqacc, out, T, C, n_head, T_pad);
    if (hs == 128) return launch_pdl(bwd_post_kernel<128>, grid, dim3(kPPThreads), 0, s, dqacc, out, T, C, n_head, T_pad);
    return cudaErrorInvalidValue;
}
cudaError_t launch_bwd_post_det_bf16(int hs, const float *part, void *dqkv, int B, int T, int C, int n_head, int T_pad,
                                     int n_slots, int window, cudaStream_t s) {
    const dim3 grid((unsigned)(B * n_head), (unsigned)(T_pad / kTile));
    auto out = static_cast<__nv_bfloat16 *>(dqkv);
    if (hs == 64)
        return launch_pdl(bwd_post_det_kernel<64>, grid, dim3(kPPThreads), 0, s, part, out, T, C, n_head, n_slots, window);
    if (hs == 128)
        return launch_pdl(bwd_post_det_kernel<128>, grid, dim3(kPPThreads), 0, s, part, out, T, C, n_head, n_slots,
                          window);
    return cudaErrorInvalidValue;
}

}  // namespace gptattn
