// fwd_sm100.cu -- bf16 causal self-attention forward for sm_100a.
//
// Computes, per (batch b, head h) and 128-row query tile i (lecture page
// "Let's build GPT: from scratch, in code, spelled out", chapters "version 3:
// adding softmax" and "version 4: self-attention"; note 6 / correction 01:20:05
// for the 1/sqrt(head_size) scale; correction 00:57:00 for the causal mask):
//     S_j = Q_i K_j^T                 (tcgen05 MMA, fp32 accumulators in TMEM)
//     online softmax of S_j * scale   (fp32, one TMEM lane = one query row per thread)
//     O  += P_j V_j                   (tcgen05 MMA, P read straight from TMEM)
// for key tiles j = 0..i only (tiles above the diagonal are skipped, the
// diagonal tile is masked element-wise), then y = O / l and lse = m + ln l.
//
// One CTA per (query tile, b, h), six warps with fixed roles:
//   warp 0      TMA producer: Q once, then K_j / V_j through a smem ring
//   warp 1      TMEM owner + MMA issuer (one elected lane)
//   warps 2..5  softmax, O rescale and epilogue (128 threads = 128 query rows)
// TMEM (512 columns): S double buffer at [0,128) and [128,256), O at [256,256+hs).
// Every barrier wait is bounded (see sm100_ptx.cuh); a timeout sets the CTA's
// abort flag and the device status word, and all roles drain and exit.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace gptattn {
namespace {

constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlabBytes = 128 * 128;  // 128 rows x 128 bytes (64 bf16 columns), one swizzle slab

template <int HS>
struct FwdCfg {
    static constexpr int kSlabs = HS / 64;
    static constexpr uint32_t kTileBytes = 128u * HS * 2u;
    static constexpr int kStages = (HS == 64) ? 3 : 2;
    static constexpr uint32_t kOffQ = 0;
    static constexpr uint32_t kOffK = kOffQ + kTileBytes;
    static constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
    static constexpr uint32_t kOffBar = kOffV + kStages * kTileBytes;
    static constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // + slack for 1024-byte alignment
    static constexpr uint32_t kColS = 0;    // S buffers at kColS + 128 * (j & 1)
    static constexpr uint32_t kColO = 256;
    // barrier slots (8 bytes each)
    static constexpr int kBarQ = 0;
    static constexpr int kBarK = 1;
    static constexpr int kBarV = kBarK + kStages;
    static constexpr int kBarE = kBarV + kStages;
    static constexpr int kBarS = kBarE + kStages;  // two
    static constexpr int kBarP = kBarS + 2;
    static constexpr int kBarO = kBarP + 1;
    static constexpr int kBarDone = kBarO + 1;
    static constexpr int kNumBars = kBarDone + 1;
    static_assert(kNumBars * 8 + 16 <= 256, "barrier area");
};

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

template <int HS>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_bf16_kernel(const __grid_constant__ CUtensorMap map_qkv, const __grid_constant__ CUtensorMap map_y,
                    float *__restrict__ lse, int B, int T, int C, int n_head, int n_qt, int *status,
                    unsigned long long budget_ns) {
    using K = FwdCfg<HS>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_base & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int BH = B * n_head;
    const int bh = blockIdx.x % BH;
    const int qt = n_qt - 1 - blockIdx.x / BH;  // longest rows first
    const int b = bh / n_head;
    const int h = bh % n_head;
    const int nkv = qt + 1;                     // causal: key tiles 0..qt

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + K::kOffBar);
    auto bar = [&](int idx) -> uint32_t { return smem_u32(&bars[idx]); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + K::kOffBar + K::kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + K::kOffBar + K::kNumBars * 8 + 4);
    const WaitGuard g{abort_flag, status, budget_ns};

    const uint32_t sQ = sbase + K::kOffQ;
    auto sK = [&](int st) -> uint32_t { return sbase + K::kOffK + st * K::kTileBytes; };
    auto sV = [&](int st) -> uint32_t { return sbase + K::kOffV + st * K::kTileBytes; };

    if (threadIdx.x == 0) {
        mbar_init(bar(K::kBarQ), 1);
        for (int s = 0; s < K::kStages; ++s) {
            mbar_init(bar(K::kBarK + s), 1);
            mbar_init(bar(K::kBarV + s), 1);
            mbar_init(bar(K::kBarE + s), 1);
        }
        mbar_init(bar(K::kBarS + 0), 1);
        mbar_init(bar(K::kBarS + 1), 1);
        mbar_init(bar(K::kBarP), 128);
        mbar_init(bar(K::kBarO), 1);
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

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_map(&map_qkv);
            tma_prefetch_map(&map_y);
            const int col_q = h * HS, col_k = C + h * HS, col_v = 2 * C + h * HS;
            mbar_arrive_expect_tx(bar(K::kBarQ), K::kTileBytes);
            for (int s = 0; s < K::kSlabs; ++s)
                tma_load_3d(sQ + s * kSlabBytes, &map_qkv, bar(K::kBarQ), col_q + 64 * s, qt * kTile, b);
            int issued = 0;
            bool ok = true;
            for (int j = 0; j < nkv; ++j) {
                const int st = j % K::kStages;
                const uint32_t ph = (uint32_t)(j / K::kStages) & 1u;
                if (j >= K::kStages && !mbar_wait(bar(K::kBarE + st), ph ^ 1u, g)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(bar(K::kBarK + st), K::kTileBytes);
                for (int s = 0; s < K::kSlabs; ++s)
                    tma_load_3d(sK(st) + s * kSlabBytes, &map_qkv, bar(K::kBarK + st), col_k + 64 * s, j * kTile, b);
                mbar_arrive_expect_tx(bar(K::kBarV + st), K::kTileBytes);
                for (int s = 0; s < K::kSlabs; ++s)
                    tma_load_3d(sV(st) + s * kSlabBytes, &map_qkv, bar(K::kBarV + st), col_v + 64 * s, j * kTile, b);
                issued = j + 1;
            }
            if (!ok || *abort_flag) {
                // let this CTA's own copies land before shared memory is released
                drain_wait(bar(K::kBarQ), 0, budget_ns);
                for (int j = (issued > K::kStages ? issued - K::kStages : 0); j < issued; ++j) {
                    const uint32_t ph = (uint32_t)(j / K::kStages) & 1u;
                    drain_wait(bar(K::kBarK + j % K::kStages), ph, budget_ns);
                    drain_wait(bar(K::kBarV + j % K::kStages), ph, budget_ns);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);  // Q, K both K-major
            constexpr uint32_t idPV = idesc_bf16_f32(128, HS, false, true);   // P from TMEM, V N-major
            bool ok = mbar_wait(bar(K::kBarQ), 0, g);
            bool any = false;
            auto issue_s = [&](int j) -> bool {
                const int st = j % K::kStages;
                const uint32_t ph = (uint32_t)(j / K::kStages) & 1u;
                if (!mbar_wait(bar(K::kBarK + st), ph, g)) return false;
                tc_fence_after();
                const uint32_t d = tmem + K::kColS + 128u * (uint32_t)(j & 1);
#pragma unroll
                for (int kk = 0; kk < HS / 16; ++kk) {
                    const uint32_t koff = (uint32_t)(kk >> 2) * kSlabBytes + (uint32_t)(kk & 3) * 32u;
                    umma_ss(d, sdesc_sw128(sQ + koff, 16, 1024), sdesc_sw128(sK(st) + koff, 16, 1024), idS,
                            kk > 0 ? 1u : 0u);
                }
                umma_commit(bar(K::kBarS + (j & 1)));
                any = true;
                return true;
            };
            auto issue_pv = [&](int j) -> bool {
                const int st = j % K::kStages;
                const uint32_t ph = (uint32_t)(j / K::kStages) & 1u;
                if (!mbar_wait(bar(K::kBarP), (uint32_t)j & 1u, g)) return false;
                if (!mbar_wait(bar(K::kBarV + st), ph, g)) return false;
                tc_fence_after();
                const uint32_t p = tmem + K::kColS + 128u * (uint32_t)(j & 1);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    umma_ts(tmem + K::kColO, p + 8u * kk, sdesc_sw128(sV(st) + kk * 2048u, kSlabBytes, 1024), idPV,
                            (j > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(bar(K::kBarE + st));
                umma_commit(bar(K::kBarO));
                return true;
            };
            for (int j = 0; j < nkv && ok; ++j) {
                ok = issue_s(j);
                if (ok && j > 0) ok = issue_pv(j - 1);
            }
            if (ok) ok = issue_pv(nkv - 1);
            if (any) {
                // all MMAs of this CTA retired before TMEM can be released
                umma_commit(bar(K::kBarDone));
                drain_wait(bar(K::kBarDone), 0, budget_ns);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax warps
        const int sp = warp & 3;                 // TMEM sub-partition this warp may access
        const int row = sp * 32 + lane;          // query row within the tile
        const uint32_t trow = tmem + ((uint32_t)(sp * 32) << 16);
        const float scale_log2 = rsqrtf((float)HS) * 1.4426950408889634f;
        float m = -INFINITY;  // running max of scaled scores (log2 units)
        float l = 0.f;        // running normaliser (fp32 weights)
        float l_r = 0.f;      // running normaliser (bf16-rounded weights)
        bool ok = true;
        for (int j = 0; j < nkv; ++j) {
            ok = warp_wait(bar(K::kBarS + (j & 1)), (uint32_t)(j >> 1) & 1u, g);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tS = trow + K::kColS + 128u * (uint32_t)(j & 1);
            uint32_t sr[128];
            tmem_ld_x32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            tmem_ld_x32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            tmem_ld_x32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
            tmem_ld_x32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
            float *s = reinterpret_cast<float *>(sr);
            if (j == qt) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c > row) s[c] = -INFINITY;
            }
            // row max with 8 independent partial maxima (no 128-long dependency chain)
            float mp[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) mp[k] = s[k];
#pragma unroll
            for (int c = 8; c < 128; ++c) mp[c & 7] = fmaxf(mp[c & 7], s[c]);
            const float mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                                   fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
            // Lazy rescaling: keep the running max unless it grows by more than
            // 8 (log2 units).  p stays <= 2^8 and l, O use the same stale max,
            // so y = O / l and lse = m + log2 l are exact; O is rescaled rarely.
            const float m_cand = mx * scale_log2;
            const bool grow = m_cand > m + 8.f;
            const float m_new = grow ? m_cand : m;
            const float alpha = grow ? ex2_approx(m - m_new) : 1.f;
            const float neg = -m_new;
            // Two row sums: of the fp32 weights (for lse) and of the bf16-rounded
            // weights the P V product actually uses (to normalise y, so that a
            // row dominated by one key returns that key's value exactly).
            float sp8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            float sr8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            uint32_t pk[64];
#pragma unroll
            for (int c = 0; c < 128; c += 2) {
                const float p0 = ex2_approx(fmaf(s[c], scale_log2, neg));
                const float p1 = ex2_approx(fmaf(s[c + 1], scale_log2, neg));
                sp8[(c >> 1) & 7] += p0 + p1;
                const uint32_t w = pack_bf16x2(p0, p1);
                sr8[(c >> 1) & 7] += bf16lo_to_f32(w) + bf16hi_to_f32(w);
                pk[c >> 1] = w;
            }
            const float sum = ((sp8[0] + sp8[1]) + (sp8[2] + sp8[3])) + ((sp8[4] + sp8[5]) + (sp8[6] + sp8[7]));
            const float sum_r = ((sr8[0] + sr8[1]) + (sr8[2] + sr8[3])) + ((sr8[4] + sr8[5]) + (sr8[6] + sr8[7]));
            tmem_st_x32(tS + 0, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
            tmem_st_x32(tS + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
            l = l * alpha + sum;
            l_r = l_r * alpha + sum_r;
            m = m_new;
            if (j > 0) {
                // rescale O once the previous P V product has landed
                ok = warp_wait(bar(K::kBarO), (uint32_t)(j - 1) & 1u, g);
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                    for (int c0 = 0; c0 < HS; c0 += 32) {
                        uint32_t o[32];
                        tmem_ld_x32(trow + K::kColO + c0, o);
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                        tmem_st_x32(trow + K::kColO + c0, o);
                    }
                }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bar(K::kBarP));
        }
        // -------------------------------------------------------- epilogue
        if (ok) ok = warp_wait(bar(K::kBarO), (uint32_t)(nkv - 1) & 1u, g);
        if (ok) {
            tc_fence_after();
            const float inv_l = 1.f / l_r;
#pragma unroll
            for (int c0 = 0; c0 < HS; c0 += 32) {
                uint32_t o[32];
                tmem_ld_x32(trow + K::kColO + c0, o);
                uint32_t w[16];
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    w[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv_l, __uint_as_float(o[2 * c + 1]) * inv_l);
                // staging tile in the Q buffer (Q is dead once the last S MMA retired)
                const uint32_t slab = sQ + (uint32_t)(c0 >> 6) * kSlabBytes + (uint32_t)row * 128u;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t chunk = (uint32_t)(((c0 & 63) >> 3) + q);
                    st_shared_v4(slab + ((chunk ^ (uint32_t)(row & 7)) << 4), w[4 * q], w[4 * q + 1], w[4 * q + 2],
                                 w[4 * q + 3]);
                }
            }
            fence_proxy_async_smem();
            const int t = qt * kTile + row;
            if (t < T) lse[(size_t)bh * (size_t)T + (size_t)t] = (m + __log2f(l)) * 0.6931471805599453f;
        }
        named_bar_sync(1, 128);
        if (warp == 2 && lane == 0 && !*abort_flag) {
            for (int s = 0; s < K::kSlabs; ++s) tma_store_3d(&map_y, sQ + s * kSlabBytes, h * HS + 64 * s, qt * kTile, b);
            bulk_commit_group();
            bulk_wait_group_0();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int HS>
cudaError_t launch_fwd_impl(const CUtensorMap &map_qkv, const CUtensorMap &map_y, float *lse, int B, int T, int C,
                            int n_head, DevCtx ctx, cudaStream_t s) {
    using K = FwdCfg<HS>;
    cudaError_t e = cudaFuncSetAttribute(fwd_bf16_kernel<HS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)K::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int n_qt = ceil_div(T, kTile);
    const long long blocks = (long long)n_qt * B * n_head;
    fwd_bf16_kernel<HS><<<dim3((unsigned)blocks), dim3(kThreads), K::kSmemBytes, s>>>(
        map_qkv, map_y, lse, B, T, C, n_head, n_qt, ctx.status, ctx.budget_ns);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_bf16(int hs, const CUtensorMap &map_qkv, const CUtensorMap &map_y, float *lse, int B, int T,
                            int C, int n_head, DevCtx ctx, cudaStream_t s) {
    if (hs == 64) return launch_fwd_impl<64>(map_qkv, map_y, lse, B, T, C, n_head, ctx, s);
    if (hs == 128) return launch_fwd_impl<128>(map_qkv, map_y, lse, B, T, C, n_head, ctx, s);
    return cudaErrorInvalidValue;
}

}  // namespace gptattn
