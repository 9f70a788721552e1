// bwd_h64_sm100.cu -- persistent bf16 causal self-attention backward, head size 64.
//
// Same mathematics as bwd_sm100.cu (chain rule through "version 3: adding
// softmax" and "version 4: self-attention" of the lecture page "Let's build
// GPT: from scratch, in code, spelled out"; P recomputed from the saved
// logsumexp):  dV += P^T dY,  dP = dY V^T,  dS = P o (dP - D),
//              dK += dS^T Q * scale,  dQ += dS K * scale.
// The workspace rows hold -D and -lse*log2(e) (negated by the preprocess kernel).
// Local window (minGPT README page, reference notes on GPT-3: locally banded
// attention): key s is seen by queries s <= t < s + window, so a key tile's
// item stops at the last query tile its band reaches and the band's far edge
// is masked element-wise like the diagonal.  window >= T is the causal case.
// Deterministic mode (n_slots > 0): instead of adding dQ_i into an fp32
// accumulator with TMA reduce-adds (whose order across CTAs varies run to run),
// each (query tile i, key tile j) partial is stored in its own slot i(i+1)/2 + j
// and the postprocess kernel sums the slots of a query tile in a fixed order.
// Dropout (inverted dropout on the weights, Philox mask of philox.cuh): the
// P^T stored for dV is the dropped, rescaled weight, and dS = P o (dP o f - D)
// with f = 1/(1-p) for kept weights, 0 for dropped ones.
//
// Schedule: one persistent CTA per SM walks a static list of work items
// (key tile j, batch b, head h), ordered longest first (small j first), in a
// snake order over the CTAs (round k takes items k*grid .. k*grid+grid-1,
// reversed on odd rounds), which evens out the causal triangle's work across
// CTAs.  Per item the CTA loops over query tiles i >= j.
//
// Warp roles (16 warps, four warpgroups; setmaxnreg moves registers from the
// first warpgroup to the last):
//   warp 0        TMA producer: K_j, V_j (double-buffered across items), and
//                 Q_i, dO_i, lse_i, D_i through a 3-stage ring
//   warp 1        TMEM owner + MMA issuer of S, dP, dV (with dropout: of all five)
//   warp 2        MMA issuer of dK, dQ (without dropout; with it, warps 2-3 draw
//                 the dropout keep words)
//   warps 4..11   softmax: TMEM sub-partition warp%4 (32 key rows), column
//                 half warp/4 - 1 (64 query columns): P^T, dS^T
//   warps 12..15  dQ drain: TMEM -> smem (fp32, swizzled) -> TMA reduce-add;
//                 and per item the dK/dV epilogue (TMEM -> bf16 -> TMA store)
// TMEM (512 columns): S^T [0,128)  dP^T [128,256)  P^T [256,320) (bf16 pairs)
//                     dV [320,384)  dK [384,448)  dQ [448,512)
// MMA order per item: S_0 dP_0 | S_1 dV_0 dP_1 | S_2 dV_1 dP_2 ... on warp 1, and
// dK_i dQ_i on warp 2 as soon as dS_i is written (with dropout warp 1 issues them
// after dP_{i+1}).
// S^T and dP^T are released as soon as the softmax warps hold them in
// registers, so the tensor pipe computes tile i+1 while tile i is in softmax.
// Every wait is bounded; roles never leave their loops early, so all named
// barriers are reached the same number of times by every thread of a role.
#include <type_traits>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace gptattn {
namespace {

constexpr int kThreads = 512;
// register budgets per thread of the four warpgroups (sum = 4 x kLaunchRegs, what the
// CTA is launched with)
constexpr int kLaunchRegs = 128;
constexpr uint32_t kRegsCtl = 96, kRegsSoftmax = 144, kRegsDrain = 128;
static_assert(kRegsCtl + 2 * kRegsSoftmax + kRegsDrain == 4 * kLaunchRegs, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlabBytes = 128 * 128;
constexpr int HS = 64;
constexpr uint32_t kTileBytes = 128u * 64u * 2u;  // one 128 x 64 bf16 tile = one slab
constexpr int kQStages = 3;
constexpr int kKVStages = 2;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffK = 0;                                   // kKVStages tiles
constexpr uint32_t kOffV = kOffK + kKVStages * kTileBytes;       // kKVStages tiles
constexpr uint32_t kOffQ = kOffV + kKVStages * kTileBytes;       // kQStages tiles
constexpr uint32_t kOffdO = kOffQ + kQStages * kTileBytes;       // kQStages tiles
constexpr uint32_t kOffdS = kOffdO + kQStages * kTileBytes;      // 128 x 128 bf16 (2 slabs)
constexpr uint32_t kOffdQ = kOffdS + 2 * kSlabBytes;             // 128 x 32 fp32 staging (1 slab)
constexpr uint32_t kOffLse = kOffdQ + kSlabBytes;                // kQStages x 128 fp32
constexpr uint32_t kOffD = kOffLse + kQStages * 512;             // kQStages x 128 fp32
constexpr uint32_t kOffBar = kOffD + kQStages * 512;
constexpr uint32_t kBarArea = 512;
// dropout keep bits, drawn ahead by warps 2 and 3: kMStages tiles of 128 key rows x 128 query bits
constexpr int kMStages = 4;
constexpr uint32_t kMaskTileBytes = 128u * 16u;
constexpr uint32_t kOffM = kOffBar + kBarArea;
template <bool kDropout>
constexpr uint32_t smem_bytes() { return kOffM + (kDropout ? kMStages * kMaskTileBytes : 0u) + 1024; }
static_assert(smem_bytes<true>() <= 227 * 1024, "shared memory");

// TMEM columns
constexpr uint32_t kColS = 0, kColdP = 128, kColP = 256, kColdV = 320, kColdK = 384, kColdQ = 448;

// barriers
constexpr int kBarKVFull = 0;                      // kKVStages
constexpr int kBarKVEmpty = kBarKVFull + kKVStages;  // kKVStages
constexpr int kBarQFull = kBarKVEmpty + kKVStages;   // kQStages
constexpr int kBarQEmpty = kBarQFull + kQStages;     // kQStages
constexpr int kBarSFull = kBarQEmpty + kQStages;
constexpr int kBarSEmpty = kBarSFull + 1;
constexpr int kBardPFull = kBarSEmpty + 1;
constexpr int kBardPEmpty = kBardPFull + 1;
constexpr int kBarPFull = kBardPEmpty + 1;
constexpr int kBarPEmpty = kBarPFull + 1;
constexpr int kBardSFull = kBarPEmpty + 1;
constexpr int kBardQFull = kBardSFull + 1;  // dQ_i done; also frees the dS buffer (dK_i ran before it)
constexpr int kBardQEmpty = kBardQFull + 1;
constexpr int kBarKdV = kBardQEmpty + 1;
constexpr int kBarAccFree = kBarKdV + 1;
constexpr int kBarDone = kBarAccFree + 1;
constexpr int kBarDoneB = kBarDone + 1;          // second issuer's last MMAs retired
constexpr int kBarMFull = kBarDoneB + 1;         // kMStages
constexpr int kBarMEmpty = kBarMFull + kMStages;  // kMStages
constexpr int kNumBars = kBarMEmpty + kMStages;
static_assert(kNumBars * 8 + 16 <= kBarArea, "barrier area");
constexpr int kMaskThreads = 64;
// MMA issuers.  Without dropout a second thread (warp 2) issues the gradient products dK and dQ
// while warp 1 issues S, dV and dP: a lone issuing thread shares its sub-partition's issue slots
// with three busy warps and runs a few times slower than the tensor pipe it feeds.  With dropout
// warps 2 and 3 draw the keep words and warp 1 issues everything.  Buffers that both issuers'
// products read are released by a commit from each (barrier count = number of issuers).
template <bool kDropout>
constexpr uint32_t kIssuers = kDropout ? 1u : 2u;

constexpr int kSoftmaxThreads = 256;
constexpr int kDrainThreads = 128;

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

// Last query tile that key tile kt's band reaches.
__device__ __forceinline__ int band_hi_tile(int kt, int window, int n_t) {
    const long long t = (long long)kt * kTile + kTile - 2 + window;  // largest key + window - 1
    return t / kTile < n_t ? (int)(t / kTile) : n_t - 1;
}

__device__ __forceinline__ int item_index(int k, int cta, int grid) {
    return (k & 1) ? (k * grid + (grid - 1 - cta)) : (k * grid + cta);
}

template <bool kDropout>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_h64_persistent(const __grid_constant__ CUtensorMap map_qkv, const __grid_constant__ CUtensorMap map_dy,
                       const __grid_constant__ CUtensorMap map_dqkv, const __grid_constant__ CUtensorMap map_dq,
                       const float *__restrict__ lse2, const float *__restrict__ Dvec, int B, int T, int C,
                       int n_head, int T_pad, int n_t, int window, int n_slots, DropoutParams dp, int *status,
                       unsigned long long budget_ns) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_base & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int wg = warp >> 2;
    const int BH = B * n_head;
    const int n_items = n_t * BH;

    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    auto bar = [&](int idx) -> uint32_t { return smem_u32(&bars[idx]); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffBar + kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffBar + kNumBars * 8 + 4);
    const WaitGuard g{abort_flag, status, budget_ns};

    auto sK = [&](int s) -> uint32_t { return sbase + kOffK + s * kTileBytes; };
    auto sV = [&](int s) -> uint32_t { return sbase + kOffV + s * kTileBytes; };
    auto sQ = [&](int s) -> uint32_t { return sbase + kOffQ + s * kTileBytes; };
    auto sdO = [&](int s) -> uint32_t { return sbase + kOffdO + s * kTileBytes; };
    const uint32_t sdS = sbase + kOffdS, sdQ = sbase + kOffdQ;
    const float *sLse = reinterpret_cast<const float *>(smem + kOffLse);
    const float *sD = reinterpret_cast<const float *>(smem + kOffD);
    auto sM = [&](int s) -> uint32_t { return sbase + kOffM + (uint32_t)s * kMaskTileBytes; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kKVStages; ++s) {
            mbar_init(bar(kBarKVFull + s), 1);
            mbar_init(bar(kBarKVEmpty + s), kIssuers<kDropout>);
        }
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(bar(kBarQFull + s), 1);
            mbar_init(bar(kBarQEmpty + s), kIssuers<kDropout>);
        }
        mbar_init(bar(kBarSFull), 1);
        mbar_init(bar(kBarSEmpty), kSoftmaxThreads);
        mbar_init(bar(kBardPFull), 1);
        mbar_init(bar(kBardPEmpty), kSoftmaxThreads);
        mbar_init(bar(kBarPFull), kSoftmaxThreads);
        mbar_init(bar(kBarPEmpty), 1);
        mbar_init(bar(kBardSFull), kSoftmaxThreads);
        mbar_init(bar(kBardQFull), 1);
        mbar_init(bar(kBardQEmpty), kDrainThreads);
        mbar_init(bar(kBarKdV), kIssuers<kDropout>);
        mbar_init(bar(kBarAccFree), kDrainThreads);
        mbar_init(bar(kBarDone), 1);
        mbar_init(bar(kBarDoneB), 1);
        for (int s = 0; s < kMStages; ++s) {
            mbar_init(bar(kBarMFull + s), kMaskThreads);
            mbar_init(bar(kBarMEmpty + s), kSoftmaxThreads);
        }
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
        regs_dec<kRegsCtl>();
        if (warp == 0) {
            // ================================================================ producer
            if (lane == 0) {
                tma_prefetch_map(&map_qkv);
                tma_prefetch_map(&map_dy);
                bool ok = true;
                int n = 0;   // items started
                int gq = 0;  // query tiles issued (ring position)
                for (int k = 0; ok; ++k, ++n) {
                    const int w = item_index(k, blockIdx.x, gridDim.x);
                    if (w >= n_items) break;
                    const int kt = w / BH, bh = w % BH, b = bh / n_head, h = bh % n_head;
                    const int kvs = n & 1;
                    if (n >= kKVStages && !(ok = mbar_wait(bar(kBarKVEmpty + kvs), (uint32_t)((n >> 1) & 1) ^ 1u, g)))
                        break;
                    mbar_arrive_expect_tx(bar(kBarKVFull + kvs), 2 * kTileBytes);
                    tma_load_3d(sK(kvs), &map_qkv, bar(kBarKVFull + kvs), C + h * HS, kt * kTile, b);
                    tma_load_3d(sV(kvs), &map_qkv, bar(kBarKVFull + kvs), 2 * C + h * HS, kt * kTile, b);
                    const int qt_end = band_hi_tile(kt, window, n_t);
                    for (int qt = kt; qt <= qt_end; ++qt, ++gq) {
                        const int st = gq % kQStages;
                        const uint32_t ph = (uint32_t)(gq / kQStages) & 1u;
                        if (gq >= kQStages && !(ok = mbar_wait(bar(kBarQEmpty + st), ph ^ 1u, g))) break;
                        const uint32_t fb = bar(kBarQFull + st);
                        mbar_arrive_expect_tx(fb, 2 * kTileBytes + 1024);
                        tma_load_3d(sQ(st), &map_qkv, fb, h * HS, qt * kTile, b);
                        tma_load_3d(sdO(st), &map_dy, fb, h * HS, qt * kTile, b);
                        const size_t rowoff = (size_t)bh * (size_t)T_pad + (size_t)qt * kTile;
                        bulk_load(sbase + kOffLse + st * 512, lse2 + rowoff, 512, fb);
                        bulk_load(sbase + kOffD + st * 512, Dvec + rowoff, 512, fb);
                    }
                }
                if (!ok || *abort_flag) {
                    // let the last copies of each buffer land before shared memory is released
                    for (int k = (n > kKVStages ? n - kKVStages : 0); k < n; ++k)
                        drain_wait(bar(kBarKVFull + (k & 1)), (uint32_t)(k >> 1) & 1u, budget_ns);
                    for (int k = (gq > kQStages ? gq - kQStages : 0); k < gq; ++k)
                        drain_wait(bar(kBarQFull + k % kQStages), (uint32_t)(k / kQStages) & 1u, budget_ns);
                }
            }
        } else if (warp == 1) {
            // ================================================================ MMA issuer
            if (lane == 0) {
                constexpr uint32_t idSS = idesc_bf16_f32(128, 128, false, false);
                constexpr uint32_t idAcc = idesc_bf16_f32(128, HS, false, true);
                constexpr uint32_t idQ = idesc_bf16_f32(128, HS, true, true);
                // Descriptors of every buffer, built once.  K-major views: rows of 128 B,
                // 8-row groups 1024 B apart.  N/M-major views: 8-row groups 1024 B apart,
                // 64-element column blocks one slab apart.  A k-step moves the start address.
                const uint64_t dK0 = sdesc_sw128(sK(0), 16, 1024), dV0 = sdesc_sw128(sV(0), 16, 1024);
                const uint64_t dQ0 = sdesc_sw128(sQ(0), 16, 1024), ddO0 = sdesc_sw128(sdO(0), 16, 1024);
                const uint64_t ddOmn0 = sdesc_sw128(sdO(0), kSlabBytes, 1024), dQmn0 = sdesc_sw128(sQ(0), kSlabBytes, 1024);
                const uint64_t dKmn0 = sdesc_sw128(sK(0), kSlabBytes, 1024);
                const uint64_t ddS = sdesc_sw128(sdS, 16, 1024), ddSmn = sdesc_sw128(sdS, kSlabBytes, 1024);
                auto at = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
                bool ok = true, any = false;
                int n = 0, gi = 0;
                int qst = 0;        // gi % kQStages, kept incrementally (no divisions on this thread)
                uint32_t qpar = 0;  // (gi / kQStages) & 1
                auto issue_S = [&](int kvs, int st) {
                    const uint64_t a = at(dK0, kvs * kTileBytes), b = at(dQ0, st * kTileBytes);
    #pragma unroll
                    for (int kk = 0; kk < HS / 16; ++kk)
                        umma_ss(tmem + kColS, at(a, kk * 32u), at(b, kk * 32u), idSS, kk > 0 ? 1u : 0u);
                    umma_commit(bar(kBarSFull));
                };
                auto issue_dP = [&](int kvs, int st) {
                    const uint64_t a = at(dV0, kvs * kTileBytes), b = at(ddO0, st * kTileBytes);
    #pragma unroll
                    for (int kk = 0; kk < HS / 16; ++kk)
                        umma_ss(tmem + kColdP, at(a, kk * 32u), at(b, kk * 32u), idSS, kk > 0 ? 1u : 0u);
                    umma_commit(bar(kBardPFull));
                };
                for (int k = 0; ok; ++k, ++n) {
                    const int w = item_index(k, blockIdx.x, gridDim.x);
                    if (w >= n_items) break;
                    const int kt = w / BH;
                    const int niter = band_hi_tile(kt, window, n_t) - kt + 1;
                    const int kvs = n & 1;
                    if (!(ok = mbar_wait(bar(kBarKVFull + kvs), (uint32_t)(n >> 1) & 1u, g))) break;
                    // first S and dP of this item
                    if (!(ok = mbar_wait(bar(kBarQFull + qst), qpar, g))) break;
                    if (gi > 0 && !(ok = mbar_wait(bar(kBarSEmpty), (uint32_t)(gi - 1) & 1u, g))) break;
                    tc_fence_after();
                    issue_S(kvs, qst);
                    any = true;
                    if (gi > 0 && !(ok = mbar_wait(bar(kBardPEmpty), (uint32_t)(gi - 1) & 1u, g))) break;
                    tc_fence_after();
                    issue_dP(kvs, qst);
                    for (int it = 0; it < niter; ++it, ++gi) {
                        const int st = qst;
                        const int st1 = qst == kQStages - 1 ? 0 : qst + 1;
                        const uint32_t qpar1 = qst == kQStages - 1 ? qpar ^ 1u : qpar;  // parity of tile gi + 1
                        const bool more = it + 1 < niter;
                        const uint32_t ph = (uint32_t)gi & 1u;
                        // The barriers this tile waits on have usually completed by the time this
                        // thread reaches them (it is the one that falls behind: it shares its
                        // sub-partition's issue slots with three busy warps, and every dependent
                        // round trip costs it hundreds of cycles).  So all of them are tested at
                        // once, and a blocking wait runs only for one that was still open.  A
                        // completed phase stays completed until this thread's own later MMAs let
                        // the next phase complete, so a set bit cannot go stale.
                        const uint32_t r1 = mbar_test4(bar(kBarQFull + st1), qpar1, bar(kBarSEmpty), ph, bar(kBarPFull),
                                                       ph, bar(kBardPEmpty), ph);
                        if (more) {  // S^T of the next query tile
                            if (!(r1 & 1u) && !(ok = mbar_wait(bar(kBarQFull + st1), qpar1, g))) break;
                            if (!(r1 & 2u) && !(ok = mbar_wait(bar(kBarSEmpty), ph, g))) break;
                            tc_fence_after();
                            issue_S(kvs, st1);
                        }
                        // dV += P^T dO
                        if (!(r1 & 4u) && !(ok = mbar_wait(bar(kBarPFull), ph, g))) break;
                        if (it == 0 && n > 0 && !(ok = mbar_wait(bar(kBarAccFree), (uint32_t)(n - 1) & 1u, g))) break;
                        tc_fence_after();
                        {
                            const uint64_t b = at(ddOmn0, st * kTileBytes);
                            const uint32_t acc = it > 0 ? 1u : 0u;
    #pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                umma_ts(tmem + kColdV, tmem + kColP + 8u * kk, at(b, kk * 2048u), idAcc, kk > 0 ? 1u : acc);
                        }
                        umma_commit(bar(kBarPEmpty));
                        // this issuer's reads of Q_i and dO_i (S_i, dP_i, dV_i) are done
                        if constexpr (!kDropout) umma_commit(bar(kBarQEmpty + st));
                        // dP^T of the next query tile, ahead of this tile's dK and dQ (which wait for
                        // this tile's dS), so the softmax warps find it ready when they reach it
                        if (more) {
                            if (!(r1 & 8u) && !(ok = mbar_wait(bar(kBardPEmpty), ph, g))) break;
                            tc_fence_after();
                            issue_dP(kvs, st1);
                        }
                        if constexpr (!kDropout) {
                            qst = st1;
                            qpar = qpar1;
                            continue;  // dK and dQ come from the second issuer
                        }
                        // dK += dS^T Q ; dQ = dS K  (gi = 0 tests the phase before the first, which
                        // counts as complete)
                        const uint32_t r2 = mbar_test4(bar(kBardSFull), ph, bar(kBardQEmpty), (uint32_t)(gi - 1) & 1u,
                                                       bar(kBardSFull), ph, bar(kBardSFull), ph);
                        if (!(r2 & 1u) && !(ok = mbar_wait(bar(kBardSFull), ph, g))) break;
                        tc_fence_after();
                        {
                            const uint64_t b = at(dQmn0, st * kTileBytes);
                            const uint32_t acc = it > 0 ? 1u : 0u;
    #pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                umma_ss(tmem + kColdK, at(ddS, (kk >> 2) * kSlabBytes + (kk & 3) * 32u), at(b, kk * 2048u),
                                        idAcc, kk > 0 ? 1u : acc);
                        }
                        // dK was the last reader of Q_i and dO_i (dQ reads dS and K): release their stage
                        umma_commit(bar(kBarQEmpty + st));
                        if (gi > 0 && !(r2 & 2u) && !(ok = mbar_wait(bar(kBardQEmpty), (uint32_t)(gi - 1) & 1u, g)))
                            break;
                        tc_fence_after();
                        {
                            const uint64_t b = at(dKmn0, kvs * kTileBytes);
    #pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                umma_ss(tmem + kColdQ, at(ddSmn, kk * 2048u), at(b, kk * 2048u), idQ, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(bar(kBardQFull));  // dQ_i retired, and dK_i before it: dS free
                        qst = st1;
                        qpar = qpar1;
                    }
                    if (!ok) break;
                    umma_commit(bar(kBarKdV));
                    umma_commit(bar(kBarKVEmpty + kvs));
                }
                if (any) {
                    umma_commit(bar(kBarDone));
                    drain_wait(bar(kBarDone), 0, budget_ns);
                }
            }
        } else {
            if constexpr (!kDropout) {
                // ================================================================ second MMA issuer (warp 2)
                if (warp == 2 && lane == 0) {
                    constexpr uint32_t idAcc = idesc_bf16_f32(128, HS, false, true);
                    constexpr uint32_t idQ = idesc_bf16_f32(128, HS, true, true);
                    const uint64_t dQmn0 = sdesc_sw128(sQ(0), kSlabBytes, 1024);
                    const uint64_t dKmn0 = sdesc_sw128(sK(0), kSlabBytes, 1024);
                    const uint64_t ddS = sdesc_sw128(sdS, 16, 1024), ddSmn = sdesc_sw128(sdS, kSlabBytes, 1024);
                    auto at = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (uint64_t)(bytes >> 4); };
                    bool ok = true, any = false;
                    int n = 0, gi = 0, qst = 0;
                    uint32_t qpar = 0;
                    for (int k = 0; ok; ++k, ++n) {
                        const int w = item_index(k, blockIdx.x, gridDim.x);
                        if (w >= n_items) break;
                        const int kt = w / BH;
                        const int niter = band_hi_tile(kt, window, n_t) - kt + 1;
                        const int kvs = n & 1;
                        if (!(ok = mbar_wait(bar(kBarKVFull + kvs), (uint32_t)(n >> 1) & 1u, g))) break;
                        for (int it = 0; it < niter; ++it, ++gi) {
                            const int st = qst;
                            const uint32_t ph = (uint32_t)gi & 1u;
                            // one batch of tests, a blocking wait only for a phase still open; none of
                            // these phases can be overtaken before this thread's own later commits
                            // (gi = 0 / n = 0 test the phase before the first, which counts as complete)
                            const uint32_t r = mbar_test4(bar(kBardSFull), ph, bar(kBardQEmpty), (uint32_t)(gi - 1) & 1u,
                                                          bar(kBarQFull + st), qpar, bar(kBarAccFree),
                                                          (uint32_t)(n - 1) & 1u);
                            if (!(r & 4u) && !(ok = mbar_wait(bar(kBarQFull + st), qpar, g))) break;
                            if (!(r & 1u) && !(ok = mbar_wait(bar(kBardSFull), ph, g))) break;
                            if (it == 0 && n > 0 && !(r & 8u) &&
                                !(ok = mbar_wait(bar(kBarAccFree), (uint32_t)(n - 1) & 1u, g)))
                                break;
                            tc_fence_after();
                            any = true;
                            {  // dK += dS^T Q
                                const uint64_t b = at(dQmn0, st * kTileBytes);
                                const uint32_t acc = it > 0 ? 1u : 0u;
    #pragma unroll
                                for (int kk = 0; kk < 8; ++kk)
                                    umma_ss(tmem + kColdK, at(ddS, (kk >> 2) * kSlabBytes + (kk & 3) * 32u),
                                            at(b, kk * 2048u), idAcc, kk > 0 ? 1u : acc);
                            }
                            umma_commit(bar(kBarQEmpty + st));  // this issuer's read of Q_i is done
                            if (gi > 0 && !(r & 2u) &&
                                !(ok = mbar_wait(bar(kBardQEmpty), (uint32_t)(gi - 1) & 1u, g)))
                                break;
                            tc_fence_after();
                            {  // dQ = dS K
                                const uint64_t b = at(dKmn0, kvs * kTileBytes);
    #pragma unroll
                                for (int kk = 0; kk < 8; ++kk)
                                    umma_ss(tmem + kColdQ, at(ddSmn, kk * 2048u), at(b, kk * 2048u), idQ,
                                            kk > 0 ? 1u : 0u);
                            }
                            umma_commit(bar(kBardQFull));  // dQ_i retired, and dK_i before it: dS free
                            qst = qst == kQStages - 1 ? 0 : qst + 1;
                            qpar = qst == 0 ? qpar ^ 1u : qpar;
                        }
                        if (!ok) break;
                        umma_commit(bar(kBarKdV));
                        umma_commit(bar(kBarKVEmpty + kvs));
                    }
                    if (any) {
                        umma_commit(bar(kBarDoneB));
                        drain_wait(bar(kBarDoneB), 0, budget_ns);
                    }
                }
            }
            // ================================================================ dropout mask (warps 2, 3)
            if constexpr (kDropout) {
                // thread -> key rows 4*kg .. 4*kg+3 and query columns 64*qh .. 64*qh+63 of every
                // mask tile, tiles in the order the softmax warps use them
                const int u = threadIdx.x - 64;
                const int kg = u >> 1, qh = u & 1;
                const uint32_t t7 = theta_low7(dp.threshold);
                bool ok = true;
                int gi = 0;
                for (int k = 0; ok; ++k) {
                    const int w = item_index(k, blockIdx.x, gridDim.x);
                    if (w >= n_items) break;
                    const int kt = w / BH, bh = w % BH;
                    const int niter = band_hi_tile(kt, window, n_t) - kt + 1;
                    for (int it = 0; it < niter; ++it, ++gi) {
                        const int ms = gi % kMStages;
                        if (gi >= kMStages &&
                            !(ok = warp_wait(bar(kBarMEmpty + ms), (uint32_t)((gi / kMStages) & 1) ^ 1u, g)))
                            break;
                        const uint32_t s0 = (uint32_t)(kt * kTile + 4 * kg);
                        const uint32_t t0 = (uint32_t)((kt + it) * kTile + 64 * qh);
                        uint32_t lo[4], hi[4];
                        if (dp.threshold >= 128u) {
                            dropout_keep32x4_keys<true>(dp.seed, t7, (uint32_t)bh, s0, t0, lo);
                            dropout_keep32x4_keys<true>(dp.seed, t7, (uint32_t)bh, s0, t0 + 32u, hi);
                        } else {
                            dropout_keep32x4_keys<false>(dp.seed, t7, (uint32_t)bh, s0, t0, lo);
                            dropout_keep32x4_keys<false>(dp.seed, t7, (uint32_t)bh, s0, t0 + 32u, hi);
                        }
                        const uint32_t dst = sM(ms) + (uint32_t)(4 * kg) * 16u + (uint32_t)qh * 8u;
#pragma unroll
                        for (int c = 0; c < 4; ++c) st_shared_v2(dst + (uint32_t)c * 16u, lo[c], hi[c]);
                        mbar_arrive(bar(kBarMFull + ms));
                    }
                }
            }
        }
    } else if (wg < 3) {
        regs_inc<kRegsSoftmax>();
        // ================================================================ softmax warps
        const int sp = warp & 3;                 // TMEM sub-partition: key rows 32*sp .. 32*sp+31
        const int half = wg - 1;                 // query columns 64*half .. 64*half+63
        const int row = sp * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(sp * 32) << 16);
        const float scale_log2 = 0.125f * 1.4426950408889634f;
        const uint64_t c2 = f32x2_pack(scale_log2, scale_log2);
        bool ok = true;
        int n = 0, gi = 0;
        for (int k = 0;; ++k, ++n) {
            const int w = item_index(k, blockIdx.x, gridDim.x);
            if (w >= n_items) break;
            const int kt = w / BH;
            const int niter = band_hi_tile(kt, window, n_t) - kt + 1;
            for (int it = 0; it < niter; ++it, ++gi) {
                const int st = gi % kQStages;
                const uint32_t ph = (uint32_t)gi & 1u;
                uint32_t keepb[2] = {0xFFFFFFFFu, 0xFFFFFFFFu};  // dropout keep bits of the 64 columns
                if constexpr (kDropout) {
                    const int ms = gi % kMStages;
                    if (ok) ok = warp_wait(bar(kBarMFull + ms), (uint32_t)(gi / kMStages) & 1u, g);
                    if (ok) {
                        const uint2 v = ld_shared_v2(sM(ms) + (uint32_t)row * 16u + (uint32_t)half * 8u);
                        keepb[0] = v.x;
                        keepb[1] = v.y;
                        mbar_arrive(bar(kBarMEmpty + ms));
                    }
                }
                if (ok) ok = warp_wait(bar(kBarQFull + st), (uint32_t)(gi / kQStages) & 1u, g);
                if (ok) ok = warp_wait(bar(kBarSFull), ph, g);
                float pf[64];  // P^T row segment, fp32
                if (ok) {
                    tc_fence_after();
                    uint32_t sr[64];
                    tmem_ld_x32_nowait(trow + kColS + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                    tmem_ld_x32_nowait(trow + kColS + 64 * half + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                    tmem_ld_wait_32(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                    tmem_ld_wait_32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                    tc_fence_before();
                    mbar_arrive(bar(kBarSEmpty));
                    const float4 *lse4 = reinterpret_cast<const float4 *>(sLse + st * 128 + 64 * half);
#pragma unroll
                    for (int c4 = 0; c4 < 16; ++c4) {
                        const float4 l = lse4[c4];
                        const int c = 4 * c4;
                        const uint64_t x01 = ffma2(f32x2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), c2,
                                                   f32x2_pack(l.x, l.y));
                        const uint64_t x23 = ffma2(f32x2_pack(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3])),
                                                   c2, f32x2_pack(l.z, l.w));
                        float x0, x1, x2, x3;
                        f32x2_unpack(x01, x0, x1);
                        f32x2_unpack(x23, x2, x3);
                        if ((c4 & 3) == 3) {  // a quarter of the exponentials on the FMA pipe
                            exp2_poly_x2(x0, x1, pf[c], pf[c + 1]);
                            exp2_poly_x2(x2, x3, pf[c + 2], pf[c + 3]);
                        } else {
                            pf[c] = ex2_approx(x0);
                            pf[c + 1] = ex2_approx(x1);
                            pf[c + 2] = ex2_approx(x2);
                            pf[c + 3] = ex2_approx(x3);
                        }
                    }
                    if (it == 0) {  // diagonal tile: query column q sees key `row` only if row <= q
#pragma unroll
                        for (int c = 0; c < 64; ++c)
                            if (64 * half + c < row) pf[c] = 0.f;
                    }
                    if (it * kTile + kTile - 1 >= window) {  // band's far edge: t sees s only if t - s < window
                        const int cut = window + row - it * kTile - 64 * half;  // columns c >= cut are masked
#pragma unroll
                        for (int c = 0; c < 64; ++c)
                            if (c >= cut) pf[c] = 0.f;
                    }
                    uint32_t pk[32];
                    if constexpr (kDropout) {  // P^T dropped with this row's 64 keep bits (already scaled)
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int cc = (2 * c) & 31;
                            pk[c] = pack_bf16x2(pf[2 * c], pf[2 * c + 1]) &
                                    keep_pair_mask(keepb[(2 * c) >> 5] << (cc >> 2), (cc >> 1) & 1);
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(pf[2 * c], pf[2 * c + 1]);
                    }
                    if (gi > 0) ok = warp_wait(bar(kBarPEmpty), (uint32_t)(gi - 1) & 1u, g);
                    if (ok) {
                        tmem_st_x32(trow + kColP + 32 * half, pk);
                        tmem_st_wait();
                        tc_fence_before();
                        mbar_arrive(bar(kBarPFull));
                    }
                }
                if (ok) ok = warp_wait(bar(kBardPFull), ph, g);
                if (ok && gi > 0) ok = warp_wait(bar(kBardQFull), (uint32_t)(gi - 1) & 1u, g);  // dS buffer free
                if (ok) {
                    tc_fence_after();
                    const float4 *D4 = reinterpret_cast<const float4 *>(sD + st * 128 + 64 * half);
                    // dS^T row `row`, query columns [64*half, 64*half+64) = slab `half`, chunks 0..7
                    const uint32_t rbase = sdS + (uint32_t)half * kSlabBytes + (uint32_t)row * 128u;
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
                        uint32_t dr[32];
                        tmem_ld_x32(trow + kColdP + 64 * half + 32 * part, dr);
                        if (part == 1) {
                            tc_fence_before();
                            mbar_arrive(bar(kBardPEmpty));
                        }
                        // dS^T = P^T o (dP^T o f - D), f the dropout factor (1 without dropout); with
                        // dropout the preprocess folded f's scale into lse and D, so pf holds P^T * scale
                        // and D / scale arrives here: dS^T = pf o (dP^T o keep - D / scale)
                        auto ds_chunk = [&](auto drop_tag) {
                            constexpr bool kDrop = decltype(drop_tag)::value;
#pragma unroll
                            for (int qq = 0; qq < 4; ++qq) {
                                const int q = 4 * part + qq;  // 16-byte chunk = 8 query columns
                                uint32_t wv[4];
#pragma unroll
                                for (int e = 0; e < 2; ++e) {
                                    const float4 d = D4[2 * q + e];
                                    const int c = 8 * q + 4 * e;      // column within the half
                                    const int cr = 8 * qq + 4 * e;    // column within this dP chunk
                                    uint32_t g[4] = {dr[cr], dr[cr + 1], dr[cr + 2], dr[cr + 3]};
                                    if constexpr (kDrop) {  // dropped columns: dP^T o f = 0
                                        const uint32_t ws = keepb[c >> 5] << ((c & 31) >> 2);
#pragma unroll
                                        for (int kk = 0; kk < 4; ++kk) g[kk] &= keep_word_mask(ws, kk);
                                    }
                                    const uint64_t g01 = f32x2_pack(__uint_as_float(g[0]), __uint_as_float(g[1]));
                                    const uint64_t g23 = f32x2_pack(__uint_as_float(g[2]), __uint_as_float(g[3]));
                                    const uint64_t a01 = fadd2(g01, f32x2_pack(d.x, d.y));
                                    const uint64_t a23 = fadd2(g23, f32x2_pack(d.z, d.w));
                                    const uint64_t s01 = fmul2(a01, f32x2_pack(pf[c], pf[c + 1]));
                                    const uint64_t s23 = fmul2(a23, f32x2_pack(pf[c + 2], pf[c + 3]));
                                    float s0, s1, s2, s3;
                                    f32x2_unpack(s01, s0, s1);
                                    f32x2_unpack(s23, s2, s3);
                                    wv[2 * e] = pack_bf16x2(s0, s1);
                                    wv[2 * e + 1] = pack_bf16x2(s2, s3);
                                }
                                st_shared_v4(rbase + (((uint32_t)q ^ (uint32_t)(row & 7)) << 4), wv[0], wv[1], wv[2],
                                             wv[3]);
                            }
                        };
                        ds_chunk(std::integral_constant<bool, kDropout>{});
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(bar(kBardSFull));
                }
            }
        }
    } else {
        // ================================================================ dQ drain warps
        regs_inc<kRegsDrain>();
        const int sp = warp & 3;
        const int row = sp * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(sp * 32) << 16);
        const bool leader = (warp == 12 && lane == 0);
        bool ok = true;
        int gi = 0;
        // 32 words as row `row` of the staging slab (128-byte swizzled); the slab's previous
        // copy-out must have read it first
        auto stage = [&](const uint32_t *v) {
            if (leader) bulk_wait_group_read_0();
            named_bar_sync(2, kDrainThreads);
            if (ok) {
                const uint32_t rbase = sdQ + (uint32_t)row * 128u;
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    st_shared_v4(rbase + (((uint32_t)q ^ (uint32_t)(row & 7)) << 4), v[4 * q], v[4 * q + 1],
                                 v[4 * q + 2], v[4 * q + 3]);
                fence_proxy_async_smem();
            }
            named_bar_sync(2, kDrainThreads);
        };
        for (int k = 0, n = 0;; ++k, ++n) {
            const int w = item_index(k, blockIdx.x, gridDim.x);
            if (w >= n_items) break;
            const int kt = w / BH, bh = w % BH;
            const int qt_end = band_hi_tile(kt, window, n_t);
            for (int qt = kt; qt <= qt_end; ++qt, ++gi) {
                if (ok) ok = warp_wait(bar(kBardQFull), (uint32_t)gi & 1u, g);
                uint32_t v[64];
                if (ok) {
                    tc_fence_after();
                    tmem_ld_x32(trow + kColdQ, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
                    tmem_ld_x32(trow + kColdQ + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
                    tc_fence_before();
                    mbar_arrive(bar(kBardQEmpty));
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {  // two 32-column halves through one 16 KB staging slab
                    stage(&v[32 * hh]);
                    if (leader && ok && !*abort_flag) {
                        if (n_slots == 0)  // add into the (b, h, query tile) rows of the accumulator
                            tma_reduce_add_2d(&map_dq, sdQ, 32 * hh, bh * T_pad + qt * kTile);
                        else  // deterministic: a slot of its own per (query tile, key tile)
                            tma_store_2d(&map_dq, sdQ, 32 * hh, (bh * n_slots + qt * (qt + 1) / 2 + kt) * kTile);
                        bulk_commit_group();
                    }
                }
            }
            // ------------------------------------------------ dK / dV epilogue of this item
            // (here rather than on the softmax warps, which go straight on to the next item):
            // TMEM -> bf16 (dK scaled) -> the staging slab -> TMA store, dV then dK
            if (ok) ok = warp_wait(bar(kBarKdV), (uint32_t)n & 1u, g);
            const int b = bh / n_head, h = bh % n_head;
#pragma unroll
            for (int which = 0; which < 2; ++which) {  // dV, then dK (scaled)
                uint32_t pv[32];
                if (ok) {
                    tc_fence_after();
                    const float mul = which == 0 ? 1.f : 0.125f;
#pragma unroll
                    for (int part = 0; part < 2; ++part) {
                        uint32_t o[32];
                        tmem_ld_x32(trow + (which == 0 ? kColdV : kColdK) + 32 * part, o);
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            pv[16 * part + c] =
                                pack_bf16x2(__uint_as_float(o[2 * c]) * mul, __uint_as_float(o[2 * c + 1]) * mul);
                    }
                    if (which == 1) {
                        tc_fence_before();
                        mbar_arrive(bar(kBarAccFree));  // the next item's dV / dK may overwrite the accumulators
                    }
                }
                stage(pv);
                if (leader && ok && !*abort_flag) {
                    tma_store_3d(&map_dqkv, sdQ, (which == 0 ? 2 * C : C) + h * HS, kt * kTile, b);
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

}  // namespace

cudaError_t launch_bwd_main_h64(const CUtensorMap &map_qkv, const CUtensorMap &map_dy, const CUtensorMap &map_dqkv,
                                const CUtensorMap &map_dq, const float *lse2, const float *D, int B, int T, int C,
                                int n_head, int T_pad, int window, int n_slots, DropoutParams dp, DevCtx ctx,
                                cudaStream_t s) {
    const bool drop = dp.threshold != 0u;
    auto kern = drop ? bwd_h64_persistent<true> : bwd_h64_persistent<false>;
    const uint32_t smem = drop ? smem_bytes<true>() : smem_bytes<false>();
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // the warpgroups' register budgets add up to the launch allocation only at kLaunchRegs per
    // thread; otherwise a setmaxnreg.inc could never be satisfied, so refuse to launch
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int n_t = ceil_div(T, kTile);
    const long long items = (long long)n_t * B * n_head;
    const int grid = (int)(items < sms ? items : sms);
    return launch_pdl(kern, dim3((unsigned)grid), dim3(kThreads), smem, s, map_qkv, map_dy, map_dqkv,
                      map_dq, lse2, D, B, T, C, n_head, T_pad, n_t, window, n_slots, dp, ctx.status, ctx.budget_ns);
}

}  // namespace gptattn
