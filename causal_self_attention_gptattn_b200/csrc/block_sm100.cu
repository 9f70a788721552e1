// block_sm100.cu -- the matrix products around the attention core of a pre-LN
// GPT block's attention sub-block (lecture page "Let's build GPT: from scratch,
// in code, spelled out", chapters "residual connections" and "layernorm (and
// its relationship to our previous batchnorm)"; the projection back into the
// residual stream after "multi-headed self-attention"):
//     xn   = LayerNorm(x) * w_ln + b_ln          (over C, eps 1e-5)
//     qkv  = xn W_attn^T + b_attn                 (c_attn: C -> 3C)
//     y    = attention(qkv)                       (the library's forward)
//     out  = x + y W_proj^T + b_proj              (c_proj: C -> C, residual add)
// Weights are stored as nn.Linear does, [out_features][in_features] (rows K-major).
//
// gemm_kernel: persistent tcgen05 GEMM, C[M][N] = A[M][K] W[N][K]^T + bias (+ R),
// bf16 in and out, fp32 accumulation in TMEM.  128 x 256 output tiles (one
// M=128 N=256 MMA per 16-wide k step), A and W slices of 64 along K through a
// 4-stage TMA ring (128-byte swizzle), two TMEM accumulators so the epilogue of
// one tile overlaps the MMAs of the next.  Warps: 0 TMA producer, 1 TMEM owner
// + MMA issuer, 2..5 epilogue (one output row per thread): TMEM -> + bias
// (+ residual, read one chunk ahead and passed through the staging tile) ->
// bf16 -> swizzled staging -> TMA store, 64 columns at a time through two
// staging tiles.  Every wait is
// bounded.
#include <type_traits>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace gptattn {
namespace {

constexpr int kGThreads = 192;
constexpr int kBM = 128, kBK = 64;
constexpr uint32_t kABytes = kBM * kBK * 2;   // 16 KB
constexpr uint32_t kStgBytes = kBM * 64 * 2;  // one 128 x 64 bf16 chunk

// Tile width along N and ring depth: 128 x 256 tiles with 4 stages, or 128 x 128 tiles
// with 6 stages (same shared memory) when the wide tiles would leave fewer than three
// per CTA.
template <int BN, int STAGES>
struct GemmShape {
    static constexpr int kBN = BN, kGStages = STAGES;
    static constexpr uint32_t kBBytes = BN * kBK * 2;
    static constexpr uint32_t kOffA = 0;
    static constexpr uint32_t kOffB = kOffA + STAGES * kABytes;
    static constexpr uint32_t kOffStg = kOffB + STAGES * kBBytes;
    static constexpr uint32_t kOffGBar = kOffStg + 2 * kStgBytes;
    static constexpr int kGBarFull = 0, kGBarEmpty = kGBarFull + STAGES, kGBarAccFull = kGBarEmpty + STAGES,
                         kGBarAccEmpty = kGBarAccFull + 2, kGBarDone = kGBarAccEmpty + 2, kGNumBars = kGBarDone + 1;
    static constexpr uint32_t kGSmemBytes = kOffGBar + 256 + 1024;
    static constexpr uint32_t kTmemCols = 2 * BN;  // two accumulators
    static_assert(kGNumBars * 8 + 16 <= 256, "barrier area");
    static_assert(kGSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kTmemCols == 256 || kTmemCols == 512, "TMEM allocation");
};
using GemmWide = GemmShape<256, 4>;
using GemmNarrow = GemmShape<128, 6>;

__device__ __forceinline__ bool warp_wait_g(uint32_t bar, uint32_t parity, const WaitGuard &g) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, g));
}

template <bool kResidual, class Shape>
__global__ void __launch_bounds__(kGThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_w,
                const __grid_constant__ CUtensorMap map_c, const __nv_bfloat16 *__restrict__ bias,
                const __nv_bfloat16 *__restrict__ resid, int M, int N, int K, int *status,
                unsigned long long budget_ns) {
    constexpr int kBN = Shape::kBN, kGStages = Shape::kGStages;
    constexpr uint32_t kBBytes = Shape::kBBytes, kOffA = Shape::kOffA, kOffB = Shape::kOffB, kOffStg = Shape::kOffStg,
                       kOffGBar = Shape::kOffGBar, kTmemCols = Shape::kTmemCols;
    constexpr int kGBarFull = Shape::kGBarFull, kGBarEmpty = Shape::kGBarEmpty, kGBarAccFull = Shape::kGBarAccFull,
                  kGBarAccEmpty = Shape::kGBarAccEmpty, kGBarDone = Shape::kGBarDone, kGNumBars = Shape::kGNumBars;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_base & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffGBar);
    auto bar = [&](int i) -> uint32_t { return smem_u32(&bars[i]); };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffGBar + kGNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffGBar + kGNumBars * 8 + 4);
    const WaitGuard g{abort_flag, status, budget_ns};
    const int tiles_n = (N + kBN - 1) / kBN, tiles_m = (M + kBM - 1) / kBM;
    const int n_tiles = tiles_m * tiles_n, nk = K / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(bar(kGBarFull + s), 1);
            mbar_init(bar(kGBarEmpty + s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(bar(kGBarAccFull + a), 1);
            mbar_init(bar(kGBarAccEmpty + a), 128);
        }
        mbar_init(bar(kGBarDone), 1);
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
    griddep_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_map(&map_a);
            tma_prefetch_map(&map_w);
            bool ok = true;
            int kc = 0;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
                const int tm = t / tiles_n, tn = t % tiles_n;
                for (int ks = 0; ks < nk; ++ks, ++kc) {
                    const int st = kc % kGStages;
                    if (kc >= kGStages &&
                        !(ok = mbar_wait(bar(kGBarEmpty + st), (uint32_t)((kc / kGStages) & 1) ^ 1u, g)))
                        break;
                    mbar_arrive_expect_tx(bar(kGBarFull + st), kABytes + kBBytes);
                    tma_load_2d(sbase + kOffA + st * kABytes, &map_a, bar(kGBarFull + st), ks * kBK, tm * kBM);
                    tma_load_2d(sbase + kOffB + st * kBBytes, &map_w, bar(kGBarFull + st), ks * kBK, tn * kBN);
                }
            }
            if (!ok || *abort_flag)
                for (int q = (kc > kGStages ? kc - kGStages : 0); q < kc; ++q) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar(kGBarFull + q % kGStages), (uint32_t)(q / kGStages) & 1u))
                        if (global_timer_ns() - t0 > budget_ns) break;
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, false, false);
            bool ok = true, any = false;
            int kc = 0, tc = 0;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++tc) {
                const int acc = tc & 1;
                if (tc >= 2 && !(ok = mbar_wait(bar(kGBarAccEmpty + acc), (uint32_t)((tc >> 1) - 1) & 1u, g))) break;
                tc_fence_after();
                for (int ks = 0; ks < nk; ++ks, ++kc) {
                    const int st = kc % kGStages;
                    if (!(ok = mbar_wait(bar(kGBarFull + st), (uint32_t)(kc / kGStages) & 1u, g))) break;
                    tc_fence_after();
                    const uint64_t da = sdesc_sw128(sbase + kOffA + st * kABytes, 16, 1024);
                    const uint64_t db = sdesc_sw128(sbase + kOffB + st * kBBytes, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        umma_ss(tmem + (uint32_t)(acc * kBN), da + (uint64_t)(kk * 2), db + (uint64_t)(kk * 2), idesc,
                                (ks > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(bar(kGBarEmpty + st));
                    any = true;
                }
                if (!ok) break;
                umma_commit(bar(kGBarAccFull + acc));
            }
            if (any) {
                umma_commit(bar(kGBarDone));
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(bar(kGBarDone), 0))
                    if (global_timer_ns() - t0 > budget_ns) break;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2..5)
        const int sp = warp & 3;
        const int row = sp * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(sp * 32) << 16);
        const bool leader = (warp == 2 && lane == 0);
        bool ok = true;
        int tc = 0, cc = 0;
        // Residual chunks are read one chunk ahead and cooperatively: lane l of the warp holds
        // 16 bytes of row sp*32 + 4i + l/8 (i = 0..7), columns 8*(l%8) .. +7 of the chunk, so
        // each load instruction covers four whole 128-byte row segments.
        const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
        auto chunks_of = [&](int tt) {
            const int rem = N - (tt % tiles_n) * kBN;
            return rem < kBN ? rem / 64 : kBN / 64;
        };
        auto load_resid = [&](int tt, int c, uint4(&dst)[8]) {
            const bool valid = tt < n_tiles;
            const int n0r = (tt % tiles_n) * kBN + c * 64;
            const int r0 = (tt / tiles_n) * kBM + sp * 32 + (lane >> 3);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = r0 + 4 * i;
                dst[i] = (valid && r < M)
                             ? *reinterpret_cast<const uint4 *>(resid + (size_t)r * N + n0r + 8 * (lane & 7))
                             : zero4;
            }
        };
        uint4 rnext[8];
        if constexpr (kResidual) load_resid(blockIdx.x, 0, rnext);
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tc) {
            const int tm = t / tiles_n, tn = t % tiles_n;
            const int acc = tc & 1;
            if (ok) ok = warp_wait_g(bar(kGBarAccFull + acc), (uint32_t)(tc >> 1) & 1u, g);
            if (ok) tc_fence_after();
            for (int ch = 0; ch < kBN / 64; ++ch, ++cc) {
                const int n0 = tn * kBN + ch * 64;
                if (n0 >= N) break;  // uniform over the 128 threads (N % 64 == 0)
                uint4 rcur[8];
                if constexpr (kResidual) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) rcur[i] = rnext[i];
                    const bool last = ch + 1 >= chunks_of(t);
                    load_resid(last ? t + (int)gridDim.x : t, last ? 0 : ch + 1, rnext);
                }
                uint32_t v[64];
                if (ok) {
                    tmem_ld_x32(trow + (uint32_t)(acc * kBN + ch * 64), *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
                    tmem_ld_x32(trow + (uint32_t)(acc * kBN + ch * 64 + 32), *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
                }
                if (ch == kBN / 64 - 1 || n0 + 64 >= N) {  // accumulator read out: the MMAs may reuse it
                    tc_fence_before();
                    mbar_arrive(bar(kGBarAccEmpty + acc));
                }
                // staging tile cc & 1 is free once the store issued two chunks ago has read it
                if (leader) bulk_wait_group_read_1();
                named_bar_sync(1, 128);
                const uint32_t stg = sbase + kOffStg + (uint32_t)(cc & 1) * kStgBytes;
                if (ok) {
                    const uint32_t rbase = stg + (uint32_t)row * 128u;
                    if constexpr (kResidual) {  // the warp's 32 residual rows into its rows of the staging tile
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const uint32_t rr = (uint32_t)(sp * 32 + 4 * i + (lane >> 3));
                            st_shared_v4(stg + rr * 128u + ((((uint32_t)lane & 7u) ^ (rr & 7u)) << 4), rcur[i].x,
                                         rcur[i].y, rcur[i].z, rcur[i].w);
                        }
                        __syncwarp();
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q) {  // 8 columns per 16-byte chunk
                        const uint4 bq = bias ? *reinterpret_cast<const uint4 *>(bias + n0 + 8 * q)
                                              : make_uint4(0u, 0u, 0u, 0u);
                        const uint32_t bw[4] = {bq.x, bq.y, bq.z, bq.w};
                        uint32_t rw[4] = {0u, 0u, 0u, 0u};
                        if constexpr (kResidual) {
                            const uint4 r4 = ld_shared_v4(rbase + (((uint32_t)q ^ (uint32_t)(row & 7)) << 4));
                            rw[0] = r4.x;
                            rw[1] = r4.y;
                            rw[2] = r4.z;
                            rw[3] = r4.w;
                        }
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float lo = __uint_as_float(v[8 * q + 2 * e]) + bf16lo_to_f32(bw[e]);
                            float hi = __uint_as_float(v[8 * q + 2 * e + 1]) + bf16hi_to_f32(bw[e]);
                            if constexpr (kResidual) {
                                lo += bf16lo_to_f32(rw[e]);
                                hi += bf16hi_to_f32(rw[e]);
                            }
                            o[e] = pack_bf16x2(lo, hi);
                        }
                        st_shared_v4(rbase + (((uint32_t)q ^ (uint32_t)(row & 7)) << 4), o[0], o[1], o[2], o[3]);
                    }
                    fence_proxy_async_smem();
                }
                named_bar_sync(1, 128);
                if (leader && ok && !*abort_flag) {
                    tma_store_2d(&map_c, stg, n0, tm * kBM);
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

// xn = (x - mean) / sqrt(var + eps) * w + b per row of C, fp32 statistics; one warp per row,
// the row held in registers (kLnMaxPerLane uint4 of 8 bf16 per lane: C <= 256 * kLnMaxPerLane).
template <int kLnMaxPerLane>
__global__ void __launch_bounds__(256) layernorm_kernel(const __nv_bfloat16 *__restrict__ x,
                                                        const __nv_bfloat16 *__restrict__ w,
                                                        const __nv_bfloat16 *__restrict__ b,
                                                        __nv_bfloat16 *__restrict__ out, int M, int C) {
    griddep_launch_dependents();
    griddep_wait();
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (row >= M) return;
    const int n8 = C / 8;
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + (size_t)row * C);
    uint4 buf[kLnMaxPerLane];
    // bf16 pair -> the two floats, packed for the paired fp32 instructions
    auto pair = [](uint32_t u) { return f32x2_pack(bf16lo_to_f32(u), bf16hi_to_f32(u)); };
    uint64_t sum2 = f32x2_pack(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kLnMaxPerLane; ++k) {
        const int i = lane + 32 * k;
        buf[k] = i < n8 ? xr[i] : make_uint4(0u, 0u, 0u, 0u);
        sum2 = fadd2(sum2, fadd2(fadd2(pair(buf[k].x), pair(buf[k].y)), fadd2(pair(buf[k].z), pair(buf[k].w))));
    }
    float s0, s1;
    f32x2_unpack(sum2, s0, s1);
    float sum = s0 + s1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float mean = sum / (float)C;
    const uint64_t negmean2 = f32x2_pack(-mean, -mean);
    uint64_t sq2 = f32x2_pack(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kLnMaxPerLane; ++k) {
        if (lane + 32 * k >= n8) continue;
        const uint32_t u[4] = {buf[k].x, buf[k].y, buf[k].z, buf[k].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint64_t d = fadd2(pair(u[e]), negmean2);
            sq2 = ffma2(d, d, sq2);
        }
    }
    f32x2_unpack(sq2, s0, s1);
    float sq = s0 + s1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    const float rstd = rsqrtf(sq / (float)C + 1e-5f);
    const uint64_t rstd2 = f32x2_pack(rstd, rstd);
    const uint4 *wr = reinterpret_cast<const uint4 *>(w), *br = reinterpret_cast<const uint4 *>(b);
    uint4 *orow = reinterpret_cast<uint4 *>(out + (size_t)row * C);
#pragma unroll
    for (int k = 0; k < kLnMaxPerLane; ++k) {
        const int i = lane + 32 * k;
        if (i >= n8) continue;
        const uint4 wq = wr[i], bq = br[i];
        const uint32_t u[4] = {buf[k].x, buf[k].y, buf[k].z, buf[k].w};
        const uint32_t wu[4] = {wq.x, wq.y, wq.z, wq.w}, bu[4] = {bq.x, bq.y, bq.z, bq.w};
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            // (x - mean) * rstd * w + b as x * a + c with a = rstd * w, c = b - mean * a
            const uint64_t a = fmul2(rstd2, pair(wu[e]));
            const uint64_t c = ffma2(negmean2, a, pair(bu[e]));
            float lo, hi;
            f32x2_unpack(ffma2(pair(u[e]), a, c), lo, hi);
            o[e] = pack_bf16x2(lo, hi);
        }
        orow[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace

namespace {
int sm_count(int *sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? 0 : -1;
}

template <class Shape>
cudaError_t launch_gemm_shape(const CUtensorMap &map_a, const CUtensorMap &map_w, const CUtensorMap &map_c,
                              const void *bias, const void *resid, int M, int N, int K, int sms, DevCtx ctx,
                              cudaStream_t s) {
    auto kern = resid ? gemm_kernel<true, Shape> : gemm_kernel<false, Shape>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Shape::kGSmemBytes);
    if (e != cudaSuccess) return e;
    const long long tiles = (long long)((M + kBM - 1) / kBM) * ((N + Shape::kBN - 1) / Shape::kBN);
    const int grid = (int)(tiles < sms ? tiles : sms);
    return launch_pdl(kern, dim3((unsigned)grid), dim3(kGThreads), Shape::kGSmemBytes, s, map_a, map_w, map_c,
                      static_cast<const __nv_bfloat16 *>(bias), static_cast<const __nv_bfloat16 *>(resid), M, N, K,
                      ctx.status, ctx.budget_ns);
}
}  // namespace

int gemm_tile_n(int M, int N) {
    int sms = 148;
    if (sm_count(&sms) != 0 || sms <= 0) sms = 148;
    const long long wide = (long long)((M + kBM - 1) / kBM) * ((N + 255) / 256);
    return wide < 3LL * sms ? 128 : 256;
}

cudaError_t launch_gemm_bf16(const CUtensorMap &map_a, const CUtensorMap &map_w, const CUtensorMap &map_c,
                             const void *bias, const void *resid, int M, int N, int K, int tile_n, DevCtx ctx,
                             cudaStream_t s) {
    int sms = 0;
    if (sm_count(&sms) != 0) return cudaErrorInvalidDevice;
    if (tile_n == 256) return launch_gemm_shape<GemmWide>(map_a, map_w, map_c, bias, resid, M, N, K, sms, ctx, s);
    if (tile_n == 128) return launch_gemm_shape<GemmNarrow>(map_a, map_w, map_c, bias, resid, M, N, K, sms, ctx, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_layernorm_bf16(const void *x, const void *w, const void *b, void *out, int M, int C,
                                  cudaStream_t s) {
    const int per_lane = (C + 255) / 256;
    auto kern = per_lane <= 1   ? layernorm_kernel<1>
                : per_lane <= 2 ? layernorm_kernel<2>
                : per_lane <= 3 ? layernorm_kernel<3>
                : per_lane <= 4 ? layernorm_kernel<4>
                : per_lane <= 8 ? layernorm_kernel<8>
                                : layernorm_kernel<16>;
    return launch_pdl(kern, dim3((unsigned)((M + 7) / 8)), dim3(256), 0, s, static_cast<const __nv_bfloat16 *>(x),
                      static_cast<const __nv_bfloat16 *>(w), static_cast<const __nv_bfloat16 *>(b),
                      static_cast<__nv_bfloat16 *>(out), M, C);
}

}  // namespace gptattn
