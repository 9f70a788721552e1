// kernels.h -- internal launch interface between the C-ABI layer (api.cu) and
// the kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "philox.cuh"

namespace gptattn {

// Per-launch device context: where a kernel records a timeout, and how long
// any single wait may last before it gives up.
struct DevCtx {
    int *status;
    unsigned long long budget_ns;
};

// Rows per tile along T used by the tensor-core kernels (queries and keys).
constexpr int kTile = 128;

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// The window the causal entry points pass: wider than any sequence, so no band
// edge ever falls inside a tile.
constexpr int kCausalWindow = 1 << 30;

// Launch with programmatic stream serialisation: the kernel's CTAs may start
// (and run their prologue) while the previous kernel of the stream finishes;
// every kernel launched this way calls griddep_wait() before touching global
// memory, so results are as with an ordinary launch.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

// ---- bf16 tensor-core path (sm_100a) --------------------------------------
// map_qkv: 3-D view (3C, T, B) of qkv, box (64, 128, 1), 128-byte swizzle.
// map_y:   3-D view (C, T, B) of y, same box.
// window: query t sees keys t-window < s <= t (kCausalWindow or any value >= T: causal);
// the head-size-128 kernels support the causal case only.
cudaError_t launch_fwd_bf16(int hs, const CUtensorMap &map_qkv, const CUtensorMap &map_y, float *lse,
                            int B, int T, int C, int n_head, int window, DropoutParams dp, DevCtx ctx,
                            cudaStream_t s);

// Head-size-64 forward with separate P buffers (same arguments as above).
cudaError_t launch_fwd_h64(const CUtensorMap &map_qkv, const CUtensorMap &map_y, float *lse, int B, int T, int C,
                           int n_head, int window, DropoutParams dp, DevCtx ctx, cudaStream_t s);

// D[bh][t] = -d_mul * sum_d y*dy, lse2[bh][t] = -lse*log2(e) + lse_bias (rows t >= T: 0 and
// -inf), dqacc zeroed.  Row stride of D/lse2 is T_pad; dqacc is [B*n_head*T_pad][hs].  Without
// dropout lse_bias = 0 and d_mul = 1; with dropout scale s, log2(s) and 1/s.
cudaError_t launch_bwd_pre_bf16(int hs, const void *y, const void *dy, const float *lse, float *D, float *lse2,
                                float *dqacc, int B, int T, int C, int n_head, int T_pad, bool zero_acc, float lse_bias,
                                float d_mul, cudaStream_t s);

// map_dy: 3-D view (C, T, B) of dy; map_dqkv: 3-D view (3C, T, B) of dqkv;
// map_dq: 2-D view (hs, B*n_head*T_pad) of dqacc (fp32), box (32, 128), 128-byte swizzle.
cudaError_t launch_bwd_main_bf16(int hs, const CUtensorMap &map_qkv, const CUtensorMap &map_dy,
                                 const CUtensorMap &map_dqkv, const CUtensorMap &map_dq, const float *lse2,
                                 const float *D, int B, int T, int C, int n_head, int T_pad, int window, int n_slots,
                                 DropoutParams dp, DevCtx ctx, cudaStream_t s);

// Persistent head-size-64 variant of the above (same arguments).
cudaError_t launch_bwd_main_h64(const CUtensorMap &map_qkv, const CUtensorMap &map_dy, const CUtensorMap &map_dqkv,
                                const CUtensorMap &map_dq, const float *lse2, const float *D, int B, int T, int C,
                                int n_head, int T_pad, int window, int n_slots, DropoutParams dp, DevCtx ctx,
                                cudaStream_t s);

// dqkv[b][t][h*hs+d] = bf16(dqacc[(b*n_head+h)*T_pad + t][d] / sqrt(hs)).
cudaError_t launch_bwd_post_bf16(int hs, const float *dqacc, void *dqkv, int B, int T, int C, int n_head,
                                 int T_pad, cudaStream_t s);

// Deterministic mode: n_slots = n_t(n_t+1)/2 partial dQ tiles per (b, h), the partial of
// (query tile i, key tile j) in rows (bh*n_slots + i(i+1)/2 + j)*128 of `part` ([rows][hs]
// fp32); the postprocess sums a query tile's partials in increasing j (head size 64).
cudaError_t launch_bwd_post_det_bf16(int hs, const float *part, void *dqkv, int B, int T, int C, int n_head, int T_pad,
                                     int n_slots, int window, cudaStream_t s);

// ---- fp32 CUDA-core path --------------------------------------------------
cudaError_t launch_fwd_f32(int hs, const float *qkv, float *y, float *lse, int B, int T, int C, int n_head, int window,
                           DropoutParams dp, cudaStream_t s);
cudaError_t launch_bwd_f32_pre(int hs, const float *y, const float *dy, float *D, int B, int T, int C,
                               int n_head, cudaStream_t s);
cudaError_t launch_bwd_f32_dq(int hs, const float *qkv, const float *dy, const float *lse, const float *D,
                              float *dqkv, int B, int T, int C, int n_head, int window, DropoutParams dp,
                              cudaStream_t s);
cudaError_t launch_bwd_f32_dkv(int hs, const float *qkv, const float *dy, const float *lse, const float *D,
                               float *dqkv, int B, int T, int C, int n_head, int window, DropoutParams dp,
                               cudaStream_t s);

// ---- decode: last position over a key/value cache (cluster of 8 CTAs per (b, h))
cudaError_t launch_decode(int hs, bool bf16, const void *qkv, void *y, float *lse, int B, int T, int T_cap, int C,
                          int n_head, cudaStream_t s);

// ---- the attention sub-block's neighbours (bf16): LayerNorm and the two linear maps
// out[M][N] = a[M][K] w[N][K]^T + bias[N] (+ resid[M][N]); bias and resid may be null.
// map_a: 2-D (K, M) view of a, box (64, 128); map_w: 2-D (K, N) view of w, box (64, tile_n);
// map_c: 2-D (N, M) view of out, box (64, 128); all 128-byte swizzle.  N % 64 == K % 64 == 0.
// tile_n (128 or 256) is the output tile width gemm_tile_n() picks for the shape.
int gemm_tile_n(int M, int N);
cudaError_t launch_gemm_bf16(const CUtensorMap &map_a, const CUtensorMap &map_w, const CUtensorMap &map_c,
                             const void *bias, const void *resid, int M, int N, int K, int tile_n, DevCtx ctx,
                             cudaStream_t s);
// out[M][C] = (x - mean) / sqrt(var + 1e-5) * w + b per row (C % 8 == 0, C <= 4096).
cudaError_t launch_layernorm_bf16(const void *x, const void *w, const void *b, void *out, int M, int C,
                                  cudaStream_t s);

// ---- bounded-wait self-test -----------------------------------------------
cudaError_t launch_selftest_timeout(DevCtx ctx, cudaStream_t s);
// ---- the backward's FMA-pipe exponential on caller data ---------------------
cudaError_t launch_selftest_exp2(const float *x, float *y, int n, cudaStream_t s);

// Kernel identifiers for the instrumentation records.
enum KernelId {
    kKFwdBf16 = 0,
    kKBwdPreBf16 = 1,
    kKBwdMainBf16 = 2,
    kKBwdPostBf16 = 3,
    kKFwdF32 = 4,
    kKBwdPreF32 = 5,
    kKBwdDqF32 = 6,
    kKBwdDkvF32 = 7,
    kKSelftest = 8,
    kKDecode = 9,
    kKLayerNorm = 10,
    kKGemm = 11,
    kKNumKernels = 12
};

}  // namespace gptattn
