// simt_f32.cu -- fp32 causal self-attention forward and backward on CUDA cores.
//
// Same function as the bf16 tensor-core path (lecture page "Let's build GPT:
// from scratch, in code, spelled out": "version 4: self-attention", causal
// mask per correction 00:57:00, 1/sqrt(head_size) per correction 01:20:05),
// kept in full fp32 (no TF32) for callers that need fp32 accuracy.  A local
// window (token t sees t-window < s <= t; minGPT README page, reference notes
// on GPT-3: locally banded attention) narrows every key or query range; the
// causal case passes window = T.  Every
// thread owns one query row (forward, dQ) or one key row (dK/dV); key or query
// rows are staged through shared memory in tiles of kRows.  Deterministic: no
// atomics.  Accurate expf/logf (no approximate intrinsics).
#include "kernels.h"
#include "philox.cuh"

namespace gptattn {
namespace {

// Dropout factor of the weight of query t for key s: 1 without dropout, else
// 1/(1 - theta/256) if the Philox mask keeps it and 0 if not.
__device__ __forceinline__ float drop_factor(const DropoutParams &dp, int bh, int t, int s) {
    if (dp.threshold == 0u) return 1.f;
    const uint32_t bits = dropout_keep4(dp.seed, dp.threshold, (uint32_t)bh, (uint32_t)t, (uint32_t)(s & ~3));
    return ((bits >> (s & 3)) & 1u) ? dp.scale : 0.f;
}

constexpr int kRows = 64;  // threads per block = rows per staged tile

template <int HS>
__device__ __forceinline__ float dot_row(const float *a, const float *b) {
    float acc = 0.f;
#pragma unroll
    for (int d = 0; d < HS; ++d) acc = fmaf(a[d], b[d], acc);
    return acc;
}

// y[b,t,h*HS+d] and lse[b,h,t] for query rows of one (b, h); the weights are
// dropped (and rescaled) in the weighted sum only, lse is the undropped one.
template <int HS>
__global__ void __launch_bounds__(kRows) fwd_f32_kernel(const float *__restrict__ qkv, float *__restrict__ y,
                                                        float *__restrict__ lse, int T, int C, int n_head, int window,
                                                        DropoutParams dp) {
    extern __shared__ float sm[];
    float *sk = sm;              // [kRows][HS]
    float *sv = sm + kRows * HS;  // [kRows][HS]
    const int bh = blockIdx.y;
    const int b = bh / n_head, h = bh % n_head;
    const int t = blockIdx.x * kRows + threadIdx.x;
    const size_t ld = (size_t)3 * C;
    const float *base = qkv + (size_t)b * T * ld + (size_t)h * HS;
    const float scale = 1.0f / sqrtf((float)HS);

    float q[HS], acc[HS];
    if (t < T) {
#pragma unroll
        for (int d = 0; d < HS; ++d) q[d] = base[(size_t)t * ld + d] * scale;
    }
#pragma unroll
    for (int d = 0; d < HS; ++d) acc[d] = 0.f;
    float m = -INFINITY, l = 0.f;

    const int last = min(T - 1, (int)(blockIdx.x * kRows + kRows - 1));  // largest query row of the block
    const int lo_t = max(0, t - window + 1);                              // first key this row sees
    const int lo_blk = max(0, (int)(blockIdx.x * kRows) - window + 1);    // first key any row of the block sees
    for (int s0 = lo_blk / kRows * kRows; s0 <= last; s0 += kRows) {
        __syncthreads();
        for (int e = threadIdx.x; e < kRows * HS; e += kRows) {
            const int r = e / HS, d = e % HS;
            const int s = s0 + r;
            sk[e] = s < T ? base[(size_t)s * ld + C + d] : 0.f;
            sv[e] = s < T ? base[(size_t)s * ld + 2 * C + d] : 0.f;
        }
        __syncthreads();
        if (t < T) {
            const int smax = min(kRows, t - s0 + 1);  // visible keys in this tile: lo_t <= s <= t
            for (int r = max(0, lo_t - s0); r < smax; ++r) {
                const float sc = dot_row<HS>(q, sk + r * HS);
                const float m_new = fmaxf(m, sc);
                const float corr = expf(m - m_new);
                const float p = expf(sc - m_new);
                l = l * corr + p;
                const float pd = p * drop_factor(dp, bh, t, s0 + r);
#pragma unroll
                for (int d = 0; d < HS; ++d) acc[d] = fmaf(acc[d], corr, pd * sv[r * HS + d]);
                m = m_new;
            }
        }
    }
    if (t < T) {
        const float inv = 1.f / l;
        float *yr = y + ((size_t)b * T + t) * (size_t)C + (size_t)h * HS;
#pragma unroll
        for (int d = 0; d < HS; ++d) yr[d] = acc[d] * inv;
        if (lse) lse[(size_t)bh * T + t] = m + logf(l);
    }
}

// D[b,h,t] = sum_d dy * y
template <int HS>
__global__ void bwd_f32_pre_kernel(const float *__restrict__ y, const float *__restrict__ dy, float *__restrict__ D,
                                   int B, int T, int C, int n_head) {
    const long long n = (long long)B * n_head * T;
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
         idx += (long long)gridDim.x * blockDim.x) {
        const int t = (int)(idx % T);
        const long long bh = idx / T;
        const int h = (int)(bh % n_head);
        const long long b = bh / n_head;
        const size_t off = ((size_t)b * T + t) * (size_t)C + (size_t)h * HS;
        float acc = 0.f;
#pragma unroll
        for (int d = 0; d < HS; ++d) acc = fmaf(y[off + d], dy[off + d], acc);
        D[idx] = acc;
    }
}

// dq[t] = scale * sum_{s<=t} P[t,s] (dy_t . v_s - D_t) k_s
template <int HS>
__global__ void __launch_bounds__(kRows) bwd_f32_dq_kernel(const float *__restrict__ qkv, const float *__restrict__ dy,
                                                           const float *__restrict__ lse, const float *__restrict__ D,
                                                           float *__restrict__ dqkv, int T, int C, int n_head,
                                                           int window, DropoutParams dp) {
    extern __shared__ float sm[];
    float *sk = sm;
    float *sv = sm + kRows * HS;
    const int bh = blockIdx.y;
    const int b = bh / n_head, h = bh % n_head;
    const int t = blockIdx.x * kRows + threadIdx.x;
    const size_t ld = (size_t)3 * C;
    const float *base = qkv + (size_t)b * T * ld + (size_t)h * HS;
    const float scale = 1.0f / sqrtf((float)HS);

    float q[HS], g[HS], acc[HS];
    float lse_t = 0.f, D_t = 0.f;
    if (t < T) {
        const float *gr = dy + ((size_t)b * T + t) * (size_t)C + (size_t)h * HS;
#pragma unroll
        for (int d = 0; d < HS; ++d) {
            q[d] = base[(size_t)t * ld + d] * scale;
            g[d] = gr[d];
        }
        lse_t = lse[(size_t)bh * T + t];
        D_t = D[(size_t)bh * T + t];
    }
#pragma unroll
    for (int d = 0; d < HS; ++d) acc[d] = 0.f;

    const int last = min(T - 1, (int)(blockIdx.x * kRows + kRows - 1));
    const int lo_t = max(0, t - window + 1);
    const int lo_blk = max(0, (int)(blockIdx.x * kRows) - window + 1);
    for (int s0 = lo_blk / kRows * kRows; s0 <= last; s0 += kRows) {
        __syncthreads();
        for (int e = threadIdx.x; e < kRows * HS; e += kRows) {
            const int r = e / HS, d = e % HS;
            const int s = s0 + r;
            sk[e] = s < T ? base[(size_t)s * ld + C + d] : 0.f;
            sv[e] = s < T ? base[(size_t)s * ld + 2 * C + d] : 0.f;
        }
        __syncthreads();
        if (t < T) {
            const int smax = min(kRows, t - s0 + 1);
            for (int r = max(0, lo_t - s0); r < smax; ++r) {
                const float p = expf(dot_row<HS>(q, sk + r * HS) - lse_t);
                const float ds = p * (dot_row<HS>(g, sv + r * HS) * drop_factor(dp, bh, t, s0 + r) - D_t);
#pragma unroll
                for (int d = 0; d < HS; ++d) acc[d] = fmaf(ds, sk[r * HS + d], acc[d]);
            }
        }
    }
    if (t < T) {
        float *out = dqkv + ((size_t)b * T + t) * ld + (size_t)h * HS;
#pragma unroll
        for (int d = 0; d < HS; ++d) out[d] = acc[d] * scale;
    }
}

// dv[s] = sum_{t>=s} P[t,s] dy_t ; dk[s] = scale * sum_{t>=s} P[t,s] (dy_t . v_s - D_t) q_t
template <int HS>
__global__ void __launch_bounds__(kRows) bwd_f32_dkv_kernel(const float *__restrict__ qkv, const float *__restrict__ dy,
                                                            const float *__restrict__ lse, const float *__restrict__ D,
                                                            float *__restrict__ dqkv, int T, int C, int n_head,
                                                            int window, DropoutParams dp) {
    extern __shared__ float sm[];
    float *sq = sm;                   // [kRows][HS] queries (pre-scaled)
    float *sg = sm + kRows * HS;      // [kRows][HS] dy rows
    float *sl = sm + 2 * kRows * HS;  // [kRows] lse
    float *sD = sl + kRows;           // [kRows] D
    const int bh = blockIdx.y;
    const int b = bh / n_head, h = bh % n_head;
    const int s = blockIdx.x * kRows + threadIdx.x;
    const size_t ld = (size_t)3 * C;
    const float *base = qkv + (size_t)b * T * ld + (size_t)h * HS;
    const float *gbase = dy + (size_t)b * T * (size_t)C + (size_t)h * HS;
    const float scale = 1.0f / sqrtf((float)HS);

    float k[HS], v[HS], dk[HS], dv[HS];
    if (s < T) {
#pragma unroll
        for (int d = 0; d < HS; ++d) {
            k[d] = base[(size_t)s * ld + C + d];
            v[d] = base[(size_t)s * ld + 2 * C + d];
        }
    }
#pragma unroll
    for (int d = 0; d < HS; ++d) dk[d] = dv[d] = 0.f;

    const int first = blockIdx.x * kRows;  // smallest key row of the block
    // last query that sees any key of the block: (largest key row) + window - 1
    const int t_end = min(T, (int)min((long long)first + kRows - 1 + window, (long long)T));
    for (int t0 = first; t0 < t_end; t0 += kRows) {
        __syncthreads();
        for (int e = threadIdx.x; e < kRows * HS; e += kRows) {
            const int r = e / HS, d = e % HS;
            const int t = t0 + r;
            sq[e] = t < T ? base[(size_t)t * ld + d] * scale : 0.f;
            sg[e] = t < T ? gbase[(size_t)t * C + d] : 0.f;
        }
        if (threadIdx.x < kRows) {
            const int t = t0 + threadIdx.x;
            sl[threadIdx.x] = t < T ? lse[(size_t)bh * T + t] : 0.f;
            sD[threadIdx.x] = t < T ? D[(size_t)bh * T + t] : 0.f;
        }
        __syncthreads();
        if (s < T) {
            const int rmin = max(0, s - t0);                                       // queries t >= s
            const int rmax = (int)min((long long)min(kRows, T - t0), (long long)s + window - t0);  // t < s + window
            for (int r = rmin; r < rmax; ++r) {
                const float p = expf(dot_row<HS>(sq + r * HS, k) - sl[r]);
                const float f = drop_factor(dp, bh, t0 + r, s);
                const float ds = p * (dot_row<HS>(sg + r * HS, v) * f - sD[r]);
                const float pd = p * f;
#pragma unroll
                for (int d = 0; d < HS; ++d) {
                    dv[d] = fmaf(pd, sg[r * HS + d], dv[d]);
                    dk[d] = fmaf(ds, sq[r * HS + d], dk[d]);  // sq already carries one factor of scale
                }
            }
        }
    }
    if (s < T) {
        float *out = dqkv + ((size_t)b * T + s) * ld + (size_t)h * HS;
#pragma unroll
        for (int d = 0; d < HS; ++d) {
            out[C + d] = dk[d];
            out[2 * C + d] = dv[d];
        }
    }
}

template <int HS>
cudaError_t launch_fwd_t(const float *qkv, float *y, float *lse, int B, int T, int C, int n_head, int window,
                         DropoutParams dp, cudaStream_t s) {
    const size_t smem = 2 * kRows * HS * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(fwd_f32_kernel<HS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    fwd_f32_kernel<HS><<<dim3(ceil_div(T, kRows), B * n_head), kRows, smem, s>>>(qkv, y, lse, T, C, n_head, window, dp);
    return cudaGetLastError();
}
template <int HS>
cudaError_t launch_dq_t(const float *qkv, const float *dy, const float *lse, const float *D, float *dqkv, int B, int T,
                        int C, int n_head, int window, DropoutParams dp, cudaStream_t s) {
    const size_t smem = 2 * kRows * HS * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(bwd_f32_dq_kernel<HS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_f32_dq_kernel<HS><<<dim3(ceil_div(T, kRows), B * n_head), kRows, smem, s>>>(qkv, dy, lse, D, dqkv, T, C, n_head, window, dp);
    return cudaGetLastError();
}
template <int HS>
cudaError_t launch_dkv_t(const float *qkv, const float *dy, const float *lse, const float *D, float *dqkv, int B, int T,
                         int C, int n_head, int window, DropoutParams dp, cudaStream_t s) {
    const size_t smem = (2 * kRows * HS + 2 * kRows) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(bwd_f32_dkv_kernel<HS>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_f32_dkv_kernel<HS><<<dim3(ceil_div(T, kRows), B * n_head), kRows, smem, s>>>(qkv, dy, lse, D, dqkv, T, C,
                                                                                     n_head, window, dp);
    return cudaGetLastError();
}

#define GPTATTN_HS_DISPATCH(hs, CALL) \
    switch (hs) {                      \
        case 16: return CALL(16);      \
        case 32: return CALL(32);      \
        case 64: return CALL(64);      \
        case 128: return CALL(128);    \
        default: return cudaErrorInvalidValue; \
    }

}  // namespace

cudaError_t launch_fwd_f32(int hs, const float *qkv, float *y, float *lse, int B, int T, int C, int n_head, int window,
                           DropoutParams dp, cudaStream_t s) {
#define CALL(H) launch_fwd_t<H>(qkv, y, lse, B, T, C, n_head, window, dp, s)
    GPTATTN_HS_DISPATCH(hs, CALL)
#undef CALL
}

cudaError_t launch_bwd_f32_pre(int hs, const float *y, const float *dy, float *D, int B, int T, int C, int n_head,
                               cudaStream_t s) {
    const long long n = (long long)B * n_head * T;
    long long blocks = (n + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
#define CALL(H) (bwd_f32_pre_kernel<H><<<(unsigned)blocks, 256, 0, s>>>(y, dy, D, B, T, C, n_head), cudaGetLastError())
    GPTATTN_HS_DISPATCH(hs, CALL)
#undef CALL
}

cudaError_t launch_bwd_f32_dq(int hs, const float *qkv, const float *dy, const float *lse, const float *D, float *dqkv,
                              int B, int T, int C, int n_head, int window, DropoutParams dp, cudaStream_t s) {
#define CALL(H) launch_dq_t<H>(qkv, dy, lse, D, dqkv, B, T, C, n_head, window, dp, s)
    GPTATTN_HS_DISPATCH(hs, CALL)
#undef CALL
}

cudaError_t launch_bwd_f32_dkv(int hs, const float *qkv, const float *dy, const float *lse, const float *D,
                               float *dqkv, int B, int T, int C, int n_head, int window, DropoutParams dp,
                               cudaStream_t s) {
#define CALL(H) launch_dkv_t<H>(qkv, dy, lse, D, dqkv, B, T, C, n_head, window, dp, s)
    GPTATTN_HS_DISPATCH(hs, CALL)
#undef CALL
}

}  // namespace gptattn
