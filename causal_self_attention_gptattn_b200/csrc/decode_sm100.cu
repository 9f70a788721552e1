// decode_sm100.cu -- attention of the last position over a key/value cache.
//
// For every (batch b, head h): the query of position T-1 attends to the keys and
// values of positions 0..T-1 (all of them visible: the causal mask hides nothing
// from the last position), which is row T-1 of the forward (lecture page "Let's
// build GPT: from scratch, in code, spelled out", chapters "version 3: adding
// softmax" and "version 4: self-attention"; the generate loop of the same page
// only reads the last position's output):
//     y[b, h] = sum_s softmax_s(q_{T-1} . k_s / sqrt(hs)) v_s,
//     lse[b, h] = ln sum_s exp(q_{T-1} . k_s / sqrt(hs)).
// The cache is the packed projection output qkv[B][T_cap][3C] (rows 0..T-1 valid).
//
// Memory-bound (each key and value row is read once), so no tensor cores: one
// thread-block cluster of 8 CTAs per (b, h) splits the keys 8 ways; in a CTA,
// HS*sizeof(elem)/16 lanes share a key row (16 bytes each), so a warp loads whole
// rows; each lane group keeps an fp32 online softmax (m, l, o) in base 2.  The
// partial states are merged within the warp (shuffles), across warps (shared
// memory) and across the cluster (distributed shared memory, read by rank 0).
// No TMA, no multicast.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace gptattn {
namespace {

constexpr int kDecThreads = 128;  // 16 CTAs per SM: the usual grids are resident in one wave
constexpr int kBatch = 4;          // key steps whose loads are issued before any of them is used
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kCluster = 8;

template <typename Elem>
__device__ __forceinline__ void unpack16(const uint4 r, float (&v)[16 / sizeof(Elem)]) {
    if constexpr (sizeof(Elem) == 2) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = bf16lo_to_f32(w[i]);
            v[2 * i + 1] = bf16hi_to_f32(w[i]);
        }
    } else {
        v[0] = __uint_as_float(r.x);
        v[1] = __uint_as_float(r.y);
        v[2] = __uint_as_float(r.z);
        v[3] = __uint_as_float(r.w);
    }
}

template <typename Elem>
__device__ __forceinline__ void load16(const Elem *p, float (&v)[16 / sizeof(Elem)]) {
    unpack16<Elem>(*reinterpret_cast<const uint4 *>(p), v);
}

// weight of a partial state with running max m against the merged max mm (base 2)
__device__ __forceinline__ float part_weight(float m, float mm) { return m == -INFINITY ? 0.f : exp2f(m - mm); }

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_peer_f32(const float *local_addr, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local_addr)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

template <typename Elem, int HS>
__global__ void __launch_bounds__(kDecThreads, 8) decode_kernel(const Elem *__restrict__ qkv, Elem *__restrict__ y,
                                                            float *__restrict__ lse, int T, int T_cap, int C,
                                                            int n_head) {
    constexpr int kE = 16 / (int)sizeof(Elem);  // elements per lane
    constexpr int kLPR = HS / kE;               // lanes per key row
    constexpr int kKPW = 32 / kLPR;             // keys per warp per step
    static_assert(kLPR >= 1 && kLPR <= 32 && 32 % kLPR == 0, "lanes per row");
    __shared__ float sm_m[kDecWarps], sm_l[kDecWarps], sm_o[kDecWarps][HS];
    __shared__ float cta_m, cta_l, cta_o[HS];

    griddep_launch_dependents();
    griddep_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = lane / kLPR, part = lane % kLPR;
    const uint32_t rank = cluster_rank();
    const int bh = blockIdx.y, b = bh / n_head, h = bh % n_head;
    const size_t row_stride = 3 * (size_t)C;
    const Elem *base = qkv + (size_t)b * T_cap * row_stride + (size_t)h * HS + (size_t)part * kE;

    // this lane's slice of the query (last position), scaled so scores come out in base 2
    float q[kE];
    load16(base + (size_t)(T - 1) * row_stride, q);
    const float qscale = rsqrtf((float)HS) * 1.4426950408889634f;
#pragma unroll
    for (int e = 0; e < kE; ++e) q[e] *= qscale;

    const int chunk = (T + kCluster - 1) / kCluster;
    const int k0 = (int)rank * chunk, k1 = min(T, k0 + chunk);
    float m = -INFINITY, l = 0.f, o[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) o[e] = 0.f;
    constexpr int kStep = kDecWarps * kKPW;  // keys the CTA covers per step
    for (int s0 = k0 + warp * kKPW; s0 < k1; s0 += kBatch * kStep) {  // warp-uniform
        uint4 kr[kBatch], vr[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int s = s0 + u * kStep + grp;
            if (s < k1) {
                kr[u] = *reinterpret_cast<const uint4 *>(base + (size_t)s * row_stride + C);
                vr[u] = *reinterpret_cast<const uint4 *>(base + (size_t)s * row_stride + 2 * C);
            }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (s0 + u * kStep >= k1) break;  // warp-uniform
            const bool valid = s0 + u * kStep + grp < k1;
            float kv[kE], vv[kE];
            unpack16<Elem>(valid ? kr[u] : make_uint4(0u, 0u, 0u, 0u), kv);
            unpack16<Elem>(valid ? vr[u] : make_uint4(0u, 0u, 0u, 0u), vv);
            float sc = 0.f;
#pragma unroll
            for (int e = 0; e < kE; ++e) sc = fmaf(q[e], kv[e], sc);
#pragma unroll
            for (int off = kLPR / 2; off > 0; off >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, off);
            if (valid) {
                const float mn = fmaxf(m, sc);
                const float alpha = part_weight(m, mn), p = exp2f(sc - mn);
                l = l * alpha + p;
#pragma unroll
                for (int e = 0; e < kE; ++e) o[e] = fmaf(p, vv[e], o[e] * alpha);
                m = mn;
            }
        }
    }
    // merge the lane groups of the warp
#pragma unroll
    for (int off = kLPR; off < 32; off <<= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, off), l2 = __shfl_xor_sync(0xffffffffu, l, off);
        const float mm = fmaxf(m, m2);
        const float a = part_weight(m, mm), a2 = part_weight(m2, mm);
        l = l * a + l2 * a2;
#pragma unroll
        for (int e = 0; e < kE; ++e) o[e] = o[e] * a + __shfl_xor_sync(0xffffffffu, o[e], off) * a2;
        m = mm;
    }
    if (lane == 0) {
        sm_m[warp] = m;
        sm_l[warp] = l;
    }
    if (grp == 0) {
#pragma unroll
        for (int e = 0; e < kE; ++e) sm_o[warp][part * kE + e] = o[e];
    }
    __syncthreads();
    // merge the warps: one thread per output dimension
    if (threadIdx.x < HS) {
        float mm = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) mm = fmaxf(mm, sm_m[w]);
        float ll = 0.f, oo = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            const float a = part_weight(sm_m[w], mm);
            ll += sm_l[w] * a;
            oo += sm_o[w][threadIdx.x] * a;
        }
        cta_o[threadIdx.x] = oo;
        if (threadIdx.x == 0) {
            cta_m = mm;
            cta_l = ll;
        }
    }
    cluster_sync();
    // rank 0 merges the cluster's partial states and writes the outputs
    if (rank == 0 && threadIdx.x < HS) {
        float pm[kCluster], mm = -INFINITY;
#pragma unroll
        for (int r = 0; r < kCluster; ++r) {
            pm[r] = ld_peer_f32(&cta_m, (uint32_t)r);
            mm = fmaxf(mm, pm[r]);
        }
        float ll = 0.f, oo = 0.f;
#pragma unroll
        for (int r = 0; r < kCluster; ++r) {
            const float a = part_weight(pm[r], mm);
            ll += ld_peer_f32(&cta_l, (uint32_t)r) * a;
            oo += ld_peer_f32(&cta_o[threadIdx.x], (uint32_t)r) * a;
        }
        const float yv = oo / ll;
        Elem *dst = y + (size_t)b * C + (size_t)h * HS + threadIdx.x;
        if constexpr (sizeof(Elem) == 2)
            *dst = __float2bfloat16_rn(yv);
        else
            *dst = yv;
        if (threadIdx.x == 0 && lse) lse[(size_t)b * n_head + h] = (mm + __log2f(ll)) * 0.6931471805599453f;
    }
    cluster_sync();  // peers keep their shared memory until rank 0 has read it
}

template <typename Elem, int HS>
cudaError_t launch_decode_impl(const Elem *qkv, Elem *y, float *lse, int B, int T, int T_cap, int C, int n_head,
                               cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kCluster, (unsigned)(B * n_head));
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, decode_kernel<Elem, HS>, qkv, y, lse, T, T_cap, C, n_head);
}

}  // namespace

cudaError_t launch_decode(int hs, bool bf16, const void *qkv, void *y, float *lse, int B, int T, int T_cap, int C,
                          int n_head, cudaStream_t s) {
    if (bf16) {
        auto q = static_cast<const __nv_bfloat16 *>(qkv);
        auto o = static_cast<__nv_bfloat16 *>(y);
        if (hs == 64) return launch_decode_impl<__nv_bfloat16, 64>(q, o, lse, B, T, T_cap, C, n_head, s);
        if (hs == 128) return launch_decode_impl<__nv_bfloat16, 128>(q, o, lse, B, T, T_cap, C, n_head, s);
        return cudaErrorInvalidValue;
    }
    auto q = static_cast<const float *>(qkv);
    auto o = static_cast<float *>(y);
    switch (hs) {
        case 16: return launch_decode_impl<float, 16>(q, o, lse, B, T, T_cap, C, n_head, s);
        case 32: return launch_decode_impl<float, 32>(q, o, lse, B, T, T_cap, C, n_head, s);
        case 64: return launch_decode_impl<float, 64>(q, o, lse, B, T, T_cap, C, n_head, s);
        case 128: return launch_decode_impl<float, 128>(q, o, lse, B, T, T_cap, C, n_head, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gptattn
