// api.cu -- the C ABI of libgptattn (declared in include/gptattn.h).
//
// Host-side responsibilities: validate every argument before anything is
// enqueued, build the TMA tensor maps that let the kernels address q, k, v of
// one head directly inside the packed qkv tensor (heads as a batch dimension,
// exercise EX1 of the lecture page "Let's build GPT: from scratch, in code,
// spelled out"), carve the caller's workspace, launch, and map CUDA errors to
// status codes.  Also owns the device status word that kernels use to report
// a bounded wait that ran out.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "gptattn.h"
#include <cmath>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace gptattn {

// Device status word: 0, or the status code of the first kernel that gave up
// on a wait since it was last read.  One per device that loads the library.
__device__ int g_device_status;

namespace {

constexpr unsigned long long kDefaultBudgetNs = 1000000000ull;  // 1 s per wait
constexpr int kMaxDevices = 64;

std::mutex g_mutex;
int *g_status_ptr[kMaxDevices] = {};
std::atomic<unsigned long long> g_launches{0};

thread_local const char *t_last_error = "no error";

gptattn_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return GPTATTN_OK;
    t_last_error = cudaGetErrorString(e);
    return GPTATTN_ERR_CUDA;
}

// A failure that is not a CUDA error code (tensor-map encoding): record why.
gptattn_status fail_cuda(const char *why) {
    t_last_error = why;
    return GPTATTN_ERR_CUDA;
}

// Device address of g_device_status for the current device (looked up once
// per device, with that device current).
cudaError_t status_ptr(int **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_device_status);
        if (e != cudaSuccess) return e;
        g_status_ptr[dev] = static_cast<int *>(p);
    }
    *out = g_status_ptr[dev];
    return cudaSuccess;
}

// ---------------------------------------------------------------------------
// Tensor maps (driver entry point fetched through the runtime, so the library
// needs no link-time dependency on libcuda).
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// bf16 tensor [B][T][W] viewed as 3-D (W, T, B); box (64, 128, 1); 128-byte
// swizzle; rows past T read as zero and are not written.
bool map_bf16_rows(CUtensorMap *m, const void *ptr, int W, int T, int B) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)W, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)W * 2u, (cuuint64_t)W * 2u * (cuuint64_t)T};
    cuuint32_t box[3] = {64, (cuuint32_t)kTile, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 matrix [rows][hs] viewed as 2-D (hs, rows); box (32, 128); 128-byte swizzle.
bool map_f32_acc(CUtensorMap *m, const void *ptr, int hs, long long rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)hs, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)hs * 4u};
    cuuint32_t box[2] = {32, (cuuint32_t)kTile};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 row-major matrix [outer][inner] viewed as 2-D (inner, outer); box (64,
// box_outer); 128-byte swizzle; out-of-range rows read as zero and are not written.
bool map_bf16_2d(CUtensorMap *m, const void *ptr, long long inner, long long outer, int box_outer) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
    cuuint64_t strides[1] = {(cuuint64_t)inner * 2u};
    cuuint32_t box[2] = {64, (cuuint32_t)box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// Validation (pure host; nothing is enqueued on failure)
// ---------------------------------------------------------------------------
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gptattn_status check_shape(int B, int T, int C, int n_head, gptattn_dtype dt, int *hs_out) {
    if (B < 0 || T < 0 || C <= 0 || n_head <= 0) return GPTATTN_ERR_INVALID_ARG;
    if (C % n_head != 0) return GPTATTN_ERR_INVALID_ARG;
    const int hs = C / n_head;
    if (dt == GPTATTN_BF16) {
        if (hs != 64 && hs != 128) return GPTATTN_ERR_UNSUPPORTED;
    } else if (dt == GPTATTN_F32) {
        if (hs != 16 && hs != 32 && hs != 64 && hs != 128) return GPTATTN_ERR_UNSUPPORTED;
    } else {
        return GPTATTN_ERR_UNSUPPORTED;
    }
    // Size limits: 3C fits a TMA dimension and an int index; grid fits in x.
    if ((long long)C * 3 > (1LL << 30)) return GPTATTN_ERR_UNSUPPORTED;
    const long long tiles = (long long)((T + kTile - 1) / kTile) * B * n_head;
    if (tiles > 0x7fffffffLL) return GPTATTN_ERR_UNSUPPORTED;
    if ((long long)B * n_head > 65535LL && dt == GPTATTN_F32) return GPTATTN_ERR_UNSUPPORTED;  // grid.y
    if (dt == GPTATTN_BF16 && (B > 65535 || (T + kTile - 1) / kTile > 65535)) return GPTATTN_ERR_UNSUPPORTED;  // grid.y
    *hs_out = hs;
    return GPTATTN_OK;
}

int padded_T(int T) { return ((T + kTile - 1) / kTile) * kTile; }

size_t align256(size_t x) { return (x + 255u) & ~(size_t)255u; }

struct BwdWorkspace {
    size_t D, lse2, dqacc, total;
};

// Partial dQ tiles per (b, h) in deterministic mode: one per (query tile i, key tile j <= i).
long long det_slots(int T) {
    const long long n_t = (T + kTile - 1) / kTile;
    return n_t * (n_t + 1) / 2;
}

BwdWorkspace workspace_layout(int B, int T, int n_head, int hs, gptattn_dtype dt, bool det = false) {
    BwdWorkspace w{};
    if (dt == GPTATTN_F32) {
        w.D = 0;
        w.total = align256((size_t)B * n_head * T * sizeof(float));
        return w;
    }
    const size_t rows = (size_t)B * n_head * padded_T(T);
    const size_t acc_rows = det ? (size_t)B * n_head * (size_t)det_slots(T) * kTile : rows;
    w.D = 0;
    w.lse2 = align256(rows * sizeof(float));
    w.dqacc = w.lse2 + align256(rows * sizeof(float));
    w.total = w.dqacc + align256(acc_rows * (size_t)hs * sizeof(float));
    return w;
}

// ---------------------------------------------------------------------------
// Instrumentation: optional CUDA events around each kernel launch.
// ---------------------------------------------------------------------------
struct ProfRecord {
    int kernel;
    cudaEvent_t start, stop;
};
struct Profiler {
    int capacity = 0;
    std::vector<ProfRecord> records;   // filled in order
    std::vector<cudaEvent_t> pool;     // reusable events
} g_prof;

cudaEvent_t prof_event() {
    if (!g_prof.pool.empty()) {
        cudaEvent_t e = g_prof.pool.back();
        g_prof.pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

template <class F>
cudaError_t run_kernel(int kernel_id, cudaStream_t s, F &&launch) {
    ProfRecord rec{kernel_id, nullptr, nullptr};
    bool recording = false;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (g_prof.capacity > 0 && (int)g_prof.records.size() < g_prof.capacity) {
            rec.start = prof_event();
            rec.stop = prof_event();
            recording = rec.start && rec.stop;
        }
    }
    if (recording) cudaEventRecord(rec.start, s);
    cudaError_t e = launch();
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (recording) {
        cudaEventRecord(rec.stop, s);
        std::lock_guard<std::mutex> lock(g_mutex);
        g_prof.records.push_back(rec);
    }
    return e;
}

// ---------------------------------------------------------------------------
// Bounded-wait self-test kernel: waits on a barrier nobody arrives at.
// ---------------------------------------------------------------------------
__global__ void selftest_timeout_kernel(int *status, unsigned long long budget_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const WaitGuard g{&abort_flag, status, budget_ns};
        (void)mbar_wait(smem_u32(&bar), 0, g);  // nothing ever completes phase 0
    }
    __syncthreads();
}

// The FMA-pipe exponential of the backward kernel, evaluated on caller data:
// y[i] = exp2_poly_x2 of x[i] (pairs of elements per thread).
__global__ void selftest_exp2_kernel(const float *__restrict__ x, float *__restrict__ y, int n) {
    const long long i = 2ll * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.f;
    float y0, y1;
    exp2_poly_x2(x0, x1, y0, y1);
    y[i] = y0;
    if (i + 1 < n) y[i + 1] = y1;
}

}  // namespace

cudaError_t launch_selftest_exp2(const float *x, float *y, int n, cudaStream_t s) {
    const long long pairs = ((long long)n + 1) / 2;
    selftest_exp2_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, s>>>(x, y, n);
    return cudaGetLastError();
}

cudaError_t launch_selftest_timeout(DevCtx ctx, cudaStream_t s) {
    selftest_timeout_kernel<<<1, 32, 0, s>>>(ctx.status, ctx.budget_ns);
    return cudaGetLastError();
}

}  // namespace gptattn

using namespace gptattn;

namespace {
// Shape checks shared by the windowed entry points: window >= 1.  Returns the
// window the kernels get (kCausalWindow when nothing is cut).
gptattn_status check_window(int window, int T, int hs, gptattn_dtype dt, int *kernel_window) {
    if (window < 1) return GPTATTN_ERR_INVALID_ARG;
    if (window >= T) {
        *kernel_window = kCausalWindow;
        return GPTATTN_OK;
    }
    *kernel_window = window;
    return GPTATTN_OK;
}

// Dropout probability -> kernel parameters (threshold theta = round(256 p), at most
// 255; a p so small that theta is 0 drops nothing).  p must be in [0, 1).
gptattn_status make_dropout(float p, unsigned long long seed, int hs, gptattn_dtype dt, DropoutParams *dp) {
    if (!(p >= 0.f && p < 1.f)) return GPTATTN_ERR_INVALID_ARG;
    // p in steps of 1/256: theta = round(256 p), at most 255; drop probability theta/256
    const double x = floor(256.0 * (double)p + 0.5);
    dp->seed = seed;
    dp->threshold = x >= 255.0 ? 255u : (uint32_t)x;
    dp->scale = dp->threshold ? (float)(1.0 / (1.0 - dp->threshold / 256.0)) : 1.f;
    return GPTATTN_OK;
}

gptattn_status fwd_impl(const void *qkv, void *y, float *lse, int B, int T, int C, int n_head, int window,
                        float dropout_p, unsigned long long seed, gptattn_dtype dt, gptattn_stream_t stream) {
    int hs = 0;
    gptattn_status st = check_shape(B, T, C, n_head, dt, &hs);
    if (st != GPTATTN_OK) return st;
    int kw = kCausalWindow;
    st = check_window(window, T, hs, dt, &kw);
    if (st != GPTATTN_OK) return st;
    DropoutParams dp{};
    st = make_dropout(dropout_p, seed, hs, dt, &dp);
    if (st != GPTATTN_OK) return st;
    if (B == 0 || T == 0) return GPTATTN_OK;
    if (!qkv || !y) return GPTATTN_ERR_INVALID_ARG;  // lse may be null: inference, not written
    if (!aligned16(qkv) || !aligned16(y) || (lse && !aligned16(lse))) return GPTATTN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    if (dt == GPTATTN_F32) {
        return from_cuda(run_kernel(kKFwdF32, s, [&] {
            return launch_fwd_f32(hs, static_cast<const float *>(qkv), static_cast<float *>(y), lse, B, T, C, n_head, kw,
                                  dp, s);
        }));
    }
    int *status = nullptr;
    cudaError_t e = status_ptr(&status);
    if (e != cudaSuccess) return from_cuda(e);
    CUtensorMap mq, my;
    if (!map_bf16_rows(&mq, qkv, 3 * C, T, B) || !map_bf16_rows(&my, y, C, T, B))
        return fail_cuda("tensor map encoding failed");
    const DevCtx ctx{status, kDefaultBudgetNs};
    return from_cuda(
        run_kernel(kKFwdBf16, s, [&] { return launch_fwd_bf16(hs, mq, my, lse, B, T, C, n_head, kw, dp, ctx, s); }));
}
}  // namespace

namespace {
// Deterministic mode on the bf16 path needs row indices of the partial-tile
// buffer that fit 32-bit TMA coordinates.
gptattn_status check_det(int B, int T, int n_head, int hs, gptattn_dtype dt) {
    if (dt != GPTATTN_BF16) return GPTATTN_OK;
    (void)hs;
    if ((long long)B * n_head * det_slots(T) * kTile > 0x7fffffffLL) return GPTATTN_ERR_UNSUPPORTED;
    return GPTATTN_OK;
}

gptattn_status bwd_impl(const void *qkv, const void *y, const float *lse, const void *dy, void *dqkv, void *workspace,
                        size_t workspace_bytes, int B, int T, int C, int n_head, int window, bool det,
                        float dropout_p, unsigned long long seed, gptattn_dtype dt, gptattn_stream_t stream) {
    int hs = 0;
    gptattn_status st = check_shape(B, T, C, n_head, dt, &hs);
    if (st != GPTATTN_OK) return st;
    int kw = kCausalWindow;
    st = check_window(window, T, hs, dt, &kw);
    if (st != GPTATTN_OK) return st;
    DropoutParams dp{};
    st = make_dropout(dropout_p, seed, hs, dt, &dp);
    if (st != GPTATTN_OK) return st;
    if (det && (st = check_det(B, T, n_head, hs, dt)) != GPTATTN_OK) return st;
    if (B == 0 || T == 0) return GPTATTN_OK;
    if (!qkv || !y || !lse || !dy || !dqkv) return GPTATTN_ERR_INVALID_ARG;
    if (!aligned16(qkv) || !aligned16(y) || !aligned16(lse) || !aligned16(dy) || !aligned16(dqkv))
        return GPTATTN_ERR_INVALID_ARG;
    const BwdWorkspace w = workspace_layout(B, T, n_head, hs, dt, det);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < w.total)
        return GPTATTN_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);

    if (dt == GPTATTN_F32) {
        const float *fq = static_cast<const float *>(qkv);
        const float *fy = static_cast<const float *>(y);
        const float *fg = static_cast<const float *>(dy);
        float *fo = static_cast<float *>(dqkv);
        float *D = reinterpret_cast<float *>(ws + w.D);
        cudaError_t e = run_kernel(kKBwdPreF32, s, [&] { return launch_bwd_f32_pre(hs, fy, fg, D, B, T, C, n_head, s); });
        if (e == cudaSuccess)
            e = run_kernel(kKBwdDqF32, s,
                           [&] { return launch_bwd_f32_dq(hs, fq, fg, lse, D, fo, B, T, C, n_head, kw, dp, s); });
        if (e == cudaSuccess)
            e = run_kernel(kKBwdDkvF32, s,
                           [&] { return launch_bwd_f32_dkv(hs, fq, fg, lse, D, fo, B, T, C, n_head, kw, dp, s); });
        return from_cuda(e);
    }

    int *status = nullptr;
    if (cudaError_t es = status_ptr(&status)) return from_cuda(es);
    const int T_pad = padded_T(T);
    float *D = reinterpret_cast<float *>(ws + w.D);
    float *lse2 = reinterpret_cast<float *>(ws + w.lse2);
    float *dqacc = reinterpret_cast<float *>(ws + w.dqacc);
    CUtensorMap mq, mdy, mdqkv, mdq;
    if (!map_bf16_rows(&mq, qkv, 3 * C, T, B) || !map_bf16_rows(&mdy, dy, C, T, B) ||
        !map_bf16_rows(&mdqkv, dqkv, 3 * C, T, B) ||
        !map_f32_acc(&mdq, dqacc, hs, det ? (long long)B * n_head * det_slots(T) * kTile : (long long)B * n_head * T_pad))
        return fail_cuda("tensor map encoding failed");
    const int n_slots = det ? (int)det_slots(T) : 0;
    const DevCtx ctx{status, kDefaultBudgetNs};
    // dropout's scale s = 256 / (256 - theta) folded into the recomputed weights (log2 s) and D (1/s)
    const float lse_bias = dp.threshold ? (float)log2(256.0 / (256.0 - dp.threshold)) : 0.f;
    const float d_mul = dp.threshold ? (float)((256.0 - dp.threshold) / 256.0) : 1.f;
    cudaError_t e = run_kernel(kKBwdPreBf16, s, [&] {
        return launch_bwd_pre_bf16(hs, y, dy, lse, D, lse2, dqacc, B, T, C, n_head, T_pad, !det, lse_bias, d_mul, s);
    });
    if (e == cudaSuccess)
        e = run_kernel(kKBwdMainBf16, s, [&] {
            return launch_bwd_main_bf16(hs, mq, mdy, mdqkv, mdq, lse2, D, B, T, C, n_head, T_pad, kw, n_slots, dp, ctx,
                                        s);
        });
    if (e == cudaSuccess)
        e = run_kernel(kKBwdPostBf16, s, [&] {
            return det ? launch_bwd_post_det_bf16(hs, dqacc, dqkv, B, T, C, n_head, T_pad, n_slots, kw, s)
                       : launch_bwd_post_bf16(hs, dqacc, dqkv, B, T, C, n_head, T_pad, s);
        });
    return from_cuda(e);
}
}  // namespace

namespace {
// Linear map checks: sizes, alignment (16 bytes: TMA bases and vector loads).
gptattn_status check_linear(const void *a, const void *w, const void *bias, const void *resid, const void *out, int M,
                            int N, int K) {
    if (M < 0 || N <= 0 || K <= 0) return GPTATTN_ERR_INVALID_ARG;
    if (N % 64 != 0 || K % 64 != 0) return GPTATTN_ERR_UNSUPPORTED;
    if (M == 0) return GPTATTN_OK;
    if (!a || !w || !out) return GPTATTN_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(w) || !aligned16(out)) return GPTATTN_ERR_INVALID_ARG;
    if ((bias && !aligned16(bias)) || (resid && !aligned16(resid))) return GPTATTN_ERR_INVALID_ARG;
    return GPTATTN_OK;
}

gptattn_status linear_impl(const void *a, const void *w, const void *bias, const void *resid, void *out, int M, int N,
                           int K, cudaStream_t s) {
    int *status = nullptr;
    if (cudaError_t es = status_ptr(&status)) return from_cuda(es);
    const int tile_n = gemm_tile_n(M, N);
    CUtensorMap ma, mw, mc;
    if (!map_bf16_2d(&ma, a, K, M, 128) || !map_bf16_2d(&mw, w, K, N, tile_n) || !map_bf16_2d(&mc, out, N, M, 128))
        return fail_cuda("tensor map encoding failed");
    const DevCtx ctx{status, kDefaultBudgetNs};
    return from_cuda(
        run_kernel(kKGemm, s, [&] { return launch_gemm_bf16(ma, mw, mc, bias, resid, M, N, K, tile_n, ctx, s); }));
}

gptattn_status check_layernorm(const void *x, const void *w, const void *b, const void *out, int M, int C) {
    if (M < 0 || C <= 0) return GPTATTN_ERR_INVALID_ARG;
    if (C % 8 != 0 || C > 4096) return GPTATTN_ERR_UNSUPPORTED;
    if (M == 0) return GPTATTN_OK;
    if (!x || !w || !b || !out) return GPTATTN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w) || !aligned16(b) || !aligned16(out)) return GPTATTN_ERR_INVALID_ARG;
    return GPTATTN_OK;
}
}  // namespace

extern "C" {

const char *gptattn_status_string(gptattn_status s) {
    switch (s) {
        case GPTATTN_OK: return "ok";
        case GPTATTN_ERR_INVALID_ARG: return "invalid argument";
        case GPTATTN_ERR_UNSUPPORTED: return "unsupported head size, dtype or size";
        case GPTATTN_ERR_CUDA: return "CUDA error";
        case GPTATTN_ERR_TIMEOUT: return "a kernel wait timed out";
        case GPTATTN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    }
    return "unknown status";
}

int gptattn_version(void) { return 100; }

const char *gptattn_last_error_string(void) { return t_last_error; }


gptattn_status gptattn_fwd(const void *qkv, void *y, float *lse, int B, int T, int C, int n_head, gptattn_dtype dt,
                           gptattn_stream_t stream) {
    return fwd_impl(qkv, y, lse, B, T, C, n_head, kCausalWindow, 0.f, 0, dt, stream);
}

gptattn_status gptattn_fwd_window(const void *qkv, void *y, float *lse, int B, int T, int C, int n_head, int window,
                                  gptattn_dtype dt, gptattn_stream_t stream) {
    return fwd_impl(qkv, y, lse, B, T, C, n_head, window, 0.f, 0, dt, stream);
}

gptattn_status gptattn_decode(const void *qkv, void *y, float *lse, int B, int T, int T_cap, int C, int n_head,
                              gptattn_dtype dt, gptattn_stream_t stream) {
    int hs = 0;
    gptattn_status st = check_shape(B, T, C, n_head, dt, &hs);
    if (st != GPTATTN_OK) return st;
    if (T_cap < T) return GPTATTN_ERR_INVALID_ARG;
    if ((long long)B * n_head > 65535LL) return GPTATTN_ERR_UNSUPPORTED;  // grid.y
    if (B == 0 || T == 0) return GPTATTN_OK;
    if (!qkv || !y) return GPTATTN_ERR_INVALID_ARG;  // lse may be null: inference, not written
    if (!aligned16(qkv) || !aligned16(y) || (lse && !aligned16(lse))) return GPTATTN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return from_cuda(run_kernel(kKDecode, s, [&] {
        return launch_decode(hs, dt == GPTATTN_BF16, qkv, y, lse, B, T, T_cap, C, n_head, s);
    }));
}

size_t gptattn_bwd_workspace_bytes(int B, int T, int C, int n_head, gptattn_dtype dt) {
    int hs = 0;
    if (check_shape(B, T, C, n_head, dt, &hs) != GPTATTN_OK) return (size_t)-1;
    if (B == 0 || T == 0) return 0;
    return workspace_layout(B, T, n_head, hs, dt).total;
}


gptattn_status gptattn_bwd(const void *qkv, const void *y, const float *lse, const void *dy, void *dqkv,
                           void *workspace, size_t workspace_bytes, int B, int T, int C, int n_head, gptattn_dtype dt,
                           gptattn_stream_t stream) {
    return bwd_impl(qkv, y, lse, dy, dqkv, workspace, workspace_bytes, B, T, C, n_head, kCausalWindow, false, 0.f, 0, dt,
                    stream);
}

gptattn_status gptattn_bwd_window(const void *qkv, const void *y, const float *lse, const void *dy, void *dqkv,
                                  void *workspace, size_t workspace_bytes, int B, int T, int C, int n_head, int window,
                                  gptattn_dtype dt, gptattn_stream_t stream) {
    return bwd_impl(qkv, y, lse, dy, dqkv, workspace, workspace_bytes, B, T, C, n_head, window, false, 0.f, 0, dt,
                    stream);
}

size_t gptattn_bwd_det_workspace_bytes(int B, int T, int C, int n_head, gptattn_dtype dt) {
    int hs = 0;
    if (check_shape(B, T, C, n_head, dt, &hs) != GPTATTN_OK) return (size_t)-1;
    if (check_det(B, T, n_head, hs, dt) != GPTATTN_OK) return (size_t)-1;
    if (B == 0 || T == 0) return 0;
    return workspace_layout(B, T, n_head, hs, dt, true).total;
}

gptattn_status gptattn_bwd_det(const void *qkv, const void *y, const float *lse, const void *dy, void *dqkv,
                               void *workspace, size_t workspace_bytes, int B, int T, int C, int n_head, int window,
                               gptattn_dtype dt, gptattn_stream_t stream) {
    return bwd_impl(qkv, y, lse, dy, dqkv, workspace, workspace_bytes, B, T, C, n_head, window, true, 0.f, 0, dt,
                    stream);
}

// Options: a zero-initialised struct (or NULL) is the plain causal call.
static gptattn_status read_opts(const gptattn_options *o, int *window, float *p, unsigned long long *seed, bool *det) {
    *window = kCausalWindow;
    *p = 0.f;
    *seed = 0;
    *det = false;
    if (!o) return GPTATTN_OK;
    if (o->window < 0) return GPTATTN_ERR_INVALID_ARG;
    if (o->window > 0) *window = o->window;
    *p = o->dropout_p;
    *seed = o->dropout_seed;
    *det = o->deterministic != 0;
    return GPTATTN_OK;
}

gptattn_status gptattn_fwd_opts(const void *qkv, void *y, float *lse, int B, int T, int C, int n_head,
                                const gptattn_options *opts, gptattn_dtype dt, gptattn_stream_t stream) {
    int window;
    float p;
    unsigned long long seed;
    bool det;
    gptattn_status st = read_opts(opts, &window, &p, &seed, &det);
    if (st != GPTATTN_OK) return st;
    return fwd_impl(qkv, y, lse, B, T, C, n_head, window, p, seed, dt, stream);
}

size_t gptattn_bwd_opts_workspace_bytes(int B, int T, int C, int n_head, const gptattn_options *opts,
                                        gptattn_dtype dt) {
    int window;
    float p;
    unsigned long long seed;
    bool det;
    if (read_opts(opts, &window, &p, &seed, &det) != GPTATTN_OK) return (size_t)-1;
    return det ? gptattn_bwd_det_workspace_bytes(B, T, C, n_head, dt) : gptattn_bwd_workspace_bytes(B, T, C, n_head, dt);
}

gptattn_status gptattn_bwd_opts(const void *qkv, const void *y, const float *lse, const void *dy, void *dqkv,
                                void *workspace, size_t workspace_bytes, int B, int T, int C, int n_head,
                                const gptattn_options *opts, gptattn_dtype dt, gptattn_stream_t stream) {
    int window;
    float p;
    unsigned long long seed;
    bool det;
    gptattn_status st = read_opts(opts, &window, &p, &seed, &det);
    if (st != GPTATTN_OK) return st;
    return bwd_impl(qkv, y, lse, dy, dqkv, workspace, workspace_bytes, B, T, C, n_head, window, det, p, seed, dt,
                    stream);
}

gptattn_status gptattn_layernorm(const void *x, const void *w, const void *b, void *out, int M, int C,
                                 gptattn_dtype dt, gptattn_stream_t stream) {
    if (dt != GPTATTN_BF16) return GPTATTN_ERR_UNSUPPORTED;
    gptattn_status st = check_layernorm(x, w, b, out, M, C);
    if (st != GPTATTN_OK || M == 0) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return from_cuda(run_kernel(kKLayerNorm, s, [&] { return launch_layernorm_bf16(x, w, b, out, M, C, s); }));
}

gptattn_status gptattn_linear(const void *a, const void *w, const void *bias, const void *resid, void *out, int M,
                              int N, int K, gptattn_dtype dt, gptattn_stream_t stream) {
    if (dt != GPTATTN_BF16) return GPTATTN_ERR_UNSUPPORTED;
    gptattn_status st = check_linear(a, w, bias, resid, out, M, N, K);
    if (st != GPTATTN_OK || M == 0) return st;
    return linear_impl(a, w, bias, resid, out, M, N, K, reinterpret_cast<cudaStream_t>(stream));
}

gptattn_status gptattn_attn_block_fwd(const void *x, const void *ln_w, const void *ln_b, const void *w_attn,
                                      const void *b_attn, const void *w_proj, const void *b_proj, void *qkv, void *y,
                                      float *lse, void *out, int B, int T, int C, int n_head, gptattn_dtype dt,
                                      gptattn_stream_t stream) {
    if (dt != GPTATTN_BF16) return GPTATTN_ERR_UNSUPPORTED;
    int hs = 0;
    gptattn_status st = check_shape(B, T, C, n_head, dt, &hs);
    if (st != GPTATTN_OK) return st;
    if ((long long)B * T > 0x7fffffffLL) return GPTATTN_ERR_UNSUPPORTED;
    const int M = B * T;
    st = check_layernorm(x, ln_w, ln_b, y, M, C);
    if (st == GPTATTN_OK) st = check_linear(y, w_attn, b_attn, nullptr, qkv, M, 3 * C, C);
    if (st == GPTATTN_OK) st = check_linear(y, w_proj, b_proj, x, out, M, C, C);
    if (st != GPTATTN_OK) return st;
    if (M == 0) return GPTATTN_OK;
    if (lse && !aligned16(lse)) return GPTATTN_ERR_INVALID_ARG;  // null: not written
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // y holds LN(x) until the attention overwrites it with the heads' outputs.
    st = from_cuda(run_kernel(kKLayerNorm, s, [&] { return launch_layernorm_bf16(x, ln_w, ln_b, y, M, C, s); }));
    if (st == GPTATTN_OK) st = linear_impl(y, w_attn, b_attn, nullptr, qkv, M, 3 * C, C, s);
    if (st == GPTATTN_OK) st = fwd_impl(qkv, y, lse, B, T, C, n_head, kCausalWindow, 0.f, 0, dt, stream);
    if (st == GPTATTN_OK) st = linear_impl(y, w_proj, b_proj, x, out, M, C, C, s);
    return st;
}

gptattn_status gptattn_get_device_status(gptattn_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaError_t e = cudaStreamSynchronize(s)) return from_cuda(e);
    int *p = nullptr;
    if (cudaError_t es = status_ptr(&p)) return from_cuda(es);
    int v = 0;
    if (cudaError_t e = cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost)) return from_cuda(e);
    const int zero = 0;
    if (cudaError_t e = cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice)) return from_cuda(e);
    return v == 0 ? GPTATTN_OK : static_cast<gptattn_status>(v);
}

gptattn_status gptattn_profile_enable(int max_records) {
    if (max_records < 0) return GPTATTN_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_mutex);
    g_prof.capacity = max_records;
    // create the events now, so recording inside a timed region allocates nothing
    const size_t want = 2u * (size_t)max_records;
    while (g_prof.pool.size() + 2u * g_prof.records.size() < want) {
        cudaEvent_t e = nullptr;
        if (cudaError_t ce = cudaEventCreate(&e)) return from_cuda(ce);
        g_prof.pool.push_back(e);
    }
    if (max_records == 0) {
        for (auto &r : g_prof.records) {
            g_prof.pool.push_back(r.start);
            g_prof.pool.push_back(r.stop);
        }
        g_prof.records.clear();
        for (cudaEvent_t e : g_prof.pool) cudaEventDestroy(e);
        g_prof.pool.clear();
    }
    return GPTATTN_OK;
}

int gptattn_profile_read(int *kernel_ids, float *ms, int capacity) {
    std::lock_guard<std::mutex> lock(g_mutex);
    int n = 0;
    for (auto &r : g_prof.records) {
        if (n < capacity && kernel_ids && ms) {
            float t = -1.f;
            if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
                t = -1.f;
            kernel_ids[n] = r.kernel;
            ms[n] = t;
            ++n;
        }
        g_prof.pool.push_back(r.start);
        g_prof.pool.push_back(r.stop);
    }
    g_prof.records.clear();
    return n;
}

const char *gptattn_kernel_name(int kernel_id) {
    static const char *names[kKNumKernels] = {
        "fwd_bf16_sm100", "bwd_pre_bf16", "bwd_bf16_sm100", "bwd_post_bf16", "fwd_f32_simt",
        "bwd_pre_f32",    "bwd_dq_f32",   "bwd_dkv_f32",    "selftest_timeout", "decode",
        "layernorm_bf16", "gemm_bf16_sm100"};
    if (kernel_id < 0 || kernel_id >= kKNumKernels) return "unknown";
    return names[kernel_id];
}

unsigned long long gptattn_launch_count(void) { return g_launches.load(); }

gptattn_status gptattn_selftest_wait_timeout(unsigned long long budget_ns, gptattn_stream_t stream) {
    if (budget_ns < 1000ull || budget_ns > 2000000000ull) return GPTATTN_ERR_INVALID_ARG;
    int *status = nullptr;
    if (cudaError_t es = status_ptr(&status)) return from_cuda(es);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const DevCtx ctx{status, budget_ns};
    return from_cuda(run_kernel(kKSelftest, s, [&] { return launch_selftest_timeout(ctx, s); }));
}

gptattn_status gptattn_selftest_exp2(const float *x, float *y, int n, gptattn_stream_t stream) {
    if (n < 0) return GPTATTN_ERR_INVALID_ARG;
    if (n == 0) return GPTATTN_OK;
    if (!x || !y || (reinterpret_cast<uintptr_t>(x) & 3u) || (reinterpret_cast<uintptr_t>(y) & 3u))
        return GPTATTN_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return from_cuda(run_kernel(kKSelftest, s, [&] { return launch_selftest_exp2(x, y, n, s); }));
}

}  // extern "C"
