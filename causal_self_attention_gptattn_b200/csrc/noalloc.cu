// noalloc.cu -- gptattn_bwd_noalloc: the backward pass for callers that cannot
// allocate device memory.
//
// gptattn_bwd needs device scratch (per-row softmax statistics and an fp32
// gradient accumulator) that its caller normally allocates.  Some callers have
// no way to do that: a plugin running inside another runtime that owns all
// device memory and hands out no allocator, or latency-critical host code that
// must not call cudaMalloc (which can synchronise the whole device).  For them
// this entry point takes its scratch from one fixed array compiled into the
// library instead.
//
// The array is a module global in device memory.  With CUDA's default lazy
// module loading a device gets it when the first call on that device looks its
// address up (which loads this file's module, so that first call does extra
// work); with eager loading, when the library's device code is loaded.  Either
// way the device holds it until the process exits.  Its host-side name is only a
// stand-in for the symbol: the device address is looked up once per device with
// cudaGetSymbolAddress (with that device current) on the first call made on
// that device, and cached.  Every call shares the array and the previous
// call's contents stay in it; the backward's first kernel rewrites every part
// of the scratch that must start at a known value (it zeroes the accumulator),
// so nothing leaks between calls.  Calls whose work overlaps on the GPU (two
// streams, or two host threads) race on the array and give wrong results.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "gptattn.h"

namespace {

constexpr size_t kScratchBytes = (size_t)GPTATTN_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_lock;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (first call per
// device does the lookup).
gptattn_status scratch_ptr(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GPTATTN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GPTATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_lock);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return GPTATTN_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return GPTATTN_OK;
}

}  // namespace

extern "C" gptattn_status gptattn_bwd_noalloc(const void *qkv, const void *y, const float *lse, const void *dy,
                                              void *dqkv, int B, int T, int C, int n_head, gptattn_dtype dt,
                                              gptattn_stream_t stream) {
    const size_t need = gptattn_bwd_workspace_bytes(B, T, C, n_head, dt);
    if (need == (size_t)-1) {
        // invalid shape: let the regular entry point report the precise status
        return gptattn_bwd(qkv, y, lse, dy, dqkv, nullptr, 0, B, T, C, n_head, dt, stream);
    }
    if (need > kScratchBytes) return GPTATTN_ERR_WORKSPACE;
    if (B == 0 || T == 0) return GPTATTN_OK;
    void *scratch = nullptr;
    const gptattn_status st = scratch_ptr(&scratch);
    if (st != GPTATTN_OK) return st;
    return gptattn_bwd(qkv, y, lse, dy, dqkv, scratch, kScratchBytes, B, T, C, n_head, dt, stream);
}
