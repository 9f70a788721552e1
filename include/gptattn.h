/*
 * gptattn.h -- C ABI of libgptattn: batched multi-head causal scaled
 * dot-product self-attention, forward and backward, on NVIDIA B200 (sm_100a).
 *
 * The operation (lecture page "Let's build GPT: from scratch, in code, spelled
 * out", chapters "version 4: self-attention", "multi-headed self-attention",
 * note 6 and the two corrections; exercise EX1 for heads as a batch dimension):
 *
 *     for every batch b and head h, with q, k, v the head's slices of qkv,
 *     S[t][s] = q_t . k_s / sqrt(hs)      for s <= t   (the future is masked)
 *     P[t][:] = softmax(S[t][:])          over the visible s <= t
 *     y_t     = sum_s P[t][s] v_s
 *     lse[t]  = ln sum_{s<=t} exp(S[t][s])   (natural log)
 *
 * Layout (all row-major, contiguous, no padding):
 *     qkv  [B][T][3C]  q = columns [0,C), k = [C,2C), v = [2C,3C); head h owns
 *                      columns [h*hs, (h+1)*hs) of each part (hs = C/n_head).
 *                      This is the output of a GPT-2 block's c_attn projection.
 *     y    [B][T][C]   heads concatenated back in the same column order.
 *     lse  [B][n_head][T]  float32 always.  The forward entry points (and
 *          gptattn_decode, gptattn_attn_block_fwd) accept lse == NULL for
 *          inference, when no backward follows: it is then not written.
 *     dy   [B][T][C], dqkv [B][T][3C]: same layouts as y and qkv.
 *
 * Element types: GPTATTN_BF16 -> qkv, y, dy, dqkv are bfloat16 (tensor-core
 * path, fp32 softmax and accumulation); GPTATTN_F32 -> they are float32 (fp32
 * CUDA-core path).  lse and the workspace are float32 in both cases.
 *
 * Supported head sizes: bf16 hs in {64, 128}; f32 hs in {16, 32, 64, 128}.
 * Scale is fixed at 1/sqrt(hs).  gptattn_fwd / gptattn_bwd are causal without
 * dropout; the _window, _det and _opts entry points below add a local window,
 * a deterministic backward and dropout on the attention weights.
 *
 * Ownership and synchronisation: every pointer is a caller-owned DEVICE
 * pointer on the current CUDA device, 16-byte aligned.  The library never
 * allocates device memory per call; the backward's scratch is the caller's
 * `workspace`.  Calls enqueue kernels on `stream` and return without
 * synchronising (stream may be NULL for the legacy default stream).  Output
 * buffers must not overlap inputs.
 *
 * Errors: arguments are validated on the host before anything is enqueued;
 * an invalid call returns a non-zero status and enqueues nothing.  A launch
 * failure returns GPTATTN_ERR_CUDA.  Kernels never trap: every internal wait
 * is bounded, and a wait that runs out makes the kernel record
 * GPTATTN_ERR_TIMEOUT in a device status word and return early (outputs are
 * then undefined); gptattn_get_device_status() reads and clears that word.
 * B == 0 or T == 0 is a valid empty call: it returns GPTATTN_OK and touches
 * nothing (pointers may then be NULL).
 */
#ifndef GPTATTN_H
#define GPTATTN_H

#include <stddef.h>

/* Only the entry points below are exported from libgptattn.so. */
#if defined(__GNUC__)
#define GPTATTN_API __attribute__((visibility("default")))
#else
#define GPTATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st *gptattn_stream_t;

typedef enum gptattn_status {
    GPTATTN_OK = 0,
    GPTATTN_ERR_INVALID_ARG = 1,  /* negative size, NULL or misaligned pointer, C % n_head != 0 */
    GPTATTN_ERR_UNSUPPORTED = 2,  /* head size or dtype outside the supported set */
    GPTATTN_ERR_CUDA = 3,         /* a CUDA runtime/driver call or a launch failed (no device included) */
    GPTATTN_ERR_TIMEOUT = 4,      /* a kernel's bounded wait ran out (reported by get_device_status) */
    GPTATTN_ERR_WORKSPACE = 5     /* workspace NULL/misaligned or smaller than gptattn_bwd_workspace_bytes */
} gptattn_status;

typedef enum gptattn_dtype {
    GPTATTN_F32 = 0,
    GPTATTN_BF16 = 1
} gptattn_dtype;

/* Forward.  Reads qkv; writes y and lse.
 * Causal self-attention forward as defined at the top of this file
 * ("version 4: self-attention" with the causal mask and 1/sqrt(hs) scale). */
GPTATTN_API gptattn_status gptattn_fwd(const void *qkv, void *y, float *lse,
                           int B, int T, int C, int n_head,
                           gptattn_dtype dt, gptattn_stream_t stream);

/* Local-window (banded) variants of gptattn_fwd / gptattn_bwd: token t sees
 * only positions t-window < s <= t (itself and the window-1 before it), the
 * locally banded attention that the minGPT README page's reference notes on
 * GPT-3 describe alternating with dense layers.  window >= 1; window >= T is
 * exactly the causal operation (the same kernels and results as gptattn_fwd /
 * gptattn_bwd).  Key tiles outside every query tile's band are skipped.
 * Supported: every head size of gptattn_fwd, any window.
 * window < 1 -> GPTATTN_ERR_INVALID_ARG.  Other arguments, layouts, the
 * workspace (gptattn_bwd_workspace_bytes) and errors as in gptattn_fwd /
 * gptattn_bwd; the backward takes the y and lse of the windowed forward. */
GPTATTN_API gptattn_status gptattn_fwd_window(const void *qkv, void *y, float *lse,
                                  int B, int T, int C, int n_head, int window,
                                  gptattn_dtype dt, gptattn_stream_t stream);
GPTATTN_API gptattn_status gptattn_bwd_window(const void *qkv, const void *y, const float *lse, const void *dy,
                                  void *dqkv, void *workspace, size_t workspace_bytes,
                                  int B, int T, int C, int n_head, int window,
                                  gptattn_dtype dt, gptattn_stream_t stream);

/* Deterministic backward (no counterpart on the pages beyond the operation:
 * a reproducibility variant of gptattn_bwd_window).  gptattn_bwd adds each
 * key tile's contribution to dQ into an fp32 accumulator with reduce-adds
 * whose order varies from run to run, so its bf16 dq can differ in the last
 * bit between runs.  This variant stores every (query tile, key tile) partial
 * of dQ in a workspace slot of its own and sums a query tile's partials in a
 * fixed order, so equal inputs give bit-identical dqkv on every run.  Same
 * arguments, semantics, support (every head size, any window) and
 * errors as gptattn_bwd_window, with a larger workspace:
 * gptattn_bwd_det_workspace_bytes() (for bf16 it adds B * n_head *
 * ceil(T/128)(ceil(T/128)+1)/2 tiles of 128 x 64 fp32; (size_t)-1 for an
 * unsupported or invalid shape).  The fp32 path has no reduce-adds and is
 * deterministic in both entry points. */
GPTATTN_API size_t gptattn_bwd_det_workspace_bytes(int B, int T, int C, int n_head, gptattn_dtype dt);
GPTATTN_API gptattn_status gptattn_bwd_det(const void *qkv, const void *y, const float *lse, const void *dy,
                               void *dqkv, void *workspace, size_t workspace_bytes,
                               int B, int T, int C, int n_head, int window,
                               gptattn_dtype dt, gptattn_stream_t stream);

/* Options for the general entry points below.  A zero-initialised struct (or
 * a NULL pointer) is the plain causal call of gptattn_fwd / gptattn_bwd.
 *   window        0: causal; > 0: local window as in gptattn_fwd_window; < 0: invalid.
 *   dropout_p     probability of dropping an attention weight, 0 <= p < 1 (else
 *                 GPTATTN_ERR_INVALID_ARG).  Inverted dropout on the weights after
 *                 the softmax (the lecture page's chapter "scaling up the model! ...
 *                 adding dropout"); lse stays the logsumexp of the undropped
 *                 scores.  p is applied in steps of 1/256: with theta = round(256 p)
 *                 (at most 255) a weight is dropped with probability theta/256 and
 *                 a kept one is scaled by 1/(1 - theta/256); p < 1/512 drops
 *                 nothing.  One Philox4x32-10 call (Salmon et al., SC 2011) covers
 *                 a 4 x 4 block of (query t, key s) pairs of batch b, head h:
 *                 counter (s/4, t/4, b*n_head+h, 0) under key (seed & 0xffffffff,
 *                 seed >> 32); weight (t, s) is kept iff byte s%4 (least
 *                 significant first) of output word t%4 is >= theta.  The backward
 *                 must get the forward's seed and p.
 *   dropout_seed  the 64-bit Philox key.
 *   deterministic backward only: bit-identical results as gptattn_bwd_det (and
 *                 its workspace size). */
typedef struct gptattn_options {
    int window;
    float dropout_p;
    unsigned long long dropout_seed;
    int deterministic;
} gptattn_options;

GPTATTN_API gptattn_status gptattn_fwd_opts(const void *qkv, void *y, float *lse,
                                int B, int T, int C, int n_head, const gptattn_options *opts,
                                gptattn_dtype dt, gptattn_stream_t stream);
/* Workspace for gptattn_bwd_opts with these options ((size_t)-1 if unsupported/invalid). */
GPTATTN_API size_t gptattn_bwd_opts_workspace_bytes(int B, int T, int C, int n_head, const gptattn_options *opts,
                                                    gptattn_dtype dt);
GPTATTN_API gptattn_status gptattn_bwd_opts(const void *qkv, const void *y, const float *lse, const void *dy,
                                void *dqkv, void *workspace, size_t workspace_bytes,
                                int B, int T, int C, int n_head, const gptattn_options *opts,
                                gptattn_dtype dt, gptattn_stream_t stream);

/* Decode: attention of the last position over a key/value cache (no
 * counterpart on the pages beyond the operation itself: it is row T-1 of
 * gptattn_fwd, the only row the pages' generate loop reads, computed without
 * the other rows).  For every batch b and head h, with q the head's query of
 * position T-1 and k_s, v_s its keys and values of positions 0..T-1 (all
 * visible to the last position):
 *     y[b][h*hs + d] = sum_s P[s] v_s[d],  P = softmax_s(q . k_s / sqrt(hs)),
 *     lse[b][h]      = ln sum_s exp(q . k_s / sqrt(hs)).
 * The cache is a packed qkv buffer [B][T_cap][3C] (same column layout as
 * gptattn_fwd's qkv, batch stride T_cap rows) of which rows 0..T-1 are read;
 * y is [B][C] (dtype dt), lse is [B][n_head] float32.  T_cap >= T; B * n_head
 * <= 65535.  Same dtypes, head sizes, pointer rules and error codes as
 * gptattn_fwd; B == 0 or T == 0 is a valid empty call.  Memory-bound; it reads
 * each key and value row once and allocates nothing. */
GPTATTN_API gptattn_status gptattn_decode(const void *qkv, void *y, float *lse,
                              int B, int T, int T_cap, int C, int n_head,
                              gptattn_dtype dt, gptattn_stream_t stream);

/* Bytes of device scratch gptattn_bwd needs for this shape (0 for an empty
 * shape; (size_t)-1 for an invalid one).  Pure host function.  No counterpart
 * on the pages: the scratch (per-row softmax statistics and an fp32 dQ
 * accumulator) belongs to this library's backward design, not to the method. */
GPTATTN_API size_t gptattn_bwd_workspace_bytes(int B, int T, int C, int n_head, gptattn_dtype dt);

/* Backward.  Given the forward's qkv, y and lse and the incoming gradient dy,
 * writes dqkv = d(sum(y o dy))/d(qkv) (chain rule through the weighted sum, the
 * row softmax and the scaled dot products; same packing as qkv).  `workspace`
 * is caller-owned device scratch of at least gptattn_bwd_workspace_bytes(...)
 * bytes, 256-byte aligned; its contents on entry are ignored and on return are
 * undefined.  Two calls that run concurrently need separate workspaces. */
GPTATTN_API gptattn_status gptattn_bwd(const void *qkv, const void *y, const float *lse, const void *dy,
                           void *dqkv, void *workspace, size_t workspace_bytes,
                           int B, int T, int C, int n_head,
                           gptattn_dtype dt, gptattn_stream_t stream);

/* Backward for callers that cannot allocate device memory (no counterpart on
 * the pages: it is a packaging variant of gptattn_bwd, not part of the
 * method).  Some callers have no allocator to call -- e.g. a plugin inside
 * another runtime that owns all device memory -- or must not call cudaMalloc
 * on their path, since it can synchronise the device.  This entry point takes
 * the same arguments as gptattn_bwd minus the workspace: the scratch comes
 * from one array of GPTATTN_NOALLOC_SCRATCH_BYTES (64 MiB) compiled into the
 * library.  The array is a module global of the library's device code: with
 * CUDA's default lazy module loading a device gets it when this entry point's
 * first call on that device loads the module (so that first call does extra
 * work), with eager loading (CUDA_MODULE_LOADING=EAGER) when the library's
 * device code is loaded; either way the device holds it until the process
 * exits.  The caller still owns and passes every input and output.
 * Returns GPTATTN_ERR_WORKSPACE, enqueueing nothing, when the shape needs more
 * scratch than that (gptattn_bwd_workspace_bytes(...) > 64 MiB).  It allocates
 * nothing: no cudaMalloc, cudaFree or allocating library routine.
 * The first call on each device looks up the array's device address (with that
 * device current), loading the module if needed, and caches it; make that
 * first call before any stream capture.  All calls share the one array and it keeps the previous call's
 * contents (the backward re-initialises what it needs); calls whose work
 * overlaps on the GPU -- on two streams or from two host threads -- race on it
 * and produce wrong results, so serialise them. */
#define GPTATTN_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
GPTATTN_API gptattn_status gptattn_bwd_noalloc(const void *qkv, const void *y, const float *lse, const void *dy,
                                               void *dqkv, int B, int T, int C, int n_head,
                                               gptattn_dtype dt, gptattn_stream_t stream);

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device: GPTATTN_OK, GPTATTN_ERR_TIMEOUT if a kernel gave up on
 * a wait since the last call, or GPTATTN_ERR_CUDA if the stream reports an
 * error.  No counterpart on the pages: error reporting of this library. */
GPTATTN_API gptattn_status gptattn_get_device_status(gptattn_stream_t stream);

/* Static human-readable name of a status code (no counterpart on the pages). */
GPTATTN_API const char *gptattn_status_string(gptattn_status s);

/* Text of the last CUDA error that made a call on this host thread return
 * GPTATTN_ERR_CUDA ("no error" if none yet).  Static string.  No counterpart
 * on the pages. */
GPTATTN_API const char *gptattn_last_error_string(void);

/* Library version, major * 10000 + minor * 100 + patch (no counterpart on the
 * pages). */
GPTATTN_API int gptattn_version(void);

/* ---- The attention sub-block of a pre-LN GPT block (bf16 only) ------------
 * minGPT README page ("卡帕西(氏)MinGPT"), GPT-2 notes: the layer norm sits at
 * the input of each sub-block; lecture page ("Let's build GPT: from scratch, in
 * code, spelled out"), chapters "multi-headed self-attention", "residual
 * connections" and "layernorm (and its relationship to our previous
 * batchnorm)".  Linear weights use nn.Linear's layout, [out_features]
 * [in_features] row-major.  All buffers are device memory owned by the caller,
 * 16-byte aligned; nothing is allocated.  dt must be GPTATTN_BF16 (else
 * GPTATTN_ERR_UNSUPPORTED).
 *
 * gptattn_layernorm: out[m][:] = (x[m][:] - mean) / sqrt(var + 1e-5) * w + b for
 *   each of the M rows of x[M][C] (population variance over the C features,
 *   fp32 statistics); w, b are [C].  C % 8 == 0 and C <= 4096
 *   (GPTATTN_ERR_UNSUPPORTED otherwise); M == 0 is a valid empty call.
 *
 * gptattn_linear: out[M][N] = a[M][K] w[N][K]^T + bias[N] (+ resid[M][N]), fp32
 *   accumulation, one rounding to bf16.  bias and resid may be NULL (no term).
 *   resid may equal out (in-place residual add); a and w must not overlap out.
 *   N % 64 == 0 and K % 64 == 0 (GPTATTN_ERR_UNSUPPORTED otherwise).
 *
 * gptattn_attn_block_fwd: for x[B][T][C],
 *     qkv = LN(x) w_attn^T + b_attn          (w_attn [3C][C], b_attn [3C])
 *     y, lse = gptattn_fwd(qkv)              (causal, as above)
 *     out = x + y w_proj^T + b_proj          (w_proj [C][C], b_proj [C])
 *   qkv [B][T][3C], y [B][T][C], lse [B][n_head][T] (float32) and out
 *   [B][T][C] are all written (qkv, y, lse are what a backward needs); y also
 *   holds LN(x) between the first two steps, so no scratch is needed.  out may
 *   equal x.  Shape rules are gptattn_fwd's (head size 64 or 128) plus the two
 *   functions above; B*T < 2^31. */
GPTATTN_API gptattn_status gptattn_layernorm(const void *x, const void *w, const void *b, void *out, int M, int C,
                                             gptattn_dtype dt, gptattn_stream_t stream);
GPTATTN_API gptattn_status gptattn_linear(const void *a, const void *w, const void *bias, const void *resid,
                                          void *out, int M, int N, int K, gptattn_dtype dt,
                                          gptattn_stream_t stream);
GPTATTN_API gptattn_status gptattn_attn_block_fwd(const void *x, const void *ln_w, const void *ln_b,
                                                  const void *w_attn, const void *b_attn, const void *w_proj,
                                                  const void *b_proj, void *qkv, void *y, float *lse, void *out,
                                                  int B, int T, int C, int n_head, gptattn_dtype dt,
                                                  gptattn_stream_t stream);

/* ---- Instrumentation (no counterpart on the pages; used by the benchmark) --
 * gptattn_profile_enable(n) with n > 0 makes later calls on the current device
 * record a pair of CUDA events around each kernel they launch, keeping up to n
 * records (n = 0 turns recording off and releases the events).  Recording adds
 * two event records per launch and nothing else.
 * gptattn_profile_read() synchronises on the recorded events and copies up to
 * `capacity` (kernel id, milliseconds) pairs, oldest first; it returns the
 * number copied and clears the record list.  gptattn_kernel_name() maps a
 * kernel id to a static name.  gptattn_launch_count() is the number of kernels
 * the library has launched since it was loaded. */
GPTATTN_API gptattn_status gptattn_profile_enable(int max_records);
GPTATTN_API int gptattn_profile_read(int *kernel_ids, float *ms, int capacity);
GPTATTN_API const char *gptattn_kernel_name(int kernel_id);
GPTATTN_API unsigned long long gptattn_launch_count(void);

/* ---- Bounded-wait self-test (no counterpart on the pages) ------------------
 * Enqueues one tiny kernel that waits, with the library's bounded-wait
 * routine, on a barrier that nothing ever completes.  After `budget_ns`
 * nanoseconds the wait gives up, the kernel records GPTATTN_ERR_TIMEOUT in the
 * device status word and returns, leaving the context usable.  Used by tests
 * to show that a lost producer ends in a status code, not a hang or a trap.
 * budget_ns must be in [1000, 2000000000]. */
GPTATTN_API gptattn_status gptattn_selftest_wait_timeout(unsigned long long budget_ns, gptattn_stream_t stream);

/* ---- Exponential self-test (no counterpart on the pages) --------------------
 * The backward kernel computes part of its softmax exponentials 2^x on the FMA
 * pipe instead of the multi-function unit: x = j + f with j = round(x), 2^f by
 * a cubic fitted on [-1/2, 1/2] by weighted least squares, j added to the
 * exponent field (Cody-Waite style range reduction).  This entry point runs
 * that routine on caller data so its accuracy can be tested: y[i] = the
 * routine's 2^x[i] for i < n.  Stated behaviour: relative error below 7.6e-5
 * for -125 <= x <= 1.5; x < -125 (including -inf) gives about 2^-125 rather
 * than 0 (the kernels zero masked weights explicitly); NaN gives NaN.  x and y
 * are device float arrays (4-byte aligned, may not overlap); n < 0 or a NULL /
 * misaligned pointer -> GPTATTN_ERR_INVALID_ARG; n == 0 is a no-op.  Enqueued
 * on `stream`, no synchronisation. */
GPTATTN_API gptattn_status gptattn_selftest_exp2(const float *x, float *y, int n, gptattn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GPTATTN_H */
