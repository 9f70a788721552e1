"""ctypes binding of libgptattn (include/gptattn.h): same function names, argument
marshalling only.  Every step of the attention runs inside the library's CUDA
kernels; there is no Python or CPU fallback.  If the shared library is missing
or fails to load, the first call raises ``LibraryNotBuilt``.

Pointer arguments accept an ``int`` address, ``None`` (NULL) or a ``torch.Tensor``
(its ``data_ptr()``); stream arguments accept an ``int`` handle, ``None`` (legacy
default stream) or a ``torch.cuda.Stream``.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgptattn.so")

GPTATTN_OK = 0
GPTATTN_ERR_INVALID_ARG = 1
GPTATTN_ERR_UNSUPPORTED = 2
GPTATTN_ERR_CUDA = 3
GPTATTN_ERR_TIMEOUT = 4
GPTATTN_ERR_WORKSPACE = 5

GPTATTN_F32 = 0
GPTATTN_BF16 = 1

# Every symbol include/gptattn.h declares.
EXPORTED = (
    "gptattn_fwd", "gptattn_fwd_window", "gptattn_bwd_window", "gptattn_bwd_det_workspace_bytes", "gptattn_bwd_det",
    "gptattn_fwd_opts", "gptattn_bwd_opts_workspace_bytes", "gptattn_bwd_opts", "gptattn_decode", "gptattn_bwd_workspace_bytes", "gptattn_bwd", "gptattn_get_device_status",
    "gptattn_status_string", "gptattn_version", "gptattn_profile_enable", "gptattn_profile_read",
    "gptattn_kernel_name", "gptattn_launch_count", "gptattn_selftest_wait_timeout", "gptattn_bwd_noalloc",
    "gptattn_last_error_string", "gptattn_layernorm", "gptattn_linear", "gptattn_attn_block_fwd",
    "gptattn_selftest_exp2",
)


class Options(ctypes.Structure):
    """gptattn_options: window (0 = causal), dropout_p, dropout_seed, deterministic."""
    _fields_ = [("window", ctypes.c_int), ("dropout_p", ctypes.c_float), ("dropout_seed", ctypes.c_ulonglong),
                ("deterministic", ctypes.c_int)]


class LibraryNotBuilt(RuntimeError):
    pass


class GptAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status == GPTATTN_ERR_CUDA:
            try:
                detail = f": {gptattn_last_error_string()}"
            except LibraryNotBuilt:
                pass
        super().__init__(f"{where}: {status_string(status)}{detail} (status {status})")


_lock = threading.Lock()
_lib = None


def lib():
    """Load libgptattn.so (once)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise LibraryNotBuilt(
                    f"{LIB_PATH} is missing: build it with `python -m causal_self_attention_gptattn_b200.build`")
            try:
                L = ctypes.CDLL(LIB_PATH)
            except OSError as e:
                raise LibraryNotBuilt(f"cannot load {LIB_PATH}: {e}") from e
            vp, i, sz, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
            L.gptattn_fwd.argtypes = [vp, vp, vp, i, i, i, i, i, st]
            L.gptattn_fwd.restype = i
            L.gptattn_fwd_window.argtypes = [vp, vp, vp, i, i, i, i, i, i, st]
            L.gptattn_fwd_window.restype = i
            L.gptattn_bwd_window.argtypes = [vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, i, st]
            L.gptattn_bwd_window.restype = i
            L.gptattn_bwd_det_workspace_bytes.argtypes = [i, i, i, i, i]
            L.gptattn_bwd_det_workspace_bytes.restype = sz
            L.gptattn_bwd_det.argtypes = [vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, i, st]
            L.gptattn_bwd_det.restype = i
            op = ctypes.POINTER(Options)
            L.gptattn_fwd_opts.argtypes = [vp, vp, vp, i, i, i, i, op, i, st]
            L.gptattn_fwd_opts.restype = i
            L.gptattn_bwd_opts_workspace_bytes.argtypes = [i, i, i, i, op, i]
            L.gptattn_bwd_opts_workspace_bytes.restype = sz
            L.gptattn_bwd_opts.argtypes = [vp, vp, vp, vp, vp, vp, sz, i, i, i, i, op, i, st]
            L.gptattn_bwd_opts.restype = i
            L.gptattn_decode.argtypes = [vp, vp, vp, i, i, i, i, i, i, st]
            L.gptattn_decode.restype = i
            L.gptattn_layernorm.argtypes = [vp, vp, vp, vp, i, i, i, st]
            L.gptattn_layernorm.restype = i
            L.gptattn_linear.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, st]
            L.gptattn_linear.restype = i
            L.gptattn_attn_block_fwd.argtypes = [vp] * 11 + [i, i, i, i, i, st]
            L.gptattn_attn_block_fwd.restype = i
            L.gptattn_bwd_workspace_bytes.argtypes = [i, i, i, i, i]
            L.gptattn_bwd_workspace_bytes.restype = sz
            L.gptattn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, st]
            L.gptattn_bwd.restype = i
            L.gptattn_get_device_status.argtypes = [st]
            L.gptattn_get_device_status.restype = i
            L.gptattn_status_string.argtypes = [i]
            L.gptattn_status_string.restype = ctypes.c_char_p
            L.gptattn_version.argtypes = []
            L.gptattn_version.restype = i
            L.gptattn_profile_enable.argtypes = [i]
            L.gptattn_profile_enable.restype = i
            L.gptattn_profile_read.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_float), i]
            L.gptattn_profile_read.restype = i
            L.gptattn_kernel_name.argtypes = [i]
            L.gptattn_kernel_name.restype = ctypes.c_char_p
            L.gptattn_launch_count.argtypes = []
            L.gptattn_launch_count.restype = ctypes.c_ulonglong
            L.gptattn_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, st]
            L.gptattn_selftest_wait_timeout.restype = i
            L.gptattn_selftest_exp2.argtypes = [vp, vp, i, st]
            L.gptattn_selftest_exp2.restype = i
            L.gptattn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, st]
            L.gptattn_bwd_noalloc.restype = i
            L.gptattn_last_error_string.argtypes = []
            L.gptattn_last_error_string.restype = ctypes.c_char_p
            _lib = L
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def gptattn_fwd(qkv, y, lse, B, T, C, n_head, dt, stream=None) -> int:
    return lib().gptattn_fwd(_ptr(qkv), _ptr(y), _ptr(lse), B, T, C, n_head, dt, _stream(stream))


def gptattn_fwd_window(qkv, y, lse, B, T, C, n_head, window, dt, stream=None) -> int:
    return lib().gptattn_fwd_window(_ptr(qkv), _ptr(y), _ptr(lse), B, T, C, n_head, window, dt, _stream(stream))


def gptattn_bwd_window(qkv, y, lse, dy, dqkv, workspace, workspace_bytes, B, T, C, n_head, window, dt,
                       stream=None) -> int:
    return lib().gptattn_bwd_window(_ptr(qkv), _ptr(y), _ptr(lse), _ptr(dy), _ptr(dqkv), _ptr(workspace),
                                    workspace_bytes, B, T, C, n_head, window, dt, _stream(stream))


def gptattn_bwd_det_workspace_bytes(B, T, C, n_head, dt) -> int:
    return lib().gptattn_bwd_det_workspace_bytes(B, T, C, n_head, dt)


def gptattn_bwd_det(qkv, y, lse, dy, dqkv, workspace, workspace_bytes, B, T, C, n_head, window, dt,
                    stream=None) -> int:
    return lib().gptattn_bwd_det(_ptr(qkv), _ptr(y), _ptr(lse), _ptr(dy), _ptr(dqkv), _ptr(workspace),
                                 workspace_bytes, B, T, C, n_head, window, dt, _stream(stream))


def _opts(opts):
    return None if opts is None else ctypes.byref(opts)


def gptattn_fwd_opts(qkv, y, lse, B, T, C, n_head, opts, dt, stream=None) -> int:
    return lib().gptattn_fwd_opts(_ptr(qkv), _ptr(y), _ptr(lse), B, T, C, n_head, _opts(opts), dt, _stream(stream))


def gptattn_bwd_opts_workspace_bytes(B, T, C, n_head, opts, dt) -> int:
    return lib().gptattn_bwd_opts_workspace_bytes(B, T, C, n_head, _opts(opts), dt)


def gptattn_bwd_opts(qkv, y, lse, dy, dqkv, workspace, workspace_bytes, B, T, C, n_head, opts, dt,
                     stream=None) -> int:
    return lib().gptattn_bwd_opts(_ptr(qkv), _ptr(y), _ptr(lse), _ptr(dy), _ptr(dqkv), _ptr(workspace),
                                  workspace_bytes, B, T, C, n_head, _opts(opts), dt, _stream(stream))


def gptattn_decode(qkv, y, lse, B, T, T_cap, C, n_head, dt, stream=None) -> int:
    return lib().gptattn_decode(_ptr(qkv), _ptr(y), _ptr(lse), B, T, T_cap, C, n_head, dt, _stream(stream))


def gptattn_layernorm(x, w, b, out, M, C, dt, stream=None) -> int:
    return lib().gptattn_layernorm(_ptr(x), _ptr(w), _ptr(b), _ptr(out), M, C, dt, _stream(stream))


def gptattn_linear(a, w, bias, resid, out, M, N, K, dt, stream=None) -> int:
    return lib().gptattn_linear(_ptr(a), _ptr(w), _ptr(bias), _ptr(resid), _ptr(out), M, N, K, dt, _stream(stream))


def gptattn_attn_block_fwd(x, ln_w, ln_b, w_attn, b_attn, w_proj, b_proj, qkv, y, lse, out, B, T, C, n_head, dt,
                           stream=None) -> int:
    return lib().gptattn_attn_block_fwd(_ptr(x), _ptr(ln_w), _ptr(ln_b), _ptr(w_attn), _ptr(b_attn), _ptr(w_proj),
                                        _ptr(b_proj), _ptr(qkv), _ptr(y), _ptr(lse), _ptr(out), B, T, C, n_head, dt,
                                        _stream(stream))


def gptattn_bwd_workspace_bytes(B, T, C, n_head, dt) -> int:
    return lib().gptattn_bwd_workspace_bytes(B, T, C, n_head, dt)


def gptattn_bwd(qkv, y, lse, dy, dqkv, workspace, workspace_bytes, B, T, C, n_head, dt, stream=None) -> int:
    return lib().gptattn_bwd(_ptr(qkv), _ptr(y), _ptr(lse), _ptr(dy), _ptr(dqkv), _ptr(workspace),
                             workspace_bytes, B, T, C, n_head, dt, _stream(stream))


def gptattn_bwd_noalloc(qkv, y, lse, dy, dqkv, B, T, C, n_head, dt, stream=None) -> int:
    """gptattn_bwd without a workspace argument, for callers that cannot allocate:
    the scratch is a fixed 64 MiB array inside the library (shared by all calls,
    so calls must not overlap on the GPU)."""
    return lib().gptattn_bwd_noalloc(_ptr(qkv), _ptr(y), _ptr(lse), _ptr(dy), _ptr(dqkv), B, T, C, n_head, dt,
                                     _stream(stream))


GPTATTN_NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


def gptattn_get_device_status(stream=None) -> int:
    return lib().gptattn_get_device_status(_stream(stream))


def gptattn_status_string(status: int) -> str:
    return lib().gptattn_status_string(status).decode()


def status_string(status: int) -> str:
    try:
        return gptattn_status_string(status)
    except LibraryNotBuilt:
        return f"status {status}"


def gptattn_last_error_string() -> str:
    return lib().gptattn_last_error_string().decode()


def gptattn_version() -> int:
    return lib().gptattn_version()


def gptattn_profile_enable(max_records: int) -> int:
    return lib().gptattn_profile_enable(max_records)


def gptattn_profile_read(capacity: int = 4096):
    """Return a list of (kernel_name, milliseconds), oldest first."""
    ids = (ctypes.c_int * capacity)()
    ms = (ctypes.c_float * capacity)()
    n = lib().gptattn_profile_read(ids, ms, capacity)
    return [(gptattn_kernel_name(ids[k]), ms[k]) for k in range(n)]


def gptattn_kernel_name(kernel_id: int) -> str:
    return lib().gptattn_kernel_name(kernel_id).decode()


def gptattn_launch_count() -> int:
    return lib().gptattn_launch_count()


def gptattn_selftest_wait_timeout(budget_ns: int, stream=None) -> int:
    return lib().gptattn_selftest_wait_timeout(budget_ns, _stream(stream))


def gptattn_selftest_exp2(x, y, n: int, stream=None) -> int:
    return lib().gptattn_selftest_exp2(_ptr(x), _ptr(y), n, _stream(stream))


def check(status: int, where: str) -> None:
    if status != GPTATTN_OK:
        raise GptAttnError(status, where)
