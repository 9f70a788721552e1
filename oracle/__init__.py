"""fp64 CPU oracle for causal multi-head self-attention (forward + backward).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only users.  The product path (the
CUDA library and its Python binding) never imports this package, and this
package imports nothing from the product.

The arithmetic lives in ``gptattn_oracle.c`` (plain loops in IEEE double, one
(batch, head) pair per OpenMP thread); this module only compiles it with gcc
and marshals numpy arrays.  See the C file's header for the passages of the
lecture page ("Let's build GPT: from scratch, in code, spelled out") that
each step follows.

Parity status: every function here is pinned by ``tests/test_oracle.py``
(closed forms, invariants, finite differences, a library special case and the
worked fixtures under ``tests/golden/``); the dropout generator (Philox4x32-10)
is pinned by its published known-answer vectors
(``tests/golden/philox4x32_10_kat.json``), its statistics and every use of the
mask.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "gptattn_oracle.c")
_LIB = os.path.join(_HERE, "libgptattn_oracle.so")
_lock = threading.Lock()
_default = None


def compile_source(src_path: str, out_path: str) -> str:
    """Compile an oracle C source into a shared library (gcc, OpenMP)."""
    tmp = out_path + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra",
           "-o", tmp, src_path, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out_path)
    return out_path


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libgptattn_oracle.so``."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(SOURCE):
        compile_source(SOURCE, _LIB)
    return _LIB


def _f64(a) -> np.ndarray:
    """Accept numpy arrays or CPU torch tensors; return a C-contiguous float64 array."""
    if hasattr(a, "detach"):
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _shape(qkv: np.ndarray, n_head: int):
    if qkv.ndim != 3 or qkv.shape[2] % 3 != 0:
        raise ValueError(f"qkv must be [B, T, 3C], got {qkv.shape}")
    B, T, C3 = qkv.shape
    C = C3 // 3
    if n_head <= 0 or C % n_head != 0:
        raise ValueError(f"C={C} is not divisible by n_head={n_head}")
    return B, T, C


class Oracle:
    """numpy front end of one compiled oracle library."""

    def __init__(self, so_path: str):
        lib = ctypes.CDLL(so_path)
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        lib.oracle_fwd.argtypes = [dp, i, i, i, i, dp, dp]
        lib.oracle_fwd.restype = i
        lib.oracle_bwd.argtypes = [dp, dp, i, i, i, i, dp]
        lib.oracle_bwd.restype = i
        lib.oracle_probs.argtypes = [dp, i, i, i, i, i, i, dp]
        lib.oracle_probs.restype = i
        lib.oracle_fwd_window.argtypes = [dp, i, i, i, i, i, dp, dp]
        lib.oracle_fwd_window.restype = i
        lib.oracle_bwd_window.argtypes = [dp, dp, i, i, i, i, i, dp]
        lib.oracle_bwd_window.restype = i
        lib.oracle_probs_window.argtypes = [dp, i, i, i, i, i, i, i, dp]
        lib.oracle_probs_window.restype = i
        u64 = ctypes.c_uint64
        lib.oracle_fwd_ex.argtypes = [dp, i, i, i, i, i, ctypes.c_double, u64, dp, dp]
        lib.oracle_fwd_ex.restype = i
        lib.oracle_bwd_ex.argtypes = [dp, dp, i, i, i, i, i, ctypes.c_double, u64, dp]
        lib.oracle_bwd_ex.restype = i
        u32p = ctypes.POINTER(ctypes.c_uint32)
        lib.oracle_philox4x32_10.argtypes = [u32p, u32p, u32p]
        lib.oracle_philox4x32_10.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = i
        lib.oracle_set_num_threads.argtypes = [i]
        lib.oracle_set_num_threads.restype = None
        self.lib = lib
        self.path = so_path

    def num_threads(self) -> int:
        return self.lib.oracle_num_threads()

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(int(n))

    def forward(self, qkv, n_head: int, window=None, dropout: float = 0.0, seed: int = 0):
        """Return (y[B,T,C], lse[B,n_head,T]) in float64.  window: local band width
        (token t sees t-window < s <= t); None = causal (every past position).
        dropout: probability of dropping an attention weight (Philox mask from seed)."""
        q = _f64(qkv)
        B, T, C = _shape(q, n_head)
        y = np.zeros((B, T, C), dtype=np.float64)
        lse = np.zeros((B, n_head, T), dtype=np.float64)
        if dropout > 0.0:
            w = max(T, 1) if window is None else int(window)
            rc = self.lib.oracle_fwd_ex(_ptr(q), B, T, C, n_head, w, float(dropout), int(seed), _ptr(y), _ptr(lse))
        elif window is None:
            rc = self.lib.oracle_fwd(_ptr(q), B, T, C, n_head, _ptr(y), _ptr(lse))
        else:
            rc = self.lib.oracle_fwd_window(_ptr(q), B, T, C, n_head, int(window), _ptr(y), _ptr(lse))
        if rc:
            raise RuntimeError(f"oracle_fwd failed with code {rc}")
        return y, lse

    def backward(self, qkv, dy, n_head: int, window=None, dropout: float = 0.0, seed: int = 0):
        """Return dqkv[B,T,3C] = d(sum(y*dy))/d(qkv) in float64 (window, dropout, seed as in forward)."""
        q = _f64(qkv)
        g = _f64(dy)
        B, T, C = _shape(q, n_head)
        if g.shape != (B, T, C):
            raise ValueError(f"dy must be {(B, T, C)}, got {g.shape}")
        dqkv = np.zeros((B, T, 3 * C), dtype=np.float64)
        if dropout > 0.0:
            w = max(T, 1) if window is None else int(window)
            rc = self.lib.oracle_bwd_ex(_ptr(q), _ptr(g), B, T, C, n_head, w, float(dropout), int(seed), _ptr(dqkv))
        elif window is None:
            rc = self.lib.oracle_bwd(_ptr(q), _ptr(g), B, T, C, n_head, _ptr(dqkv))
        else:
            rc = self.lib.oracle_bwd_window(_ptr(q), _ptr(g), B, T, C, n_head, int(window), _ptr(dqkv))
        if rc:
            raise RuntimeError(f"oracle_bwd failed with code {rc}")
        return dqkv

    def philox(self, ctr, key):
        """Philox4x32-10 of a 4-word counter under a 2-word key (four uint32 words)."""
        c = (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in ctr])
        k = (ctypes.c_uint32 * 2)(*[int(x) & 0xFFFFFFFF for x in key])
        o = (ctypes.c_uint32 * 4)()
        self.lib.oracle_philox4x32_10(c, k, o)
        return [int(x) for x in o]

    def probs(self, qkv, n_head: int, b: int, h: int, window=None):
        """Return the T x T attention weights of batch b, head h (window as in forward)."""
        q = _f64(qkv)
        B, T, C = _shape(q, n_head)
        P = np.zeros((T, T), dtype=np.float64)
        if window is None:
            rc = self.lib.oracle_probs(_ptr(q), B, T, C, n_head, int(b), int(h), _ptr(P))
        else:
            rc = self.lib.oracle_probs_window(_ptr(q), B, T, C, n_head, int(window), int(b), int(h), _ptr(P))
        if rc:
            raise RuntimeError(f"oracle_probs failed with code {rc}")
        return P


def default() -> Oracle:
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def num_threads() -> int:
    return default().num_threads()


def set_num_threads(n: int) -> None:
    default().set_num_threads(n)


def forward(qkv, n_head: int, window=None, dropout: float = 0.0, seed: int = 0):
    return default().forward(qkv, n_head, window, dropout, seed)


def backward(qkv, dy, n_head: int, window=None, dropout: float = 0.0, seed: int = 0):
    return default().backward(qkv, dy, n_head, window, dropout, seed)


def philox(ctr, key):
    return default().philox(ctr, key)


def probs(qkv, n_head: int, b: int, h: int, window=None):
    return default().probs(qkv, n_head, b, h, window)
