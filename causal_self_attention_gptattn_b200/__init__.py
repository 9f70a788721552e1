"""libgptattn for NVIDIA B200: batched multi-head causal self-attention,
forward and backward, in hand-written sm_100a kernels behind a C ABI.

``gptattn``   -- the ctypes binding (same names as include/gptattn.h).
``attention`` -- a torch.autograd wrapper for users holding torch tensors:
                 ``y = attention(qkv, n_head)`` with qkv[B, T, 3C] on a CUDA
                 device (bf16 or fp32); gradients flow to qkv.  PyTorch only
                 allocates memory and supplies the stream; the kernels do the
                 arithmetic.
``workloads`` -- seeded synthetic inputs of the benchmark shapes.
"""
from __future__ import annotations

from . import gptattn  # noqa: F401

__all__ = ["gptattn", "attention", "forward", "backward"]


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return gptattn.GPTATTN_BF16
    if t.dtype == torch.float32:
        return gptattn.GPTATTN_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


def forward(qkv, n_head: int):
    """Return (y[B,T,C], lse[B,n_head,T] fp32) for a CUDA tensor qkv[B,T,3C]."""
    import torch
    if not qkv.is_cuda:
        raise ValueError("qkv must be a CUDA tensor (there is no CPU path)")
    qkv = qkv.contiguous()
    B, T, C3 = qkv.shape
    C = C3 // 3
    y = torch.empty(B, T, C, dtype=qkv.dtype, device=qkv.device)
    lse = torch.empty(B, n_head, T, dtype=torch.float32, device=qkv.device)
    st = torch.cuda.current_stream(qkv.device)
    gptattn.check(gptattn.gptattn_fwd(qkv, y, lse, B, T, C, n_head, _dtype_code(qkv), st), "gptattn_fwd")
    return y, lse


def backward(qkv, y, lse, dy, n_head: int):
    """Return dqkv[B,T,3C] given the forward's qkv, y, lse and the gradient dy."""
    import torch
    qkv, y, lse, dy = qkv.contiguous(), y.contiguous(), lse.contiguous(), dy.contiguous()
    B, T, C3 = qkv.shape
    C = C3 // 3
    dt = _dtype_code(qkv)
    dqkv = torch.empty_like(qkv)
    nbytes = gptattn.gptattn_bwd_workspace_bytes(B, T, C, n_head, dt)
    if nbytes == (1 << 64) - 1:
        raise ValueError("invalid shape for gptattn_bwd")
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=qkv.device)
    st = torch.cuda.current_stream(qkv.device)
    gptattn.check(gptattn.gptattn_bwd(qkv, y, lse, dy, dqkv, ws, nbytes, B, T, C, n_head, dt, st), "gptattn_bwd")
    return dqkv


def attention(qkv, n_head: int):
    """Causal multi-head self-attention of packed qkv[B,T,3C] -> y[B,T,C], differentiable."""
    import torch

    class _Attn(torch.autograd.Function):
        @staticmethod
        def forward(ctx, x):
            y, lse = forward(x, n_head)
            ctx.save_for_backward(x, y, lse)
            return y

        @staticmethod
        def backward(ctx, dy):
            x, y, lse = ctx.saved_tensors
            return backward(x, y, lse, dy, n_head)

    return _Attn.apply(qkv)
