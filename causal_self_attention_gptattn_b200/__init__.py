"""libgptattn for NVIDIA B200: batched multi-head causal self-attention,
forward and backward, in hand-written sm_100a kernels behind a C ABI.

``gptattn``   -- the ctypes binding (same names as include/gptattn.h).
``attention`` -- a torch.autograd wrapper for users holding torch tensors:
                 ``y = attention(qkv, n_head)`` with qkv[B, T, 3C] on a CUDA
                 device (bf16 or fp32); gradients flow to qkv.  Options: a
                 local window, dropout on the attention weights (seeded
                 Philox mask), a deterministic backward.  PyTorch only
                 allocates memory and supplies the stream; the kernels do the
                 arithmetic.
``attn_block_forward`` -- the pre-LN attention sub-block (LayerNorm, c_attn,
                 attention, c_proj + residual) in one call.
``workloads`` -- seeded synthetic inputs of the benchmark shapes.
"""
from __future__ import annotations

from . import gptattn  # noqa: F401

__all__ = ["gptattn", "attention", "forward", "backward", "attn_block_forward"]


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return gptattn.GPTATTN_BF16
    if t.dtype == torch.float32:
        return gptattn.GPTATTN_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")


def _opts(window, dropout_p, seed, deterministic):
    return gptattn.Options(window=int(window or 0), dropout_p=float(dropout_p), dropout_seed=int(seed) & (2**64 - 1),
                           deterministic=1 if deterministic else 0)


def forward(qkv, n_head: int, window=None, dropout_p: float = 0.0, seed: int = 0, need_lse: bool = True):
    """Return (y[B,T,C], lse[B,n_head,T] fp32) for a CUDA tensor qkv[B,T,3C].

    window: token t sees t-window < s <= t (None: every past token); dropout_p, seed: dropout on
    the attention weights with the Philox mask of that seed; need_lse=False (inference) returns
    lse=None and skips writing it."""
    import torch
    if not qkv.is_cuda:
        raise ValueError("qkv must be a CUDA tensor (there is no CPU path)")
    qkv = qkv.contiguous()
    B, T, C3 = qkv.shape
    C = C3 // 3
    y = torch.empty(B, T, C, dtype=qkv.dtype, device=qkv.device)
    lse = torch.empty(B, n_head, T, dtype=torch.float32, device=qkv.device) if need_lse else None
    st = torch.cuda.current_stream(qkv.device)
    o = _opts(window, dropout_p, seed, False)
    gptattn.check(gptattn.gptattn_fwd_opts(qkv, y, lse, B, T, C, n_head, o, _dtype_code(qkv), st), "gptattn_fwd_opts")
    return y, lse


def backward(qkv, y, lse, dy, n_head: int, window=None, dropout_p: float = 0.0, seed: int = 0,
             deterministic: bool = False):
    """Return dqkv[B,T,3C] given the forward's qkv, y, lse (and its window, dropout_p, seed) and
    the gradient dy; deterministic=True gives bit-identical results on every run."""
    import torch
    qkv, y, lse, dy = qkv.contiguous(), y.contiguous(), lse.contiguous(), dy.contiguous()
    B, T, C3 = qkv.shape
    C = C3 // 3
    dt = _dtype_code(qkv)
    dqkv = torch.empty_like(qkv)
    o = _opts(window, dropout_p, seed, deterministic)
    nbytes = gptattn.gptattn_bwd_opts_workspace_bytes(B, T, C, n_head, o, dt)
    if nbytes == (1 << 64) - 1:
        raise ValueError("invalid shape or options for the backward")
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=qkv.device)
    st = torch.cuda.current_stream(qkv.device)
    gptattn.check(gptattn.gptattn_bwd_opts(qkv, y, lse, dy, dqkv, ws, nbytes, B, T, C, n_head, o, dt, st),
                  "gptattn_bwd_opts")
    return dqkv


def attention(qkv, n_head: int, window=None, dropout_p: float = 0.0, seed=None, deterministic: bool = False):
    """Causal multi-head self-attention of packed qkv[B,T,3C] -> y[B,T,C], differentiable.

    With dropout_p > 0 and seed None a fresh seed is drawn from torch's CPU generator for the
    call; the backward reuses it, so both passes see the same mask."""
    import torch
    if dropout_p > 0.0 and seed is None:
        seed = int(torch.randint(0, 2**62, (1,)).item())
    seed = 0 if seed is None else int(seed)

    class _Attn(torch.autograd.Function):
        @staticmethod
        def forward(ctx, x):
            y, lse = forward(x, n_head, window, dropout_p, seed)
            ctx.save_for_backward(x, y, lse)
            return y

        @staticmethod
        def backward(ctx, dy):
            x, y, lse = ctx.saved_tensors
            return backward(x, y, lse, dy, n_head, window, dropout_p, seed, deterministic)

    return _Attn.apply(qkv)


def attn_block_forward(x, ln_w, ln_b, w_attn, b_attn, w_proj, b_proj, n_head: int):
    """Forward of a pre-LN block's attention sub-block for bf16 CUDA tensors:
    out = x + c_proj(attention(c_attn(LayerNorm(x)))), weights in nn.Linear layout.
    Returns (out, qkv, y, lse)."""
    import torch
    if not x.is_cuda or x.dtype != torch.bfloat16:
        raise ValueError("x must be a bfloat16 CUDA tensor")
    x = x.contiguous()
    B, T, C = x.shape
    dev = x.device
    qkv = torch.empty(B, T, 3 * C, dtype=x.dtype, device=dev)
    y = torch.empty(B, T, C, dtype=x.dtype, device=dev)
    lse = torch.empty(B, n_head, T, dtype=torch.float32, device=dev)
    out = torch.empty_like(x)
    p = [t.contiguous() for t in (ln_w, ln_b, w_attn, b_attn, w_proj, b_proj)]
    gptattn.check(gptattn.gptattn_attn_block_fwd(x, *p, qkv, y, lse, out, B, T, C, n_head, gptattn.GPTATTN_BF16,
                                                 torch.cuda.current_stream(dev)), "gptattn_attn_block_fwd")
    return out, qkv, y, lse
