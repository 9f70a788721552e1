"""fp64 CPU oracle for the attention sub-block of a pre-LN GPT block (forward).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only users.  It shares nothing with
the CUDA library.

What it computes, step by step, with the passage each step follows:

  - minGPT README page ("卡帕西(氏)MinGPT"), reference notes on GPT-2: the
    layer norm sits at the input of each sub-block (pre-activation residual
    network), so the sub-block is  out = x + proj(attn(c_attn(LN(x)))).
  - "Let's build GPT: from scratch, in code, spelled out" (lecture page),
    chapter "layernorm (and its relationship to our previous batchnorm)":
    each token's feature row (not the batch column) is normalised to zero mean
    and unit variance, then scaled and shifted by learned per-feature gains and
    biases.  Read as the biased (population) variance with eps = 1e-5 added
    under the square root, the defaults of PyTorch's nn.LayerNorm, which the
    lecture's model uses; the page gives no eps.
  - same page, chapter "multi-headed self-attention": one linear map produces
    the queries, keys and values of all heads (here packed as q | k | v along
    the feature axis, head h in columns [h*hs, (h+1)*hs) of each), and after
    the heads are concatenated a second linear map projects back to C.
  - same page, chapter "residual connections": the sub-block's output is added
    to its input (the residual stream is x itself, not the normalised x).
  - the attention core is the oracle's own causal attention (``oracle.forward``).

Linear maps use nn.Linear's convention: weight [out_features][in_features],
out = x @ W^T + b.  All arithmetic is IEEE double (numpy); the only library
primitive is the matrix product.
"""
from __future__ import annotations

import numpy as np

LN_EPS = 1e-5


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().double().numpy()
    return np.asarray(a, dtype=np.float64)


def layernorm(x, w, b, eps: float = LN_EPS) -> np.ndarray:
    """Normalise each row of x[..., C] over its C features; then * w + b."""
    x, w, b = _f64(x), _f64(w), _f64(b)
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)   # population variance
    return (x - mean) / np.sqrt(var + eps) * w + b


def linear(x, w, b=None) -> np.ndarray:
    """x[..., K] @ w[N, K]^T (+ b[N])."""
    x, w = _f64(x), _f64(w)
    out = x @ w.T
    if b is not None:
        out = out + _f64(b)
    return out


def attn_block_forward(x, ln_w, ln_b, w_attn, b_attn, w_proj, b_proj, n_head: int, attention=None):
    """Return (out, qkv, y, lse) of the sub-block for x[B, T, C].

    qkv = c_attn(LN(x)) [B, T, 3C];  y, lse = causal attention of qkv;
    out = x + c_proj(y).  ``attention`` defaults to the oracle's forward."""
    if attention is None:
        from . import forward as attention
    x = _f64(x)
    xn = layernorm(x, ln_w, ln_b)
    qkv = linear(xn, w_attn, b_attn)
    y, lse = attention(qkv, n_head)
    out = x + linear(y, w_proj, b_proj)
    return out, qkv, y, lse
