"""Pins of the attention sub-block oracle (``oracle/block.py``).

Each ``pin_*`` takes a module-like object with ``layernorm``, ``linear`` and
``attn_block_forward`` and the attention oracle front end, and raises
AssertionError when the block oracle disagrees with a closed form or a library
special case.  ``tests/test_block_oracle.py`` runs them on the real block
oracle and on copies with planted mistakes.

Passages: the minGPT README page's GPT-2 notes (layer norm at the input of
each sub-block), and the lecture page ("Let's build GPT: from scratch, in
code, spelled out") chapters "layernorm (and its relationship to our previous
batchnorm)", "multi-headed self-attention" and "residual connections".  The
eps = 1e-5 and the population variance are the reading of the layer norm
that PyTorch's nn.LayerNorm fixes (the pages give neither).
"""
from __future__ import annotations

import math

import numpy as np
import torch

EPS = 1e-5


def _rng(seed):
    return np.random.default_rng(seed)


def pin_ln_two_point_closed_form(blk, orc):
    """Row (c+a, c-a): mean c, population variance a^2, so the normalised row
    is (+-a) / sqrt(a^2 + eps); then gain and bias per feature.  a = 0.01 makes
    eps matter (a^2 = 1e-4): 0.01 / sqrt(1.1e-4) = 0.95346..."""
    a, c = 0.01, 3.25
    x = np.array([[c + a, c - a]])
    w = np.array([2.0, -3.0])
    b = np.array([0.5, -1.0])
    n = a / math.sqrt(a * a + EPS)
    out = blk.layernorm(x, w, b)
    assert np.allclose(out, [[2.0 * n + 0.5, -3.0 * -n - 1.0]], rtol=0, atol=1e-12)


def pin_ln_row_moments(blk, orc):
    """Unit gain, zero bias: every row has mean 0 and population variance
    var/(var+eps), whatever the row's own mean and scale (a token's features
    are normalised, not a feature across tokens)."""
    r = _rng(31)
    x = r.standard_normal((7, 48)) * r.uniform(0.05, 4.0, (7, 1)) + r.uniform(-5, 5, (7, 1))
    out = blk.layernorm(x, np.ones(48), np.zeros(48))
    var = x.var(axis=1)
    assert np.abs(out.mean(axis=1)).max() < 1e-12
    assert np.allclose(out.var(axis=1), var / (var + EPS), rtol=1e-12, atol=0)


def pin_ln_constant_row(blk, orc):
    """A constant row has nothing to normalise: the output is the bias."""
    x = np.full((3, 8), 0.75)
    b = np.arange(8) * 0.5 - 1.0
    out = blk.layernorm(x, np.full(8, 7.0), b)
    assert np.array_equal(out, np.broadcast_to(b, (3, 8)))


def pin_linear_permutation(blk, orc):
    """W[n][k] = 1 iff k = perm[n] selects input feature perm[n] for output n
    (out = x W^T + b, nn.Linear's weight layout); a cyclic shift is not its own
    inverse, so the transposed product gives a different answer."""
    K = 6
    perm = np.roll(np.arange(K), 1)
    W = np.zeros((K, K))
    W[np.arange(K), perm] = 1.0
    x = _rng(32).standard_normal((4, K))
    b = np.arange(K) * 0.25
    assert np.array_equal(blk.linear(x, W, b), x[:, perm] + b)


def pin_linear_library(blk, orc):
    """torch.nn.functional.linear in fp64 on rectangular shapes."""
    r = _rng(33)
    x, W, b = r.standard_normal((5, 3, 24)), r.standard_normal((40, 24)), r.standard_normal(40)
    ref = torch.nn.functional.linear(torch.tensor(x), torch.tensor(W), torch.tensor(b)).numpy()
    assert np.abs(blk.linear(x, W, b) - ref).max() < 1e-12


def _params(r, C):
    return dict(ln_w=1.0 + 0.2 * r.standard_normal(C), ln_b=0.1 * r.standard_normal(C),
                w_attn=r.standard_normal((3 * C, C)) / math.sqrt(C), b_attn=0.1 * r.standard_normal(3 * C),
                w_proj=r.standard_normal((C, C)) / math.sqrt(C), b_proj=0.1 * r.standard_normal(C))


def pin_block_zero_projection(blk, orc):
    """With a zero output projection the sub-block adds only its bias to the
    residual stream: out = x + b_proj exactly (the stream is x, not LN(x))."""
    B, T, C, nh = 2, 9, 16, 2
    r = _rng(34)
    x = r.standard_normal((B, T, C)) + 2.0
    p = _params(r, C)
    p["w_proj"] = np.zeros((C, C))
    out, _, _, _ = blk.attn_block_forward(x, n_head=nh, attention=orc.forward, **p)
    assert np.array_equal(out, x + p["b_proj"])


def pin_block_prefix_average(blk, orc):
    """c_attn = [0; 0; I] (zero queries and keys, values = LN(x)) and c_proj = I:
    all visible scores are equal, so each position averages the normalised rows
    of itself and the past: out[t] = x[t] + mean_{s<=t} LN(x)[s].  LN(x) here is
    written out per row with the two-point-pinned formula."""
    B, T, C, nh = 2, 11, 12, 3
    r = _rng(35)
    x = r.standard_normal((B, T, C)) * 1.5 + 0.7
    ln_w, ln_b = 1.0 + 0.3 * r.standard_normal(C), 0.2 * r.standard_normal(C)
    w_attn = np.zeros((3 * C, C))
    w_attn[2 * C:] = np.eye(C)
    out, qkv, _, _ = blk.attn_block_forward(x, ln_w, ln_b, w_attn, np.zeros(3 * C), np.eye(C), np.zeros(C),
                                            n_head=nh, attention=orc.forward)
    for bi in range(B):
        xn = np.empty((T, C))
        for t in range(T):
            row = x[bi, t]
            mu = sum(row) / C
            var = sum((v - mu) ** 2 for v in row) / C
            xn[t] = [(row[k] - mu) / math.sqrt(var + EPS) * ln_w[k] + ln_b[k] for k in range(C)]
        for t in range(T):
            expect = x[bi, t] + xn[:t + 1].mean(axis=0)
            assert np.allclose(out[bi, t], expect, rtol=0, atol=1e-12)
        assert np.abs(qkv[bi, :, :2 * C]).max() == 0.0


def pin_block_library_special_case(blk, orc):
    """PyTorch in fp64: layer_norm (eps 1e-5) -> linear -> causal
    scaled_dot_product_attention over the heads -> linear, plus x."""
    B, T, C, nh = 2, 21, 24, 3
    hs = C // nh
    r = _rng(36)
    x = r.standard_normal((B, T, C)) * 2.0 - 0.5
    p = _params(r, C)
    t = {k: torch.tensor(v) for k, v in p.items()}
    xt = torch.tensor(x)
    F = torch.nn.functional
    xn = F.layer_norm(xt, (C,), t["ln_w"], t["ln_b"], eps=EPS)
    qkv = F.linear(xn, t["w_attn"], t["b_attn"])
    q, k, v = qkv.split(C, dim=2)
    heads = lambda a: a.view(B, T, nh, hs).transpose(1, 2)
    y = F.scaled_dot_product_attention(heads(q), heads(k), heads(v), is_causal=True).transpose(1, 2).reshape(B, T, C)
    ref = xt + F.linear(y, t["w_proj"], t["b_proj"])
    out, qkv_o, y_o, _ = blk.attn_block_forward(x, n_head=nh, attention=orc.forward, **p)
    assert np.abs(qkv_o - qkv.numpy()).max() < 1e-12
    assert np.abs(y_o - y.numpy()).max() < 1e-12
    assert np.abs(out - ref.numpy()).max() < 1e-12


def pin_block_regression_fixture(blk, orc):
    """Regression fixture written by tests/golden/make_golden.py from this oracle:
    catches any later change to the block oracle's arithmetic."""
    import json
    import os
    fx = json.load(open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "block_small_seeded.json")))
    p = {k: np.array(fx[k]) for k in ("ln_w", "ln_b", "w_attn", "b_attn", "w_proj", "b_proj")}
    out, qkv, y, lse = blk.attn_block_forward(np.array(fx["x"]), n_head=fx["n_head"], attention=orc.forward, **p)
    for got, key in ((out, "out"), (qkv, "qkv"), (y, "y"), (lse, "lse")):
        assert np.allclose(got, fx[key], rtol=0, atol=1e-12), key


def pin_block_empty(blk, orc):
    """T = 0: nothing to compute, shapes preserved."""
    C = 8
    p = _params(_rng(37), C)
    out, qkv, y, lse = blk.attn_block_forward(np.zeros((2, 0, C)), n_head=2, attention=orc.forward, **p)
    assert out.shape == (2, 0, C) and qkv.shape == (2, 0, 3 * C) and y.shape == (2, 0, C)


BLOCK_PINS = [
    pin_ln_two_point_closed_form,
    pin_ln_row_moments,
    pin_ln_constant_row,
    pin_linear_permutation,
    pin_linear_library,
    pin_block_zero_projection,
    pin_block_prefix_average,
    pin_block_library_special_case,
    pin_block_empty,
    pin_block_regression_fixture,
]
