"""Parity of the attention sub-block's CUDA path (LayerNorm, the two linear maps
and the whole pre-LN sub-block) with the fp64 oracle, through the C ABI.

Tolerances (derived from the arithmetic; inputs are bf16, accumulation fp32,
each output rounded once to bf16, relative rounding error <= 2^-9):
  layernorm, linear: |out - ref| <= 2^-8 * |ref| + 2e-3 * rms(ref)
  sub-block, step by step (each step fed the GPU's own bf16 input): qkv and
    out as linear; y within 2e-2 and lse within 1e-2 (the attention bounds)
  sub-block end to end (oracle fed only x and the weights): the bf16
    intermediates (LN(x), qkv, y) add their roundings: max |err| <= 3e-2 * max|ref|
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
import oracle.block as block
from causal_self_attention_gptattn_b200 import gptattn as ga
from gpu_helpers import Guarded
from causal_self_attention_gptattn_b200.workloads import block_inputs

pytestmark = pytest.mark.gpu
BF = ga.GPTATTN_BF16


def _dev():
    return torch.device("cuda", 0)


def _f64(t):
    return t.detach().cpu().double().numpy()


def _close_linear(got, ref, what):
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2e-3 * math.sqrt(float((ref ** 2).mean()) + 1e-30)
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of tolerance, worst {err.max():.3g}"


@pytest.mark.parametrize("M,C", [(1000, 768), (7, 64), (33, 1024), (130, 4096), (1, 2048)])
def test_layernorm_parity(M, C):
    r = np.random.default_rng(100 + C)
    x = torch.tensor(r.standard_normal((M, C)) * 1.7 + 0.4).to(torch.bfloat16)
    w = torch.tensor(1.0 + 0.2 * r.standard_normal(C)).to(torch.bfloat16)
    b = torch.tensor(0.1 * r.standard_normal(C)).to(torch.bfloat16)
    out = Guarded(M * C, torch.bfloat16, _dev())
    s = torch.cuda.current_stream()
    ga.check(ga.gptattn_layernorm(x.to(_dev()), w.to(_dev()), b.to(_dev()), out.view, M, C, BF, s), "layernorm")
    torch.cuda.synchronize()
    assert out.intact()
    ref = block.layernorm(_f64(x), _f64(w), _f64(b))
    _close_linear(_f64(out.view).reshape(M, C), ref, "layernorm")


@pytest.mark.parametrize("M,N,K,with_bias,with_resid", [
    (300, 2304, 768, True, False),    # c_attn at C = 768, ragged M
    (300, 768, 768, True, True),      # c_proj with the residual
    (128, 64, 64, False, False),      # one tile, one chunk
    (1, 192, 128, True, True),        # a single row
    (517, 320, 1024, False, True),    # N not a multiple of the tile width
    (20000, 768, 256, True, True),    # enough tiles for the 128 x 256 shape (the smaller ones use 128 x 128)
])
def test_linear_parity(M, N, K, with_bias, with_resid):
    r = np.random.default_rng(M * 7 + N + K)
    a = torch.tensor(r.standard_normal((M, K))).to(torch.bfloat16)
    w = torch.tensor(r.standard_normal((N, K)) / math.sqrt(K)).to(torch.bfloat16)
    bias = torch.tensor(r.standard_normal(N)).to(torch.bfloat16) if with_bias else None
    resid = torch.tensor(r.standard_normal((M, N))).to(torch.bfloat16) if with_resid else None
    out = Guarded(M * N, torch.bfloat16, _dev())
    s = torch.cuda.current_stream()
    ga.check(ga.gptattn_linear(a.to(_dev()), w.to(_dev()), None if bias is None else bias.to(_dev()),
                               None if resid is None else resid.to(_dev()), out.view, M, N, K, BF, s), "linear")
    torch.cuda.synchronize()
    assert out.intact()
    ref = block.linear(_f64(a), _f64(w), None if bias is None else _f64(bias))
    if resid is not None:
        ref = ref + _f64(resid)
    _close_linear(_f64(out.view).reshape(M, N), ref, "linear")


def test_linear_in_place_residual():
    M, N, K = 260, 512, 256
    r = np.random.default_rng(5)
    a = torch.tensor(r.standard_normal((M, K))).to(torch.bfloat16)
    w = torch.tensor(r.standard_normal((N, K)) / math.sqrt(K)).to(torch.bfloat16)
    bias = torch.tensor(r.standard_normal(N)).to(torch.bfloat16)
    x = torch.tensor(r.standard_normal((M, N))).to(torch.bfloat16)
    xd = x.to(_dev()).contiguous()
    ga.check(ga.gptattn_linear(a.to(_dev()), w.to(_dev()), bias.to(_dev()), xd, xd, M, N, K, BF,
                               torch.cuda.current_stream()), "linear in place")
    torch.cuda.synchronize()
    ref = block.linear(_f64(a), _f64(w), _f64(bias)) + _f64(x)
    _close_linear(_f64(xd), ref, "linear in place")


def _run_block(x, p, n_head):
    B, T, C = x.shape
    dev = _dev()
    d = {k: v.to(dev).contiguous() for k, v in p.items()}
    qkv = Guarded(B * T * 3 * C, torch.bfloat16, dev)
    y = Guarded(B * T * C, torch.bfloat16, dev)
    lse = Guarded(B * n_head * T, torch.float32, dev)
    out = Guarded(B * T * C, torch.bfloat16, dev)
    ga.check(ga.gptattn_attn_block_fwd(x.to(dev), d["ln_w"], d["ln_b"], d["w_attn"], d["b_attn"], d["w_proj"],
                                       d["b_proj"], qkv.view, y.view, lse.view, out.view, B, T, C, n_head, BF,
                                       torch.cuda.current_stream()), "attn_block_fwd")
    torch.cuda.synchronize()
    for g in (qkv, y, lse, out):
        assert g.intact()
    return (_f64(qkv.view).reshape(B, T, 3 * C), _f64(y.view).reshape(B, T, C),
            _f64(lse.view).reshape(B, n_head, T), _f64(out.view).reshape(B, T, C))


def _check_block(x, p, n_head, qkv, y, lse, out, rows=None):
    """Step by step on the GPU's own intermediates, then end to end."""
    xf = _f64(x)
    pf = {k: _f64(v) for k, v in p.items()}
    sel = slice(None) if rows is None else rows
    ln = block.layernorm(xf[:, sel], pf["ln_w"], pf["ln_b"])
    # c_attn from the exact LN: the GPU rounds LN(x) to bf16 first, which the
    # linear bound absorbs only after rounding the oracle's LN the same way
    ln_b16 = torch.tensor(ln).to(torch.bfloat16).double().numpy()
    _close_linear(qkv[:, sel], block.linear(ln_b16, pf["w_attn"], pf["b_attn"]), "c_attn")
    y_ref, lse_ref = oracle.forward(qkv, n_head)
    assert np.abs(y[:, sel] - y_ref[:, sel]).max() <= 2e-2
    assert np.abs(lse[:, :, sel] - lse_ref[:, :, sel]).max() <= 1e-2
    _close_linear(out[:, sel], xf[:, sel] + block.linear(y[:, sel], pf["w_proj"], pf["b_proj"]), "c_proj")
    if rows is None:
        ref, _, _, _ = block.attn_block_forward(xf, n_head=n_head, attention=oracle.forward, **pf)
        assert np.abs(out - ref).max() <= 3e-2 * np.abs(ref).max()


@pytest.mark.parametrize("B,T,C,n_head", [(2, 300, 768, 12), (1, 257, 256, 2), (3, 128, 128, 2), (1, 1, 768, 12)])
def test_attn_block_parity(B, T, C, n_head):
    x, p = block_inputs(B, T, C, seed=B * 1000 + T + C)
    qkv, y, lse, out = _run_block(x, p, n_head)
    _check_block(x, p, n_head, qkv, y, lse, out)


def test_attn_block_full_size_sampled():
    """GPT-2 124M attention sub-block at B=16, T=1024: step-by-step parity for
    batch element 5 (every row, all heads) -- the oracle's attention over one
    batch element takes about a second."""
    B, T, C, n_head = 16, 1024, 768, 12
    x, p = block_inputs(B, T, C, seed=124)
    qkv, y, lse, out = _run_block(x, p, n_head)
    b = 5
    _check_block(x[b:b + 1], p, n_head, qkv[b:b + 1], y[b:b + 1], lse[b:b + 1], out[b:b + 1], rows=slice(None))
    assert np.isfinite(out).all()
