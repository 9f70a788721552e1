"""GPU parity of attention dropout (gptattn_fwd_opts / gptattn_bwd_opts) against
the fp64 oracle with the same Philox4x32-10 mask; the GPU's generator and the
oracle's are separate implementations of the published definition."""
import math

import numpy as np
import pytest
import torch

import oracle
from causal_self_attention_gptattn_b200 import gptattn as ga
from causal_self_attention_gptattn_b200.workloads import make_inputs
from gpu_helpers import compare, run_fwd_bwd

pytestmark = pytest.mark.gpu


def ref(qkv, dy, n_head, p, seed, window=None):
    pf = float(np.float32(p))  # the library takes p as float32
    y, lse = oracle.forward(qkv, n_head, window=window, dropout=pf, seed=seed)
    return y, lse, oracle.backward(qkv, dy, n_head, window=window, dropout=pf, seed=seed)


@pytest.mark.parametrize("B,T,n_head,hs,p", [(2, 77, 2, 32, 0.1), (1, 130, 2, 64, 0.5), (1, 65, 1, 128, 0.3),
                                             (2, 40, 4, 16, 0.9)])
def test_dropout_fp32(B, T, n_head, hs, p):
    qkv, dy = make_inputs(B, T, n_head, hs, dtype=torch.float32, seed=1300 + T)
    seed = (11 << 32) | (T * 7919)
    got = run_fwd_bwd(qkv, dy, n_head, opts=ga.Options(dropout_p=p, dropout_seed=seed))
    compare(got, ref(qkv, dy, n_head, p, seed), torch.float32, f"fp32 dropout {p}")


@pytest.mark.parametrize("B,T,n_head,hs,p,window", [(2, 300, 2, 64, 0.1, 0), (1, 384, 2, 64, 0.3, 0),
                                                    (2, 129, 1, 64, 0.5, 0), (1, 520, 2, 64, 0.2, 200),
                                                    (1, 1000, 1, 64, 0.1, 0), (1, 300, 2, 128, 0.1, 0),
                                                    (2, 257, 1, 128, 0.6, 0), (1, 520, 2, 128, 0.2, 200),
                                                    (1, 640, 1, 128, 0.3, 0)])
def test_dropout_bf16(B, T, n_head, hs, p, window):
    qkv, dy = make_inputs(B, T, n_head, hs, dtype=torch.bfloat16, seed=1400 + T + hs)
    seed = 0xDEADBEEF00000000 + T
    got = run_fwd_bwd(qkv, dy, n_head, opts=ga.Options(window=window, dropout_p=p, dropout_seed=seed))
    compare(got, ref(qkv, dy, n_head, p, seed, window=window or None), torch.bfloat16, f"bf16 dropout {p} w {window}")


@pytest.mark.parametrize("hs", [64, 128])
@pytest.mark.parametrize("p", [0.37, 0.7])  # theta = 95 and 179: both sides of 128
def test_dropout_mask_bits_match_the_oracle_generator(p, hs):
    """Zero queries and v = identity expose every weight's dropout factor in y
    (forward); dy[t] = e_t exposes it in dV[s, t] = P[t, s] f[t, s] (backward).
    Both kept sets must equal the oracle generator's decision bit for bit."""
    T, n_head, seed = hs, 2, 0x0123456789ABCDEF
    C = n_head * hs
    qkv = torch.zeros(1, T, 3 * C)
    qkv[0, :, C:2 * C] = torch.randn(T, C, generator=torch.Generator().manual_seed(5))
    dy = torch.zeros(1, T, C)
    for h in range(n_head):
        qkv[0, :, 2 * C + h * hs:2 * C + (h + 1) * hs] = torch.eye(T)
        dy[0, :, h * hs:(h + 1) * hs] = torch.eye(T)
    thr = min(255, math.floor(256.0 * float(np.float32(p)) + 0.5))  # theta = round(256 p)
    for dtype in ((torch.float32, torch.bfloat16) if hs == 64 else (torch.bfloat16,)):
        y, _, dqkv = run_fwd_bwd(qkv.to(dtype), dy.to(dtype), n_head, opts=ga.Options(dropout_p=p, dropout_seed=seed))
        for h in range(n_head):
            for t in range(T):
                for s in range(t + 1):
                    r = oracle.philox([s // 4, t // 4, h, 0], [seed & 0xFFFFFFFF, seed >> 32])
                    kept = ((r[t % 4] >> (8 * (s % 4))) & 0xFF) >= thr
                    assert kept == (y[0, t, h * hs + s] > 0), ("forward", str(dtype), h, t, s)
                    assert kept == (dqkv[0, s, 2 * C + h * hs + t] > 0), ("backward", str(dtype), h, t, s)


def test_dropout_zero_is_the_plain_path_and_seeds_matter():
    qkv, dy = make_inputs(2, 200, 2, 64, dtype=torch.bfloat16, seed=1500)
    a = run_fwd_bwd(qkv, dy, 2)
    b = run_fwd_bwd(qkv, dy, 2, opts=ga.Options(dropout_p=0.0, dropout_seed=99))
    for x, z in zip(a, b):
        assert np.array_equal(x, z)
    c1 = run_fwd_bwd(qkv, dy, 2, opts=ga.Options(dropout_p=0.2, dropout_seed=5))
    c2 = run_fwd_bwd(qkv, dy, 2, opts=ga.Options(dropout_p=0.2, dropout_seed=5))
    c3 = run_fwd_bwd(qkv, dy, 2, opts=ga.Options(dropout_p=0.2, dropout_seed=6))
    assert np.array_equal(c1[0], c2[0]) and np.array_equal(c1[1], a[1])  # lse is the undropped one
    assert not np.array_equal(c1[0], c3[0])


@pytest.mark.parametrize("hs", [64, 128])
def test_dropout_with_deterministic_backward_is_repeatable(hs):
    qkv, dy = make_inputs(1, 640, 2, hs, dtype=torch.bfloat16, seed=1600 + hs)
    o = ga.Options(dropout_p=0.25, dropout_seed=77, deterministic=1)
    g1 = run_fwd_bwd(qkv, dy, 2, opts=o)[2]
    g2 = run_fwd_bwd(qkv, dy, 2, opts=o)[2]
    assert np.array_equal(g1, g2)
    compare(run_fwd_bwd(qkv, dy, 2, opts=o), ref(qkv, dy, 2, 0.25, 77), torch.bfloat16, "dropout + deterministic")
