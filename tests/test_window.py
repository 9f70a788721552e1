"""GPU parity of the local-window (banded) entry points against the fp64
oracle's windowed forward and backward: token t sees t-window < s <= t."""
import numpy as np
import pytest
import torch

import oracle
from causal_self_attention_gptattn_b200.workloads import WORKLOADS, make_inputs, workload_inputs
from gpu_helpers import compare, run_fwd_bwd, select_heads

pytestmark = pytest.mark.gpu


def oracle_window(qkv, dy, n_head, window):
    y, lse = oracle.forward(qkv, n_head, window=window)
    return y, lse, oracle.backward(qkv, dy, n_head, window=window)


@pytest.mark.parametrize("B,T,n_head,hs,window", [(2, 77, 2, 32, 5), (1, 130, 2, 64, 64), (1, 200, 1, 16, 1),
                                                  (2, 65, 1, 128, 200), (1, 150, 2, 64, 97)])
def test_window_fp32(B, T, n_head, hs, window):
    qkv, dy = make_inputs(B, T, n_head, hs, dtype=torch.float32, seed=800 + T + window)
    got = run_fwd_bwd(qkv, dy, n_head, window=window)
    compare(got, oracle_window(qkv, dy, n_head, window), torch.float32, f"fp32 window {window}")


# bands narrower than, equal to and wider than a tile, edges inside and on tile boundaries, ragged T
BF16 = [(2, 300, 2, 1), (1, 384, 2, 128), (1, 520, 2, 100), (2, 1000, 1, 300), (1, 256, 2, 129),
        (1, 200, 1, 255), (1, 777, 2, 640), (2, 129, 1, 2), (1, 64, 2, 17)]


@pytest.mark.parametrize("B,T,n_head,window", BF16)
def test_window_bf16(B, T, n_head, window):
    qkv, dy = make_inputs(B, T, n_head, 64, dtype=torch.bfloat16, seed=900 + T + window)
    got = run_fwd_bwd(qkv, dy, n_head, window=window)
    compare(got, oracle_window(qkv, dy, n_head, window), torch.bfloat16, f"bf16 T={T} window {window}")


# head size 128 (the long-context shape): bands inside a tile, across tiles, ragged T
BF16_H128 = [(1, 300, 2, 1), (2, 520, 1, 100), (1, 384, 2, 128), (1, 777, 1, 300), (2, 200, 2, 255)]


@pytest.mark.parametrize("B,T,n_head,window", BF16_H128)
def test_window_bf16_head128(B, T, n_head, window):
    qkv, dy = make_inputs(B, T, n_head, 128, dtype=torch.bfloat16, seed=960 + T + window)
    got = run_fwd_bwd(qkv, dy, n_head, window=window)
    compare(got, oracle_window(qkv, dy, n_head, window), torch.bfloat16, f"bf16 hs128 T={T} window {window}")


def test_window_bf16_head128_long_context_sampled_heads():
    """The GPT-3-style long-context shape (B=4, T=2048, 16 heads of 128) with a 512-token band, the
    sparse layer of the alternating pattern; sampled heads against the oracle.  Inputs are N(0,1):
    with the workload's doubled qkv (sharp softmax) the band leaves so few keys per row that the
    bf16 rounding of the weights and of y alone gives y errors of 2.5-2.9e-2, above the 2e-2 the
    causal configurations are held to (a CPU emulation of that arithmetic shows the same)."""
    w = WORKLOADS[5]
    qkv, dy = make_inputs(w.B, w.T, w.n_head, w.hs, dtype=torch.bfloat16, seed=1005)
    y, lse, dqkv = run_fwd_bwd(qkv, dy, w.n_head, window=512)
    batches, heads = [0, w.B - 1], [0, 15]
    q_s = select_heads(qkv[batches].double().numpy(), w.n_head, 3, heads)
    g_s = select_heads(dy[batches].double().numpy(), w.n_head, 1, heads)
    ref = oracle_window(q_s, g_s, len(heads), 512)
    got = (select_heads(y[batches], w.n_head, 1, heads), lse[batches][:, heads],
           select_heads(dqkv[batches], w.n_head, 3, heads))
    compare(got, ref, torch.bfloat16, "long_context window 512")


def test_window_at_least_T_is_the_causal_path():
    """window >= T takes exactly the causal kernels: y, lse, dK and dV bit-identical.  dQ is
    summed over key tiles by fp32 reduce-adds whose order is not fixed (the deterministic
    backward is the bitwise-reproducible one), so it is held to one bf16 rounding step."""
    B, T, nh, hs = 2, 333, 2, 64
    C = nh * hs
    qkv, dy = make_inputs(B, T, nh, hs, dtype=torch.bfloat16, seed=950)
    a = run_fwd_bwd(qkv, dy, nh)
    for other in (run_fwd_bwd(qkv, dy, nh, window=T), run_fwd_bwd(qkv, dy, nh, window=10**6)):
        for x, z in zip(a[:2], other[:2]):  # y, lse
            assert np.array_equal(x, z)
        assert np.array_equal(a[2][..., C:], other[2][..., C:])  # dK, dV
        dq_a, dq_o = a[2][..., :C], other[2][..., :C]
        assert np.allclose(dq_a, dq_o, rtol=2.0 ** -7, atol=1e-6 * np.abs(dq_a).max()), \
            np.abs(dq_a - dq_o).max()


def test_window_band_locality():
    """Changing tokens before a query's band leaves that query's y and lse bit-identical."""
    T, w = 700, 200
    qkv, dy = make_inputs(1, T, 2, 64, dtype=torch.bfloat16, seed=951)
    y0, l0, _ = run_fwd_bwd(qkv, dy, 2, window=w)
    q2 = qkv.clone()
    t = 650
    q2[:, :t - w + 1] = torch.randn(q2[:, :t - w + 1].shape, generator=torch.Generator().manual_seed(4)).to(q2.dtype)
    y1, l1, _ = run_fwd_bwd(q2, dy, 2, window=w)
    assert np.array_equal(y0[:, t:], y1[:, t:])
    assert np.array_equal(l0[:, :, t:], l1[:, :, t:])


def test_window_bf16_full_size_sampled_heads():
    """GPT-2 124M shape with a 256-token band (the GPT-3 layer pattern's sparse layer);
    the oracle on two sampled batches and three heads."""
    w = WORKLOADS[3]
    qkv, dy = workload_inputs(w)
    y, lse, dqkv = run_fwd_bwd(qkv, dy, w.n_head, window=256)
    batches, heads = [0, w.B - 1], [0, 5, 11]
    q_s = select_heads(qkv[batches].double().numpy(), w.n_head, 3, heads)
    g_s = select_heads(dy[batches].double().numpy(), w.n_head, 1, heads)
    ref = oracle_window(q_s, g_s, len(heads), 256)
    got = (select_heads(y[batches], w.n_head, 1, heads), lse[batches][:, heads],
           select_heads(dqkv[batches], w.n_head, 3, heads))
    compare(got, ref, torch.bfloat16, "gpt2_124m window 256")
