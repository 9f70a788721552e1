"""GPU parity of gptattn_decode (the last position over a key/value cache)
against the fp64 oracle's forward, whose row T-1 is the same function."""
import numpy as np
import pytest
import torch

import oracle
from causal_self_attention_gptattn_b200 import gptattn as ga
from causal_self_attention_gptattn_b200.workloads import WORKLOADS, make_inputs, workload_inputs
from gpu_helpers import TOL_BF16_LSE, TOL_BF16_Y, TOL_F32, Guarded

pytestmark = pytest.mark.gpu


def run_decode(qkv_cpu, n_head, T, T_cap=None):
    """qkv_cpu: [B, T_cap, 3C] host tensor; rows >= T are never to be read."""
    dev = torch.device("cuda", 0)
    B, Tc, C3 = qkv_cpu.shape
    C = C3 // 3
    dt = ga.GPTATTN_BF16 if qkv_cpu.dtype == torch.bfloat16 else ga.GPTATTN_F32
    qkv = qkv_cpu.to(dev).contiguous()
    y = Guarded(B * C, qkv_cpu.dtype, dev)
    lse = Guarded(B * n_head, torch.float32, dev)
    s = torch.cuda.current_stream(dev)
    ga.check(ga.gptattn_decode(qkv, y.view, lse.view, B, T, Tc if T_cap is None else T_cap, C, n_head, dt, s),
             "gptattn_decode")
    assert ga.gptattn_get_device_status(s) == ga.GPTATTN_OK
    assert y.intact() and lse.intact(), "write outside an output buffer"
    return (y.view.view(B, C).double().cpu().numpy(), lse.view.view(B, n_head).double().cpu().numpy())


def oracle_last_row(qkv_valid, n_head):
    y, lse = oracle.forward(qkv_valid, n_head)
    return y[:, -1, :], lse[:, :, -1]


def check(got, ref, dtype, what):
    y, lse = got
    ry, rl = ref
    assert np.isfinite(y).all() and np.isfinite(lse).all(), what
    ey, el = float(np.abs(y - ry).max()), float(np.abs(lse - rl).max())
    if dtype == torch.float32:
        assert ey <= TOL_F32 and el <= TOL_F32, f"{what}: y {ey:.3e} lse {el:.3e}"
    else:
        assert ey <= TOL_BF16_Y and el <= TOL_BF16_LSE, f"{what}: y {ey:.3e} lse {el:.3e}"


@pytest.mark.parametrize("B,T,n_head,hs", [(2, 1, 2, 64), (2, 2, 2, 64), (1, 9, 3, 64), (2, 128, 2, 64),
                                           (1, 1000, 2, 64), (2, 1031, 1, 128), (1, 7, 2, 128)])
def test_decode_bf16(B, T, n_head, hs):
    qkv, _ = make_inputs(B, T, n_head, hs, dtype=torch.bfloat16, seed=500 + T + hs)
    check(run_decode(qkv, n_head, T), oracle_last_row(qkv, n_head), torch.bfloat16, f"bf16 {B},{T},{n_head},{hs}")


@pytest.mark.parametrize("B,T,n_head,hs", [(2, 1, 4, 16), (1, 33, 2, 32), (2, 200, 2, 64), (1, 77, 1, 128)])
def test_decode_fp32(B, T, n_head, hs):
    qkv, _ = make_inputs(B, T, n_head, hs, dtype=torch.float32, seed=600 + T + hs)
    check(run_decode(qkv, n_head, T), oracle_last_row(qkv, n_head), torch.float32, f"fp32 {B},{T},{n_head},{hs}")


@pytest.mark.parametrize("dtype,hs", [(torch.bfloat16, 64), (torch.float32, 32)])
def test_decode_reads_only_valid_rows(dtype, hs):
    """A cache with capacity T_cap > T: rows T..T_cap-1 hold NaN and must not be read."""
    B, T, T_cap, n_head = 2, 150, 256, 2
    qkv, _ = make_inputs(B, T, n_head, hs, dtype=dtype, seed=701)
    cache = torch.full((B, T_cap, qkv.shape[2]), float("nan"), dtype=dtype)
    cache[:, :T] = qkv
    check(run_decode(cache, n_head, T, T_cap), oracle_last_row(qkv, n_head), dtype, "cache with NaN tail")


def test_decode_sharp_softmax():
    qkv, _ = make_inputs(2, 300, 2, 64, dtype=torch.float32, seed=702)
    qkv[..., :256] *= 4.0  # q and k of both heads: sharp scores
    qkv = qkv.to(torch.bfloat16)
    check(run_decode(qkv, 2, 300), oracle_last_row(qkv, 2), torch.bfloat16, "sharp softmax")


@pytest.mark.parametrize("idx", [3, 4])
def test_decode_full_workload_sampled_batches(idx):
    """The GPT-2 shapes at full size; the oracle is run on two sampled sequences."""
    w = WORKLOADS[idx]
    qkv, _ = workload_inputs(w)
    y, lse = run_decode(qkv, w.n_head, w.T)
    for b in (0, w.B - 1):
        ry, rl = oracle_last_row(qkv[b:b + 1], w.n_head)
        check((y[b:b + 1], lse[b:b + 1]), (ry, rl), torch.bfloat16, f"{w.name} batch {b}")


def test_decode_matches_forward_last_row_on_gpu():
    """The two CUDA paths agree on the last position (same function, different kernels)."""
    from gpu_helpers import run_fwd_bwd
    qkv, dy = make_inputs(2, 257, 2, 64, dtype=torch.bfloat16, seed=703)
    fy, flse, _ = run_fwd_bwd(qkv, dy, 2)
    dy_, dlse = run_decode(qkv, 2, 257)
    assert np.abs(dy_ - fy[:, -1, :]).max() <= TOL_BF16_Y
    assert np.abs(dlse - flse[:, :, -1]).max() <= TOL_BF16_LSE
