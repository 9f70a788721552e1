"""GPU checks of gptattn_bwd_det: parity with the fp64 oracle (causal and local
window), bit-identical dqkv on repeated runs, agreement with gptattn_bwd."""
import numpy as np
import pytest
import torch

import oracle
from causal_self_attention_gptattn_b200 import gptattn as ga
from causal_self_attention_gptattn_b200.workloads import WORKLOADS, make_inputs, workload_inputs
from gpu_helpers import Guarded, compare, run_fwd_bwd, select_heads

pytestmark = pytest.mark.gpu


def run_det(qkv_cpu, dy_cpu, n_head, window=10**9, reps=1):
    """Forward (windowed entry point) then the deterministic backward `reps` times
    into fresh buffers; returns (y, lse, [dqkv per rep]) as float64 numpy, plus the
    raw bf16/fp32 dqkv tensors for bitwise comparison."""
    dev = torch.device("cuda", 0)
    dtype = qkv_cpu.dtype
    dt = ga.GPTATTN_BF16 if dtype == torch.bfloat16 else ga.GPTATTN_F32
    B, T, C3 = qkv_cpu.shape
    C = C3 // 3
    qkv = qkv_cpu.to(dev).contiguous()
    dy = dy_cpu.to(dev).contiguous()
    y = torch.empty(B, T, C, dtype=dtype, device=dev)
    lse = torch.empty(B, n_head, T, dtype=torch.float32, device=dev)
    s = torch.cuda.current_stream(dev)
    ga.check(ga.gptattn_fwd_window(qkv, y, lse, B, T, C, n_head, window, dt, s), "gptattn_fwd_window")
    nbytes = ga.gptattn_bwd_det_workspace_bytes(B, T, C, n_head, dt)
    raws = []
    for r in range(reps):
        ws = torch.full((max(nbytes, 256),), 0x55 + r, dtype=torch.uint8, device=dev)  # stale contents differ per run
        out = Guarded(B * T * 3 * C, dtype, dev)
        ga.check(ga.gptattn_bwd_det(qkv, y, lse, dy, out.view, ws, nbytes, B, T, C, n_head, window, dt, s),
                 "gptattn_bwd_det")
        assert ga.gptattn_get_device_status(s) == ga.GPTATTN_OK
        assert out.intact(), "write outside dqkv"
        raws.append(out.view.view(B, T, 3 * C).clone())
    yy = y.double().cpu().numpy()
    ll = lse.double().cpu().numpy()
    return yy, ll, [r.double().cpu().numpy() for r in raws], raws


@pytest.mark.parametrize("B,T,n_head,window", [(2, 300, 2, 10**9), (1, 1000, 2, 10**9), (2, 520, 2, 200),
                                               (1, 129, 3, 10**9), (1, 64, 1, 1)])
def test_det_bf16_parity(B, T, n_head, window):
    qkv, dy = make_inputs(B, T, n_head, 64, dtype=torch.bfloat16, seed=1100 + T)
    y, lse, (g,), _ = run_det(qkv, dy, n_head, window)
    w = None if window >= T else window
    ry, rl = oracle.forward(qkv, n_head, window=w)
    rg = oracle.backward(qkv, dy, n_head, window=w)
    compare((y, lse, g), (ry, rl, rg), torch.bfloat16, f"det T={T} window {window}")


@pytest.mark.parametrize("B,T,n_head,window", [(1, 300, 2, 10**9), (2, 520, 1, 200), (1, 129, 2, 10**9)])
def test_det_bf16_head128_parity_and_repeatable(B, T, n_head, window):
    qkv, dy = make_inputs(B, T, n_head, 128, dtype=torch.bfloat16, seed=1150 + T)
    y, lse, gs, raws = run_det(qkv, dy, n_head, window, reps=2)
    assert torch.equal(raws[1].view(torch.int16), raws[0].view(torch.int16)), "deterministic backward differs"
    w = None if window >= T else window
    ry, rl = oracle.forward(qkv, n_head, window=w)
    rg = oracle.backward(qkv, dy, n_head, window=w)
    compare((y, lse, gs[0]), (ry, rl, rg), torch.bfloat16, f"det hs128 T={T} window {window}")


def test_det_bf16_bitwise_repeatable_at_full_size():
    """GPT-2 124M shape: three runs give bit-identical dqkv; they agree with the
    reduce-add backward within tolerance; sampled heads agree with the oracle."""
    w = WORKLOADS[3]
    qkv, dy = workload_inputs(w)
    y, lse, gs, raws = run_det(qkv, dy, w.n_head, reps=3)
    for r in raws[1:]:
        assert torch.equal(r.view(torch.int16), raws[0].view(torch.int16)), "deterministic backward differs between runs"
    _, _, g_atomic = run_fwd_bwd(qkv, dy, w.n_head)
    scale = np.abs(g_atomic).max()
    assert np.abs(gs[0] - g_atomic).max() <= 1e-2 * scale
    batches, heads = [0, w.B - 1], [0, 7]
    q_s = select_heads(qkv[batches].double().numpy(), w.n_head, 3, heads)
    g_s = select_heads(dy[batches].double().numpy(), w.n_head, 1, heads)
    ry, rl = oracle.forward(q_s, len(heads))
    rg = oracle.backward(q_s, g_s, len(heads))
    got = (select_heads(y[batches], w.n_head, 1, heads), lse[batches][:, heads],
           select_heads(gs[0][batches], w.n_head, 3, heads))
    compare(got, (ry, rl, rg), torch.bfloat16, "det gpt2_124m")


def test_det_fp32_equals_regular_path():
    """The fp32 path has no reduce-adds: both entry points give the same bits."""
    qkv, dy = make_inputs(2, 150, 2, 32, dtype=torch.float32, seed=1200)
    _, _, (g,), _ = run_det(qkv, dy, 2)
    _, _, g2 = run_fwd_bwd(qkv, dy, 2)
    assert np.array_equal(g, g2)
