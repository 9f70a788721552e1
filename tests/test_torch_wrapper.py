"""The package's torch front end (`attention`, `forward`, `backward`,
`attn_block_forward`): the same results as the C entry points it marshals
for, and gradients that flow through autograd to qkv."""
import numpy as np
import pytest
import torch

import causal_self_attention_gptattn_b200 as pkg
import oracle
from causal_self_attention_gptattn_b200 import gptattn as ga
from causal_self_attention_gptattn_b200.workloads import block_inputs, make_inputs
from gpu_helpers import TOL_BF16_DQKV_REL, TOL_BF16_Y, TOL_F32

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda", 0)


def test_attention_autograd_matches_oracle_fp32_and_bf16():
    for dtype, hs, tol_y in ((torch.float32, 32, TOL_F32), (torch.bfloat16, 64, TOL_BF16_Y)):
        B, T, nh = 2, 150, 2
        qkv_c, dy_c = make_inputs(B, T, nh, hs, dtype=dtype, seed=91)
        qkv = qkv_c.to(_dev()).requires_grad_(True)
        y = pkg.attention(qkv, nh)
        y.backward(dy_c.to(_dev()))
        ry, _ = oracle.forward(qkv_c, nh)
        rg = oracle.backward(qkv_c, dy_c, nh)
        assert np.abs(y.detach().double().cpu().numpy() - ry).max() <= tol_y
        err = np.abs(qkv.grad.double().cpu().numpy() - rg).max()
        assert err <= (TOL_F32 if dtype == torch.float32 else TOL_BF16_DQKV_REL * np.abs(rg).max())


def test_window_and_deterministic_options_match_the_c_calls():
    B, T, nh, hs, W = 2, 300, 3, 64, 100
    C = nh * hs
    qkv_c, dy_c = make_inputs(B, T, nh, hs, dtype=torch.bfloat16, seed=92)
    qkv, dy = qkv_c.to(_dev()), dy_c.to(_dev())
    x = qkv.clone().requires_grad_(True)
    y = pkg.attention(x, nh, window=W, deterministic=True)
    y.backward(dy)
    s = torch.cuda.current_stream()
    y2 = torch.empty_like(y)
    lse2 = torch.empty(B, nh, T, dtype=torch.float32, device=_dev())
    ga.check(ga.gptattn_fwd_window(qkv, y2, lse2, B, T, C, nh, W, ga.GPTATTN_BF16, s), "fwd_window")
    nb = ga.gptattn_bwd_det_workspace_bytes(B, T, C, nh, ga.GPTATTN_BF16)
    ws = torch.empty(nb, dtype=torch.uint8, device=_dev())
    g2 = torch.empty_like(qkv)
    ga.check(ga.gptattn_bwd_det(qkv, y2, lse2, dy, g2, ws, nb, B, T, C, nh, W, ga.GPTATTN_BF16, s), "bwd_det")
    torch.cuda.synchronize()
    assert torch.equal(y.detach(), y2)
    assert torch.equal(x.grad, g2)


def test_dropout_option_uses_one_mask_for_both_passes():
    B, T, nh, hs, p, seed = 2, 200, 2, 64, 0.2, 12345
    qkv_c, dy_c = make_inputs(B, T, nh, hs, dtype=torch.bfloat16, seed=93)
    x = qkv_c.to(_dev()).requires_grad_(True)
    y = pkg.attention(x, nh, dropout_p=p, seed=seed)
    y.backward(dy_c.to(_dev()))
    ry, _ = oracle.forward(qkv_c, nh, dropout=p, seed=seed)
    rg = oracle.backward(qkv_c, dy_c, nh, dropout=p, seed=seed)
    assert np.abs(y.detach().double().cpu().numpy() - ry).max() <= TOL_BF16_Y
    assert np.abs(x.grad.double().cpu().numpy() - rg).max() <= TOL_BF16_DQKV_REL * np.abs(rg).max()


def test_inference_forward_without_lse():
    qkv = make_inputs(2, 130, 2, 64, dtype=torch.bfloat16, seed=94)[0].to(_dev())
    y1, lse1 = pkg.forward(qkv, 2)
    y2, lse2 = pkg.forward(qkv, 2, need_lse=False)
    torch.cuda.synchronize()
    assert lse2 is None and lse1.shape == (2, 2, 130)
    assert torch.equal(y1, y2)


def test_attn_block_forward_matches_the_c_call():
    B, T, C, nh = 2, 130, 256, 4
    x, p = block_inputs(B, T, C, seed=95)
    d = {k: v.to(_dev()) for k, v in p.items()}
    xd = x.to(_dev())
    out, qkv, y, lse = pkg.attn_block_forward(xd, d["ln_w"], d["ln_b"], d["w_attn"], d["b_attn"], d["w_proj"],
                                              d["b_proj"], nh)
    out2 = torch.empty_like(out)
    qkv2, y2, lse2 = torch.empty_like(qkv), torch.empty_like(y), torch.empty_like(lse)
    ga.check(ga.gptattn_attn_block_fwd(xd, d["ln_w"], d["ln_b"], d["w_attn"], d["b_attn"], d["w_proj"], d["b_proj"],
                                       qkv2, y2, lse2, out2, B, T, C, nh, ga.GPTATTN_BF16,
                                       torch.cuda.current_stream()), "attn_block_fwd")
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(qkv, qkv2) and torch.equal(y, y2) and torch.equal(lse, lse2)
