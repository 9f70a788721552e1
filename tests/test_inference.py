"""Inference calls: the forward entry points, decode and the attention sub-block
accept lse == NULL (no backward follows) and then write everything else exactly
as with an lse buffer."""
import pytest
import torch

from causal_self_attention_gptattn_b200 import gptattn as ga
from causal_self_attention_gptattn_b200.workloads import block_inputs, make_inputs

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda", 0)


@pytest.mark.parametrize("dtype,hs,T", [(torch.bfloat16, 64, 300), (torch.bfloat16, 128, 257), (torch.float32, 32, 77)])
def test_forward_without_lse(dtype, hs, T):
    B, nh = 2, 3
    C = nh * hs
    dt = ga.GPTATTN_BF16 if dtype == torch.bfloat16 else ga.GPTATTN_F32
    qkv = make_inputs(B, T, nh, hs, dtype=dtype, seed=77)[0].to(_dev())
    y1 = torch.empty(B, T, C, dtype=dtype, device=_dev())
    y2 = torch.full_like(y1, 3.0)
    lse = torch.empty(B, nh, T, dtype=torch.float32, device=_dev())
    s = torch.cuda.current_stream()
    ga.check(ga.gptattn_fwd(qkv, y1, lse, B, T, C, nh, dt, s), "fwd with lse")
    ga.check(ga.gptattn_fwd(qkv, y2, None, B, T, C, nh, dt, s), "fwd without lse")
    if hs == 64 or dtype == torch.float32:
        y3 = torch.full_like(y1, 3.0)
        ga.check(ga.gptattn_fwd_window(qkv, y3, None, B, T, C, nh, 100, dt, s), "windowed fwd without lse")
        y4 = torch.empty_like(y1)
        ga.check(ga.gptattn_fwd_window(qkv, y4, lse, B, T, C, nh, 100, dt, s), "windowed fwd with lse")
        torch.cuda.synchronize()
        assert torch.equal(y3, y4)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    ga.check(ga.gptattn_get_device_status(s), "status")


def test_decode_without_lse():
    B, T, nh, hs = 3, 517, 12, 64
    C = nh * hs
    qkv = make_inputs(B, T, nh, hs, dtype=torch.bfloat16, seed=78)[0].to(_dev())
    y1 = torch.empty(B, C, dtype=torch.bfloat16, device=_dev())
    y2 = torch.full_like(y1, 3.0)
    lse = torch.empty(B, nh, dtype=torch.float32, device=_dev())
    s = torch.cuda.current_stream()
    ga.check(ga.gptattn_decode(qkv, y1, lse, B, T, T, C, nh, ga.GPTATTN_BF16, s), "decode with lse")
    ga.check(ga.gptattn_decode(qkv, y2, None, B, T, T, C, nh, ga.GPTATTN_BF16, s), "decode without lse")
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_attn_block_without_lse():
    B, T, C, nh = 2, 200, 256, 4
    x, p = block_inputs(B, T, C, seed=79)
    d = {k: v.to(_dev()) for k, v in p.items()}
    xd = x.to(_dev())
    outs = []
    for with_lse in (True, False):
        qkv = torch.empty(B, T, 3 * C, dtype=torch.bfloat16, device=_dev())
        y = torch.empty(B, T, C, dtype=torch.bfloat16, device=_dev())
        lse = torch.empty(B, nh, T, dtype=torch.float32, device=_dev()) if with_lse else None
        out = torch.empty(B, T, C, dtype=torch.bfloat16, device=_dev())
        ga.check(ga.gptattn_attn_block_fwd(xd, d["ln_w"], d["ln_b"], d["w_attn"], d["b_attn"], d["w_proj"],
                                           d["b_proj"], qkv, y, lse, out, B, T, C, nh, ga.GPTATTN_BF16,
                                           torch.cuda.current_stream()), "attn_block_fwd")
        outs.append(out)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
