"""gptattn_bwd_noalloc: the backward for callers that cannot allocate device
memory (for example a plugin inside a runtime that owns all device memory).
Its scratch is a fixed array inside the library, so this checks, through the C
ABI, that two calls in a row give the same dqkv as the regular gptattn_bwd with
a caller-allocated workspace (within the bf16 / fp32 parity tolerances), and
that shapes needing more scratch than the array holds are refused.

Kept in a file of its own that pytest collects last."""
import pytest
import torch

from causal_self_attention_gptattn_b200 import gptattn as ga
from causal_self_attention_gptattn_b200.workloads import make_inputs
from gpu_helpers import TOL_BF16_DQKV_REL, TOL_F32

pytestmark = pytest.mark.gpu


def _fwd(qkv, B, T, C, nh, dt, s):
    y = torch.empty(B, T, C, dtype=qkv.dtype, device=qkv.device)
    lse = torch.empty(B, nh, T, dtype=torch.float32, device=qkv.device)
    ga.check(ga.gptattn_fwd(qkv, y, lse, B, T, C, nh, dt, s), "gptattn_fwd")
    return y, lse


@pytest.mark.parametrize("B,T,nh,hs,dtype", [(2, 300, 3, 64, torch.bfloat16), (1, 257, 2, 128, torch.bfloat16),
                                             (2, 70, 4, 16, torch.float32)])
def test_noalloc_matches_workspace_backward(B, T, nh, hs, dtype):
    dev = torch.device("cuda", 0)
    s = torch.cuda.current_stream(dev)
    dt = ga.GPTATTN_BF16 if dtype == torch.bfloat16 else ga.GPTATTN_F32
    C = nh * hs
    qkv_c, dy_c = make_inputs(B, T, nh, hs, dtype=dtype, seed=99 + T)
    qkv, dy = qkv_c.to(dev), dy_c.to(dev)
    y, lse = _fwd(qkv, B, T, C, nh, dt, s)

    ref = torch.empty_like(qkv)
    nbytes = ga.gptattn_bwd_workspace_bytes(B, T, C, nh, dt)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    ga.check(ga.gptattn_bwd(qkv, y, lse, dy, ref, ws, nbytes, B, T, C, nh, dt, s), "gptattn_bwd")

    scale = ref.float().abs().max().item()
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16_DQKV_REL * scale
    for call in range(2):  # the shared scratch keeps the previous call's contents
        out = torch.full_like(qkv, float("nan"))
        ga.check(ga.gptattn_bwd_noalloc(qkv, y, lse, dy, out, B, T, C, nh, dt, s), "gptattn_bwd_noalloc")
        ga.check(ga.gptattn_get_device_status(s), "device status")
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= tol, f"call {call}: max |noalloc - bwd| = {err:.3e} > {tol:.3e}"


def test_noalloc_refuses_shapes_beyond_its_scratch():
    B, T, nh, hs = 16, 2048, 16, 128       # needs far more than 64 MiB of scratch
    C = nh * hs
    assert ga.gptattn_bwd_workspace_bytes(B, T, C, nh, ga.GPTATTN_BF16) > ga.GPTATTN_NOALLOC_SCRATCH_BYTES
    before = ga.gptattn_launch_count()
    x = torch.zeros(16, device="cuda")
    rc = ga.gptattn_bwd_noalloc(x, x, x, x, x, B, T, C, nh, ga.GPTATTN_BF16, torch.cuda.current_stream())
    assert rc == ga.GPTATTN_ERR_WORKSPACE
    assert ga.gptattn_launch_count() == before
