"""Run the CUDA path through the C ABI on torch-allocated buffers with guard bands,
and compare with the fp64 oracle."""
from __future__ import annotations

import numpy as np
import torch

from causal_self_attention_gptattn_b200 import gptattn as ga

GUARD = 4096          # elements of guard band on each side of every output buffer
FILL = {torch.bfloat16: 7.0, torch.float32: -7.0}

# Tolerances (written here, used by every parity test):
#   fp32 path: max |err| <= 1e-4 for y, lse and dqkv
#   bf16 path: max |err| <= 2e-2 for y; max |err| <= 5e-2 * max|ref| for dqkv;
#              lse max |err| <= 1e-2
TOL_F32 = 1e-4
TOL_BF16_Y = 2e-2
TOL_BF16_DQKV_REL = 5e-2
TOL_BF16_LSE = 1e-2


class Guarded:
    """A flat device buffer with sentinel-filled bands before and after the view."""

    def __init__(self, n: int, dtype, device):
        self.fill = FILL[dtype]
        self.buf = torch.full((n + 2 * GUARD,), self.fill, dtype=dtype, device=device)
        self.view = self.buf[GUARD:GUARD + n]

    def intact(self) -> bool:
        lo = self.buf[:GUARD]
        hi = self.buf[GUARD + self.view.numel():]
        return bool((lo == self.fill).all().item() and (hi == self.fill).all().item())


def run_fwd_bwd(qkv_cpu: torch.Tensor, dy_cpu: torch.Tensor, n_head: int, stream=None, window=None, opts=None):
    """Forward + backward through the C ABI (the local-window entry points when
    window is given, the options entry points when opts is given).  Returns
    float64 numpy (y, lse, dqkv)."""
    dev = torch.device("cuda", 0)
    dtype = qkv_cpu.dtype
    dt = ga.GPTATTN_BF16 if dtype == torch.bfloat16 else ga.GPTATTN_F32
    B, T, C3 = qkv_cpu.shape
    C = C3 // 3
    qkv = qkv_cpu.to(dev).contiguous()
    dy = dy_cpu.to(dev).contiguous()
    y = Guarded(B * T * C, dtype, dev)
    lse = Guarded(B * n_head * T, torch.float32, dev)
    dqkv = Guarded(B * T * 3 * C, dtype, dev)
    nbytes = (ga.gptattn_bwd_workspace_bytes(B, T, C, n_head, dt) if opts is None
              else ga.gptattn_bwd_opts_workspace_bytes(B, T, C, n_head, opts, dt))
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    if opts is not None:
        ga.check(ga.gptattn_fwd_opts(qkv, y.view, lse.view, B, T, C, n_head, opts, dt, s), "gptattn_fwd_opts")
        ga.check(ga.gptattn_bwd_opts(qkv, y.view, lse.view, dy, dqkv.view, ws, nbytes, B, T, C, n_head, opts, dt, s),
                 "gptattn_bwd_opts")
    elif window is None:
        ga.check(ga.gptattn_fwd(qkv, y.view, lse.view, B, T, C, n_head, dt, s), "gptattn_fwd")
        ga.check(ga.gptattn_bwd(qkv, y.view, lse.view, dy, dqkv.view, ws, nbytes, B, T, C, n_head, dt, s),
                 "gptattn_bwd")
    else:
        ga.check(ga.gptattn_fwd_window(qkv, y.view, lse.view, B, T, C, n_head, window, dt, s), "gptattn_fwd_window")
        ga.check(ga.gptattn_bwd_window(qkv, y.view, lse.view, dy, dqkv.view, ws, nbytes, B, T, C, n_head, window, dt,
                                       s), "gptattn_bwd_window")
    rc = ga.gptattn_get_device_status(s)
    assert rc == ga.GPTATTN_OK, ga.status_string(rc)
    assert y.intact() and lse.intact() and dqkv.intact(), "write outside an output buffer"
    out_y = y.view.view(B, T, C).double().cpu().numpy()
    out_lse = lse.view.view(B, n_head, T).double().cpu().numpy()
    out_dqkv = dqkv.view.view(B, T, 3 * C).double().cpu().numpy()
    return out_y, out_lse, out_dqkv


def select_heads(x: np.ndarray, n_head: int, parts: int, heads) -> np.ndarray:
    """Keep only the given heads' columns of a [B, T, parts*C] array (column order kept)."""
    B, T, W = x.shape
    C = W // parts
    hs = C // n_head
    v = x.reshape(B, T, parts, n_head, hs)[:, :, :, list(heads)]
    return v.reshape(B, T, parts * len(heads) * hs)


def compare(got, ref, dtype, what=""):
    """Assert the tolerances above; returns (y_err, lse_err, dqkv_err, dqkv_scale)."""
    y, lse, dqkv = got
    ry, rlse, rdqkv = ref
    ey = float(np.abs(y - ry).max()) if ry.size else 0.0
    el = float(np.abs(lse - rlse).max()) if rlse.size else 0.0
    eg = float(np.abs(dqkv - rdqkv).max()) if rdqkv.size else 0.0
    sg = float(np.abs(rdqkv).max()) if rdqkv.size else 0.0
    assert np.isfinite(y).all() and np.isfinite(lse).all() and np.isfinite(dqkv).all(), what
    if dtype == torch.float32:
        assert ey <= TOL_F32, f"{what} y err {ey:.3e}"
        assert el <= TOL_F32, f"{what} lse err {el:.3e}"
        assert eg <= TOL_F32, f"{what} dqkv err {eg:.3e}"
    else:
        assert ey <= TOL_BF16_Y, f"{what} y err {ey:.3e}"
        assert el <= TOL_BF16_LSE, f"{what} lse err {el:.3e}"
        assert eg <= TOL_BF16_DQKV_REL * sg, f"{what} dqkv err {eg:.3e} vs scale {sg:.3e}"
    return ey, el, eg, sg
