"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and validates arguments before touching the device."""
import ctypes
import os
import re

import pytest

from causal_self_attention_gptattn_b200 import gptattn as ga

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gptattn.h")

FAKE = 0x7f0000000000  # 16-byte aligned address that is never dereferenced


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gptattn_[a-z_0-9]+)\s*\(", text)))


def test_library_builds_and_loads():
    from causal_self_attention_gptattn_b200 import build
    build.build()
    assert os.path.exists(ga.LIB_PATH)
    assert ga.gptattn_version() == 100


def test_exports_every_declared_symbol():
    names = declared_functions()
    assert set(names) == set(ga.EXPORTED), names
    raw = ctypes.CDLL(ga.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), f"{n} not exported"


def test_only_c_abi_symbols_are_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", ga.LIB_PATH], capture_output=True, text=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if " T " in line}
    ours = {s for s in syms if s.startswith("gptattn_")}
    assert ours == set(declared_functions())


def test_status_strings():
    for code in range(6):
        assert ga.gptattn_status_string(code)
    assert ga.gptattn_kernel_name(2) == "bwd_bf16_sm100"
    assert ga.gptattn_kernel_name(99) == "unknown"


@pytest.mark.parametrize("B,T,C,nh,dt,want", [
    (-1, 4, 128, 2, ga.GPTATTN_BF16, ga.GPTATTN_ERR_INVALID_ARG),
    (1, -4, 128, 2, ga.GPTATTN_BF16, ga.GPTATTN_ERR_INVALID_ARG),
    (1, 4, 0, 2, ga.GPTATTN_BF16, ga.GPTATTN_ERR_INVALID_ARG),
    (1, 4, 128, 0, ga.GPTATTN_BF16, ga.GPTATTN_ERR_INVALID_ARG),
    (1, 4, 130, 4, ga.GPTATTN_BF16, ga.GPTATTN_ERR_INVALID_ARG),     # C % n_head != 0
    (1, 4, 96, 3, ga.GPTATTN_BF16, ga.GPTATTN_ERR_UNSUPPORTED),      # hs = 32 on bf16
    (1, 4, 96, 4, ga.GPTATTN_F32, ga.GPTATTN_ERR_UNSUPPORTED),       # hs = 24 on fp32
    (1, 4, 256, 1, ga.GPTATTN_BF16, ga.GPTATTN_ERR_UNSUPPORTED),     # hs = 256
    (1, 4, 128, 2, 7, ga.GPTATTN_ERR_UNSUPPORTED),                   # bad dtype code
])
def test_fwd_shape_validation(B, T, C, nh, dt, want):
    assert ga.gptattn_fwd(FAKE, FAKE, FAKE, B, T, C, nh, dt, None) == want


def test_null_and_misaligned_pointers_rejected():
    args = (2, 8, 128, 2, ga.GPTATTN_BF16, None)
    assert ga.gptattn_fwd(None, FAKE, FAKE, *args) == ga.GPTATTN_ERR_INVALID_ARG
    assert ga.gptattn_fwd(FAKE, None, FAKE, *args) == ga.GPTATTN_ERR_INVALID_ARG
    assert ga.gptattn_fwd(FAKE, FAKE, FAKE + 4, *args) == ga.GPTATTN_ERR_INVALID_ARG  # lse misaligned (NULL is allowed)
    assert ga.gptattn_fwd(FAKE + 8, FAKE, FAKE, *args) == ga.GPTATTN_ERR_INVALID_ARG
    assert ga.gptattn_fwd(FAKE, FAKE + 2, FAKE, *args) == ga.GPTATTN_ERR_INVALID_ARG
    ws = ga.gptattn_bwd_workspace_bytes(2, 8, 128, 2, ga.GPTATTN_BF16)
    assert ga.gptattn_bwd(FAKE, FAKE, FAKE, None, FAKE, FAKE, ws, *args) == ga.GPTATTN_ERR_INVALID_ARG
    assert ga.gptattn_bwd(FAKE, FAKE, None, FAKE, FAKE, FAKE, ws, *args) == ga.GPTATTN_ERR_INVALID_ARG  # bwd needs lse
    assert ga.gptattn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE + 4, FAKE, ws, *args) == ga.GPTATTN_ERR_INVALID_ARG


def test_workspace_checks():
    args = (2, 200, 128, 2, ga.GPTATTN_BF16, None)
    ws = ga.gptattn_bwd_workspace_bytes(2, 200, 128, 2, ga.GPTATTN_BF16)
    # D + lse*log2e (B*nh*T_pad floats each) + dQ accumulator (B*nh*T_pad*hs floats), 256-byte aligned parts
    T_pad = 256
    rows = 2 * 2 * T_pad
    assert ws == rows * 4 + rows * 4 + rows * 64 * 4
    assert ga.gptattn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws - 1, *args) == ga.GPTATTN_ERR_WORKSPACE
    assert ga.gptattn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, None, ws, *args) == ga.GPTATTN_ERR_WORKSPACE
    assert ga.gptattn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 16, ws, *args) == ga.GPTATTN_ERR_WORKSPACE
    assert ga.gptattn_bwd_workspace_bytes(2, 64, 64, 4, ga.GPTATTN_F32) == 2 * 4 * 64 * 4
    assert ga.gptattn_bwd_workspace_bytes(2, 64, 65, 4, ga.GPTATTN_F32) == (1 << 64) - 1
    assert ga.gptattn_bwd_workspace_bytes(0, 64, 64, 4, ga.GPTATTN_F32) == 0


def test_empty_calls_are_noops():
    for dt, C in ((ga.GPTATTN_BF16, 128), (ga.GPTATTN_F32, 64)):
        assert ga.gptattn_fwd(None, None, None, 0, 16, C, 2, dt, None) == ga.GPTATTN_OK
        assert ga.gptattn_fwd(None, None, None, 3, 0, C, 2, dt, None) == ga.GPTATTN_OK
        assert ga.gptattn_bwd(None, None, None, None, None, None, 0, 0, 16, C, 2, dt, None) == ga.GPTATTN_OK


def test_selftest_budget_range():
    assert ga.gptattn_selftest_wait_timeout(10, None) == ga.GPTATTN_ERR_INVALID_ARG
    assert ga.gptattn_selftest_wait_timeout(3 * 10**9, None) == ga.GPTATTN_ERR_INVALID_ARG


def test_profile_enable_rejects_negative():
    assert ga.gptattn_profile_enable(-1) == ga.GPTATTN_ERR_INVALID_ARG
    assert ga.gptattn_profile_enable(0) == ga.GPTATTN_OK
    assert ga.gptattn_profile_read(8) == []


def test_decode_validation():
    bf, f32 = ga.GPTATTN_BF16, ga.GPTATTN_F32
    assert ga.gptattn_decode(FAKE, FAKE, FAKE, 2, 9, 8, 128, 2, bf, None) == ga.GPTATTN_ERR_INVALID_ARG  # T > T_cap
    assert ga.gptattn_decode(FAKE, FAKE, FAKE, 2, 8, 8, 96, 3, bf, None) == ga.GPTATTN_ERR_UNSUPPORTED  # hs = 32 on bf16
    assert ga.gptattn_decode(FAKE, FAKE, FAKE, 2, 8, 8, 96, 4, f32, None) == ga.GPTATTN_ERR_UNSUPPORTED  # hs = 24
    assert ga.gptattn_decode(FAKE, FAKE, FAKE, 40000, 8, 8, 128, 2, bf, None) == ga.GPTATTN_ERR_UNSUPPORTED  # grid.y
    assert ga.gptattn_decode(None, FAKE, FAKE, 2, 8, 8, 128, 2, bf, None) == ga.GPTATTN_ERR_INVALID_ARG
    assert ga.gptattn_decode(FAKE, FAKE + 2, FAKE, 2, 8, 8, 128, 2, bf, None) == ga.GPTATTN_ERR_INVALID_ARG
    assert ga.gptattn_decode(None, None, None, 0, 8, 8, 128, 2, bf, None) == ga.GPTATTN_OK
    assert ga.gptattn_decode(None, None, None, 2, 0, 8, 128, 2, f32, None) == ga.GPTATTN_OK
    assert ga.gptattn_kernel_name(9) == "decode"


def test_window_validation():
    bf, f32 = ga.GPTATTN_BF16, ga.GPTATTN_F32
    assert ga.gptattn_fwd_window(FAKE, FAKE, FAKE, 2, 8, 128, 2, 0, bf, None) == ga.GPTATTN_ERR_INVALID_ARG
    assert ga.gptattn_fwd_window(FAKE, FAKE, FAKE, 2, 8, 128, 2, -3, f32, None) == ga.GPTATTN_ERR_INVALID_ARG
    ws = ga.gptattn_bwd_workspace_bytes(2, 300, 256, 2, bf)
    assert ga.gptattn_bwd_window(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, 2, 300, 256, 2, 0, bf,
                                 None) == ga.GPTATTN_ERR_INVALID_ARG
    # bf16 head size 128 takes any window: a bad pointer, not the shape, is what is refused here
    assert ga.gptattn_fwd_window(FAKE + 2, FAKE, FAKE, 2, 300, 256, 2, 100, bf, None) == ga.GPTATTN_ERR_INVALID_ARG
    assert ga.gptattn_fwd_window(None, None, None, 0, 8, 128, 2, 4, bf, None) == ga.GPTATTN_OK
    assert ga.gptattn_bwd_window(None, None, None, None, None, None, 0, 2, 0, 64, 4, 4, f32, None) == ga.GPTATTN_OK


def test_deterministic_backward_workspace_and_validation():
    bf, f32 = ga.GPTATTN_BF16, ga.GPTATTN_F32
    B, T, C, nh = 2, 300, 128, 2  # 3 query tiles -> 6 partial tiles per (b, h)
    rows = B * nh * 384
    base = rows * 4 + rows * 4
    assert ga.gptattn_bwd_det_workspace_bytes(B, T, C, nh, bf) == base + B * nh * 6 * 128 * 64 * 4
    assert ga.gptattn_bwd_det_workspace_bytes(B, T, C, nh, f32) == ga.gptattn_bwd_workspace_bytes(B, T, C, nh, f32)
    # head size 128: D, lse*log2e and 6 partial tiles of 128 x 128 fp32 per (b, h)
    assert ga.gptattn_bwd_det_workspace_bytes(B, T, 256, nh, bf) == base + B * nh * 6 * 128 * 128 * 4
    ws = ga.gptattn_bwd_det_workspace_bytes(B, T, C, nh, bf)
    assert ga.gptattn_bwd_det(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws - 1, B, T, C, nh, 10**6, bf,
                              None) == ga.GPTATTN_ERR_WORKSPACE
    # head size 128 needs its own (larger) workspace
    assert ga.gptattn_bwd_det(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, B, T, 256, nh, 10**6, bf,
                              None) == ga.GPTATTN_ERR_WORKSPACE
    assert ga.gptattn_bwd_det(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, B, T, C, nh, 0, bf,
                              None) == ga.GPTATTN_ERR_INVALID_ARG
    assert ga.gptattn_bwd_det(None, None, None, None, None, None, 0, 0, T, C, nh, 1, bf, None) == ga.GPTATTN_OK


def test_options_validation():
    bf, f32 = ga.GPTATTN_BF16, ga.GPTATTN_F32
    O = ga.Options
    args = (2, 8, 128, 2)
    assert ga.gptattn_fwd_opts(FAKE, FAKE, FAKE, *args, O(window=-1), bf, None) == ga.GPTATTN_ERR_INVALID_ARG
    assert ga.gptattn_fwd_opts(FAKE, FAKE, FAKE, *args, O(dropout_p=1.0), bf, None) == ga.GPTATTN_ERR_INVALID_ARG
    assert ga.gptattn_fwd_opts(FAKE, FAKE, FAKE, *args, O(dropout_p=-0.1), f32, None) == ga.GPTATTN_ERR_INVALID_ARG
    # bf16 dropout at head size 128 is accepted (an empty batch launches nothing)
    assert ga.gptattn_fwd_opts(None, None, None, 0, 8, 256, 2, O(dropout_p=0.1), bf, None) == ga.GPTATTN_OK
    assert ga.gptattn_fwd_opts(None, None, None, 0, 8, 128, 2, None, bf, None) == ga.GPTATTN_OK
    assert ga.gptattn_bwd_opts_workspace_bytes(*args, None, bf) == ga.gptattn_bwd_workspace_bytes(*args, bf)
    assert ga.gptattn_bwd_opts_workspace_bytes(*args, O(deterministic=1), bf) == \
        ga.gptattn_bwd_det_workspace_bytes(*args, bf)
    assert ga.gptattn_bwd_opts_workspace_bytes(*args, O(window=-2), bf) == (1 << 64) - 1


def test_block_validation():
    BF, F32 = ga.GPTATTN_BF16, ga.GPTATTN_F32
    OK, INV, UNS = 0, ga.GPTATTN_ERR_INVALID_ARG, ga.GPTATTN_ERR_UNSUPPORTED
    # layernorm: C % 8, C <= 4096, bf16 only, pointers
    assert ga.gptattn_layernorm(FAKE, FAKE, FAKE, FAKE, 4, 12, BF) == UNS
    assert ga.gptattn_layernorm(FAKE, FAKE, FAKE, FAKE, 4, 4104, BF) == UNS
    assert ga.gptattn_layernorm(FAKE, FAKE, FAKE, FAKE, 4, 768, F32) == UNS
    assert ga.gptattn_layernorm(None, FAKE, FAKE, FAKE, 4, 768, BF) == INV
    assert ga.gptattn_layernorm(FAKE + 2, FAKE, FAKE, FAKE, 4, 768, BF) == INV
    assert ga.gptattn_layernorm(FAKE, FAKE, FAKE, FAKE, -1, 768, BF) == INV
    assert ga.gptattn_layernorm(None, None, None, None, 0, 768, BF) == OK
    # linear: N % 64, K % 64, pointers; bias and resid optional but aligned
    assert ga.gptattn_linear(FAKE, FAKE, FAKE, None, FAKE, 8, 96, 64, BF) == UNS
    assert ga.gptattn_linear(FAKE, FAKE, FAKE, None, FAKE, 8, 64, 32, BF) == UNS
    assert ga.gptattn_linear(FAKE, FAKE, FAKE, None, FAKE, 8, 64, 64, F32) == UNS
    assert ga.gptattn_linear(None, FAKE, FAKE, None, FAKE, 8, 64, 64, BF) == INV
    assert ga.gptattn_linear(FAKE, FAKE, FAKE + 8, None, FAKE, 8, 64, 64, BF) == INV
    assert ga.gptattn_linear(FAKE, FAKE, None, FAKE + 4, FAKE, 8, 64, 64, BF) == INV
    assert ga.gptattn_linear(FAKE, FAKE, None, None, FAKE, 8, 0, 64, BF) == INV
    assert ga.gptattn_linear(None, None, None, None, None, 0, 64, 64, BF) == OK
    # block: attention shape rules + the two above
    args = [FAKE] * 11
    assert ga.gptattn_attn_block_fwd(*args, 2, 16, 96, 3, BF) == UNS      # head size 32
    assert ga.gptattn_attn_block_fwd(*args, 2, 16, 768, 12, F32) == UNS
    assert ga.gptattn_attn_block_fwd(*args[:9], FAKE + 4, FAKE, 2, 16, 768, 12, BF) == INV   # lse misaligned
    assert ga.gptattn_attn_block_fwd(*args[:5], FAKE + 2, *args[6:], 2, 16, 768, 12, BF) == INV   # w_proj
    assert ga.gptattn_attn_block_fwd(*([None] * 11), 0, 16, 768, 12, BF) == OK
    assert ga.gptattn_attn_block_fwd(*([None] * 11), 2, 0, 768, 12, BF) == OK


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="needs a machine without a usable CUDA device")
def test_cuda_failure_maps_to_status_and_message():
    """Fault injection from the environment: with no usable device, every call that passes validation
    fails in the CUDA runtime, returns GPTATTN_ERR_CUDA and leaves the runtime's message readable."""
    assert ga.gptattn_fwd(FAKE, FAKE, FAKE, 2, 8, 128, 2, ga.GPTATTN_BF16, None) == ga.GPTATTN_ERR_CUDA
    assert ga.gptattn_last_error_string() not in ("", "no error")
    assert ga.gptattn_fwd(FAKE, FAKE, FAKE, 2, 8, 64, 4, ga.GPTATTN_F32, None) == ga.GPTATTN_ERR_CUDA
    ws = ga.gptattn_bwd_workspace_bytes(2, 8, 128, 2, ga.GPTATTN_BF16)
    assert ga.gptattn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, 2, 8, 128, 2, ga.GPTATTN_BF16, None) == \
        ga.GPTATTN_ERR_CUDA
    assert ga.gptattn_linear(FAKE, FAKE, None, None, FAKE, 8, 64, 64, ga.GPTATTN_BF16, None) == ga.GPTATTN_ERR_CUDA
    assert ga.gptattn_get_device_status(None) == ga.GPTATTN_ERR_CUDA
