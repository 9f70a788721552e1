"""Seeded synthetic inputs for causal self-attention, shared by tests and bench.

This module holds input recipes only -- none of the attention arithmetic.  The
same arrays feed both the CUDA path and the fp64 oracle, so it is the one
module the two sides have in common.

Shapes follow the pages' workloads:
  * ``fp32_tiny``      -- B=2, T=64, 4 heads of 16 (C=64), fp32: a small case the
                          oracle finishes instantly (the nanoGPT README's CPU run uses
                          4 heads, 64-token context).
  * ``baby_gpt``       -- B=64, T=256, 6 heads of 64 (C=384): the shape of the
                          README's char-level "baby GPT" config.  Its qkv is the
                          projection of layer-normed activations, LN(x) @ W with
                          x ~ N(0,1), W ~ N(0, 0.02^2) (the minGPT notes' init),
                          computed in fp32 and rounded to bf16.
  * ``gpt2_124m``      -- B=16, T=1024, 12 heads of 64 (C=768): GPT-2 124M.
  * ``gpt2_1p5b``      -- B=8, T=1024, 25 heads of 64 (C=1600): GPT-2 1.5B.
  * ``long_context``   -- B=4, T=2048, 16 heads of 128 (C=2048): GPT-3-style
                          2048-token window; qkv ~ 2*N(0,1) for a sharper softmax.
For all of them dy ~ N(0,1).  Values are drawn in fp32 from a CPU
``torch.Generator`` seeded with 1000 + config index (draw order: x then W, or
qkv; then dy) and cast to the compute dtype afterwards.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int
    name: str
    dtype: str          # "f32" or "bf16"
    B: int
    T: int
    n_head: int
    hs: int
    recipe: str = "iid"     # "iid" or "ln_proj"
    qkv_scale: float = 1.0

    @property
    def C(self) -> int:
        return self.n_head * self.hs

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def flops_fwd(self) -> float:
        """Causal forward FLOPs, counted as half of the dense 2 matmuls."""
        return 2.0 * self.B * self.n_head * self.T * self.T * self.hs

    def flops_bwd(self) -> float:
        """Causal backward FLOPs (5 matmuls, half of dense)."""
        return 2.5 * self.flops_fwd()

    def flops_fwd_bwd(self) -> float:
        return 3.5 * self.flops_fwd()

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "T": self.T, "n_head": self.n_head,
                "head_size": self.hs, "C": self.C, "dtype": self.dtype}


WORKLOADS = {
    1: Workload(1, "fp32_tiny", "f32", 2, 64, 4, 16),
    2: Workload(2, "baby_gpt", "bf16", 64, 256, 6, 64, recipe="ln_proj"),
    3: Workload(3, "gpt2_124m", "bf16", 16, 1024, 12, 64),
    4: Workload(4, "gpt2_1p5b", "bf16", 8, 1024, 25, 64),
    5: Workload(5, "long_context", "bf16", 4, 2048, 16, 128, qkv_scale=2.0),
}


def by_name(name: str) -> Workload:
    for w in WORKLOADS.values():
        if w.name == name:
            return w
    raise KeyError(name)


def make_inputs(B: int, T: int, n_head: int, hs: int, dtype=torch.bfloat16, seed: int = 0,
                recipe: str = "iid", qkv_scale: float = 1.0):
    """Return (qkv[B,T,3C], dy[B,T,C]) on the CPU in ``dtype``."""
    C = n_head * hs
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    if recipe == "ln_proj":
        x = torch.randn(B, T, C, generator=g, dtype=torch.float32)
        W = torch.randn(C, 3 * C, generator=g, dtype=torch.float32) * 0.02
        xn = torch.nn.functional.layer_norm(x, (C,), eps=1e-5)
        qkv = xn @ W
    elif recipe == "iid":
        qkv = torch.randn(B, T, 3 * C, generator=g, dtype=torch.float32)
    else:
        raise ValueError(recipe)
    if qkv_scale != 1.0:
        qkv = qkv * qkv_scale
    dy = torch.randn(B, T, C, generator=g, dtype=torch.float32)
    return qkv.to(dtype).contiguous(), dy.to(dtype).contiguous()


def workload_inputs(w: Workload, B: int | None = None, T: int | None = None):
    """Seeded inputs of a named workload (optionally with B or T overridden)."""
    return make_inputs(B if B is not None else w.B, T if T is not None else w.T, w.n_head, w.hs,
                       dtype=w.torch_dtype, seed=1000 + w.index, recipe=w.recipe,
                       qkv_scale=w.qkv_scale)


def block_inputs(B: int, T: int, C: int, seed: int = 0):
    """Seeded inputs of the pre-LN attention sub-block, bf16 on the CPU:
    x[B,T,C] ~ N(0,1); LayerNorm gain 1 + 0.1 N(0,1) and bias 0.1 N(0,1);
    c_attn weight [3C][C] and c_proj weight [C][C] ~ N(0,1)/sqrt(C) (so the
    projected queries and keys are O(1) and the softmax is not flat); both
    biases 0.1 N(0,1).  Draw order: x, ln_w, ln_b, w_attn, b_attn, w_proj, b_proj."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    rn = lambda *shape: torch.randn(*shape, generator=g, dtype=torch.float32)
    x = rn(B, T, C)
    p = {"ln_w": 1.0 + 0.1 * rn(C), "ln_b": 0.1 * rn(C),
         "w_attn": rn(3 * C, C) / C ** 0.5, "b_attn": 0.1 * rn(3 * C),
         "w_proj": rn(C, C) / C ** 0.5, "b_proj": 0.1 * rn(C)}
    return x.to(torch.bfloat16).contiguous(), {k: v.to(torch.bfloat16).contiguous() for k, v in p.items()}
