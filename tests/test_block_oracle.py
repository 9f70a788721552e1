"""Pins of the attention sub-block oracle, and planted mistakes in copies of it
(on the CPU) that each must trip at least one pin."""
import importlib.util

import numpy as np
import pytest

import oracle.block as block
from block_pins import BLOCK_PINS

SRC = open(block.__file__).read()

# (name, original text, mutated text) -- each original occurs exactly once
MUTANTS = [
    ("ln_unbiased_variance", "var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)",
     "var = ((x - mean) ** 2).sum(axis=-1, keepdims=True) / (x.shape[-1] - 1)"),
    ("ln_eps_dropped", "np.sqrt(var + eps)", "np.sqrt(var)"),
    ("ln_eps_outside_sqrt", "np.sqrt(var + eps)", "(np.sqrt(var) + eps)"),
    ("ln_over_tokens", "mean = x.mean(axis=-1, keepdims=True)", "mean = x.mean(axis=-2, keepdims=True)"),
    ("ln_gain_dropped", "eps) * w + b", "eps) + b"),
    ("ln_bias_dropped", "eps) * w + b", "eps) * w"),
    ("linear_transposed", "out = x @ w.T", "out = x @ w"),
    ("linear_bias_dropped", "out = out + _f64(b)", "out = out"),
    ("residual_on_normalised", "out = x + linear(y, w_proj, b_proj)", "out = xn + linear(y, w_proj, b_proj)"),
    ("residual_dropped", "out = x + linear(y, w_proj, b_proj)", "out = linear(y, w_proj, b_proj)"),
    ("post_norm", "qkv = linear(xn, w_attn, b_attn)", "qkv = linear(x, w_attn, b_attn)"),
]


@pytest.mark.parametrize("pin", BLOCK_PINS, ids=[p.__name__ for p in BLOCK_PINS])
def test_block_pin(orc, pin):
    pin(block, orc)


def _load_mutant(tmp_path, name, text):
    path = tmp_path / f"block_{name}.py"
    path.write_text(text)
    spec = importlib.util.spec_from_file_location(f"block_mutant_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.filterwarnings("ignore::RuntimeWarning")  # broken copies may average empty slices
@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_block_mutant_is_caught(orc, tmp_path, name, old, new):
    assert SRC.count(old) == 1, f"mutation anchor for {name} not unique"
    mutant = _load_mutant(tmp_path, name, SRC.replace(old, new))
    failed = []
    with np.errstate(all="ignore"):
        for pin in BLOCK_PINS:
            try:
                pin(mutant, orc)
            except (AssertionError, ValueError, FloatingPointError):
                failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
