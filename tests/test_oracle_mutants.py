"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that
each one trips at least one pin -- evidence that the pins constrain every
step: the scale, the mask, the softmax shift, operand order and the backward
terms."""

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = open(oracle.SOURCE).read()

# (name, original text, mutated text) -- each original occurs exactly once
MUTANTS = [
    ("scale_by_sqrt_C", "Pt[s] = acc * scale;", "Pt[s] = acc * (1.0 / sqrt((double)C));"),
    ("scale_dropped", "Pt[s] = acc * scale;", "Pt[s] = acc;"),
    ("lse_missing_max", "lse_row[t] = m + log(l);", "lse_row[t] = log(l);"),
    ("scores_transposed",
     "acc += qkv_at(qkv, T, C, hs, b, t, 0, h, d) * qkv_at(qkv, T, C, hs, b, s, 1, h, d);",
     "acc += qkv_at(qkv, T, C, hs, b, s, 0, h, d) * qkv_at(qkv, T, C, hs, b, t, 1, h, d);"),
    ("output_sums_keys", "acc += Pt[s] * drop_factor(dr, bh, t, s) * qkv_at(qkv, T, C, hs, b, s, 2, h, d);",
     "acc += Pt[s] * drop_factor(dr, bh, t, s) * qkv_at(qkv, T, C, hs, b, s, 1, h, d);"),
    ("future_leaks", "for (int s = t + 1; s < T; ++s) Pt[s] = 0.0;",
     "for (int s = t + 1; s < T; ++s) Pt[s] = (s == t + 1) ? 1e-3 : 0.0;"),
    ("softmax_jacobian_sign", "dSt[s] = Pt[s] * (dSt[s] - rowdot);", "dSt[s] = Pt[s] * (dSt[s] + rowdot);"),
    ("softmax_jacobian_dropped", "dSt[s] = Pt[s] * (dSt[s] - rowdot);", "dSt[s] = Pt[s] * dSt[s];"),
    ("dP_uses_keys",
     "acc += dyb[(size_t)t * ld_dy + d] * qkv_at(qkv, T, C, hs, b, s, 2, h, d);",
     "acc += dyb[(size_t)t * ld_dy + d] * qkv_at(qkv, T, C, hs, b, s, 1, h, d);"),
    ("dV_transposed_P", "acc += P[(size_t)t * (size_t)T + s] * drop_factor(&dr, b * n_head + h, t, s) *",
     "acc += P[(size_t)s * (size_t)T + t] * drop_factor(&dr, b * n_head + h, t, s) *"),
    ("dQ_uses_queries",
     "acc += dS[(size_t)t * (size_t)T + s] * qkv_at(qkv, T, C, hs, b, s, 1, h, d);",
     "acc += dS[(size_t)t * (size_t)T + s] * qkv_at(qkv, T, C, hs, b, s, 0, h, d);"),
    ("dK_missing_scale", "dk[(size_t)s * ld_dqkv + d] = acc * scale;", "dk[(size_t)s * ld_dqkv + d] = acc;"),
    ("dropout_scale_missing", "? 1.0 / (1.0 - theta / 256.0) : 0.0;", "? 1.0 : 0.0;"),
    ("dropout_scale_unquantised", "? 1.0 / (1.0 - theta / 256.0) : 0.0;", "? 1.0 / (1.0 - dr->p) : 0.0;"),
    ("dropout_block_transposed", "return ((r[t & 3] >> (8 * (s & 3))) & 0xFFu) >= theta;",
     "return ((r[s & 3] >> (8 * (t & 3))) & 0xFFu) >= theta;"),
    ("dropout_mask_ignored_in_dP", "acc *= drop_factor(&dr, b * n_head + h, t, s);", "acc *= 1.0 / (1.0 - dr.p);"),
    ("band_one_key_too_many", "return t - window + 1 > 0 ? t - window + 1 : 0;", "return t - window > 0 ? t - window : 0;"),
    ("band_last_query_dropped", "return s + window - 1 < T - 1 ? s + window - 1 : T - 1;",
     "return s + window - 2 < T - 1 ? s + window - 2 : T - 1;"),
    ("dK_transposed_dS",
     "acc += dS[(size_t)t * (size_t)T + s] * qkv_at(qkv, T, C, hs, b, t, 0, h, d);",
     "acc += dS[(size_t)s * (size_t)T + t] * qkv_at(qkv, T, C, hs, b, t, 0, h, d);"),
    # the dropout generator: mistakes that keep its output uniform, so only the
    # published known-answer vectors can catch them
    ("philox_nine_rounds", "for (int round = 0; round < 10; ++round)", "for (int round = 0; round < 9; ++round)"),
    ("philox_multipliers_swapped", "const uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)c0;",
     "const uint64_t p0 = (uint64_t)PHILOX_M1 * (uint64_t)c0;"),
    ("philox_key_schedule_swapped", "k0 += PHILOX_W0;", "k0 += PHILOX_W1;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    assert SRC.count(old) == 1, f"mutation anchor for {name} not unique"
    src = tmp_path / f"{name}.c"
    src.write_text(SRC.replace(old, new))
    so = oracle.compile_source(str(src), str(tmp_path / f"{name}.so"))
    mutant = oracle.Oracle(so)
    failed = []
    for pin in ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, RuntimeError, ValueError, FloatingPointError):
            failed.append(pin.__name__)
            break
    assert failed, f"mutant {name} passed every pin"
