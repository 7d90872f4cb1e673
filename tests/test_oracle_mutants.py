"""The oracle's pins catch plausible mistakes: each case compiles a copy of
zero_oracle.c with one mistake planted (on the CPU, in a temporary
directory), runs the named pin against it and expects that pin to fail."""
import os

import pytest

import oracle
from oracle import build as obuild

import test_oracle_adam as A
import test_oracle_adam_invariants as I
import test_oracle_bf16 as B
import test_oracle_reduce as R

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "zero_oracle.c")

MUTANTS = [
    ("bf16 truncates instead of rounding",
     "  if (d_tz < d_aw) return toward_zero;\n  if (d_aw < d_tz) return away;",
     "  return toward_zero;",
     lambda: R.test_mean_exact_when_accumulation_exact(8)),
    ("ties round up instead of to even",
     "  return (toward_zero & 1u) ? away : toward_zero;",
     "  return away;",
     lambda: B.test_bf16_rne_worked_cases(1.0 + 2.0**-8, 0x3F80)),
    ("rank order reversed",
     "    for (int32_t r = 0; r < n_ranks; ++r) acc = acc + zo_bf16_to_f32(rank_grads[r][i]);\n    out[i] = acc;",
     "    for (int32_t r = n_ranks - 1; r >= 0; --r) acc = acc + zo_bf16_to_f32(rank_grads[r][i]);\n    out[i] = acc;",
     R.test_rank_order_matters_and_is_zero_to_n_minus_1),
    ("mean not divided by N",
     "    out[i] = zo_bf16_rne(acc * inv_n);",
     "    out[i] = zo_bf16_rne(acc);",
     lambda: R.test_mean_exact_when_accumulation_exact(4)),
    ("bias correction of m dropped",
     "    const float mh = mi / bc1;\n    const float vh = vi / bc2;\n    const float den = sqrtf(vh) + eps_f;\n    const float ratio = mh / den;\n    const float upd = lr_f * ratio;\n    p = p - upd;\n    master[i] = p;\n    m[i] = mi;\n    v[i] = vi;\n    if (p_out) p_out[i] = zo_bf16_rne(p);\n  }\n}\n\n/*\n * The same Adam",
     "    const float mh = mi;\n    const float vh = vi / bc2;\n    const float den = sqrtf(vh) + eps_f;\n    const float ratio = mh / den;\n    const float upd = lr_f * ratio;\n    p = p - upd;\n    master[i] = p;\n    m[i] = mi;\n    v[i] = vi;\n    if (p_out) p_out[i] = zo_bf16_rne(p);\n  }\n}\n\n/*\n * The same Adam",
     lambda: A.test_adam_matches_torch_adamw(0.0)),
    ("update sign flipped",
     "    p = p - upd;\n    master[i] = p;\n    m[i] = mi;\n    v[i] = vi;\n    if (p_out) p_out[i] = zo_bf16_rne(p);\n  }\n}\n\n/*\n * The same Adam",
     "    p = p + upd;\n    master[i] = p;\n    m[i] = mi;\n    v[i] = vi;\n    if (p_out) p_out[i] = zo_bf16_rne(p);\n  }\n}\n\n/*\n * The same Adam",
     A.test_first_step_moves_each_weight_by_lr_against_the_gradient_sign),
    ("beta2 used for the first moment",
     "    float a = b1 * m[i];\n    float b = omb1 * gi;\n    const float mi = a + b;\n    const float gg = gi * gi;\n    a = b2 * v[i];\n    b = omb2 * gg;\n    const float vi = a + b;\n    const float mh = mi / bc1;\n    const float vh = vi / bc2;\n    const float den = sqrtf(vh) + eps_f;\n    const float ratio = mh / den;\n    const float upd = lr_f * ratio;\n    p = p - upd;\n    master[i] = p;\n    m[i] = mi;\n    v[i] = vi;\n    if (p_out) p_out[i] = zo_bf16_rne(p);\n  }\n}\n\n/*\n * The same Adam",
     "    float a = b2 * m[i];\n    float b = omb1 * gi;\n    const float mi = a + b;\n    const float gg = gi * gi;\n    a = b2 * v[i];\n    b = omb2 * gg;\n    const float vi = a + b;\n    const float mh = mi / bc1;\n    const float vh = vi / bc2;\n    const float den = sqrtf(vh) + eps_f;\n    const float ratio = mh / den;\n    const float upd = lr_f * ratio;\n    p = p - upd;\n    master[i] = p;\n    m[i] = mi;\n    v[i] = vi;\n    if (p_out) p_out[i] = zo_bf16_rne(p);\n  }\n}\n\n/*\n * The same Adam",
     lambda: A.test_adam_matches_torch_adamw(0.0)),
    ("eps inside the square root",
     "    const float den = sqrtf(vh) + eps_f;\n    const float ratio = mh / den;\n    const float upd = lr_f * ratio;\n    p = p - upd;\n    master[i] = p;\n    m[i] = mi;\n    v[i] = vi;\n    if (p_out) p_out[i] = zo_bf16_rne(p);\n  }\n}\n\n/*\n * The same Adam",
     "    const float den = sqrtf(vh + eps_f);\n    const float ratio = mh / den;\n    const float upd = lr_f * ratio;\n    p = p - upd;\n    master[i] = p;\n    m[i] = mi;\n    v[i] = vi;\n    if (p_out) p_out[i] = zo_bf16_rne(p);\n  }\n}\n\n/*\n * The same Adam",
     A.test_first_step_moves_each_weight_by_lr_against_the_gradient_sign),
    ("weight decay dropped",
     "    const float gi = zo_bf16_to_f32(g[i]);\n    float p = master[i];\n    p = p * decay;",
     "    const float gi = zo_bf16_to_f32(g[i]);\n    float p = master[i];",
     A.test_weight_decay_alone_scales_weights_by_one_minus_lr_wd),
    ("second moment from |g| instead of g^2",
     "    const float gg = gi * gi;\n    a = b2 * v[i];\n    b = omb2 * gg;\n    const float vi = a + b;\n    const float mh = mi / bc1;\n    const float vh = vi / bc2;\n    const float den = sqrtf(vh) + eps_f;\n    const float ratio = mh / den;\n    const float upd = lr_f * ratio;\n    p = p - upd;\n    master[i] = p;\n    m[i] = mi;\n    v[i] = vi;\n    if (p_out) p_out[i] = zo_bf16_rne(p);\n  }\n}\n\n/*\n * The same Adam",
     "    const float gg = fabsf(gi);\n    a = b2 * v[i];\n    b = omb2 * gg;\n    const float vi = a + b;\n    const float mh = mi / bc1;\n    const float vh = vi / bc2;\n    const float den = sqrtf(vh) + eps_f;\n    const float ratio = mh / den;\n    const float upd = lr_f * ratio;\n    p = p - upd;\n    master[i] = p;\n    m[i] = mi;\n    v[i] = vi;\n    if (p_out) p_out[i] = zo_bf16_rne(p);\n  }\n}\n\n/*\n * The same Adam",
     lambda: I.test_power_of_two_gradient_scale_leaves_the_update_bits_unchanged(3, 0.0)),
    ("square root of the second moment dropped",
     "    const float den = sqrtf(vh) + eps_f;\n    const float ratio = mh / den;\n    const float upd = lr_f * ratio;\n    p = p - upd;\n    master[i] = p;\n    m[i] = mi;\n    v[i] = vi;\n    if (p_out) p_out[i] = zo_bf16_rne(p);\n  }\n}\n\n/*\n * The same Adam",
     "    const float den = vh + eps_f;\n    const float ratio = mh / den;\n    const float upd = lr_f * ratio;\n    p = p - upd;\n    master[i] = p;\n    m[i] = mi;\n    v[i] = vi;\n    if (p_out) p_out[i] = zo_bf16_rne(p);\n  }\n}\n\n/*\n * The same Adam",
     lambda: I.test_power_of_two_gradient_scale_leaves_the_update_bits_unchanged(-1, 0.0)),
    ("first moment from |g|",
     "    float b = omb1 * gi;\n    const float mi = a + b;\n    const float gg = gi * gi;\n    a = b2 * v[i];\n    b = omb2 * gg;\n    const float vi = a + b;\n    const float mh = mi / bc1;\n    const float vh = vi / bc2;\n    const float den = sqrtf(vh) + eps_f;\n    const float ratio = mh / den;\n    const float upd = lr_f * ratio;\n    p = p - upd;\n    master[i] = p;\n    m[i] = mi;\n    v[i] = vi;\n    if (p_out) p_out[i] = zo_bf16_rne(p);\n  }\n}\n\n/*\n * The same Adam",
     "    float b = omb1 * fabsf(gi);\n    const float mi = a + b;\n    const float gg = gi * gi;\n    a = b2 * v[i];\n    b = omb2 * gg;\n    const float vi = a + b;\n    const float mh = mi / bc1;\n    const float vh = vi / bc2;\n    const float den = sqrtf(vh) + eps_f;\n    const float ratio = mh / den;\n    const float upd = lr_f * ratio;\n    p = p - upd;\n    master[i] = p;\n    m[i] = mi;\n    v[i] = vi;\n    if (p_out) p_out[i] = zo_bf16_rne(p);\n  }\n}\n\n/*\n * The same Adam",
     lambda: I.test_negated_gradients_negate_weights_and_first_moment_exactly(0.0)),
    ("bias-correction power off by one step",
     "  for (int64_t k = 0; k < t; ++k) {\n    p1 = p1 * beta1;",
     "  for (int64_t k = 0; k < t - 1; ++k) {\n    p1 = p1 * beta1;",
     A.test_bias_correction_scalars),
]


@pytest.mark.parametrize("name,old,new,pin", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pin_catches_planted_mistake(tmp_path, name, old, new, pin):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for '{name}' not found exactly once"
    mutant = tmp_path / "zero_oracle_mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = obuild.build(src=str(mutant), out=str(tmp_path / "libzero_oracle_mutant.so"))
    with oracle.use_library(lib):
        with pytest.raises(AssertionError):
            pin()
    # and the unmutated oracle passes the same pin
    pin()


# --- mistakes planted in the oracle's plan and collectives (Python side) ---

import numpy as np  # noqa: E402

import test_oracle_stages as S  # noqa: E402


def test_pins_catch_a_gather_that_skips_rank_zero(monkeypatch):
    real = oracle.all_gather

    def broken(param_shards, plan_, lo, hi, rank_out, out_base=0):
        saved = rank_out[0].copy()
        real(param_shards, plan_, lo, hi, rank_out, out_base)
        rank_out[0][...] = saved

    monkeypatch.setattr(oracle, "all_gather", broken)
    with pytest.raises(AssertionError):
        S.test_all_gather_inverts_partition_and_rs_equals_ar_slice()


def test_pins_catch_a_reduce_scatter_to_the_wrong_owner(monkeypatch):
    def broken(rank_grads, plan_, lo, hi, grad_shards):
        n = plan_.n_ranks
        for r in range(n):
            olo, ohi = plan_.owned(r)
            a, b = max(lo, olo), min(hi, ohi)
            if a < b:
                grad_shards[(r + 1) % n][a - olo:b - olo] = oracle.reduce_mean([g[a:b] for g in rank_grads])

    monkeypatch.setattr(oracle, "reduce_scatter", broken)
    with pytest.raises(AssertionError):
        S.test_all_gather_inverts_partition_and_rs_equals_ar_slice()


def test_pins_catch_a_bucket_schedule_that_drops_an_interval(monkeypatch):
    real = oracle.bucket_schedule
    monkeypatch.setattr(oracle, "bucket_schedule", lambda p: real(p)[:-1] if len(real(p)) > 1 else real(p))
    with pytest.raises(AssertionError):
        S.test_bucket_schedule_worked_example()
