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

import test_oracle_clip as C  # noqa: E402
import test_oracle_f16 as F  # noqa: E402

# Each arithmetic mistake is planted once: the oracle has one rank-order sum
# (rank_sum) and one update loop (zo_adam_ex, which zo_adam and zo_adam_coef
# call).  The update's mistakes are checked through each entry point's own
# pins -- the plain bf16 update (zo_adam), the clipped one (zo_adam_coef) and
# the binary16 one with a loss scale (zo_adam_ex) -- and every listed pin must
# fail; the last mistakes break the forwarding of the entry points.
def CLIP_PIN():
    C.test_active_clip_matches_torch_clip_grad_norm_and_adamw()
    C.test_three_clipped_steps_match_torch()


def F16_PIN():
    F.test_fp16_adam_matches_torch_adamw_on_unscaled_gradient()
    F.test_fp16_three_steps_match_torch_adamw()


MUTANTS = [
    ("bf16 truncates instead of rounding",
     "  if (d_tz < d_aw) return toward_zero;\n  if (d_aw < d_tz) return away;",
     "  return toward_zero;",
     [lambda: R.test_mean_exact_when_accumulation_exact(8)]),
    ("ties round up instead of to even",
     "  return (toward_zero & 1u) ? away : toward_zero;",
     "  return away;",
     [lambda: B.test_bf16_rne_worked_cases(1.0 + 2.0**-8, 0x3F80)]),
    ("rank order reversed",
     "  for (int32_t r = 0; r < n_ranks; ++r) acc = acc + fmt_to_f32(fmt, rank_grads[r][i]);",
     "  for (int32_t r = n_ranks - 1; r >= 0; --r) acc = acc + fmt_to_f32(fmt, rank_grads[r][i]);",
     [R.test_rank_order_matters_and_is_zero_to_n_minus_1]),
    ("mean not divided by N",
     "rank_sum(fmt, n_ranks, rank_grads, i) * inv_n)",
     "rank_sum(fmt, n_ranks, rank_grads, i))",
     [lambda: R.test_mean_exact_when_accumulation_exact(4), lambda: F.test_f16_mean_exact_when_accumulation_exact(4)]),
    ("bias correction of m dropped",
     "    const float mh = mi / bc1;",
     "    const float mh = mi;",
     [lambda: A.test_adam_matches_torch_adamw(0.0), CLIP_PIN, F16_PIN]),
    ("update sign flipped",
     "    p = p - upd;",
     "    p = p + upd;",
     [A.test_first_step_moves_each_weight_by_lr_against_the_gradient_sign, CLIP_PIN, F16_PIN]),
    ("beta2 used for the first moment",
     "    float a = b1 * m[i];",
     "    float a = b2 * m[i];",
     [lambda: A.test_adam_matches_torch_adamw(0.0), CLIP_PIN, F16_PIN]),
    ("eps inside the square root",
     "    const float den = sqrtf(vh) + eps_f;",
     "    const float den = sqrtf(vh + eps_f);",
     [A.test_first_step_moves_each_weight_by_lr_against_the_gradient_sign, CLIP_PIN, F16_PIN]),
    ("weight decay dropped",
     "    p = p * decay;\n",
     "",
     [A.test_weight_decay_alone_scales_weights_by_one_minus_lr_wd, CLIP_PIN, F16_PIN]),
    ("second moment from |g| instead of g^2",
     "    const float gg = gi * gi;",
     "    const float gg = fabsf(gi);",
     [lambda: I.test_power_of_two_gradient_scale_leaves_the_update_bits_unchanged(3, 0.0), CLIP_PIN, F16_PIN]),
    ("square root of the second moment dropped",
     "    const float den = sqrtf(vh) + eps_f;",
     "    const float den = vh + eps_f;",
     [lambda: I.test_power_of_two_gradient_scale_leaves_the_update_bits_unchanged(-1, 0.0), CLIP_PIN, F16_PIN]),
    ("first moment from |g|",
     "    float b = omb1 * gi;",
     "    float b = omb1 * fabsf(gi);",
     [lambda: I.test_negated_gradients_negate_weights_and_first_moment_exactly(0.0), CLIP_PIN, F16_PIN]),
    ("bias-correction power off by one step",
     "  for (int64_t k = 0; k < t; ++k) {\n    p1 = p1 * beta1;",
     "  for (int64_t k = 0; k < t - 1; ++k) {\n    p1 = p1 * beta1;",
     [A.test_bias_correction_scalars]),
    ("clipping coefficient not forwarded by zo_adam_coef",
     "zo_adam_ex(ZO_BF16, n, g, 1.0f, coef,",
     "zo_adam_ex(ZO_BF16, n, g, 1.0f, 1.0f,",
     [CLIP_PIN]),
    ("loss scale not applied",
     "    if (inv_scale != 1.0f) gi = gi * inv_scale;\n",
     "",
     [F16_PIN]),
    ("averaged gradient rounded to bf16 whatever the format",
     "out[i] = fmt_rne(fmt, rank_sum(fmt, n_ranks, rank_grads, i) * inv_n);",
     "out[i] = zo_bf16_rne(rank_sum(fmt, n_ranks, rank_grads, i) * inv_n);",
     [lambda: F.test_f16_mean_exact_when_accumulation_exact(2)]),
    ("parameters rounded to bf16 whatever the format",
     "    if (p_out) p_out[i] = fmt_rne(fmt, p);",
     "    if (p_out) p_out[i] = zo_bf16_rne(p);",
     [F16_PIN]),
]


@pytest.mark.parametrize("name,old,new,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pin_catches_planted_mistake(tmp_path, name, old, new, pins):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for '{name}' not found exactly once"
    mutant = tmp_path / "zero_oracle_mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = obuild.build(src=str(mutant), out=str(tmp_path / "libzero_oracle_mutant.so"))
    with oracle.use_library(lib):
        for pin in pins:
            with pytest.raises(AssertionError):
                pin()
    # and the unmutated oracle passes the same pins
    for pin in pins:
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
