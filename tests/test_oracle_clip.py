"""Pins for the oracle's optional global-norm clip and overflow skip (not on
the pages; the usual mixed-precision conventions): an inactive clip changes
nothing, an active clip matches torch.nn.utils.clip_grad_norm_ followed by
AdamW, the clipped gradient's norm is the limit, a skipped step changes no
state and does not advance t, and every ZeRO stage still equals plain DP."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads as W

STAGES = (oracle.STAGE_DP, oracle.STAGE_Z1, oracle.STAGE_Z2, oracle.STAGE_Z3)


def _setup(numel, layer, n_ranks, bucket, seed, dist):
    p = oracle.plan(numel, layer, n_ranks, bucket)
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, synth.base(seed, synth.STREAM_MASTER, 0, 0),
                       W.MASTER_DIST, as_f32=True)

    def g(t, r):
        return W.host_padded(p.offset, p.numel, p.psi_pad, synth.base(seed, synth.STREAM_GRAD, t, r), dist)

    return p, m0, g


def test_inactive_clip_is_bitwise_no_clip():
    p, m0, g = _setup([3000, 1000], [0, 1], 4, 1024, 31, synth.Dist(synth.NORMAL, 1e-2))
    hp = oracle.AdamHP(weight_decay=0.01)
    a, ra = oracle.run(p, oracle.STAGE_Z2, m0, g, 3, hp)
    b, rb = oracle.run(p, oracle.STAGE_Z2, m0, g, 3, hp, clip_norm=1e9)
    assert all(r.coef == 1.0 for r in rb)
    va, vb = oracle.full_view(p, 2, a), oracle.full_view(p, 2, b)
    for k in va:
        assert np.array_equal(va[k], vb[k])


def test_clip_coefficient_definition():
    assert oracle.clip_coef(10.0, 20.0) == 1.0
    assert oracle.clip_coef(1000.0, 1000.0) == 1.0      # 1 - 1e-9 rounds to 1.0f: no clip
    assert oracle.clip_coef(10.0, 10.0) == float(np.float32(1 - 2.0**-23))  # 1 - 1e-7 rounds below 1
    assert oracle.clip_coef(4.0, 1.0) == float(np.float32(1.0 / (4.0 + 1e-6)))
    assert oracle.clip_coef(0.0, 1.0) == 1.0


def test_active_clip_matches_torch_clip_grad_norm_and_adamw():
    """One step, every element, against torch: clip_grad_norm_ on the averaged
    gradient (as fp32 values), then AdamW.  torch computes the norm in fp32,
    so the coefficients differ by a few fp32 ulp: tolerances reflect that."""
    p, m0, g = _setup([20000], [0], 4, 20000, 32, synth.Dist(synth.NORMAL, 1e-2))
    hp = oracle.AdamHP(lr=1e-3, weight_decay=0.01)
    ranks, reps = oracle.run(p, oracle.STAGE_Z2, m0, g, 1, hp, clip_norm=0.05)
    assert reps[0].coef < 0.5
    view = oracle.full_view(p, oracle.STAGE_Z2, ranks)
    gavg = oracle.bf16_to_f32(view["grad"])
    w = torch.nn.Parameter(torch.from_numpy(m0.copy()))
    w.grad = torch.from_numpy(gavg.copy())
    total = torch.nn.utils.clip_grad_norm_([w], 0.05, foreach=False)
    assert math.isclose(float(total), reps[0].grad_norm, rel_tol=1e-4)  # torch sums in fp32
    opt = torch.optim.AdamW([w], lr=hp.lr, betas=(hp.beta1, hp.beta2), eps=hp.eps, weight_decay=0.01,
                            foreach=False, fused=False)
    opt.step()
    np.testing.assert_allclose(view["m"], opt.state[w]["exp_avg"].numpy(), rtol=1e-5, atol=1e-11)
    np.testing.assert_allclose(view["v"], opt.state[w]["exp_avg_sq"].numpy(), rtol=1e-5, atol=1e-15)
    d_or = view["master"].astype(np.float64) - m0
    d_tc = w.detach().numpy().astype(np.float64) - m0
    assert np.all(np.abs(d_or - d_tc) <= 1e-4 * np.abs(d_tc) + np.spacing(np.abs(view["master"])) + 1e-10)


def test_clipped_gradient_has_the_limit_norm():
    p, m0, g = _setup([50000], [0], 2, 50000, 33, synth.Dist(synth.NORMAL, 1e-2))
    _, reps = oracle.run(p, oracle.STAGE_Z2, m0, g, 1, oracle.AdamHP(), clip_norm=0.1)
    norm, coef = reps[0].grad_norm, reps[0].coef
    assert norm > 0.1
    # ||coef * g|| = coef * norm = max_norm * norm / (norm + 1e-6), up to fp32 rounding of coef
    assert math.isclose(coef * norm, 0.1 * norm / (norm + 1e-6), rel_tol=2 ** -23)


def test_overflow_skip_changes_nothing_and_keeps_t():
    numel, layer = [4000, 96], [0, 1]
    p, m0, g = _setup(numel, layer, 4, 512, 34, synth.Dist(synth.NORMAL, 1e-2))
    bad = lambda k, r: (lambda a: (a.__setitem__(7, 0x7F80), a)[1])(g(k, r)) if (k == 2 and r == 1) else g(k, r)
    hp = oracle.AdamHP()
    for stage in STAGES:
        ranks, reps = oracle.run(p, stage, m0, bad, 3, hp, skip_nonfinite=True)
        assert [r.skipped for r in reps] == [False, True, False]
        assert reps[1].nonfinite == 1
        # reference: the same steps without the bad one, the third call at t = 2
        ref_ranks = oracle.init_states(p, stage, m0)
        oracle.step(p, stage, ref_ranks, lambda _t, r: g(1, r), 1, hp)
        oracle.step(p, stage, ref_ranks, lambda _t, r: g(3, r), 2, hp)
        a, b = oracle.full_view(p, stage, ranks), oracle.full_view(p, stage, ref_ranks)
        for k in ("master", "m", "v", "params"):
            assert np.array_equal(a[k], b[k]), (stage, k)


@pytest.mark.parametrize("clip", [0.05, 1e9])
def test_stages_agree_under_clip_and_skip(clip):
    numel, layer = W.transformer_layers(2, 16, 64)
    p, m0, g = _setup(numel, layer, 3, 1024, 35, synth.Dist(synth.NORMAL, 1e-2, zero_mod=9))
    hp = oracle.AdamHP(weight_decay=0.01)
    views = []
    for stage in STAGES:
        ranks, reps = oracle.run(p, stage, m0, g, 3, hp, clip_norm=clip, skip_nonfinite=True)
        views.append(oracle.full_view(p, stage, ranks))
    for v in views[1:]:
        for k in ("master", "m", "v", "params", "grad"):
            assert np.array_equal(v[k], views[0][k]), k


def test_three_clipped_steps_match_torch():
    """Three clipped steps against torch (clip_grad_norm_ on each step's
    averaged gradient, then AdamW): from the second step on the moments are
    non-zero, so a mistake in how the old moments enter the update shows
    (step one starts from m = v = 0 and cannot see it)."""
    p, m0, g = _setup([20000], [0], 4, 20000, 34, synth.Dist(synth.NORMAL, 1e-2))
    hp = oracle.AdamHP(lr=1e-3, weight_decay=0.01)
    w = torch.nn.Parameter(torch.from_numpy(m0.copy()))
    opt = torch.optim.AdamW([w], lr=hp.lr, betas=(hp.beta1, hp.beta2), eps=hp.eps, weight_decay=0.01,
                            foreach=False, fused=False)
    for steps in (1, 2, 3):
        ranks, reps = oracle.run(p, oracle.STAGE_Z2, m0, g, steps, hp, clip_norm=0.05)
        assert reps[-1].coef < 0.5
        view = oracle.full_view(p, oracle.STAGE_Z2, ranks)
        w.grad = torch.from_numpy(oracle.bf16_to_f32(view["grad"]).copy())
        torch.nn.utils.clip_grad_norm_([w], 0.05, foreach=False)
        opt.step()
        np.testing.assert_allclose(view["m"], opt.state[w]["exp_avg"].numpy(), rtol=1e-4, atol=1e-10)
        np.testing.assert_allclose(view["v"], opt.state[w]["exp_avg_sq"].numpy(), rtol=1e-4, atol=1e-14)
        np.testing.assert_allclose(view["master"], w.detach().numpy(), rtol=1e-6, atol=1e-6)
        w.data.copy_(torch.from_numpy(view["master"].copy()))  # keep the two on the oracle's weights
