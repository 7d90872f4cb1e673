"""Pins for the oracle's IEEE binary16 path (fp16 gradients and parameters
with a loss scale): conversions against numpy's float16 (IEEE round to
nearest even) exhaustively, hand-worked overflow / tie / subnormal cases,
exact means, bitwise invariance under power-of-two loss scales, overflow
detection, and agreement with torch's AdamW on the unscaled gradient."""
import math
import multiprocessing as mp

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads as W

CHUNK = 1 << 26


def _check_chunks(chunks):
    import os
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle as o

    bad = []
    for c in chunks:
        u = np.arange(c * CHUNK, (c + 1) * CHUNK, dtype=np.uint64).astype(np.uint32)
        f = u.view(np.float32)
        got = o.f16_rne(f)
        with np.errstate(over="ignore"):
            ref = f.astype(np.float16).view(np.uint16)
        nan_in = np.isnan(f)
        mism = (got != ref) & ~nan_in
        got_nan = ((got & 0x7C00) == 0x7C00) & ((got & 0x03FF) != 0)
        if np.any(mism):
            i = int(np.flatnonzero(mism)[0])
            bad.append((int(u[i]), int(got[i]), int(ref[i])))
        if np.any(nan_in & ~got_nan):
            bad.append(("nan", int(np.flatnonzero(nan_in & ~got_nan)[0])))
    return bad


def test_f16_rne_exhaustive_vs_numpy():
    n_chunks = (1 << 32) // CHUNK
    workers = max(1, min(16, mp.cpu_count()))
    parts = [list(range(k, n_chunks, workers)) for k in range(workers)]
    with mp.get_context("spawn").Pool(workers) as pool:
        bad = [b for r in pool.map(_check_chunks, parts) for b in r]
    assert not bad, bad[:5]


def test_f16_to_f32_all_patterns():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.f16_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    both_nan = np.isnan(got) & np.isnan(ref)
    assert np.array_equal(got.view(np.uint32)[~both_nan], ref.view(np.uint32)[~both_nan])
    assert np.array_equal(np.isnan(got), np.isnan(ref))


@pytest.mark.parametrize("x,expect", [
    (65504.0, 0x7BFF), (65519.99, 0x7BFF), (65520.0, 0x7C00), (-65520.0, 0xFC00),
    (1.0 + 2.0**-11, 0x3C00), (1.0 + 3 * 2.0**-11, 0x3C02), (2.0**-24, 0x0001), (2.0**-25, 0x0000),
    (3 * 2.0**-25, 0x0002), (2.0**-14 - 2.0**-25, 0x0400), (-0.0, 0x8000), (float("inf"), 0x7C00),
])
def test_f16_rne_worked_cases(x, expect):
    assert int(oracle.f16_rne(np.array([x], np.float32))[0]) == expect


@pytest.mark.parametrize("n_ranks", [1, 2, 4, 8, 16])
def test_f16_mean_exact_when_accumulation_exact(n_ranks):
    rng = np.random.default_rng(700 + n_ranks)
    mant = rng.integers(1024, 2048, size=(n_ranks, 4096))
    exp = rng.integers(-6, 2, size=(n_ranks, 4096)) - 10
    vals = (rng.choice([-1.0, 1.0], size=mant.shape) * mant * np.exp2(exp)).astype(np.float16)
    exact = np.array([math.fsum(vals[:, i].astype(np.float64)) / n_ranks for i in range(vals.shape[1])])
    expect = exact.astype(np.float32).astype(np.float16).view(np.uint16)
    got = oracle.reduce_mean_fmt([vals[r].view(np.uint16) for r in range(n_ranks)], oracle.F16)
    assert np.array_equal(got, expect)


def _setup(numel, layer, n_ranks, bucket, seed, sigma, positive=False):
    p = oracle.plan(numel, layer, n_ranks, bucket)
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, synth.base(seed, synth.STREAM_MASTER, 0, 0),
                       W.MASTER_DIST, as_f32=True)
    rng = np.random.default_rng(seed)
    grads = {}

    def g(k, r, scale=1.0):
        key = (k, r)
        if key not in grads:
            if positive:  # magnitudes in [2^-10, 2^-5]: every average is a normal binary16
                x = np.exp2(rng.uniform(-10.0, -5.0, size=p.psi_pad)).astype(np.float32)
            else:
                x = rng.normal(0.0, sigma, size=p.psi_pad).astype(np.float32)
            x[~p.real_mask()] = 0
            grads[key] = oracle.f16_rne(x)
        base = oracle.f16_to_f32(grads[key]).astype(np.float64) * scale
        return oracle.f16_rne(base.astype(np.float32))

    return p, m0, g


def test_power_of_two_loss_scale_changes_no_bit():
    """Gradients S times larger with loss scale S (S = 2^10; positive
    gradients so that no average is a binary16 subnormal, where the unscaled
    run would lose precision -- the reason loss scaling exists): every state
    equals the unscaled run bit for bit."""
    p, m0, g = _setup([6000, 1000], [0, 1], 4, 2048, 71, 1e-2, positive=True)
    hp = oracle.AdamHP(weight_decay=0.01)
    a, ra = oracle.run(p, oracle.STAGE_Z2, m0, lambda k, r: g(k, r), 3, hp, fmt=oracle.F16)
    b, rb = oracle.run(p, oracle.STAGE_Z2, m0, lambda k, r: g(k, r, 1024.0), 3, hp, fmt=oracle.F16,
                       loss_scale=1024.0)
    va, vb = oracle.full_view(p, 2, a), oracle.full_view(p, 2, b)
    for k in ("master", "m", "v", "params"):
        assert np.array_equal(va[k], vb[k]), k
    for x, y in zip(ra, rb):
        assert math.isclose(x.grad_norm, y.grad_norm, rel_tol=1e-15)


def test_fp16_overflow_is_detected_and_skipped():
    p, m0, g = _setup([4000], [0], 2, 4000, 72, 1e-2)
    hp = oracle.AdamHP()
    huge = lambda k, r: g(k, r, 1e7 if k == 2 else 1.0)  # 1e7 * 1e-2 overflows binary16 on some elements
    ranks, reps = oracle.run(p, oracle.STAGE_Z2, m0, huge, 3, hp, skip_nonfinite=True, fmt=oracle.F16)
    assert [r.skipped for r in reps] == [False, True, False] and reps[1].nonfinite > 0


def test_fp16_adam_matches_torch_adamw_on_unscaled_gradient():
    p, m0, g = _setup([20000], [0], 4, 20000, 73, 1e-2)
    hp = oracle.AdamHP(lr=1e-3, weight_decay=0.01)
    S = 256.0
    ranks, reps = oracle.run(p, oracle.STAGE_Z2, m0, lambda k, r: g(k, r, S), 1, hp, fmt=oracle.F16,
                             loss_scale=S)
    view = oracle.full_view(p, oracle.STAGE_Z2, ranks)
    gavg = oracle.f16_to_f32(view["grad"]) / np.float32(S)
    w = torch.nn.Parameter(torch.from_numpy(m0.copy()))
    w.grad = torch.from_numpy(gavg.astype(np.float32))
    opt = torch.optim.AdamW([w], lr=hp.lr, betas=(hp.beta1, hp.beta2), eps=hp.eps, weight_decay=0.01,
                            foreach=False, fused=False)
    opt.step()
    np.testing.assert_allclose(view["m"], opt.state[w]["exp_avg"].numpy(), rtol=2e-6, atol=1e-9)
    np.testing.assert_allclose(view["v"], opt.state[w]["exp_avg_sq"].numpy(), rtol=2e-6, atol=1e-13)
    # the update itself: the weights' change against torch's (torch orders
    # the same operations differently, hence a relative bound, not bits)
    d_or = view["master"].astype(np.float64) - m0
    d_tc = w.detach().numpy().astype(np.float64) - m0
    assert np.all(np.abs(d_or - d_tc) <= 1e-4 * np.abs(d_tc) + np.spacing(np.abs(view["master"])) + 1e-10)
    assert np.array_equal(view["params"], oracle.f16_rne(view["master"]))
    assert math.isclose(reps[0].grad_norm, float(np.sqrt(np.sum(gavg.astype(np.float64) ** 2))), rel_tol=1e-12)


@pytest.mark.parametrize("scale", [1.0, 512.0])
def test_fp16_stages_agree(scale):
    numel, layer = W.transformer_layers(2, 16, 64)
    p, m0, g = _setup(numel, layer, 3, 1024, 74, 1e-2)
    hp = oracle.AdamHP(weight_decay=0.01)
    views = []
    for stage in (oracle.STAGE_DP, oracle.STAGE_Z1, oracle.STAGE_Z2, oracle.STAGE_Z3):
        ranks, _ = oracle.run(p, stage, m0, lambda k, r: g(k, r, scale), 3, hp, fmt=oracle.F16, loss_scale=scale,
                              clip_norm=0.05)
        views.append(oracle.full_view(p, stage, ranks))
    for v in views[1:]:
        for k in ("master", "m", "v", "params", "grad"):
            assert np.array_equal(v[k], views[0][k]), k


def test_fp16_three_steps_match_torch_adamw():
    """Three binary16 steps with loss scale 256 against torch's AdamW on the
    unscaled averaged gradients: the second and third steps start from
    non-zero moments, so a mistake in how the old moments enter shows."""
    p, m0, g = _setup([20000], [0], 4, 20000, 74, 1e-2)
    hp = oracle.AdamHP(lr=1e-3, weight_decay=0.01)
    S = 256.0
    w = torch.nn.Parameter(torch.from_numpy(m0.copy()))
    opt = torch.optim.AdamW([w], lr=hp.lr, betas=(hp.beta1, hp.beta2), eps=hp.eps, weight_decay=0.01,
                            foreach=False, fused=False)
    for steps in (1, 2, 3):
        ranks, _ = oracle.run(p, oracle.STAGE_Z2, m0, lambda k, r: g(k, r, S), steps, hp, fmt=oracle.F16,
                              loss_scale=S)
        view = oracle.full_view(p, oracle.STAGE_Z2, ranks)
        w.grad = torch.from_numpy((oracle.f16_to_f32(view["grad"]) / np.float32(S)).astype(np.float32))
        opt.step()
        np.testing.assert_allclose(view["m"], opt.state[w]["exp_avg"].numpy(), rtol=1e-4, atol=1e-10)
        np.testing.assert_allclose(view["v"], opt.state[w]["exp_avg_sq"].numpy(), rtol=1e-4, atol=1e-14)
        np.testing.assert_allclose(view["master"], w.detach().numpy(), rtol=1e-6, atol=1e-6)
        w.data.copy_(torch.from_numpy(view["master"].copy()))
