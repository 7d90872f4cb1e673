"""Pins for the oracle's Adam update: an independent implementation
(torch.optim.AdamW on CPU, fp32, single-tensor path) with an algebraically
equal but differently ordered formula, and the special cases the textbook
definition fixes exactly."""
import numpy as np
import pytest
import torch

import oracle


def _bf16(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def _f32(h: np.ndarray) -> np.ndarray:
    return torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).float().numpy()


@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_adam_matches_torch_adamw(wd):
    """Five steps of bias-corrected Adam with decoupled weight decay, against
    torch.optim.AdamW.  The op order differs (torch scales by lr/bc1 and
    divides sqrt(v) by sqrt(bc2)), so this pins the formula -- every term,
    sign and index -- not the rounding."""
    rng = np.random.default_rng(11 + int(wd * 100))
    n = 100000
    hp = oracle.AdamHP(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=wd)
    master = rng.normal(0.0, 0.02, size=n).astype(np.float32)
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    p_t = torch.nn.Parameter(torch.from_numpy(master.copy()))
    opt = torch.optim.AdamW([p_t], lr=hp.lr, betas=(hp.beta1, hp.beta2), eps=hp.eps,
                            weight_decay=wd, foreach=False, fused=False)
    for t in range(1, 6):
        g16 = _bf16(rng.normal(0.0, 1e-2, size=n).astype(np.float32))
        before = master.copy()
        # both sides start the step from the same weights and moments
        with torch.no_grad():
            p_t.copy_(torch.from_numpy(master))
        if t > 1:
            opt.state[p_t]["exp_avg"].copy_(torch.from_numpy(m))
            opt.state[p_t]["exp_avg_sq"].copy_(torch.from_numpy(v))
        params = oracle.adam(g16, master, m, v, hp, t)
        p_t.grad = torch.from_numpy(_f32(g16))
        opt.step()
        st = opt.state[p_t]
        # torch forms m by lerp (m + w (g - m)): near-cancelling m differ by a
        # few ulp of |g| (~1e-2), so the absolute floor is 1e-9
        np.testing.assert_allclose(m, st["exp_avg"].numpy(), rtol=2e-6, atol=1e-9)
        np.testing.assert_allclose(v, st["exp_avg_sq"].numpy(), rtol=2e-6, atol=1e-13)
        # the update itself (tiny next to the weight) to a relative 1e-4, plus
        # one fp32 ulp of the weight for the final rounding of p - update
        d_or = master.astype(np.float64) - before
        d_tc = p_t.detach().numpy().astype(np.float64) - before
        ulp_w = np.spacing(np.abs(master)).astype(np.float64)
        # the 1e-9 floor on m above propagates into the update as lr*dm/sqrt(vhat)
        vhat = v.astype(np.float64) / (1.0 - hp.beta2**t)
        from_m = hp.lr * 1e-9 / (np.sqrt(vhat) + hp.eps)
        assert np.all(np.abs(d_or - d_tc) <= 1e-4 * np.abs(d_tc) + ulp_w + from_m)
        assert np.array_equal(params, _bf16(master))


def test_zero_gradient_from_zero_moments_leaves_weights_unchanged():
    rng = np.random.default_rng(12)
    master = rng.normal(0.0, 0.02, size=1000).astype(np.float32)
    ref = master.copy()
    m = np.zeros_like(master)
    v = np.zeros_like(master)
    g = np.zeros(1000, np.uint16)
    for t in range(1, 4):
        oracle.adam(g, master, m, v, oracle.AdamHP(), t)
    assert np.array_equal(master, ref) and not m.any() and not v.any()


def test_first_step_moves_each_weight_by_lr_against_the_gradient_sign():
    """t = 1 from m = v = 0: mh = g and vh = g^2 up to rounding, so the step is
    -lr * g / (|g| + eps) ~ -lr * sign(g) when |g| >> eps."""
    rng = np.random.default_rng(13)
    n = 50000
    hp = oracle.AdamHP(lr=1e-3)
    master = rng.normal(0.0, 0.02, size=n).astype(np.float32)
    before = master.astype(np.float64)
    g16 = _bf16(rng.normal(0.0, 1e-2, size=n).astype(np.float32))
    g16[g16 == 0] = 0x3C00  # no zero gradients here
    g16[g16 == 0x8000] = 0x3C00
    oracle.adam(g16, master, np.zeros(n, np.float32), np.zeros(n, np.float32), hp, 1)
    step = master.astype(np.float64) - before
    gv = _f32(g16).astype(np.float64)
    expect = -hp.lr * np.sign(gv)
    # exact step: -lr * g/(|g| + eps) = -lr sign(g) (1 - eps/(|g| + eps)); plus
    # fp32 rounding of the bias-corrected moments (a few ulp, relative) and
    # of the new weight (one ulp of |w|)
    bound = hp.lr * hp.eps / np.abs(gv) + 1e-6 * hp.lr + 2 * np.spacing(np.abs(master))
    assert np.all(np.abs(step - expect) <= bound)


def test_weight_decay_alone_scales_weights_by_one_minus_lr_wd():
    hp = oracle.AdamHP(lr=0.5, weight_decay=0.5)  # decay factor 0.75, exact
    master = np.array([1.0, -2.0, 0.25, 3.0], np.float32)
    oracle.adam(np.zeros(4, np.uint16), master, np.zeros(4, np.float32), np.zeros(4, np.float32),
                hp, 1)
    assert np.array_equal(master, np.array([0.75, -1.5, 0.1875, 2.25], np.float32))


def test_bias_correction_scalars():
    """bc = 1 - beta^t: t = 1 gives 1 - beta, t = 3 gives 1 - beta^3, large t
    tends to 1; each derived scalar is rounded once from binary64."""
    hp = oracle.AdamHP(lr=0.5, beta1=0.5, beta2=0.75, eps=0.25, weight_decay=0.5)
    s1 = oracle.adam_scalars(hp, 1)
    assert list(s1) == [0.5, 0.75, 0.5, 0.25, 0.5, 0.25, 0.75, 0.5, 0.25]
    s3 = oracle.adam_scalars(hp, 3)
    assert s3[4] == np.float32(0.875) and s3[5] == np.float32(1 - 27 / 64)
    s_big = oracle.adam_scalars(oracle.AdamHP(), 100000)
    assert s_big[4] == np.float32(1.0) and s_big[5] == np.float32(1.0)
    # the decimal hyper-parameters are used, not their fp32 roundings
    s_dec = oracle.adam_scalars(oracle.AdamHP(beta2=0.999), 1)
    assert s_dec[3] == np.float32(0.001) and s_dec[3] != np.float32(1.0 - float(np.float32(0.999)))
