"""Exact invariants of bias-corrected Adam that pin the oracle's update
without restating it.

Binary floating point rounds a product, quotient or square root the same way
at every power-of-two scale (away from overflow and subnormals), so:

* with eps = 0, multiplying every gradient by 2^k multiplies the first moment
  by 2^k and the second by 4^k exactly; the bias-corrected ratio
  m_hat / sqrt(v_hat) -- and so every weight and bf16 parameter -- keeps its
  bits.  A second moment not built from g^2, a missing square root or the
  two moments swapped all break this;
* rounding is symmetric about zero, so from zero weights without weight
  decay, negating every gradient negates the first moment and every weight
  bit for bit and leaves the second moment as it is.  A first moment built
  from |g|, or a term whose sign does not follow the gradient's, breaks it.

Both hold for the textbook definition of Adam with decoupled weight decay
(the update each owner applies to its shard in the ZeRO stages of "ZERO训练技术",
sections "ZeRO-1" to "ZeRO-3", part "3. 更新")."""
import numpy as np
import pytest
import torch

import oracle


def _bf16(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def _f32(h: np.ndarray) -> np.ndarray:
    return torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).float().numpy()


def _grads(rng, n, steps):
    """bf16 gradients ~N(0, 1e-2) with no zeros (eps = 0 would divide 0 by 0)."""
    out = []
    for _ in range(steps):
        g = _bf16(rng.normal(0.0, 1e-2, size=n).astype(np.float32))
        g[(g == 0) | (g == 0x8000)] = 0x3C23  # 0.00995...
        out.append(g)
    return out


def _scaled(g16: np.ndarray, k: int) -> np.ndarray:
    s = _bf16(_f32(g16) * np.float32(2.0**k))
    assert np.array_equal(_f32(s), _f32(g16) * np.float32(2.0**k))  # exact in bf16
    return s


def _run(grads, master0, hp):
    master = master0.copy()
    m = np.zeros_like(master)
    v = np.zeros_like(master)
    params = None
    for t, g in enumerate(grads, start=1):
        params = oracle.adam(g, master, m, v, hp, t)
    return master, m, v, params


@pytest.mark.parametrize("k", [-6, -1, 3])
@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_power_of_two_gradient_scale_leaves_the_update_bits_unchanged(k, wd):
    rng = np.random.default_rng(40 + k)
    n, steps = 20000, 4
    hp = oracle.AdamHP(lr=1e-3, beta1=0.9, beta2=0.999, eps=0.0, weight_decay=wd)
    master0 = rng.normal(0.0, 0.02, size=n).astype(np.float32)
    grads = _grads(rng, n, steps)
    base = _run(grads, master0, hp)
    scaled = _run([_scaled(g, k) for g in grads], master0, hp)
    assert np.array_equal(scaled[0], base[0])                                # weights
    assert np.array_equal(scaled[3], base[3])                                # bf16 parameters
    assert np.array_equal(scaled[1], base[1] * np.float32(2.0**k))           # m scales by 2^k
    assert np.array_equal(scaled[2], base[2] * np.float32(4.0**k))           # v scales by 4^k
    # the invariant is not vacuous: the weights moved
    assert np.count_nonzero(base[0] != master0) > n // 2


def test_with_eps_the_scale_invariance_breaks_where_eps_matters():
    """eps > 0 is the one term that does not scale: with gradients shrunk
    until sqrt(v_hat) is comparable to eps, the update changes -- the check
    above is sensitive to the term it sets to zero."""
    rng = np.random.default_rng(47)
    n = 5000
    hp = oracle.AdamHP(lr=1e-3, eps=1e-8)
    master0 = rng.normal(0.0, 0.02, size=n).astype(np.float32)
    grads = _grads(rng, n, 2)
    base = _run(grads, master0, hp)
    tiny = _run([_scaled(g, -20) for g in grads], master0, hp)  # |g| ~ 1e-8
    assert not np.array_equal(tiny[0], base[0])


@pytest.mark.parametrize("eps", [0.0, 1e-8])
def test_negated_gradients_negate_weights_and_first_moment_exactly(eps):
    rng = np.random.default_rng(48)
    n, steps = 20000, 5
    hp = oracle.AdamHP(lr=1e-3, eps=eps, weight_decay=0.0)
    grads = _grads(rng, n, steps)
    zero = np.zeros(n, np.float32)
    base = _run(grads, zero, hp)
    neg = _run([g ^ np.uint16(0x8000) for g in grads], zero, hp)  # flip the bf16 sign bit
    assert np.array_equal(neg[0], -base[0])
    assert np.array_equal(neg[1], -base[1])
    assert np.array_equal(neg[2], base[2])
    assert np.array_equal(neg[3], base[3] ^ np.uint16(0x8000))
    assert np.all(base[2] > 0) and np.count_nonzero(base[0]) == n
