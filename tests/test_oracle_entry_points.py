"""The oracle's update and reduction entry points agree bit for bit where
their inputs coincide.  There is one update loop (zo_adam_ex) and one
rank-order sum; zo_adam, zo_adam_coef and zo_reduce_mean reach them with
fixed arguments, and these pins check that forwarding: the plain bf16 update
equals the clipped one at an inactive coefficient and the general one at
inv_scale = coef = 1, the clipped one equals the general one at the same
coefficient, and the bf16 mean equals the format-generic mean at bf16 ([T]
sections "ZeRO-1" to "ZeRO-3", part "3. 更新", and section "ZeRO-2" for the
mean)."""
import ctypes

import numpy as np
import pytest

import oracle


def _inputs(seed, n=20000):
    rng = np.random.default_rng(seed)
    g32 = (rng.standard_normal(n) * 1e-2).astype(np.float32)
    g = oracle.bf16_rne(g32)
    master = (rng.standard_normal(n) * 0.02).astype(np.float32)
    m = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    v = (np.abs(rng.standard_normal(n)) * 1e-5).astype(np.float32)
    return g, master, m, v


def _bits(*arrays):
    return [np.ascontiguousarray(a).view(np.uint8).tobytes() for a in arrays]


@pytest.mark.parametrize("t", [1, 2, 7])
@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_plain_clipped_and_general_updates_agree(t, wd):
    hp = oracle.AdamHP(lr=1e-3, weight_decay=wd)
    g, master, m, v = _inputs(100 + t)
    runs = []
    for kind in ("plain", "coef1", "coef_big", "ex"):
        a, b, c = master.copy(), m.copy(), v.copy()
        if kind == "plain":
            p = oracle.adam(g, a, b, c, hp, t)
        elif kind == "coef1":
            p = oracle.adam_coef(g, 1.0, a, b, c, hp, t)
        elif kind == "coef_big":
            p = oracle.adam_coef(g, 3.5, a, b, c, hp, t)
        else:
            p = oracle.adam_ex(g, oracle.BF16, 1.0, 1.0, a, b, c, hp, t)
        runs.append(_bits(a, b, c, p))
    assert all(r == runs[0] for r in runs[1:])


@pytest.mark.parametrize("coef", [0.5, 0.123, 0.999])
def test_clipped_update_equals_general_update_at_the_same_coefficient(coef):
    hp = oracle.AdamHP(lr=1e-3, weight_decay=0.01)
    g, master, m, v = _inputs(200)
    a1, b1, c1 = master.copy(), m.copy(), v.copy()
    p1 = oracle.adam_coef(g, coef, a1, b1, c1, hp, 3)
    a2, b2, c2 = master.copy(), m.copy(), v.copy()
    p2 = oracle.adam_ex(g, oracle.BF16, 1.0, coef, a2, b2, c2, hp, 3)
    assert _bits(a1, b1, c1, p1) == _bits(a2, b2, c2, p2)
    # and an active coefficient does change the update
    a3, b3, c3 = master.copy(), m.copy(), v.copy()
    oracle.adam(g, a3, b3, c3, hp, 3)
    assert _bits(b1) != _bits(b3)


@pytest.mark.parametrize("n_ranks", [1, 2, 5, 8])
def test_bf16_mean_equals_format_generic_mean_at_bf16(n_ranks):
    rng = np.random.default_rng(300 + n_ranks)
    reps = [oracle.bf16_rne((rng.standard_normal(30000) * 1e-2).astype(np.float32)) for _ in range(n_ranks)]
    a = oracle.reduce_mean(reps)
    lib = oracle._load()
    b = np.empty_like(a)
    arr = (ctypes.c_void_p * n_ranks)(*[r.ctypes.data for r in reps])
    lib.zo_reduce_mean_fmt(oracle.BF16, n_ranks, a.size, arr, b.ctypes.data)
    assert np.array_equal(a, b)
