"""Pins for the oracle's rank-order reduction (the "reduce" of reduce-scatter
and all-reduce): exact sums where binary32 accumulation is exact, the
recursive-summation error bound otherwise, and the special cases the
definition fixes."""
import math

import numpy as np
import pytest
import torch

import oracle

U32 = 2.0**-24  # unit roundoff of binary32


def _torch_bf16_bits(x32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x32, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def _bf16_from_f32(x: np.ndarray) -> np.ndarray:
    """bf16 patterns of values already representable in bf16 (upper halves)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0)
    return (u >> 16).astype(np.uint16)


def _narrow_range_bf16(rng, n_ranks, n, e0):
    """bf16 values in +-[2^e0, 2^(e0+8)): every rank-order fp32 partial sum of
    up to 64 of them is exact (at most 8 + 8 + 6 significant bits)."""
    mant = rng.integers(128, 256, size=(n_ranks, n))            # 8-bit significand
    exp = rng.integers(e0, e0 + 8, size=(n_ranks, n)) - 7
    sign = rng.choice([-1.0, 1.0], size=(n_ranks, n))
    return (sign * mant * np.exp2(exp)).astype(np.float32)


@pytest.mark.parametrize("n_ranks", [1, 2, 4, 8, 16, 64])
def test_mean_exact_when_accumulation_exact(n_ranks):
    """Power-of-two N: sum and 1/N scaling are exact, so the averaged bf16 is
    the exact mean (math.fsum) rounded once to bf16 -- taken here from torch."""
    rng = np.random.default_rng(1000 + n_ranks)
    vals = _narrow_range_bf16(rng, n_ranks, 4096, e0=-10)
    exact = np.array([math.fsum(vals[:, i].astype(np.float64)) / n_ranks
                      for i in range(vals.shape[1])])
    assert np.all(exact.astype(np.float32).astype(np.float64) == exact)
    expect = _torch_bf16_bits(exact.astype(np.float32))
    got = oracle.reduce_mean([_bf16_from_f32(vals[r]) for r in range(n_ranks)])
    assert np.array_equal(got, expect)


@pytest.mark.parametrize("n_ranks", [1, 2, 3, 5, 7, 8, 9, 16, 64])
def test_rank_sum_within_recursive_summation_bound(n_ranks):
    """|fl(sum) - sum| <= (N-1) u sum|g| for rank-order binary32 accumulation
    (Higham, Accuracy and Stability of Numerical Algorithms, eq. 4.4)."""
    rng = np.random.default_rng(2000 + n_ranks)
    g = rng.normal(0.0, 1e-2, size=(n_ranks, 20000)).astype(np.float32)
    g16 = [_torch_bf16_bits(g[r]) for r in range(n_ranks)]
    gv = np.stack([oracle.bf16_to_f32(a) for a in g16]).astype(np.float64)
    got = oracle.rank_sum_f32(g16).astype(np.float64)
    exact = np.array([math.fsum(gv[:, i]) for i in range(gv.shape[1])])
    bound = (n_ranks - 1) * U32 * np.abs(gv).sum(axis=0) * (1 + 1e-6)
    assert np.all(np.abs(got - exact) <= bound)


@pytest.mark.parametrize("n_ranks", list(range(1, 10)) + [16, 64])
def test_mean_within_bf16_half_ulp_of_exact(n_ranks):
    """The averaged bf16 lies within half a bf16 ulp of the exact mean plus the
    accumulation and 1/N rounding errors (a bound, any N)."""
    rng = np.random.default_rng(3000 + n_ranks)
    g = rng.normal(0.0, 1e-2, size=(n_ranks, 20000)).astype(np.float32)
    g16 = [_torch_bf16_bits(g[r]) for r in range(n_ranks)]
    gv = np.stack([oracle.bf16_to_f32(a) for a in g16]).astype(np.float64)
    exact = np.array([math.fsum(gv[:, i]) for i in range(gv.shape[1])]) / n_ranks
    got = oracle.bf16_to_f32(oracle.reduce_mean(g16)).astype(np.float64)
    absmean = np.abs(gv).sum(axis=0) / n_ranks
    acc_err = (n_ranks - 1) * U32 * absmean + 2 * U32 * absmean
    half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(got), 1e-38))) - 8)
    assert np.all(np.abs(got - exact) <= half_ulp + 2 * acc_err + 1e-45)


@pytest.mark.parametrize("n_ranks", list(range(1, 10)) + [16, 64])
def test_identical_replicas_mean_is_replica(n_ranks):
    rng = np.random.default_rng(4000 + n_ranks)
    g = _torch_bf16_bits(rng.normal(0.0, 1.0, size=50000).astype(np.float32))
    g[g == 0x8000] = 0  # -0 becomes +0 under a +0 accumulator; tested separately
    got = oracle.reduce_mean([g] * n_ranks)
    assert np.array_equal(got, g)


def test_opposite_pairs_cancel_exactly():
    rng = np.random.default_rng(5)
    g = _torch_bf16_bits(rng.normal(0.0, 1.0, size=10000).astype(np.float32))
    neg = g ^ np.uint16(0x8000)
    got = oracle.reduce_mean([g, neg, neg ^ np.uint16(0x8000), neg])
    assert np.all(got == 0)


def test_single_rank_is_identity_and_negative_zero_becomes_positive():
    rng = np.random.default_rng(6)
    g = _torch_bf16_bits(rng.normal(0.0, 1.0, size=10000).astype(np.float32))
    g[:3] = [0x8000, 0x0000, 0x8000]
    got = oracle.reduce_mean([g])
    expect = g.copy()
    expect[expect == 0x8000] = 0
    assert np.array_equal(got, expect)


def test_rank_order_matters_and_is_zero_to_n_minus_1():
    """(1 + 2^-24) + ... in rank order: 2^24 + 1 + 1 != 1 + 1 + 2^24 in binary32."""
    big = _bf16_from_f32(np.array([2.0**24], np.float32))
    one = _bf16_from_f32(np.array([1.0], np.float32))
    s_fwd = oracle.rank_sum_f32([big, one, one])[0]
    s_rev = oracle.rank_sum_f32([one, one, big])[0]
    assert s_fwd == np.float32(2.0**24)            # each +1 is lost to rounding (tie -> even)
    assert s_rev == np.float32(2.0**24 + 2.0)


def test_nonfinite_and_sumsq():
    g = _bf16_from_f32(np.array([3.0, -4.0, 0.0, 0.5], np.float32))
    assert oracle.sumsq(g) == 25.25
    assert oracle.count_nonfinite(g) == 0
    g2 = np.concatenate([g, np.array([0x7F80, 0xFFC1, 0x7F7F], np.uint16)])
    assert oracle.count_nonfinite(g2) == 2


def test_sumsq_matches_fsum_within_fp64_bound():
    rng = np.random.default_rng(8)
    g = _torch_bf16_bits(rng.normal(0.0, 1e-2, size=200000).astype(np.float32))
    x = oracle.bf16_to_f32(g).astype(np.float64)
    exact = math.fsum(x * x)  # each square is exact in binary64 (8-bit significands)
    n = x.size
    assert abs(oracle.sumsq(g) - exact) <= (n - 1) * 2.0**-53 * exact
