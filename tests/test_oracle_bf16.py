"""Pins for the oracle's bf16 conversions against an independent implementation
(torch's CPU float->bfloat16 conversion), exhaustively over all 2^32 fp32
bit patterns.  NaN inputs must give a NaN (payloads may differ)."""
import multiprocessing as mp

import numpy as np
import pytest

CHUNK = 1 << 26


def _check_chunks(chunks):
    import sys
    import os

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch

    import oracle

    torch.set_num_threads(1)
    bad = []
    for c in chunks:
        u = np.arange(c * CHUNK, (c + 1) * CHUNK, dtype=np.uint64).astype(np.uint32)
        f = u.view(np.float32)
        got = oracle.bf16_rne(f)
        ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        nan_in = np.isnan(f)
        got_nan = (got & 0x7F80) == 0x7F80
        got_nan &= (got & 0x007F) != 0
        mism = (got != ref) & ~nan_in
        if np.any(mism):
            i = int(np.flatnonzero(mism)[0])
            bad.append((int(u[i]), int(got[i]), int(ref[i])))
        if np.any(nan_in & ~got_nan):
            i = int(np.flatnonzero(nan_in & ~got_nan)[0])
            bad.append((int(u[i]), int(got[i]), -1))
    return bad


def test_bf16_rne_exhaustive_vs_torch():
    n_chunks = (1 << 32) // CHUNK
    workers = max(1, min(16, mp.cpu_count()))
    parts = [list(range(k, n_chunks, workers)) for k in range(workers)]
    ctx = mp.get_context("spawn")
    with ctx.Pool(workers) as pool:
        results = pool.map(_check_chunks, parts)
    bad = [b for r in results for b in r]
    assert not bad, f"first mismatches (bits, oracle, torch): {bad[:5]}"


def test_bf16_to_f32_all_patterns():
    import torch

    import oracle

    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_to_f32(h)
    ref = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).float().numpy()
    both_nan = np.isnan(got) & np.isnan(ref)
    assert np.array_equal(got.view(np.uint32)[~both_nan], ref.view(np.uint32)[~both_nan])
    assert np.array_equal(np.isnan(got), np.isnan(ref))


@pytest.mark.parametrize(
    "x,expect",
    [
        (1.0, 0x3F80),
        (1.0 + 2.0**-8, 0x3F80),             # tie -> even (down)
        (1.0 + 3 * 2.0**-8, 0x3F82),         # tie -> even (up)
        (1.0 + 2.0**-8 + 2.0**-20, 0x3F81),  # just above the tie
        (-1.0 - 2.0**-8, 0xBF80),
        (3.3895313892515355e38, 0x7F7F),     # largest finite bf16
        (3.4028234663852886e38, 0x7F80),     # fp32 max rounds to +inf
        (float("inf"), 0x7F80),
        (-0.0, 0x8000),
        (2.0**-133, 0x0001),                 # smallest bf16 subnormal
        (2.0**-134, 0x0000),                 # half of it: tie -> even (0)
        (3 * 2.0**-134, 0x0002),             # 1.5 ulp: tie -> even (2)
    ],
)
def test_bf16_rne_worked_cases(x, expect):
    """Hand-worked IEEE roundTiesToEven cases on the 8-bit significand."""
    import oracle

    assert int(oracle.bf16_rne(np.array([x], dtype=np.float32))[0]) == expect
