"""Shared helpers for the tests: seeded input fills (host and device), the
oracle's reference run for a workload, and ulp-distance comparisons."""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

import synth
from synth import workloads as W

# Tolerances of the CUDA path against the oracle (stated for the method):
# reduced gradient shards and all indexing bit-exact; fp32 master/m/v within
# 2 ulp (relative 2.4e-7); bf16 parameters within 1 bf16 ulp.
F32_ULP_TOL = 2
F32_REL_TOL = 2.4e-7
BF16_ULP_TOL = 1


# ------------------------------------------------------------ comparisons ----

def _ordered(bits: np.ndarray, width: int) -> np.ndarray:
    """Map IEEE patterns to integers whose difference counts ulps."""
    b = bits.astype(np.int64)
    sign = 1 << (width - 1)
    return np.where(b & sign, -(b & (sign - 1)), b)


def f32_ulp_dist(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, np.float32)
    b = np.ascontiguousarray(b, np.float32)
    d = np.abs(_ordered(a.view(np.uint32), 32) - _ordered(b.view(np.uint32), 32))
    both_nan = np.isnan(a) & np.isnan(b)
    return np.where(both_nan, 0, d)


def bf16_ulp_dist(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a).view(np.uint16)
    b = np.ascontiguousarray(b).view(np.uint16)
    nan_a = ((a & 0x7F80) == 0x7F80) & ((a & 0x7F) != 0)
    nan_b = ((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)
    d = np.abs(_ordered(a, 16) - _ordered(b, 16))
    return np.where(nan_a & nan_b, 0, d)


def assert_f32_close(got: np.ndarray, ref: np.ndarray, what: str):
    d = f32_ulp_dist(got, ref)
    rel = np.abs(got.astype(np.float64) - ref.astype(np.float64)) / np.maximum(np.abs(ref.astype(np.float64)), 1e-300)
    ok = (d <= F32_ULP_TOL) | (rel <= F32_REL_TOL)
    if not np.all(ok):
        i = int(np.flatnonzero(~ok)[0])
        raise AssertionError(f"{what}: {int((~ok).sum())} elements beyond 2 ulp; first at {i}: "
                             f"got {got[i]!r} ref {ref[i]!r} ({int(d[i])} ulp)")


def assert_bf16_close(got: np.ndarray, ref: np.ndarray, what: str):
    d = bf16_ulp_dist(got, ref)
    if np.any(d > BF16_ULP_TOL):
        i = int(np.flatnonzero(d > BF16_ULP_TOL)[0])
        raise AssertionError(f"{what}: {int((d > BF16_ULP_TOL).sum())} elements beyond 1 bf16 ulp; "
                             f"first at {i}: got {hex(int(got.view(np.uint16)[i]))} ref {hex(int(ref.view(np.uint16)[i]))}")


def assert_bits_equal(got: np.ndarray, ref: np.ndarray, what: str):
    g = np.ascontiguousarray(got).view(np.uint8)
    r = np.ascontiguousarray(ref).view(np.uint8)
    if not np.array_equal(g, r):
        gg = np.ascontiguousarray(got).reshape(-1)
        rr = np.ascontiguousarray(ref).reshape(-1)
        bad = np.flatnonzero(gg.view(np.uint8 if gg.itemsize == 1 else f"u{gg.itemsize}") !=
                             rr.view(np.uint8 if rr.itemsize == 1 else f"u{rr.itemsize}"))
        raise AssertionError(f"{what}: {bad.size} elements differ; first at {int(bad[0])}: "
                             f"got {gg[bad[0]]!r} ref {rr[bad[0]]!r}")


# ------------------------------------------------------------ input fills ----

def real_segments(offsets: Sequence[int], numel: Sequence[int], lo: int, hi: int):
    """(a, b) flat ranges of real elements inside [lo, hi), in order."""
    out = []
    for off, n in zip(offsets, numel):
        a, b = max(lo, off), min(hi, off + n)
        if a < b:
            out.append((a, b))
    return out


class DeviceFill:
    """Device-side seeded fills for a workload (pads are written as 0)."""

    def __init__(self, w: W.Workload, offsets: Sequence[int], psi_pad: int, f16: bool = False):
        self.w, self.offsets, self.psi_pad = w, list(offsets), psi_pad
        self.fill16 = synth.dev_f16 if f16 else synth.dev_bf16
        self.has_pads = any(o + n != e for o, n, e in zip(self.offsets, w.numel, self.offsets[1:] + [psi_pad]))

    def grads_into(self, step: int, rank: int, lo: int, hi: int, buf_ptr: int, buf_tensor, stream: int):
        """Write flat elements [lo, hi) of rank's step-`step` gradient at buf_ptr
        (buf_tensor: the int16 torch view starting at buf_ptr, for zeroing)."""
        b = W.grad_base(self.w, step, rank)
        segs = real_segments(self.offsets, self.w.numel, lo, hi)
        if self.has_pads:
            import torch

            with torch.cuda.stream(torch.cuda.ExternalStream(stream) if stream else torch.cuda.default_stream()):
                buf_tensor[: hi - lo].zero_()
        for a, e in segs:
            self.fill16(b, a, e - a, self.w.grad_dist, buf_ptr + 2 * (a - lo), stream)

    def master_into(self, master_ptr: int, master_tensor, stream: int):
        b = W.master_base(self.w)
        if self.has_pads:
            master_tensor.zero_()
        for a, e in real_segments(self.offsets, self.w.numel, 0, self.psi_pad):
            synth.dev_f32(b, a, e - a, W.MASTER_DIST, master_ptr + 4 * a, stream)


def host_grads(w: W.Workload, offsets, psi_pad: int, step: int, rank: int) -> np.ndarray:
    return W.host_padded(offsets, w.numel, psi_pad, W.grad_base(w, step, rank), w.grad_dist)


def host_master(w: W.Workload, offsets, psi_pad: int) -> np.ndarray:
    return W.host_padded(offsets, w.numel, psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)


def sample_indices(offsets, numel, psi_pad: int, shard: int, n_ranks: int, n_random: int,
                   seed: int = 1234, intervals: Sequence[tuple] = ()) -> np.ndarray:
    """Random real elements plus every boundary that can go wrong: both ends of
    each tensor, each shard and each schedule interval."""
    rng = np.random.default_rng(seed)
    real = [(o, o + n) for o, n in zip(offsets, numel) if n > 0]
    picks = []
    for a, b in real:
        picks += [a, a + 1, b - 2, b - 1]
    for r in range(n_ranks + 1):
        for d in (-2, -1, 0, 1):
            picks.append(r * shard + d)
    for lo, hi in intervals:
        picks += [lo - 1, lo, hi - 1, hi]
    lens = np.array([b - a for a, b in real], dtype=np.float64)
    which = rng.choice(len(real), size=n_random, p=lens / lens.sum())
    starts = np.array([real[k][0] for k in which])
    spans = np.array([real[k][1] - real[k][0] for k in which])
    picks += list(starts + (rng.random(n_random) * spans).astype(np.int64))
    idx = np.array(sorted(set(int(i) for i in picks if 0 <= i < psi_pad)), dtype=np.int64)
    mask = np.zeros(idx.size, dtype=bool)
    for a, b in real:
        mask |= (idx >= a) & (idx < b)
    return idx[mask]


def oracle_sampled(w: W.Workload, idx: np.ndarray, steps: int):
    """Plain-DP result of the sampled elements after ``steps`` steps."""
    import oracle

    m0 = synth.host_f32_at(W.master_base(w), idx, W.MASTER_DIST)
    per_step = []
    for t in range(1, steps + 1):
        per_step.append(np.stack([synth.host_bf16_at(W.grad_base(w, t, r), idx, w.grad_dist)
                                  for r in range(w.n_ranks)]))
    hp = oracle.AdamHP(**w.hyper.__dict__)
    out = oracle.trajectory_at(m0, per_step, hp)
    last = per_step[-1]
    g = oracle.reduce_mean([last[r] for r in range(last.shape[0])])
    out["grad"] = g
    return out


def to_np(t) -> np.ndarray:
    import torch

    a = t.detach().cpu()
    if a.dtype == torch.int16:
        return a.numpy().view(np.uint16)
    return a.numpy()
