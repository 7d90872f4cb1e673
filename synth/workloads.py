"""Synthetic workload recipes for the ZeRO optimizer step.

Each recipe fixes the parameter list (tensor sizes grouped into layers), the
number of logical data-parallel ranks N, the ZeRO stage(s), the bucket size,
the seeds and the value distributions of the per-rank gradients and of the
initial fp32 master weights, the Adam hyper-parameters and the step count.
Nothing here computes any part of the optimizer step.

Shapes follow the pages' and the benchmark's transformer-shaped parameter
lists: per layer LayerNorm-1 gain/bias, qkv weight and bias, attention
projection weight and bias, LayerNorm-2 gain/bias, MLP up weight and bias,
MLP down weight and bias.  No dataset is involved: every value is drawn from
the counter-based generator in this package.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np

from . import NORMAL, STREAM_GRAD, STREAM_MASTER, UNIFORM, Dist, base, host_bf16, host_f16, host_f32

SEED0 = 0x5EED0000


def transformer_layers(n_layers: int, hidden: int, mlp: int) -> tuple:
    """(numel list, layer id list) of a stack of pre-LN transformer blocks."""
    per_layer = [hidden, hidden,                 # LN1 gain, bias
                 hidden * 3 * hidden, 3 * hidden,  # qkv weight, bias
                 hidden * hidden, hidden,          # attention projection weight, bias
                 hidden, hidden,                   # LN2 gain, bias
                 hidden * mlp, mlp,                # MLP up weight, bias
                 mlp * hidden, hidden]             # MLP down weight, bias
    numel, layer = [], []
    for l in range(n_layers):
        numel += per_layer
        layer += [l] * len(per_layer)
    return numel, layer


@dataclass(frozen=True)
class Hyper:
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.0


@dataclass
class Workload:
    name: str
    numel: List[int]
    layer_id: List[int]
    n_ranks: int
    stages: Sequence[int]
    bucket_elems: Optional[int]        # None = one bucket spanning everything
    grad_dist: Dist
    master_dist: Dist
    steps: int
    hyper: Hyper
    seed: int
    notes: str = ""

    @property
    def psi(self) -> int:
        return int(sum(self.numel))


MASTER_DIST = Dist(NORMAL, 0.02)


def flat_1m_n4() -> Workload:
    """Flat 1,048,576 params as 4 tensors of 512x512, N = 4, ZeRO-2, one bucket."""
    return Workload("flat-1M-4x512x512-N4-zero2", [512 * 512] * 4, [0, 1, 2, 3], 4, (2,), None,
                    Dist(NORMAL, 1e-3), MASTER_DIST, 3, Hyper(), SEED0 + 1)


def gpt_85m_n8() -> Workload:
    """12 layers, hidden 768 (85,054,464 params), N = 8, DP/ZeRO-1/2/3, 1% zero grads, wd 0.01."""
    numel, layer = transformer_layers(12, 768, 3072)
    return Workload("transformer-12L-h768-85M-N8", numel, layer, 8, (0, 1, 2, 3), None,
                    Dist(NORMAL, 1e-2, zero_mod=100), MASTER_DIST, 5, Hyper(weight_decay=0.01),
                    SEED0 + 2)


def gpt_1p2b_n8() -> Workload:
    """24 layers, hidden 2048 (1,208,598,528 params), N = 8, ZeRO-2, 200M-element bucket."""
    numel, layer = transformer_layers(24, 2048, 8192)
    return Workload("transformer-24L-h2048-1.2B-N8-zero2-bucket200M", numel, layer, 8, (2,),
                    200_000_000, Dist(NORMAL, 1e-2), MASTER_DIST, 3, Hyper(), SEED0 + 3)


def gpt_6p4b_n64() -> Workload:
    """32 layers, hidden 4096 (6,444,154,880 params), N = 64, ZeRO-3, one layer live."""
    numel, layer = transformer_layers(32, 4096, 16384)
    return Workload("transformer-32L-h4096-6.4B-N64-zero3", numel, layer, 64, (3,), None,
                    Dist(NORMAL, 1e-2), MASTER_DIST, 2, Hyper(), SEED0 + 4)


def flat_sweep(elems: int, n_ranks: int) -> Workload:
    """Flat buffer of ``elems`` params, ZeRO-2, one bucket, grads U(-1e-2, 1e-2)."""
    return Workload(f"flat-sweep-E{elems}-N{n_ranks}", [elems], [0], n_ranks, (2,), None,
                    Dist(UNIFORM, 1e-2), MASTER_DIST, 1, Hyper(), SEED0 + 5)


SWEEP_ELEMS = [1024 * 4**k for k in range(11)]    # 1K .. 1G
SWEEP_RANKS = [2, 4, 8, 16, 64]


# ----------------------------------------------------------- host fills ----

def grad_base(w: Workload, step: int, rank: int) -> int:
    return base(w.seed, STREAM_GRAD, step, rank)


def master_base(w: Workload) -> int:
    return base(w.seed, STREAM_MASTER, 0, 0)


def host_padded(offsets: Sequence[int], numel: Sequence[int], psi_pad: int, b: int, dist: Dist,
                as_f32: bool = False, f16: bool = False) -> np.ndarray:
    """Values for a padded flat layout: element at flat position i draws
    index i; pad positions (between tensors and at the tail) are 0.  16-bit
    patterns are bf16 unless ``f16``."""
    out = np.zeros(psi_pad, dtype=np.float32 if as_f32 else np.uint16)
    fill = host_f32 if as_f32 else (host_f16 if f16 else host_bf16)
    for off, n in zip(offsets, numel):
        if n:
            out[off:off + n] = fill(b, off, n, dist)
    return out
