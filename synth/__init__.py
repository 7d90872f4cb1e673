"""Seeded synthetic inputs for the ZeRO optimizer step.

This module holds the counter-based generator (SplitMix64, Steele, Lea &
Flood 2014) that both the CUDA path's tests/bench and the CPU oracle draw
their inputs from.  It contains none of the optimizer step's arithmetic: it
only produces gradient replicas and initial master weights.

Host draws come from ``libsynth_host.so`` (plain C); device draws from
``libsynth_dev.so`` (a CUDA fill kernel).  Both evaluate the same definition
in ``synth_gen.h`` and must agree bit for bit.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
NORMAL = 0
UNIFORM = 1

_host = None
_dev = None


def _load_host():
    global _host
    if _host is None:
        path = os.path.join(_HERE, "libsynth_host.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run __graft_entry__.build() first")
        lib = ctypes.CDLL(path)
        u64, i64, u32, i32, f64 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_uint32, ctypes.c_int, ctypes.c_double
        lib.synth_host_base.restype = u64
        lib.synth_host_base.argtypes = [u64, u32, u32, u32]
        for name in ("synth_host_fill_bf16", "synth_host_fill_f32"):
            fn = getattr(lib, name)
            fn.restype = None
            fn.argtypes = [u64, i64, i64, i32, f64, u32, ctypes.c_void_p]
        for name in ("synth_host_fill_f16",):
            fn = getattr(lib, name)
            fn.restype = None
            fn.argtypes = [u64, i64, i64, i32, f64, u32, ctypes.c_void_p]
        for name in ("synth_host_gather_bf16", "synth_host_gather_f32", "synth_host_gather_f16"):
            fn = getattr(lib, name)
            fn.restype = None
            fn.argtypes = [u64, ctypes.c_void_p, i64, i32, f64, u32, ctypes.c_void_p]
        _host = lib
    return _host


def _load_dev():
    global _dev
    if _dev is None:
        path = os.path.join(_HERE, "libsynth_dev.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run __graft_entry__.build() first")
        lib = ctypes.CDLL(path)
        u64, i64, u32, i32, f64 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_uint32, ctypes.c_int, ctypes.c_double
        lib.synth_dev_base.restype = u64
        lib.synth_dev_base.argtypes = [u64, u32, u32, u32]
        for name in ("synth_dev_fill_bf16", "synth_dev_fill_f32", "synth_dev_fill_f16"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [u64, i64, i64, i32, f64, u32, ctypes.c_void_p, ctypes.c_void_p]
        _dev = lib
    return _dev


@dataclass(frozen=True)
class Dist:
    """A value distribution: ``kind`` NORMAL (sigma) or UNIFORM (half-width a),
    with an optional exact-zero fraction 1/zero_mod (0 = none)."""

    kind: int
    width: float
    zero_mod: int = 0

    @property
    def scale(self) -> float:
        if self.kind == NORMAL:
            return self.width * math.sqrt(3.0) / float(1 << 24)
        return float(self.width)


# Stream ids: one per kind of input so that draws never collide.
STREAM_GRAD = 1
STREAM_MASTER = 2


def base(seed: int, stream: int, step: int, rank: int) -> int:
    return int(_load_host().synth_host_base(seed, stream, step, rank))


def host_bf16(b: int, idx0: int, n: int, dist: Dist) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    if n:
        _load_host().synth_host_fill_bf16(b, idx0, n, dist.kind, dist.scale, dist.zero_mod,
                                          out.ctypes.data)
    return out


def host_f16(b: int, idx0: int, n: int, dist: Dist) -> np.ndarray:
    """Binary16 patterns (uint16): the fp32 values truncated toward zero."""
    out = np.empty(n, dtype=np.uint16)
    if n:
        _load_host().synth_host_fill_f16(b, idx0, n, dist.kind, dist.scale, dist.zero_mod, out.ctypes.data)
    return out


def host_f16_at(b: int, idx: np.ndarray, dist: Dist) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    out = np.empty(idx.size, dtype=np.uint16)
    if idx.size:
        _load_host().synth_host_gather_f16(b, idx.ctypes.data, idx.size, dist.kind, dist.scale,
                                           dist.zero_mod, out.ctypes.data)
    return out


def host_f32(b: int, idx0: int, n: int, dist: Dist) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    if n:
        _load_host().synth_host_fill_f32(b, idx0, n, dist.kind, dist.scale, dist.zero_mod,
                                         out.ctypes.data)
    return out


def host_bf16_at(b: int, idx: np.ndarray, dist: Dist) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    out = np.empty(idx.size, dtype=np.uint16)
    if idx.size:
        _load_host().synth_host_gather_bf16(b, idx.ctypes.data, idx.size, dist.kind, dist.scale,
                                            dist.zero_mod, out.ctypes.data)
    return out


def host_f32_at(b: int, idx: np.ndarray, dist: Dist) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    out = np.empty(idx.size, dtype=np.float32)
    if idx.size:
        _load_host().synth_host_gather_f32(b, idx.ctypes.data, idx.size, dist.kind, dist.scale,
                                           dist.zero_mod, out.ctypes.data)
    return out


def dev_bf16(b: int, idx0: int, n: int, dist: Dist, out_ptr: int, stream: int) -> None:
    """Fill ``n`` bf16 values (as uint16) at device pointer ``out_ptr``."""
    rc = _load_dev().synth_dev_fill_bf16(b, idx0, n, dist.kind, dist.scale, dist.zero_mod,
                                         out_ptr, stream)
    if rc != 0:
        raise RuntimeError(f"synth_dev_fill_bf16 failed with cudaError {rc}")


def dev_f16(b: int, idx0: int, n: int, dist: Dist, out_ptr: int, stream: int) -> None:
    rc = _load_dev().synth_dev_fill_f16(b, idx0, n, dist.kind, dist.scale, dist.zero_mod, out_ptr, stream)
    if rc != 0:
        raise RuntimeError(f"synth_dev_fill_f16 failed with cudaError {rc}")


def dev_f32(b: int, idx0: int, n: int, dist: Dist, out_ptr: int, stream: int) -> None:
    rc = _load_dev().synth_dev_fill_f32(b, idx0, n, dist.kind, dist.scale, dist.zero_mod,
                                        out_ptr, stream)
    if rc != 0:
        raise RuntimeError(f"synth_dev_fill_f32 failed with cudaError {rc}")
