"""CPU oracle for the ZeRO optimizer step over N logical data-parallel ranks.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference leg may import this package.  The
product library never calls it, and it imports nothing from the product: it
shares no code, header, table or helper with the CUDA path.  The only thing
both sides share is the seeded input generator in ``synth``.

What it computes, and where each piece comes from (three web pages on ZeRO):
  [T]  "ZERO训练技术" (wqh011128.github.io)
  [M]  "ZeRO：从优化器状态到残差状态的显存优化" (xuesongtap.github.io)
  [Q]  mstx.cn post 475, a ZeRO interview write-up

* ``plan``            -- the N-way contiguous ownership partition ([T] section
                         "ZeRO-1", part "optimizer state 怎么切分") and the
                         fixed-size bucket schedule ([M] section 3.3 "CB").
* ``all_reduce`` / ``reduce_scatter`` / ``all_gather`` -- the three
                         collectives as literal copies between per-rank arrays
                         ([T] sections "ZeRO-1" and "ZeRO-2"; [Q] sections 三, 四).
* ``run``             -- plain DP and the ZeRO-1/2/3 step flows ([T] sections
                         "先立一个基线", "ZeRO-1", "ZeRO-2", "ZeRO-3").
* ``state_bytes`` / ``mem_model`` -- per-rank model-state bytes ([Q] section
                         六 table; [M] section 5 worked example).
* ``comm_elems``      -- logical communication volume per rank ([M] section 2;
                         [Q] sections 三.3, 五.4).

The per-element arithmetic (bf16 rounding, the rank-order reduction, Adam)
lives in ``zero_oracle.c``; its readings of the pages are stated there.

Pinned by ``tests/test_oracle_*.py``: exhaustive bf16 rounding against
torch's CPU conversion, reduction against exact sums and error bounds, Adam
against ``torch.optim.AdamW``, stage equivalence with plain DP, bucket
invariance, brute force on tiny sizes, and the pages' closed forms and worked
numbers.  ``grad_norm`` has no exact external pin beyond an fp64 error bound
against ``math.fsum`` and is compared to the CUDA path within a tolerance.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field
from typing import Callable, List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None
_lib_path = None  # an alternative build, for the tests that plant mistakes in the oracle

STAGE_DP, STAGE_Z1, STAGE_Z2, STAGE_Z3 = 0, 1, 2, 3
BF16, F16 = 0, 1  # 16-bit storage formats of gradients and parameters
GRANULE = 8  # every tensor starts on an 8-element boundary (a stated layout choice)


class use_library:
    """Context manager: run the oracle on another build of zero_oracle.c (the
    mutation tests compile copies with a planted mistake)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib, _lib_path
        self.saved = (_lib, _lib_path)
        _lib, _lib_path = None, self.path
        return self

    def __exit__(self, *exc):
        global _lib, _lib_path
        _lib, _lib_path = self.saved
        return False


def _load():
    global _lib
    if _lib is None:
        path = _lib_path or os.path.join(_HERE, "libzero_oracle.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run __graft_entry__.build() first")
        lib = ctypes.CDLL(path)
        vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
        lib.zo_bf16_rne.restype = ctypes.c_uint16
        lib.zo_bf16_rne.argtypes = [f32]
        lib.zo_bf16_to_f32.restype = f32
        lib.zo_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.zo_bf16_rne_array.restype = None
        lib.zo_bf16_rne_array.argtypes = [i64, vp, vp]
        lib.zo_bf16_to_f32_array.restype = None
        lib.zo_bf16_to_f32_array.argtypes = [i64, vp, vp]
        lib.zo_reduce_mean.restype = None
        lib.zo_reduce_mean.argtypes = [i32, i64, vp, vp]
        lib.zo_rank_sum_f32.restype = None
        lib.zo_rank_sum_f32.argtypes = [i32, i64, vp, vp]
        lib.zo_adam_scalars.restype = None
        f64 = ctypes.c_double
        lib.zo_adam_scalars.argtypes = [f64, f64, f64, f64, f64, i64, vp]
        lib.zo_adam.restype = None
        lib.zo_adam.argtypes = [i64, vp, vp, vp, vp, vp, f64, f64, f64, f64, f64, i64]
        lib.zo_adam_coef.restype = None
        lib.zo_adam_coef.argtypes = [i64, vp, f32, vp, vp, vp, vp, f64, f64, f64, f64, f64, i64]
        lib.zo_f16_rne.restype = ctypes.c_uint16
        lib.zo_f16_rne.argtypes = [f32]
        lib.zo_f16_to_f32.restype = f32
        lib.zo_f16_to_f32.argtypes = [ctypes.c_uint16]
        lib.zo_f16_rne_array.restype = None
        lib.zo_f16_rne_array.argtypes = [i64, vp, vp]
        lib.zo_f16_to_f32_array.restype = None
        lib.zo_f16_to_f32_array.argtypes = [i64, vp, vp]
        lib.zo_reduce_mean_fmt.restype = None
        lib.zo_reduce_mean_fmt.argtypes = [ctypes.c_int, i32, i64, vp, vp]
        lib.zo_adam_ex.restype = None
        lib.zo_adam_ex.argtypes = [ctypes.c_int, i64, vp, f32, f32, vp, vp, vp, vp, f64, f64, f64, f64, f64, i64]
        lib.zo_sumsq_fmt.restype = ctypes.c_double
        lib.zo_sumsq_fmt.argtypes = [ctypes.c_int, i64, vp]
        lib.zo_count_nonfinite_fmt.restype = i64
        lib.zo_count_nonfinite_fmt.argtypes = [ctypes.c_int, i64, vp]
        lib.zo_sumsq.restype = ctypes.c_double
        lib.zo_sumsq.argtypes = [i64, vp]
        lib.zo_count_nonfinite.restype = i64
        lib.zo_count_nonfinite.argtypes = [i64, vp]
        _lib = lib
    return _lib


# ------------------------------------------------------------ elementwise ----

def bf16_rne(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), IEEE round to nearest even,
    overflow to infinity.  The 2-byte format of the gradients and parameter
    copies that the pages account everywhere ([M] section 1, memory
    composition; [Q] sections 二, 四.2, 五.2); the pages name no rounding, and
    round-to-nearest-even is the reading taken."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    if x.size:
        _load().zo_bf16_rne_array(x.size, x.ctypes.data, out.ctypes.data)
    return out


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32, exact (the 2-byte format of [M] section 1)."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, dtype=np.float32)
    if h.size:
        _load().zo_bf16_to_f32_array(h.size, h.ctypes.data, out.ctypes.data)
    return out


def f16_rne(x: np.ndarray) -> np.ndarray:
    """fp32 -> IEEE binary16 bit patterns (uint16), round to nearest even,
    overflow to infinity, subnormals kept.  The FP16 the pages name for
    gradients and parameters ([M] section 1) as the alternative storage
    format to bf16."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    if x.size:
        _load().zo_f16_rne_array(x.size, x.ctypes.data, out.ctypes.data)
    return out


def f16_to_f32(h: np.ndarray) -> np.ndarray:
    """IEEE binary16 bit patterns -> fp32, exact ([M] section 1's FP16)."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, dtype=np.float32)
    if h.size:
        _load().zo_f16_to_f32_array(h.size, h.ctypes.data, out.ctypes.data)
    return out


def fmt_rne(x: np.ndarray, fmt: int) -> np.ndarray:
    """``bf16_rne`` or ``f16_rne`` by the storage format."""
    return f16_rne(x) if fmt == F16 else bf16_rne(x)


def fmt_to_f32(h: np.ndarray, fmt: int) -> np.ndarray:
    """``bf16_to_f32`` or ``f16_to_f32`` by the storage format."""
    return f16_to_f32(h) if fmt == F16 else bf16_to_f32(h)


def _ptr_array(arrays: Sequence[np.ndarray]):
    ptrs = (ctypes.c_void_p * len(arrays))()
    for r, a in enumerate(arrays):
        ptrs[r] = a.ctypes.data
    return ptrs


def reduce_mean(rank_slices: Sequence[np.ndarray]) -> np.ndarray:
    """Averaged bf16 gradient of N equal-length rank slices (uint16 arrays):
    the reduction of [T] section "ZeRO-2" (reduce-scatter of the ranks'
    gradients, averaged over the N ranks).  The pages fix neither order nor
    precision; the reading taken: a binary32 sum from +0 in rank order
    0..N-1, multiplied by the binary32 reciprocal of N, rounded to bf16."""
    rank_slices = [np.ascontiguousarray(a, dtype=np.uint16) for a in rank_slices]
    n = rank_slices[0].size
    assert all(a.size == n for a in rank_slices)
    out = np.empty(n, dtype=np.uint16)
    if n:
        _load().zo_reduce_mean(len(rank_slices), n, _ptr_array(rank_slices), out.ctypes.data)
    return out


def reduce_mean_fmt(rank_slices: Sequence[np.ndarray], fmt: int) -> np.ndarray:
    """reduce_mean for either 16-bit format (the bf16 path is reduce_mean):
    [T] section "ZeRO-2"'s averaged gradient, the mean rounded once to the
    storage format."""
    if fmt == BF16:
        return reduce_mean(rank_slices)
    rank_slices = [np.ascontiguousarray(a, dtype=np.uint16) for a in rank_slices]
    n = rank_slices[0].size
    out = np.empty(n, dtype=np.uint16)
    if n:
        _load().zo_reduce_mean_fmt(fmt, len(rank_slices), n, _ptr_array(rank_slices), out.ctypes.data)
    return out


def rank_sum_f32(rank_slices: Sequence[np.ndarray]) -> np.ndarray:
    """The binary32 rank-order sum inside ``reduce_mean``, before the mean
    ([T] section "ZeRO-2", the reduce of the reduce-scatter)."""
    rank_slices = [np.ascontiguousarray(a, dtype=np.uint16) for a in rank_slices]
    n = rank_slices[0].size
    out = np.empty(n, dtype=np.float32)
    if n:
        _load().zo_rank_sum_f32(len(rank_slices), n, _ptr_array(rank_slices), out.ctypes.data)
    return out


@dataclass(frozen=True)
class AdamHP:
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.0


def adam_scalars(hp: AdamHP, t: int) -> np.ndarray:
    """float32[9]: beta1, beta2, 1-beta1, 1-beta2, bc1, bc2, decay, lr, eps.
    The per-step scalars of bias-corrected Adam with decoupled weight decay,
    the optimizer every page names without writing it out ([T] sections
    "ZeRO-1" to "ZeRO-3", part "3. 更新"; the definition is Kingma & Ba's
    Algorithm 1 plus Loshchilov & Hutter's decoupled decay): each formed in
    binary64 from the hyper-parameters (beta^t by t multiplications) and
    rounded once to binary32."""
    out = np.empty(9, dtype=np.float32)
    _load().zo_adam_scalars(hp.lr, hp.beta1, hp.beta2, hp.eps, hp.weight_decay, t,
                            out.ctypes.data)
    return out


def adam(g: np.ndarray, master: np.ndarray, m: np.ndarray, v: np.ndarray, hp: AdamHP,
         t: int) -> np.ndarray:
    """In-place Adam on fp32 master/m/v from the bf16 grad g; returns the bf16 params.

    The owner's update of its shard in every ZeRO stage ([T] sections
    "ZeRO-1" to "ZeRO-3", part "3. 更新"), on the fp32 master weights and
    moments the pages keep per parameter ([M] section 1: 4 + 4 + 4 bytes),
    followed by the cast of the new master to the 2-byte parameter copy."""
    assert master.dtype == np.float32 and m.dtype == np.float32 and v.dtype == np.float32
    assert master.flags.c_contiguous and m.flags.c_contiguous and v.flags.c_contiguous
    g = np.ascontiguousarray(g, dtype=np.uint16)
    n = g.size
    assert master.size == n and m.size == n and v.size == n
    out = np.empty(n, dtype=np.uint16)
    if n:
        _load().zo_adam(n, g.ctypes.data, master.ctypes.data, m.ctypes.data, v.ctypes.data,
                        out.ctypes.data, hp.lr, hp.beta1, hp.beta2, hp.eps, hp.weight_decay, t)
    return out


def adam_coef(g: np.ndarray, coef: float, master: np.ndarray, m: np.ndarray, v: np.ndarray, hp: AdamHP,
              t: int) -> np.ndarray:
    """Adam with the averaged gradient scaled by a clipping coefficient
    (applied only when coef < 1): ``adam``'s update ([T] sections "ZeRO-1" to
    "ZeRO-3", part "3. 更新") on fp32(g) * coef.  Clipping itself is not on
    the pages; see ``clip_coef``."""
    g = np.ascontiguousarray(g, dtype=np.uint16)
    n = g.size
    assert master.size == n and m.size == n and v.size == n
    out = np.empty(n, dtype=np.uint16)
    if n:
        _load().zo_adam_coef(n, g.ctypes.data, float(np.float32(coef)), master.ctypes.data, m.ctypes.data,
                             v.ctypes.data, out.ctypes.data, hp.lr, hp.beta1, hp.beta2, hp.eps, hp.weight_decay, t)
    return out


def adam_ex(g: np.ndarray, fmt: int, inv_scale: float, coef: float, master: np.ndarray, m: np.ndarray,
            v: np.ndarray, hp: AdamHP, t: int) -> np.ndarray:
    """Adam for either format with a loss-scale unscale (inv_scale != 1) and a
    clipping coefficient (applied when < 1); returns the 16-bit params.
    ``adam``'s update ([T] sections "ZeRO-1" to "ZeRO-3", part "3. 更新") on
    the FP16 storage the pages name ([M] section 1), whose gradients carry the
    loss scale that fp16 training needs (not on the pages): fp32(g) times
    fp32(1/S), then the coefficient, each one binary32 multiplication."""
    g = np.ascontiguousarray(g, dtype=np.uint16)
    n = g.size
    out = np.empty(n, dtype=np.uint16)
    if n:
        _load().zo_adam_ex(fmt, n, g.ctypes.data, float(np.float32(inv_scale)), float(np.float32(coef)),
                           master.ctypes.data, m.ctypes.data, v.ctypes.data, out.ctypes.data,
                           hp.lr, hp.beta1, hp.beta2, hp.eps, hp.weight_decay, t)
    return out


def sumsq_fmt(g: np.ndarray, fmt: int) -> float:
    """Sum of squares of a 16-bit gradient in binary64, in element order: the
    squared norm for the clip and overflow checks (not on the pages)."""
    g = np.ascontiguousarray(g, dtype=np.uint16)
    return float(_load().zo_sumsq_fmt(fmt, g.size, g.ctypes.data)) if g.size else 0.0


def count_nonfinite_fmt(g: np.ndarray, fmt: int) -> int:
    """Number of infinite or NaN elements of a 16-bit gradient (the overflow
    check; not on the pages)."""
    g = np.ascontiguousarray(g, dtype=np.uint16)
    return int(_load().zo_count_nonfinite_fmt(fmt, g.size, g.ctypes.data)) if g.size else 0


CLIP_EPS = 1e-6


def clip_coef(grad_norm: float, max_norm: float) -> float:
    """Global-norm clipping coefficient (not on the pages; the usual
    convention): c = max_norm / (norm + 1e-6) in binary64, rounded once to
    binary32; 1 when that is not below 1 (no clipping)."""
    c = float(np.float32(max_norm / (grad_norm + CLIP_EPS)))
    return c if c < 1.0 else 1.0


def sumsq(g: np.ndarray) -> float:
    """``sumsq_fmt`` for bf16 (not on the pages: the gradient norm's square)."""
    g = np.ascontiguousarray(g, dtype=np.uint16)
    return float(_load().zo_sumsq(g.size, g.ctypes.data)) if g.size else 0.0


def count_nonfinite(g: np.ndarray) -> int:
    """``count_nonfinite_fmt`` for bf16 (the overflow check; not on the pages)."""
    g = np.ascontiguousarray(g, dtype=np.uint16)
    return int(_load().zo_count_nonfinite(g.size, g.ctypes.data)) if g.size else 0


# ------------------------------------------------------------------- plan ----

def _roundup(x: int, m: int) -> int:
    return (x + m - 1) // m * m


@dataclass
class Plan:
    """Flat layout of a parameter list cut into N owned segments.

    Reading of "cut the parameter vector into N parts" ([T] section "ZeRO-1",
    part "optimizer state 怎么切分"): tensors are laid end to end in list
    order, each starting on an 8-element boundary; the flat length is padded
    up to a multiple of 8N so the N segments are equal and contiguous; rank r
    owns [r*S, (r+1)*S).  Pad elements hold 0 everywhere.
    """

    numel: List[int]
    layer_id: List[int]
    n_ranks: int
    bucket_elems: int
    offset: List[int] = field(default_factory=list)   # start of each tensor
    slot_end: List[int] = field(default_factory=list)  # end of each tensor's padded slot
    psi: int = 0          # real parameter count
    psi_pad: int = 0      # padded flat length
    shard: int = 0        # S = psi_pad / N
    layers: List[tuple] = field(default_factory=list)   # (layer id, lo, hi), list order
    buckets: List[tuple] = field(default_factory=list)  # (lo, hi), in schedule order

    def owner(self, i: int) -> int:
        return i // self.shard

    def owned(self, r: int) -> tuple:
        return (r * self.shard, (r + 1) * self.shard)

    def real_mask(self) -> np.ndarray:
        mask = np.zeros(self.psi_pad, dtype=bool)
        for off, n in zip(self.offset, self.numel):
            mask[off:off + n] = True
        return mask


def plan(numel: Sequence[int], layer_id: Sequence[int], n_ranks: int, bucket_elems: int) -> Plan:
    """The flat layout, the N-way ownership partition ([T] section "ZeRO-1",
    part "optimizer state 怎么切分"; reading in ``Plan``), the layers' flat
    ranges ([T] section "ZeRO-3", one layer gathered at a time) and the
    fixed-size buffer schedule (``bucket_schedule``: [M] section 3.3 "CB")."""
    assert n_ranks >= 1 and bucket_elems > 0 and bucket_elems % GRANULE == 0
    assert len(numel) == len(layer_id) and len(numel) >= 1
    assert all(n >= 0 for n in numel)
    assert all(a <= b for a, b in zip(layer_id, layer_id[1:]))
    p = Plan(list(numel), list(layer_id), n_ranks, bucket_elems)
    cursor = 0
    for n in numel:
        p.offset.append(cursor)
        cursor = _roundup(cursor + n, GRANULE)
    flat = cursor
    p.psi = int(sum(numel))
    p.psi_pad = _roundup(max(flat, 1), GRANULE * n_ranks)
    p.shard = p.psi_pad // n_ranks
    # each tensor's padded slot runs to the next tensor's start; the last one
    # also takes the tail padding up to psi_pad
    p.slot_end = p.offset[1:] + [p.psi_pad]
    # layers: maximal runs of equal layer id (contiguous in the flat space)
    k = 0
    while k < len(numel):
        j = k
        while j + 1 < len(numel) and layer_id[j + 1] == layer_id[k]:
            j += 1
        p.layers.append((layer_id[k], p.offset[k], p.slot_end[j]))
        k = j + 1
    p.buckets = bucket_schedule(p)
    return p


def bucket_schedule(p: Plan) -> List[tuple]:
    """Fixed-size buffer schedule ([M] section 3.3 "CB"; [T] section "ZeRO-2",
    part "2. 反向"): gradients become ready layer by layer from the last layer
    back, so tensors are walked in reverse list order and packed into the
    current interval while it stays within ``bucket_elems``; when the next
    tensor does not fit, the interval is flushed.  A tensor slot larger than
    the buffer is cut into buffer-sized chunks from its end, each its own
    interval (the last, lowest chunk may be shorter).
    """
    out: List[tuple] = []
    cur: Optional[list] = None  # [lo, hi]
    B = p.bucket_elems
    for k in reversed(range(len(p.numel))):
        a, b = p.offset[k], p.slot_end[k]
        size = b - a
        if size == 0:
            continue
        if size > B:
            if cur is not None:
                out.append(tuple(cur))
                cur = None
            e = b
            while e - a > B:
                out.append((e - B, e))
                e -= B
            out.append((a, e))
        elif cur is not None and (cur[1] - cur[0]) + size <= B:
            cur[0] = a
        else:
            if cur is not None:
                out.append(tuple(cur))
            cur = [a, b]
    if cur is not None:
        out.append(tuple(cur))
    return out


# ------------------------------------------------------------ collectives ----

def all_reduce(rank_grads: Sequence[np.ndarray], lo: int, hi: int, fmt: int = BF16) -> None:
    """All-reduce of [lo, hi) in place ([T] section "ZeRO-1", part "2. 反向"):
    every rank's replica receives the same averaged gradient."""
    g = reduce_mean_fmt([a[lo:hi] for a in rank_grads], fmt)
    for a in rank_grads:
        a[lo:hi] = g


def reduce_scatter(rank_grads: Sequence[np.ndarray], plan_: Plan, lo: int, hi: int,
                   grad_shards: List[np.ndarray], fmt: int = BF16) -> None:
    """Reduce-scatter of [lo, hi) ([T] section "ZeRO-2", part "reduce-scatter
    是什么"): rank r receives only the reduced values of the elements it owns,
    written into its shard array (indexed from r*S)."""
    for r in range(plan_.n_ranks):
        olo, ohi = plan_.owned(r)
        a, b = max(lo, olo), min(hi, ohi)
        if a >= b:
            continue
        grad_shards[r][a - olo:b - olo] = reduce_mean_fmt([g[a:b] for g in rank_grads], fmt)


def all_gather(param_shards: Sequence[np.ndarray], plan_: Plan, lo: int, hi: int,
               rank_out: Sequence[np.ndarray], out_base: int = 0) -> None:
    """All-gather of [lo, hi) ([T] section "ZeRO-1", part "all-gather 是什么"):
    each rank contributes the part of its owned shard inside [lo, hi) and
    every destination receives the concatenation.  ``rank_out[q]`` is indexed
    from flat position ``out_base``."""
    for r in range(plan_.n_ranks):
        olo, ohi = plan_.owned(r)
        a, b = max(lo, olo), min(hi, ohi)
        if a >= b:
            continue
        piece = param_shards[r][a - olo:b - olo]
        for q in range(len(rank_out)):
            rank_out[q][a - out_base:b - out_base] = piece


# ----------------------------------------------------------- step flows ----

GradFn = Callable[[int, int], np.ndarray]  # (step, rank) -> uint16[psi_pad], pads 0


@dataclass
class RankState:
    params: Optional[np.ndarray] = None   # bf16 full replica (DP/Z1/Z2) or shard (Z3)
    grads: Optional[np.ndarray] = None    # bf16 full (DP/Z1) or owned shard (Z2/Z3)
    master: Optional[np.ndarray] = None   # fp32, full (DP) or owned shard
    m: Optional[np.ndarray] = None
    v: Optional[np.ndarray] = None


@dataclass
class StepReport:
    grad_norm: float
    nonfinite: int
    gathered: Optional[List[List[np.ndarray]]] = None  # Z3: per layer (schedule order), per rank
    skipped: bool = False
    coef: float = 1.0


def init_states(plan_: Plan, stage: int, master0: np.ndarray, fmt: int = BF16) -> List[RankState]:
    """Every rank starts from the same fp32 master (pads 0), m = v = 0 and the
    16-bit parameter copy equal to the master rounded to the format: plain
    DP's identical replicas ([T] section "先立一个基线"), each ZeRO stage
    keeping of the fp32 states only the owned shard ([T] sections "ZeRO-1"
    to "ZeRO-3") and stage 3 only the owned parameter shard."""
    assert master0.dtype == np.float32 and master0.size == plan_.psi_pad
    p16 = fmt_rne(master0, fmt)
    ranks = []
    for r in range(plan_.n_ranks):
        lo, hi = plan_.owned(r)
        st = RankState()
        if stage == STAGE_DP:
            st.master = master0.copy()
        else:
            st.master = master0[lo:hi].copy()
        st.m = np.zeros_like(st.master)
        st.v = np.zeros_like(st.master)
        st.params = p16[lo:hi].copy() if stage == STAGE_Z3 else p16.copy()
        ranks.append(st)
    return ranks


def step(plan_: Plan, stage: int, ranks: List[RankState], grads: GradFn, t: int,
         hp: AdamHP, clip_norm: float = 0.0, skip_nonfinite: bool = False, fmt: int = BF16,
         loss_scale: float = 1.0) -> StepReport:
    """One optimizer step, t >= 1, following the pages' flow for ``stage``:
    every gradient is reduced (and scattered) first, then each rank updates
    what it owns, then the parameters are gathered.

    Options that are not on the pages (a global-norm clip and an overflow
    skip): the norm of the whole averaged gradient is known after the
    reduction, before any update.  With ``skip_nonfinite`` a step whose
    averaged gradient holds an Inf or NaN changes no state (the caller does not
    advance t); with ``clip_norm`` > 0 every rank's Adam uses the gradient
    times clip_coef(norm, clip_norm).

    ``fmt`` = F16 stores gradients and parameters as IEEE binary16; with a
    ``loss_scale`` S the ranks' gradients are S times the true ones: the
    averaged gradient is rounded to the format still scaled, the update first
    multiplies it by fp32(1/S), and the reported norm (and the clip) is that
    of the unscaled gradient, sqrt(sum g^2) / S."""
    N, S = plan_.n_ranks, plan_.shard
    generic = fmt != BF16 or loss_scale != 1.0
    inv_scale = float(np.float32(1.0 / loss_scale))
    local = [grads(t, r).astype(np.uint16, copy=True) for r in range(N)]
    assert all(a.size == plan_.psi_pad for a in local)

    def update(g, st):
        if generic:
            return adam_ex(g, fmt, inv_scale, coef, st.master, st.m, st.v, hp, t)
        if coef < 1.0:
            return adam_coef(g, coef, st.master, st.m, st.v, hp, t)
        return adam(g, st.master, st.m, st.v, hp, t)

    if stage in (STAGE_DP, STAGE_Z1):
        # backward ends with a full all-reduce; every rank keeps the full grad
        for lo, hi in plan_.buckets:
            all_reduce(local, lo, hi, fmt)
        for r in range(N):
            ranks[r].grads = local[r]
        g_full = local[0]
    else:
        shards = [np.zeros(S, dtype=np.uint16) for _ in range(N)]
        if stage == STAGE_Z2:
            # layer-by-layer reduce-scatter through the fixed-size buffer
            for lo, hi in plan_.buckets:
                reduce_scatter(local, plan_, lo, hi, shards, fmt)
        else:
            # per layer, last to first: reduce-scatter the layer's gradient
            for _, lo, hi in reversed(plan_.layers):
                reduce_scatter(local, plan_, lo, hi, shards, fmt)
        for r in range(N):
            ranks[r].grads = shards[r]
        g_full = np.concatenate(shards)
    if generic:
        norm = float(np.sqrt(sumsq_fmt(g_full, fmt))) / loss_scale
        nonfinite = count_nonfinite_fmt(g_full, fmt)
    else:
        norm = float(np.sqrt(sumsq(g_full)))
        nonfinite = count_nonfinite(g_full)
    if skip_nonfinite and nonfinite > 0:
        return StepReport(grad_norm=norm, nonfinite=nonfinite, skipped=True)
    coef = clip_coef(norm, clip_norm) if clip_norm > 0 else 1.0
    if stage == STAGE_DP:
        # every rank runs the identical update on its full replica
        for r in range(N):
            ranks[r].params = update(local[r], ranks[r])
        return StepReport(grad_norm=norm, nonfinite=nonfinite, coef=coef)
    if stage in (STAGE_Z1, STAGE_Z2):
        # each rank updates only its owned shard, then all-gather
        new_shards = []
        for r in range(N):
            lo, hi = plan_.owned(r)
            new_shards.append(update(ranks[r].grads[lo:hi] if stage == STAGE_Z1 else ranks[r].grads, ranks[r]))
        all_gather(new_shards, plan_, 0, plan_.psi_pad, [ranks[r].params for r in range(N)])
        return StepReport(grad_norm=norm, nonfinite=nonfinite, coef=coef)
    assert stage == STAGE_Z3
    for r in range(N):
        ranks[r].params = update(ranks[r].grads, ranks[r])
    # per layer, the all-gather of the updated shards into a temporary
    # full-layer buffer on every rank, released after use
    gathered = []
    for _, lo, hi in reversed(plan_.layers):
        tmp = [np.zeros(hi - lo, dtype=np.uint16) for _ in range(N)]
        all_gather([ranks[r].params for r in range(N)], plan_, lo, hi, tmp, out_base=lo)
        gathered.append(tmp)
    return StepReport(grad_norm=norm, nonfinite=nonfinite, gathered=gathered, coef=coef)


def run(plan_: Plan, stage: int, master0: np.ndarray, grads: GradFn, steps: int, hp: AdamHP,
        clip_norm: float = 0.0, skip_nonfinite: bool = False, fmt: int = BF16, loss_scale: float = 1.0):
    """``steps`` optimizer steps; gradients for call k come from grads(k, r).
    Each step follows ``step``'s flow for the stage ([T] sections
    "先立一个基线", "ZeRO-1", "ZeRO-2", "ZeRO-3").  A skipped step (the
    overflow skip, not on the pages) does not advance the Adam step counter
    t, so the Adam step number of call k is 1 + (calls before it that were
    not skipped)."""
    ranks = init_states(plan_, stage, master0, fmt)
    reports = []
    t = 0
    for k in range(1, steps + 1):
        rep = step(plan_, stage, ranks, lambda _t, r, k=k: grads(k, r), t + 1, hp, clip_norm, skip_nonfinite,
                   fmt, loss_scale)
        if not rep.skipped:
            t += 1
        reports.append(rep)
    return ranks, reports


def full_view(plan_: Plan, stage: int, ranks: List[RankState]) -> dict:
    """Assemble the flat master/m/v/params/grad (psi_pad each) from the ranks:
    owned shards concatenated in rank order (rank 0's copy for DP) -- the
    inverse of the ownership partition of [T] section "ZeRO-1"."""
    if stage == STAGE_DP:
        r0 = ranks[0]
        return dict(master=r0.master, m=r0.m, v=r0.v, params=r0.params, grad=r0.grads)
    cat = lambda name: np.concatenate([getattr(r, name) for r in ranks])
    out = dict(master=cat("master"), m=cat("m"), v=cat("v"))
    out["params"] = cat("params") if stage == STAGE_Z3 else ranks[0].params
    if stage == STAGE_Z1:
        out["grad"] = ranks[0].grads
    else:
        out["grad"] = cat("grads")
    return out


# ---------------------------------------------------- sampled trajectories ----

def trajectory_at(master0: np.ndarray, rank_grads_per_step: Sequence[np.ndarray], hp: AdamHP,
                  t0: int = 1) -> dict:
    """Plain-DP result for a sample of elements, which every ZeRO stage must
    reproduce ([T] sections "ZeRO-1"/"ZeRO-2"/"ZeRO-3": sharding the state
    does not change the update).  ``rank_grads_per_step[s]`` is uint16[N, k]
    for step t0 + s; ``master0`` is float32[k].  Returns the final master, m,
    v, bf16 params and the last step's averaged bf16 grad."""
    master = np.ascontiguousarray(master0, dtype=np.float32).copy()
    m = np.zeros_like(master)
    v = np.zeros_like(master)
    params = bf16_rne(master)
    g = np.zeros(master.size, dtype=np.uint16)
    for s, rg in enumerate(rank_grads_per_step):
        g = reduce_mean([rg[r] for r in range(rg.shape[0])])
        params = adam(g, master, m, v, hp, t0 + s)
    return dict(master=master, m=m, v=v, params=params, grad=g)


# ------------------------------------------------- memory and communication ----

def state_bytes(plan_: Plan, stage: int) -> tuple:
    """Per-rank long-lived model-state bytes (params, grads, optimizer states)
    for a mixed-precision Adam run ([Q] sections 二, 三.2, 四.2, 五.2; [M]
    section 1): 16-bit params and grads at 2 B, fp32 master/m/v at 12 B; each
    stage shards one more of the three ([T] section "一张总对比表")."""
    P, S = plan_.psi_pad, plan_.shard
    return {
        STAGE_DP: (2 * P, 2 * P, 12 * P),
        STAGE_Z1: (2 * P, 2 * P, 12 * S),
        STAGE_Z2: (2 * P, 2 * S, 12 * S),
        STAGE_Z3: (2 * S, 2 * S, 12 * S),
    }[stage]


def mem_model(psi: float, n_ranks: int) -> dict:
    """The pages' per-card model-state totals in bytes, written out term by
    term (16-bit params 2, 16-bit grads 2, fp32 master/m/v 12 per param, each
    sharded over N where the stage shards it)."""
    return {
        STAGE_DP: 2 * psi + 2 * psi + 12 * psi,
        STAGE_Z1: 2 * psi + 2 * psi + 12 * psi / n_ranks,
        STAGE_Z2: 2 * psi + 2 * psi / n_ranks + 12 * psi / n_ranks,
        STAGE_Z3: 2 * psi / n_ranks + 2 * psi / n_ranks + 12 * psi / n_ranks,
    }


def comm_elems(plan_: Plan, stage: int) -> dict:
    """Logical elements each rank sends per step, ring convention: a
    reduce-scatter or an all-gather of P elements over N ranks sends
    P(N-1)/N, an all-reduce twice that.  DP: one all-reduce.  ZeRO-1: an
    all-reduce and the parameter all-gather ([T] section "ZeRO-1"; [Q] section
    三.3).  ZeRO-2: reduce-scatter plus the all-gather.  ZeRO-3: a parameter
    all-gather in the forward, another in the backward, and the gradient
    reduce-scatter ([Q] section 五.4, 七)."""
    P, N = plan_.psi_pad, plan_.n_ranks
    one = P * (N - 1) // N
    return {
        STAGE_DP: dict(all_reduce=2 * one, reduce_scatter=0, all_gather=0),
        STAGE_Z1: dict(all_reduce=2 * one, reduce_scatter=0, all_gather=one),
        STAGE_Z2: dict(all_reduce=0, reduce_scatter=one, all_gather=one),
        STAGE_Z3: dict(all_reduce=0, reduce_scatter=one, all_gather=2 * one),
    }[stage]
