"""B200 (sm_100a) ZeRO optimizer step over N logical data-parallel ranks.

The compute lives in ``libzero_sm.so`` (hand-written CUDA behind a C ABI,
declared in ``include/zero_sm.h``).  This module only marshals arguments:

* the raw C functions, under their C names (``zero_init``, ``zero_step``, ...),
  loaded with ctypes;
* ``ZeroOptimizer``, which sizes and allocates the arenas with torch (device
  memory is torch's; the library never allocates), binds them, and exposes
  the entry points with tensors and Python callables.

Importing raises if the native library is missing: there is no CPU or
PyTorch fallback for any step of the path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzero_sm.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                      "(the ZeRO step has no fallback implementation)")

lib = ctypes.CDLL(LIB_PATH)

# ------------------------------------------------------------------ C ABI ----

ZERO_OK, ZERO_EINVAL, ZERO_ENOMEM, ZERO_ECUDA, ZERO_ESTATE, ZERO_ENOTIMPL, ZERO_EGUARD = range(7)
STATUS_NAMES = {0: "ZERO_OK", 1: "ZERO_EINVAL", 2: "ZERO_ENOMEM", 3: "ZERO_ECUDA", 4: "ZERO_ESTATE",
                5: "ZERO_ENOTIMPL", 6: "ZERO_EGUARD"}
ZERO_STAGE_DP, ZERO_STAGE_1, ZERO_STAGE_2, ZERO_STAGE_3 = 0, 1, 2, 3
ZERO_MAX_RANKS = 128
(ZERO_ARENA_STATES, ZERO_ARENA_PARAMS, ZERO_ARENA_GRADS, ZERO_ARENA_GRAD_SHARDS, ZERO_ARENA_GATHER,
 ZERO_ARENA_SCRATCH, ZERO_NUM_ARENAS) = range(7)
ZERO_OPT_KEEP_GRAD_SHARDS, ZERO_OPT_REPLICA_PAD, ZERO_OPT_BLOCKS_PER_SM, ZERO_OPT_TIMING, ZERO_OPT_KERNEL = 1, 2, 3, 4, 5
ZERO_KERNEL_AUTO, ZERO_KERNEL_REGISTER, ZERO_KERNEL_TMA, ZERO_KERNEL_BULK = 0, 1, 2, 3
ZERO_OPT_GRAD_BUFFERS = 6
ZERO_OPT_TMA_GROUPS = 7
ZERO_OPT_TMA_STAGES = 8
ZERO_OPT_TMA_CTAS_PER_SM = 9
ZERO_OPT_DTYPE = 10
ZERO_OPT_PIPELINE = 11
ZERO_OPT_PDL = 12
ZERO_OPT_TMA_TILE = 13
ZERO_OPT_TMA_WARPS = 14
ZERO_OPT_WAIT_LIMIT_NS = 15
ZERO_OPT_STORE_HINT = 16
ZERO_OPT_GUARD = 17
ZERO_OPT_NVTX = 18
ZERO_OPT_LAYERED = 19
ZERO_DTYPE_BF16, ZERO_DTYPE_F16 = 0, 1
(ZERO_VIEW_MASTER, ZERO_VIEW_EXP_AVG, ZERO_VIEW_EXP_AVG_SQ, ZERO_VIEW_PARAM, ZERO_VIEW_GRAD_SHARD,
 ZERO_VIEW_GRAD_BUF, ZERO_VIEW_GATHER) = range(7)


class zero_layout(ctypes.Structure):
    _fields_ = [("n_tensors", ctypes.c_int32), ("numel", ctypes.POINTER(ctypes.c_int64)),
                ("layer_id", ctypes.POINTER(ctypes.c_int32))]


class zero_adam_hparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double), ("beta2", ctypes.c_double),
                ("eps", ctypes.c_double), ("weight_decay", ctypes.c_double)]


class zero_sizes(ctypes.Structure):
    _fields_ = [("psi", ctypes.c_int64), ("psi_pad", ctypes.c_int64), ("shard", ctypes.c_int64),
                ("max_layer", ctypes.c_int64), ("replica_pitch", ctypes.c_int64),
                ("n_buckets", ctypes.c_int32), ("n_layers", ctypes.c_int32),
                ("arena_bytes", ctypes.c_int64 * ZERO_NUM_ARENAS)]


class zero_step_stats(ctypes.Structure):
    _fields_ = [("grad_norm", ctypes.c_double), ("nonfinite", ctypes.c_int64), ("step", ctypes.c_int64),
                ("comm_elems", ctypes.c_int64 * 3), ("clip_coef", ctypes.c_double), ("skipped", ctypes.c_int64)]


zero_grad_fn = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                ctypes.c_int64, ctypes.POINTER(ctypes.c_void_p), ctypes.c_void_p)
zero_gather_fn = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                  ctypes.c_int64, ctypes.POINTER(ctypes.c_void_p), ctypes.c_void_p)

_vp, _i32, _i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
_PTRS = ctypes.POINTER(ctypes.c_void_p)
_SIGS = {
    "zero_version": (_i32, []),
    "zero_init": (_i32, [ctypes.POINTER(zero_layout), _i32, _i32, _i64, ctypes.POINTER(_vp)]),
    "zero_set_option": (_i32, [_vp, _i32, _i64]),
    "zero_buffer_sizes": (_i32, [_vp, ctypes.POINTER(zero_sizes)]),
    "zero_tensor_offsets": (_i32, [_vp, ctypes.POINTER(_i64), _i32]),
    "zero_buckets": (_i32, [_vp, ctypes.POINTER(_i64), _i32, ctypes.POINTER(_i32)]),
    "zero_layers": (_i32, [_vp, ctypes.POINTER(_i64), _i32, ctypes.POINTER(_i32)]),
    "zero_bind": (_i32, [_vp, _PTRS]),
    "zero_set_hparams": (_i32, [_vp, ctypes.POINTER(zero_adam_hparams)]),
    "zero_load_master": (_i32, [_vp, _vp, _vp]),
    "zero_import_state": (_i32, [_vp, _vp, _vp, _vp, _i64, _i64, _vp]),
    "zero_get_step": (_i32, [_vp, ctypes.POINTER(_i64)]),
    "zero_set_step": (_i32, [_vp, _i64]),
    "zero_view": (_i32, [_vp, _i32, _i32, ctypes.POINTER(_vp), ctypes.POINTER(_i64)]),
    "zero_state_bytes": (_i32, [_vp, _i32, ctypes.POINTER(_i64)]),
    "zero_comm_elems": (_i32, [_vp, ctypes.POINTER(_i64)]),
    "zero_reduce_scatter": (_i32, [_vp, _i64, _i64, _PTRS, _vp]),
    "zero_all_reduce": (_i32, [_vp, _i64, _i64, _PTRS, _vp]),
    "zero_adam_shard": (_i32, [_vp, _i32, _i64, _vp]),
    "zero_all_gather": (_i32, [_vp, _i64, _i64, _PTRS, _vp]),
    "zero_step": (_i32, [_vp, zero_grad_fn, _vp, zero_gather_fn, _vp, _vp,
                         ctypes.POINTER(zero_step_stats)]),
    "zero_step_resident": (_i32, [_vp, _PTRS, zero_gather_fn, _vp, _vp,
                                  ctypes.POINTER(zero_step_stats)]),
    "zero_kernel_timing": (_i32, [_vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i64),
                                  ctypes.POINTER(ctypes.c_double)]),
    "zero_launch_count": (_i32, [_vp, ctypes.POINTER(_i64)]),
    "zero_set_clip": (_i32, [_vp, ctypes.c_double, _i32]),
    "zero_set_loss_scale": (_i32, [_vp, ctypes.c_double]),
    "zero_set_pipeline_streams": (_i32, [_vp, _vp, _vp]),
    "zero_fused_config": (_i32, [_vp, ctypes.POINTER(_i32), ctypes.POINTER(_i32), ctypes.POINTER(_i32)]),
    "zero_fused_tile": (_i32, [_vp, ctypes.POINTER(_i32)]),
    "zero_probe_pattern": (_i32, [_vp, _PTRS, _vp]),
    "zero_read_stats": (_i32, [_vp, _vp, ctypes.POINTER(zero_step_stats)]),
    "zero_check_guards": (_i32, [_vp, _vp, ctypes.POINTER(ctypes.c_int64)]),
    "zero_fused_step_static": (_i32, [_i32, _i64, _PTRS, _vp, _vp, _vp, _PTRS,
                                      ctypes.POINTER(zero_adam_hparams), _i64, _vp, _vp]),
    "zero_dist_init": (_i32, [ctypes.POINTER(zero_layout), _i32, _i32, _i32, ctypes.POINTER(_vp)]),
    "zero_dist_sizes": (_i32, [_vp, ctypes.POINTER(_i64), ctypes.POINTER(_i64)]),
    "zero_dist_tensor_offsets": (_i32, [_vp, ctypes.POINTER(_i64), _i32]),
    "zero_dist_bind": (_i32, [_vp, _PTRS]),
    "zero_dist_export": (_i32, [_vp, _vp]),
    "zero_dist_open_peers": (_i32, [_vp, _vp]),
    "zero_dist_set_hparams": (_i32, [_vp, ctypes.POINTER(zero_adam_hparams)]),
    "zero_dist_load_master": (_i32, [_vp, _vp, _vp]),
    "zero_dist_step": (_i32, [_vp, _vp]),
    "zero_dist_step_layer": (_i32, [_vp, _i32, _i32, _vp]),
    "zero_dist_adam_shard": (_i32, [_vp, _vp, _vp]),
    "zero_dist_read_partial": (_i32, [_vp, _vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i64),
                                      ctypes.POINTER(_i64)]),
    "zero_dist_view": (_i32, [_vp, _i32, ctypes.POINTER(_vp), ctypes.POINTER(_i64)]),
    "zero_dist_combine_partials": (_i32, [_i32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i64),
                                          ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i64)]),
    "zero_dist_last_error": (ctypes.c_char_p, [_vp]),
    "zero_dist_destroy": (None, [_vp]),
    "zero_last_error": (ctypes.c_char_p, [_vp]),
    "zero_destroy": (None, [_vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args
    globals()[_name] = _fn

__all__ = list(_SIGS) + ["ZeroOptimizer", "ZeroDist", "AdamHParams", "ZeroError", "lib", "LIB_PATH",
                         "options_from_config", "exchange_records", "rank_ordered_norm", "ordered_step"]
ZERO_DIST_ARENA_GRAD, ZERO_DIST_ARENA_PARAM, ZERO_DIST_ARENA_STATES, ZERO_DIST_ARENA_SCRATCH = 0, 1, 2, 3
ZERO_DIST_ARENA_GATHER = 4
ZERO_DIST_NUM_ARENAS = 5
ZERO_DIST_HANDLE_BYTES = 256


class ZeroError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def _ptr_array(ptrs: Sequence[int]):
    arr = (ctypes.c_void_p * len(ptrs))()
    for i, p in enumerate(ptrs):
        arr[i] = int(p)
    return arr


# ------------------------------------------------------------ Python API ----

@dataclass(frozen=True)
class AdamHParams:
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.0


def options_from_config(cfg: dict) -> dict:
    """``ZeroOptimizer`` keyword arguments from a DeepSpeed-style JSON config.

    Reads the keys of the fixed-buffer snippet in "ZeRO：从优化器状态到残差状态
    的显存优化" section 3.3 "CB" -- ``reduce_bucket_size``,
    ``allgather_bucket_size`` (elements) and ``communication_data_type`` --
    and the ZeRO ``stage``, either at the top level or under
    ``zero_optimization``; every other key is left alone.

    * ``reduce_bucket_size`` -> ``bucket_elems``, rounded up to a multiple of 8
      (the granule every interval starts on).
    * ``allgather_bucket_size``: the fused step gathers each interval in the
      pass that reduces and updates it, so the gather bucket is the reduce
      bucket; a different value raises ``ValueError`` instead of being
      silently ignored (alone, it sets the bucket).
    * ``communication_data_type``: "fp16" -> ZERO_DTYPE_F16, "bf16" /
      "bfloat16" -> ZERO_DTYPE_BF16; anything else raises ``ValueError``
      (the gradients and parameter copies are 16-bit here).
    * ``stage``: 1, 2 or 3; 0 (plain data parallelism) raises, as
      ``zero_init`` has no stage 0.
    """
    z = cfg.get("zero_optimization", {}) if isinstance(cfg.get("zero_optimization"), dict) else {}

    def key(name):
        return z[name] if name in z else cfg.get(name)

    out = {}
    stage = key("stage")
    if stage is not None:
        if int(stage) not in (1, 2, 3):
            raise ValueError(f"stage {stage}: the library implements ZeRO stages 1, 2 and 3")
        out["stage"] = int(stage)
    rb, ab = key("reduce_bucket_size"), key("allgather_bucket_size")
    if rb is not None and ab is not None and int(float(rb)) != int(float(ab)):
        raise ValueError(f"allgather_bucket_size {ab} != reduce_bucket_size {rb}: the fused step gathers "
                         "each interval as it reduces it, so the two buckets are one")
    bucket = rb if rb is not None else ab
    if bucket is not None:
        b = int(float(bucket))
        if b <= 0:
            raise ValueError(f"bucket size {bucket} must be positive")
        out["bucket_elems"] = (b + 7) // 8 * 8
    dt = key("communication_data_type")
    if dt is not None:
        name = str(dt).lower()
        if name in ("fp16", "float16", "half"):
            out["dtype"] = ZERO_DTYPE_F16
        elif name in ("bf16", "bfloat16"):
            out["dtype"] = ZERO_DTYPE_BF16
        else:
            raise ValueError(f"communication_data_type {dt!r}: gradients and parameters are bf16 or fp16")
    return out


class ZeroOptimizer:
    """One ZeRO context over ``n_ranks`` logical ranks on the current CUDA device.

    ``numel``/``layer_id``: the parameter list (flat order, non-decreasing
    layer ids).  ``bucket_elems`` defaults to one bucket spanning everything.
    Arenas are torch uint8 tensors owned by this object.
    """

    def __init__(self, numel: Sequence[int], layer_id: Sequence[int], n_ranks: int, stage: int,
                 bucket_elems: Optional[int] = None, hparams: AdamHParams = AdamHParams(),
                 keep_grad_shards: bool = True, replica_pad: int = 0, blocks_per_sm: int = 0,
                 kernel: int = ZERO_KERNEL_AUTO, grad_buffers: bool = True, tma_groups: int = 0,
                 tma_stages: int = 0, tma_ctas_per_sm: int = 0, dtype: int = ZERO_DTYPE_BF16,
                 pipeline: int = 0, tma_tile: int = 0, tma_warps: int = 0, guard: int = 0, device=None):
        import torch

        self._torch = torch
        self.n_ranks, self.stage = int(n_ranks), int(stage)
        n = len(numel)
        self._numel = (ctypes.c_int64 * n)(*[int(x) for x in numel])
        self._layer = (ctypes.c_int32 * n)(*[int(x) for x in layer_id])
        lay = zero_layout(n, self._numel, self._layer)
        # None / 0: the library's one bucket spanning the padded flat space
        self.bucket_elems = 0 if bucket_elems is None else int(bucket_elems)
        ctx = ctypes.c_void_p()
        st = zero_init(ctypes.byref(lay), self.n_ranks, self.stage, self.bucket_elems, ctypes.byref(ctx))
        if st != ZERO_OK:
            raise ZeroError(st, "zero_init", zero_last_error(None).decode())
        self.ctx = ctx
        if not keep_grad_shards:
            self._check(zero_set_option(ctx, ZERO_OPT_KEEP_GRAD_SHARDS, 0), "zero_set_option")
        if replica_pad:
            self._check(zero_set_option(ctx, ZERO_OPT_REPLICA_PAD, int(replica_pad)), "zero_set_option")
        if blocks_per_sm:
            self._check(zero_set_option(ctx, ZERO_OPT_BLOCKS_PER_SM, int(blocks_per_sm)), "zero_set_option")
        if kernel:
            self._check(zero_set_option(ctx, ZERO_OPT_KERNEL, int(kernel)), "zero_set_option")
        if not grad_buffers:
            self._check(zero_set_option(ctx, ZERO_OPT_GRAD_BUFFERS, 0), "zero_set_option")
        if tma_groups:
            self._check(zero_set_option(ctx, ZERO_OPT_TMA_GROUPS, int(tma_groups)), "zero_set_option")
        if tma_stages:
            self._check(zero_set_option(ctx, ZERO_OPT_TMA_STAGES, int(tma_stages)), "zero_set_option")
        if dtype != ZERO_DTYPE_BF16:
            self._check(zero_set_option(ctx, ZERO_OPT_DTYPE, int(dtype)), "zero_set_option")
        if tma_ctas_per_sm:
            self._check(zero_set_option(ctx, ZERO_OPT_TMA_CTAS_PER_SM, int(tma_ctas_per_sm)), "zero_set_option")
        if tma_tile:
            self._check(zero_set_option(ctx, ZERO_OPT_TMA_TILE, int(tma_tile)), "zero_set_option")
        if tma_warps:
            self._check(zero_set_option(ctx, ZERO_OPT_TMA_WARPS, int(tma_warps)), "zero_set_option")
        if pipeline:
            self._check(zero_set_option(ctx, ZERO_OPT_PIPELINE, int(pipeline)), "zero_set_option")
        if guard:
            self._check(zero_set_option(ctx, ZERO_OPT_GUARD, int(guard)), "zero_set_option")
        self.pipeline = int(pipeline)
        self.sizes = zero_sizes()
        self._check(zero_buffer_sizes(ctx, ctypes.byref(self.sizes)), "zero_buffer_sizes")
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.device = dev
        self.arenas = []
        ptrs = (ctypes.c_void_p * ZERO_NUM_ARENAS)()
        for k in range(ZERO_NUM_ARENAS):
            nb = int(self.sizes.arena_bytes[k])
            t = torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None
            self.arenas.append(t)
            ptrs[k] = t.data_ptr() if t is not None else None
        with torch.cuda.device(dev):
            self._check(zero_bind(ctx, ptrs), "zero_bind")
            if self.pipeline:
                # torch's pooled streams, which torch never destroys: its own
                # bookkeeping (pinned-memory blocks remember the streams they
                # were copied on) may refer to them after this context is gone
                self._cb_stream = torch.cuda.Stream(device=dev)
                self._k_stream = torch.cuda.Stream(device=dev, priority=-64) if self.pipeline == 2 else None
                self._check(zero_set_pipeline_streams(ctx, self._cb_stream.cuda_stream,
                                                      self._k_stream.cuda_stream if self._k_stream else None),
                            "zero_set_pipeline_streams")
        self.set_hparams(hparams)
        self._keep = []  # callbacks alive during a call

    # -- plumbing --
    def _check(self, st: int, where: str):
        if st != ZERO_OK:
            raise ZeroError(st, where, zero_last_error(self.ctx).decode())

    def _stream(self, stream=None) -> int:
        if stream is None:
            return self._torch.cuda.current_stream(self.device).cuda_stream
        return int(getattr(stream, "cuda_stream", stream))

    def close(self):
        if getattr(self, "ctx", None):
            zero_destroy(self.ctx)
            self.ctx = None
            self.arenas = []

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- plan --
    @property
    def psi(self) -> int:
        return int(self.sizes.psi)

    @property
    def psi_pad(self) -> int:
        return int(self.sizes.psi_pad)

    @property
    def shard(self) -> int:
        return int(self.sizes.shard)

    def offsets(self) -> List[int]:
        n = len(self._numel)
        out = (ctypes.c_int64 * n)()
        self._check(zero_tensor_offsets(self.ctx, out, n), "zero_tensor_offsets")
        return list(out)

    def buckets(self) -> List[tuple]:
        n = ctypes.c_int32()
        self._check(zero_buckets(self.ctx, None, 0, ctypes.byref(n)), "zero_buckets")
        out = (ctypes.c_int64 * (2 * n.value))()
        self._check(zero_buckets(self.ctx, out, n.value, ctypes.byref(n)), "zero_buckets")
        return [(out[2 * k], out[2 * k + 1]) for k in range(n.value)]

    def layers(self) -> List[tuple]:
        n = ctypes.c_int32()
        self._check(zero_layers(self.ctx, None, 0, ctypes.byref(n)), "zero_layers")
        out = (ctypes.c_int64 * (3 * n.value))()
        self._check(zero_layers(self.ctx, out, n.value, ctypes.byref(n)), "zero_layers")
        return [(int(out[3 * k]), out[3 * k + 1], out[3 * k + 2]) for k in range(n.value)]

    def state_bytes(self, rank: int) -> tuple:
        out = (ctypes.c_int64 * 3)()
        self._check(zero_state_bytes(self.ctx, rank, out), "zero_state_bytes")
        return tuple(out)

    def comm_elems(self) -> tuple:
        out = (ctypes.c_int64 * 3)()
        self._check(zero_comm_elems(self.ctx, out), "zero_comm_elems")
        return tuple(out)

    # -- views --
    def _tensor_at(self, ptr: int, n: int, dtype):
        torch = self._torch
        esize = torch.empty((), dtype=dtype).element_size()
        for a in self.arenas:
            if a is None:
                continue
            base = a.data_ptr()
            if base <= ptr and ptr + n * esize <= base + a.numel():
                off = ptr - base
                return a[off:off + n * esize].view(dtype)
        raise ValueError("pointer outside the bound arenas")

    def view(self, what: int, rank: int = 0):
        """torch view (uint16 for bf16 patterns, float32 for states) of a buffer."""
        torch = self._torch
        p = ctypes.c_void_p()
        n = ctypes.c_int64()
        self._check(zero_view(self.ctx, what, rank, ctypes.byref(p), ctypes.byref(n)), "zero_view")
        dtype = torch.float32 if what in (ZERO_VIEW_MASTER, ZERO_VIEW_EXP_AVG, ZERO_VIEW_EXP_AVG_SQ) else torch.int16
        return self._tensor_at(p.value, n.value, dtype)

    # -- state --
    def set_hparams(self, hp: AdamHParams):
        h = zero_adam_hparams(hp.lr, hp.beta1, hp.beta2, hp.eps, hp.weight_decay)
        self._check(zero_set_hparams(self.ctx, ctypes.byref(h)), "zero_set_hparams")
        self.hparams = hp

    def load_master(self, master=None, stream=None):
        """master: float32 CUDA tensor of psi_pad values, or None when the
        master view has been written in place."""
        ptr = None if master is None else master.data_ptr()
        if master is not None:
            assert master.dtype == self._torch.float32 and master.is_cuda and master.numel() == self.psi_pad
        self._check(zero_load_master(self.ctx, ptr, self._stream(stream)), "zero_load_master")

    def export_state(self) -> dict:
        """Copies of the flat fp32 state (psi_pad each) and the step counter."""
        return dict(master=self.view(ZERO_VIEW_MASTER).clone(), exp_avg=self.view(ZERO_VIEW_EXP_AVG).clone(),
                    exp_avg_sq=self.view(ZERO_VIEW_EXP_AVG_SQ).clone(), t=self.t)

    def import_state(self, state: dict, stream=None):
        """Resume from ``export_state()`` of any context over the same parameter list."""
        n = min(int(state["master"].numel()), self.psi_pad)
        self._check(zero_import_state(self.ctx, state["master"].data_ptr(), state["exp_avg"].data_ptr(),
                                      state["exp_avg_sq"].data_ptr(), n, int(state["t"]),
                                      self._stream(stream)), "zero_import_state")

    @property
    def t(self) -> int:
        v = ctypes.c_int64()
        self._check(zero_get_step(self.ctx, ctypes.byref(v)), "zero_get_step")
        return v.value

    @t.setter
    def t(self, value: int):
        self._check(zero_set_step(self.ctx, int(value)), "zero_set_step")

    # -- the step --
    @staticmethod
    def _stats_dict(s: zero_step_stats) -> dict:
        return dict(grad_norm=s.grad_norm, nonfinite=int(s.nonfinite), step=int(s.step),
                    comm_elems=tuple(s.comm_elems), clip_coef=s.clip_coef, skipped=bool(s.skipped))

    def _wrap_gather(self, gather_fn):
        if gather_fn is None:
            return zero_gather_fn()

        def cb(user, layer, lo, hi, bufs, stream):
            try:
                r = gather_fn(int(layer), int(lo), int(hi), [bufs[i] for i in range(self.n_ranks)], stream)
                return int(r or 0)
            except Exception as exc:  # a Python error must not unwind through C
                self._cb_error = exc
                return 1

        return zero_gather_fn(cb)

    def step(self, grad_fn: Optional[Callable] = None, gather_fn: Optional[Callable] = None,
             stats: bool = False, stream=None):
        """grad_fn(step, lo, hi, rank_buf_ptrs, stream) fills the ranks' buffers;
        gather_fn(layer, lo, hi, rank_buf_ptrs, stream) consumes a stage-3
        gathered layer.  Returns the statistics dict when ``stats``."""
        self._cb_error = None
        if grad_fn is None:
            gcb = zero_grad_fn()
        else:
            def g(user, t, lo, hi, bufs, stream_):
                try:
                    r = grad_fn(int(t), int(lo), int(hi), [bufs[i] for i in range(self.n_ranks)], stream_)
                    return int(r or 0)
                except Exception as exc:
                    self._cb_error = exc
                    return 1
            gcb = zero_grad_fn(g)
        acb = self._wrap_gather(gather_fn)
        out = zero_step_stats()
        st = zero_step(self.ctx, gcb, None, acb, None, self._stream(stream),
                       ctypes.byref(out) if stats else None)
        if self._cb_error is not None:
            raise self._cb_error
        self._check(st, "zero_step")
        return self._stats_dict(out) if stats else None

    def step_resident(self, rank_grads, gather_fn: Optional[Callable] = None, stats: bool = False,
                      stream=None):
        """rank_grads: N CUDA tensors (or one [N, psi_pad] tensor) of bf16 patterns."""
        ptrs = _ptr_array([g.data_ptr() for g in rank_grads])
        self._cb_error = None
        acb = self._wrap_gather(gather_fn)
        out = zero_step_stats()
        st = zero_step_resident(self.ctx, ptrs, acb, None, self._stream(stream),
                                ctypes.byref(out) if stats else None)
        if self._cb_error is not None:
            raise self._cb_error
        self._check(st, "zero_step_resident")
        return self._stats_dict(out) if stats else None

    def set_clip(self, max_norm: float = 0.0, skip_nonfinite: bool = False):
        """Global-norm clipping (max_norm > 0) and overflow skip; see zero_set_clip."""
        self._check(zero_set_clip(self.ctx, float(max_norm), 1 if skip_nonfinite else 0), "zero_set_clip")

    def set_loss_scale(self, scale: float):
        """The ranks' gradients are ``scale`` times the true ones; see zero_set_loss_scale."""
        self._check(zero_set_loss_scale(self.ctx, float(scale)), "zero_set_loss_scale")

    def fused_config(self) -> dict:
        k, g, s = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        self._check(zero_fused_config(self.ctx, ctypes.byref(k), ctypes.byref(g), ctypes.byref(s)),
                    "zero_fused_config")
        tile = ctypes.c_int32()
        self._check(zero_fused_tile(self.ctx, ctypes.byref(tile)), "zero_fused_tile")
        return dict(kernel={1: "register", 2: "tma", 3: "bulk"}[k.value], groups=g.value, stages=s.value,
                    tile=tile.value)

    def set_staged(self, tile: int = 0, warps: int = 0, stages: int = 0):
        """Tile, consumer warps and ring depth of the staged kernels (0 = the library's choice)."""
        self._check(zero_set_option(self.ctx, ZERO_OPT_TMA_TILE, int(tile)), "zero_set_option")
        self._check(zero_set_option(self.ctx, ZERO_OPT_TMA_WARPS, int(warps)), "zero_set_option")
        self._check(zero_set_option(self.ctx, ZERO_OPT_TMA_STAGES, int(stages)), "zero_set_option")

    def probe_pattern(self, rank_grads, stream=None):
        """The movement-only twin of the step's bulk-store launches (zero_probe_pattern)."""
        ptrs = (ctypes.c_void_p * self.n_ranks)(*[int(g.data_ptr()) for g in rank_grads])
        self._check(zero_probe_pattern(self.ctx, ptrs, self._stream(stream)), "zero_probe_pattern")

    def set_kernel(self, kernel: int):
        self._check(zero_set_option(self.ctx, ZERO_OPT_KERNEL, int(kernel)), "zero_set_option")

    def set_store_hint(self, on):
        """Bulk-store kernel: L2 evict-first hint on its stores (True / False;
        None = the library's choice; ZERO_OPT_STORE_HINT)."""
        v = -1 if on is None else (1 if on else 0)
        self._check(zero_set_option(self.ctx, ZERO_OPT_STORE_HINT, v), "zero_set_option")

    def set_wait_limit(self, ns: int):
        """Limit of the staged kernels' ring waits in ns (0: one non-blocking test; see ZERO_OPT_WAIT_LIMIT_NS)."""
        self._check(zero_set_option(self.ctx, ZERO_OPT_WAIT_LIMIT_NS, int(ns)), "zero_set_option")

    def set_pdl(self, on: bool):
        """Programmatic dependent launch between a callback-free step's fused launches (default on)."""
        self._check(zero_set_option(self.ctx, ZERO_OPT_PDL, 1 if on else 0), "zero_set_option")

    def set_timing(self, on: bool):
        self._check(zero_set_option(self.ctx, ZERO_OPT_TIMING, 1 if on else 0), "zero_set_option")

    def kernel_timing(self) -> dict:
        """Fused-kernel launches recorded since the last call: device ms,
        launch count, modelled bytes."""
        ms = ctypes.c_double()
        n = ctypes.c_int64()
        b = ctypes.c_double()
        self._check(zero_kernel_timing(self.ctx, ctypes.byref(ms), ctypes.byref(n), ctypes.byref(b)),
                    "zero_kernel_timing")
        return dict(ms=ms.value, launches=n.value, model_bytes=b.value)

    def launch_count(self) -> int:
        """Kernels this context has enqueued since it was created."""
        n = ctypes.c_int64()
        self._check(zero_launch_count(self.ctx, ctypes.byref(n)), "zero_launch_count")
        return n.value

    def check_guards(self, stream=None) -> dict:
        """Check the arenas' guard bytes (ZERO_OPT_GUARD; waits for the
        stream).  Returns {"changed": bytes, "arena": first's arena, "offset":
        its byte offset} ({0, -1, -1} when clean, "message" naming the row or
        tail otherwise); other failures raise."""
        out = (ctypes.c_int64 * 3)()
        st = zero_check_guards(self.ctx, self._stream(stream), out)
        if st not in (ZERO_OK, ZERO_EGUARD):
            self._check(st, "zero_check_guards")
        res = dict(changed=out[0], arena=out[1], offset=out[2])
        if st == ZERO_EGUARD:
            res["message"] = zero_last_error(self.ctx).decode()
        return res

    def set_layered(self, on: bool):
        """A callback-free stage-3 step as one launch over its layers (ZERO_OPT_LAYERED, default on)."""
        self._check(zero_set_option(self.ctx, ZERO_OPT_LAYERED, 1 if on else 0), "zero_set_option")

    def set_nvtx(self, on: bool):
        """NVTX ranges per step, launch and unfused call on the domain "zero_sm" (ZERO_OPT_NVTX)."""
        self._check(zero_set_option(self.ctx, ZERO_OPT_NVTX, 1 if on else 0), "zero_set_option")

    def set_guard(self, mode: int):
        """1: guards checked on request; 2: also after every step (ZERO_OPT_GUARD; the
        context must have been made with guard bytes)."""
        self._check(zero_set_option(self.ctx, ZERO_OPT_GUARD, int(mode)), "zero_set_option")

    def read_stats(self, stream=None) -> dict:
        out = zero_step_stats()
        self._check(zero_read_stats(self.ctx, self._stream(stream), ctypes.byref(out)), "zero_read_stats")
        return self._stats_dict(out)

    # -- unfused parts --
    def reduce_scatter(self, lo: int, hi: int, rank_grads: Optional[Sequence[int]] = None, stream=None):
        ptrs = None if rank_grads is None else _ptr_array(rank_grads)
        self._check(zero_reduce_scatter(self.ctx, lo, hi, ptrs, self._stream(stream)), "zero_reduce_scatter")

    def all_reduce(self, lo: int, hi: int, rank_grads: Optional[Sequence[int]] = None, stream=None):
        ptrs = None if rank_grads is None else _ptr_array(rank_grads)
        self._check(zero_all_reduce(self.ctx, lo, hi, ptrs, self._stream(stream)), "zero_all_reduce")

    def adam_shard(self, rank: int, t: int = 0, stream=None):
        """Adam on rank's shard (-1 = all) for step t; t = 0 takes the
        context's counter + 1 and, with rank = -1, advances the counter."""
        self._check(zero_adam_shard(self.ctx, rank, t, self._stream(stream)), "zero_adam_shard")

    def all_gather(self, lo: int, hi: int, rank_out: Optional[Sequence[int]] = None, stream=None):
        ptrs = None if rank_out is None else _ptr_array(rank_out)
        self._check(zero_all_gather(self.ctx, lo, hi, ptrs, self._stream(stream)), "zero_all_gather")


# ------------------------------------------------ one logical rank per GPU ----
#
# Host-side plumbing of the rank-per-GPU step (zero_dist_* in
# include/zero_sm.h): the exchange of the ranks' IPC records, the ordering
# of a step between the ranks (barriers around the kernel), and the global
# gradient norm from the ranks' partial sums.  These three helpers take the
# torch.distributed module and group, so that they run as written over gloo
# on CPU.

def exchange_records(dist, record: bytes, group=None) -> List[bytes]:
    """Every rank's export record, in rank order (all_gather_object)."""
    if len(record) != ZERO_DIST_HANDLE_BYTES:
        raise ValueError(f"a rank's record is {ZERO_DIST_HANDLE_BYTES} bytes, got {len(record)}")
    out: List = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, record, group=group)
    for q, r in enumerate(out):
        if not isinstance(r, (bytes, bytearray)) or len(r) != ZERO_DIST_HANDLE_BYTES:
            raise RuntimeError(f"rank {q} sent a malformed record")
    return [bytes(r) for r in out]


def rank_ordered_norm(dist, sumsq: float, nonfinite: int, group=None):
    """(global norm, non-finite count) from the ranks' partial sums, added in
    rank order 0..N-1 in binary64 (every rank gets the same bits)."""
    world = dist.get_world_size(group)
    parts: List = [None] * world
    dist.all_gather_object(parts, (float(sumsq), int(nonfinite)), group=group)
    sq = (ctypes.c_double * world)(*[p[0] for p in parts])
    nf = (ctypes.c_int64 * world)(*[p[1] for p in parts])
    norm, total = ctypes.c_double(), ctypes.c_int64()
    st = zero_dist_combine_partials(world, sq, nf, ctypes.byref(norm), ctypes.byref(total))
    if st != ZERO_OK:
        raise ZeroError(st, "zero_dist_combine_partials", "bad partials")
    return norm.value, total.value


def ordered_step(dist, sync: Callable[[], None], launch: Callable[[], None], group=None):
    """The cross-rank order of one step: this rank's pending work on its
    replicas done and every rank past that point (barrier) before the
    launch; the launch done and every rank past that point before return."""
    sync()
    dist.barrier(group=group)
    launch()
    sync()
    dist.barrier(group=group)


class ZeroDist:
    """Rank ``dist.get_rank(group)`` of a ZeRO step with one logical rank per
    GPU (stage 1, 2 or 3): allocates this rank's arenas with torch on ``device``,
    binds them, exchanges IPC records with the other ranks and opens theirs.
    Every call below is collective (every rank calls it, in the same order)."""

    def __init__(self, numel: Sequence[int], layer_id: Sequence[int], stage: int = ZERO_STAGE_2,
                 hparams: AdamHParams = AdamHParams(), group=None, device=None):
        import torch
        import torch.distributed as dist

        self._torch, self._dist, self.group = torch, dist, group
        self.world, self.rank = dist.get_world_size(group), dist.get_rank(group)
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        n = len(numel)
        self._numel = (ctypes.c_int64 * n)(*[int(x) for x in numel])
        self._layer = (ctypes.c_int32 * n)(*[int(x) for x in layer_id])
        lay = zero_layout(n, self._numel, self._layer)
        ctx = ctypes.c_void_p()
        st = zero_dist_init(ctypes.byref(lay), self.world, self.rank, int(stage), ctypes.byref(ctx))
        if st != ZERO_OK:
            raise ZeroError(st, "zero_dist_init", zero_dist_last_error(None).decode())
        self.ctx, self.stage = ctx, int(stage)
        plan = (ctypes.c_int64 * 3)()
        ab = (ctypes.c_int64 * ZERO_DIST_NUM_ARENAS)()
        self._check(zero_dist_sizes(ctx, plan, ab), "zero_dist_sizes")
        self.psi, self.psi_pad, self.shard = int(plan[0]), int(plan[1]), int(plan[2])
        self.arenas = [torch.empty(int(ab[k]), dtype=torch.uint8, device=self.device) if int(ab[k]) else None
                       for k in range(ZERO_DIST_NUM_ARENAS)]
        ptrs = (ctypes.c_void_p * ZERO_DIST_NUM_ARENAS)(*[a.data_ptr() if a is not None else None
                                                          for a in self.arenas])
        with torch.cuda.device(self.device):
            self._check(zero_dist_bind(ctx, ptrs), "zero_dist_bind")
            if self.world > 1:
                rec = ctypes.create_string_buffer(ZERO_DIST_HANDLE_BYTES)
                self._check(zero_dist_export(ctx, rec), "zero_dist_export")
                records = exchange_records(dist, rec.raw, group)
                allrec = ctypes.create_string_buffer(b"".join(records), ZERO_DIST_HANDLE_BYTES * self.world)
                self._check(zero_dist_open_peers(ctx, allrec), "zero_dist_open_peers")
                dist.barrier(group=group)  # every rank has mapped every other before anyone writes
        hp = zero_adam_hparams(hparams.lr, hparams.beta1, hparams.beta2, hparams.eps, hparams.weight_decay)
        self._check(zero_dist_set_hparams(ctx, ctypes.byref(hp)), "zero_dist_set_hparams")

    def _check(self, st: int, where: str):
        if st != ZERO_OK:
            raise ZeroError(st, where, zero_dist_last_error(self.ctx).decode())

    def _stream(self) -> int:
        return self._torch.cuda.current_stream(self.device).cuda_stream

    def _sync(self):
        self._torch.cuda.current_stream(self.device).synchronize()

    def offsets(self) -> List[int]:
        out = (ctypes.c_int64 * len(self._numel))()
        self._check(zero_dist_tensor_offsets(self.ctx, out, len(self._numel)), "zero_dist_tensor_offsets")
        return list(out)

    def view(self, what: int):
        """Tensor view of ZERO_VIEW_MASTER/_EXP_AVG/_EXP_AVG_SQ (the owned
        shard) or ZERO_VIEW_PARAM/ZERO_VIEW_GRAD_BUF (this rank's replicas)."""
        ptr, n = ctypes.c_void_p(), ctypes.c_int64()
        self._check(zero_dist_view(self.ctx, int(what), ctypes.byref(ptr), ctypes.byref(n)), "zero_dist_view")
        dt = self._torch.float32 if what in (ZERO_VIEW_MASTER, ZERO_VIEW_EXP_AVG, ZERO_VIEW_EXP_AVG_SQ) \
            else self._torch.int16
        item = 4 if dt == self._torch.float32 else 2
        arena = self.arenas[ZERO_DIST_ARENA_STATES if item == 4 else
                            ZERO_DIST_ARENA_PARAM if what == ZERO_VIEW_PARAM else
                            ZERO_DIST_ARENA_GATHER if what == ZERO_VIEW_GATHER else ZERO_DIST_ARENA_GRAD]
        off = (ptr.value - arena.data_ptr())
        return arena[off: off + item * n.value].view(dt)

    def load_master(self, master_full):
        """master_full: fp32 CUDA tensor of psi_pad values on this rank's device."""
        ordered_step(self._dist, self._sync,
                     lambda: self._check(zero_dist_load_master(self.ctx, master_full.data_ptr(), self._stream()),
                                         "zero_dist_load_master"), self.group)

    def step(self, stats: bool = False):
        """One step; with ``stats`` the global gradient norm and non-finite
        count (rank-ordered sum of the ranks' partials) and the step number."""
        ordered_step(self._dist, self._sync,
                     lambda: self._check(zero_dist_step(self.ctx, self._stream()), "zero_dist_step"), self.group)
        if not stats:
            return None
        sq, nf, t = ctypes.c_double(), ctypes.c_int64(), ctypes.c_int64()
        self._check(zero_dist_read_partial(self.ctx, self._stream(), ctypes.byref(sq), ctypes.byref(nf),
                                           ctypes.byref(t)), "zero_dist_read_partial")
        norm, nft = rank_ordered_norm(self._dist, sq.value, nf.value, self.group)
        return {"grad_norm": norm, "nonfinite": nft, "step": t.value}

    def step_layer(self, layer: int, last: bool, stats: bool = False):
        """Stage 3: one layer of the step (every rank's GRAD buffer holds the
        layer's gradient); ``last`` completes the step.  Statistics as step()."""
        ordered_step(self._dist, self._sync,
                     lambda: self._check(zero_dist_step_layer(self.ctx, int(layer), 1 if last else 0, self._stream()),
                                         "zero_dist_step_layer"), self.group)
        if not (stats and last):
            return None
        sq, nf, t = ctypes.c_double(), ctypes.c_int64(), ctypes.c_int64()
        self._check(zero_dist_read_partial(self.ctx, self._stream(), ctypes.byref(sq), ctypes.byref(nf),
                                           ctypes.byref(t)), "zero_dist_read_partial")
        norm, nft = rank_ordered_norm(self._dist, sq.value, nf.value, self.group)
        return {"grad_norm": norm, "nonfinite": nft, "step": t.value}

    def adam_shard(self, grad_shard):
        """Adam on the owned shard from an already reduced bf16 shard (S
        values): the update of a step whose collectives are NCCL calls."""
        self._check(zero_dist_adam_shard(self.ctx, grad_shard.data_ptr(), self._stream()), "zero_dist_adam_shard")

    def close(self):
        if getattr(self, "ctx", None):
            self._sync()
            self._dist.barrier(group=self.group)  # no peer still writes this rank's replicas
            zero_dist_destroy(self.ctx)
            self.ctx = None
