#!/usr/bin/env python
"""Throughput of the fused ZeRO optimizer step on B200.

Default workload: 24 transformer layers of hidden 2048 (1,208,598,528
params), N = 8 logical data-parallel ranks in one GPU's HBM, ZeRO-2 with the
fixed 200,000,000-element bucket schedule.  One step = one reduce-scatter +
Adam + all-gather pass over every parameter (7 fused kernel launches), the
8 gradient replicas already resident in HBM.

Prints one JSON line (rank 0): params/s for the whole job, the fused
kernel's achieved HBM bandwidth against the measured copy peak, the same
metric end to end through the C ABI with gradients copied from pinned host
memory, and the CPU oracle timed on a bounded sample of the same workload.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With --gpus N > 1 (launched by torch.distributed.run, one process per GPU)
every GPU runs its own full job (independent replicas of the workload; the
step has no inter-GPU exchange): weak scaling, time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "fused ZeRO step params/sec (1 B200); achieved HBM GB/s vs ~8 TB/s roofline"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
_CSRC = os.path.join(ROOT, "zero_sharded_optimizer_sm_b200", "csrc")
# the sources each fused kernel is compiled from (kernels.cuh holds only
# declarations and argument structs)
# the files a fused kernel's device code comes from (its traffic record is
# void once any of them changes)
KERNEL_SOURCES = {"tma": [os.path.join(_CSRC, f) for f in ("fused_tma.cu", "tma_pipe.cuh", "device_math.cuh",
                                                            "kernels.cuh")],
                  "register": [os.path.join(_CSRC, f) for f in ("kernels.cu", "device_math.cuh", "kernels.cuh")],
                  "bulk": [os.path.join(_CSRC, f) for f in ("fused_bulk.cu", "tma_pipe.cuh", "device_math.cuh",
                                                            "kernels.cuh", "layered_walk.cuh")]}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "fused_step_traffic.json")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) leg")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the CPU oracle leg")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--blocks-per-sm", type=int, default=0)
    ap.add_argument("--kernel", choices=("auto", "register", "tma", "bulk"), default="auto",
                    help="fused-step kernel (auto = the library's choice for this N)")
    ap.add_argument("--replica-pad", type=int, default=0)
    ap.add_argument("--tile", type=int, default=0, help="bulk-store kernel: elements per tile (0 = library's choice)")
    ap.add_argument("--warps", type=int, default=0, help="bulk-store kernel: consumer warps (0 = library's choice)")
    ap.add_argument("--ring", type=int, default=0, help="staged kernels: ring depth (0 = library's choice)")
    ap.add_argument("--no-pdl", action="store_true",
                    help="launch the step's fused kernels plainly (no programmatic dependent launch)")
    ap.add_argument("--no-layered", action="store_true",
                    help="stage 3: one launch per layer instead of the layered launch over all layers")
    ap.add_argument("--sweep", action="store_true",
                    help="flat-buffer sweep instead of the bench line: 1K..1G elements (x4) x N in "
                         "{2,4,8,16,64}, fused step vs unfused reduce-scatter + Adam + all-gather; one "
                         "JSON line per cell")
    ap.add_argument("--sweep-max-gb", type=float, default=150.0)
    ap.add_argument("--stages", action="store_true",
                    help="ZeRO-1/2/3 fused-step throughput on the 1.2B (N=8) and 85M (N=8) workloads "
                         "and ZeRO-3 on the 6.4B (N=64) workload; one JSON line per cell")
    ap.add_argument("--overlap", action="store_true",
                    help="ZERO_OPT_PIPELINE: step time with the gradient producer (the seeded "
                         "generator standing in for the backward) run in order vs one interval ahead "
                         "on the context's stream, on the 1.2B and 85M workloads; one JSON line per cell")
    ap.add_argument("--ref-sample-elems", type=int, default=0,
                    help="reference arm: elements per oracle step (0 = sized to about a minute)")
    ap.add_argument("--clip", type=float, default=0.0,
                    help="global-norm clip at this norm with the overflow skip on: the two-pass step "
                         "(reduce everything, read the norm, then Adam + broadcast)")
    ap.add_argument("--dtype", choices=("bf16", "f16"), default="bf16",
                    help="16-bit storage of gradients and parameters (f16: IEEE binary16 with loss scale 1024)")
    ap.add_argument("--stage", type=int, choices=(1, 2, 3), default=2,
                    help="ZeRO stage of the bench line (the benchmark is stage 2)")
    ap.add_argument("--rank-per-gpu", action="store_true",
                    help="ZeRO with one logical rank per GPU (zero_dist_*: N = --gpus processes, each GPU "
                         "holding its gradient and parameter replicas and its fp32 shard); one JSON line "
                         "from rank 0")
    ap.add_argument("--arm", choices=("fused", "nccl"), default="fused",
                    help="with --rank-per-gpu: the library's fused peer-memory kernel, or NCCL "
                         "reduce-scatter + the library's shard update + NCCL all-gather")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="gpt-1.2b",
                    help="gpt-1.2b: the benchmark workload; flat-32m: a 33.5M-param flat buffer, "
                         "N = 8, one bucket (2 GB on the device); flat-8m-n64: 8.4M params, N = 64 "
                         "(3 GB on the device); the small ones are for profiler captures")
    return ap.parse_args(argv)


# ------------------------------------------------------------ environment ----

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import datetime

    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(value: float, dist, device) -> float:
    """Largest value over all ranks (every rank calls this the same number of times)."""
    if dist is None:
        return value
    import torch

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist):
    if dist is not None:
        dist.barrier()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_sources_digest(kernel: str) -> str:
    h = hashlib.sha256()
    for path in KERNEL_SOURCES[kernel]:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_for_current_kernel(kernel: str, key: str, elems_per_launch: float):
    """Per-launch DRAM bytes from the committed ncu summary for this kernel
    configuration, scaled to this launch size, or None when the kernel's
    sources changed since the capture (or there is no capture)."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)[key]
        if rec.get("sources_sha256") != kernel_sources_digest(kernel):
            return None
        return rec["dram_bytes_per_elem"] * elems_per_launch
    except Exception:
        return None


def nvsmi_index(device_index: int) -> int:
    """nvidia-smi's index of CUDA device `device_index`: the two numberings
    differ when CUDA_VISIBLE_DEVICES selects or reorders devices, so the GPU
    is matched by its PCI domain, bus and device numbers (the CUDA index when
    nothing matches)."""
    try:
        import torch

        p = torch.cuda.get_device_properties(device_index)
        want = (int(p.pci_domain_id), int(p.pci_bus_id), int(p.pci_device_id))
        out = subprocess.run(["nvidia-smi", "--query-gpu=index,pci.bus_id", "--format=csv,noheader"],
                             capture_output=True, text=True, timeout=30).stdout
        for line in out.splitlines():
            idx, bus = [x.strip() for x in line.split(",")[:2]]
            dom, b, dev_fn = bus.split(":")
            if (int(dom, 16), int(b, 16), int(dev_fn.split(".")[0], 16)) == want:
                return int(idx)
    except Exception:
        pass
    return device_index


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "nvidia_smi_index": self.gpu}


# ---------------------------------------------------------------- workload ----

def _gpt_1p2b():
    from synth import workloads as W

    return W.gpt_1p2b_n8()


def _gpt_85m():
    from synth import workloads as W

    w = W.gpt_85m_n8()
    w.bucket_elems = 20_000_000
    return w


def _flat_32m():
    from synth import workloads as W

    w = W.flat_sweep(1 << 25, 8)
    w.bucket_elems = 1 << 25
    return w


def _flat_8m_n64():
    from synth import workloads as W

    w = W.flat_sweep(1 << 23, 64)
    w.bucket_elems = 1 << 23
    return w


WORKLOADS = {"gpt-1.2b": _gpt_1p2b, "gpt-85m": _gpt_85m, "flat-32m": _flat_32m, "flat-8m-n64": _flat_8m_n64}
_ARGS = None


def workload():
    return WORKLOADS[_ARGS.workload if _ARGS is not None else "gpt-1.2b"]()


def fused_kernel_name(fc: dict, n_ranks: int, layered: bool = False) -> str:
    """The fused kernel a context launches, from its zero_fused_config
    (layered: a callback-free stage-3 step as one launch over its layers)."""
    if fc["kernel"] == "bulk":
        if n_ranks > 16:
            return "fused_bulk_chunked_kernel"
        return "fused_bulk_layered_kernel" if layered else "fused_bulk_kernel"
    if fc["kernel"] != "tma":
        return "fused_step_kernel"
    if n_ranks > 16:
        return "fused_step_chunked_kernel"
    return "fused_step_tma_wide_kernel" if fc["groups"] == 3 else "fused_step_tma_kernel"


def bench_stage() -> int:
    return _ARGS.stage if _ARGS is not None else 2


def oracle_stage(stage: int) -> int:
    import oracle

    return {1: oracle.STAGE_Z1, 2: oracle.STAGE_Z2, 3: oracle.STAGE_Z3}[stage]


def usable_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


_SLICE_BARRIER = None


def _slice_init(barrier):
    global _SLICE_BARRIER
    _SLICE_BARRIER = barrier


def _oracle_slice(job):
    """One worker of the parallel oracle timing (a spawned process): literal
    steps of the oracle on flat elements [a, a + n) of the workload (their
    values are the workload's: every input is drawn by its flat index), timed
    after all workers have their inputs."""
    import numpy as np

    import oracle
    import synth
    from synth import workloads as W

    w, stage, a, n, warmup, steps = job
    p = oracle.plan([n], [0], w.n_ranks, w.bucket_elems or (1 << 40))
    m0 = np.zeros(p.psi_pad, np.float32)
    m0[:n] = synth.host_f32(W.master_base(w), a, n, W.MASTER_DIST)
    grads = []
    for r in range(w.n_ranks):
        g = np.zeros(p.psi_pad, np.uint16)
        g[:n] = synth.host_bf16(W.grad_base(w, 1, r), a, n, w.grad_dist)
        grads.append(g)
    st = oracle_stage(stage)
    ranks = oracle.init_states(p, st, m0)
    hp = oracle.AdamHP(**w.hyper.__dict__)
    t = 0
    for _ in range(warmup):
        t += 1
        oracle.step(p, st, ranks, lambda t_, r: grads[r], t, hp)
    if _SLICE_BARRIER is not None:
        _SLICE_BARRIER.wait()
    t0 = time.perf_counter()
    for _ in range(steps):
        t += 1
        oracle.step(p, st, ranks, lambda t_, r: grads[r], t, hp)
    return n, time.perf_counter() - t0


def oracle_parallel(w, stage: int, total: int, warmup: int, steps: int, procs: int):
    """The oracle as it stands over `total` leading elements, split into
    `procs` contiguous slices timed in as many spawned processes, released
    together by a barrier.  Returns (params/s, seconds per step of the
    slowest slice, elements)."""
    import multiprocessing as mp

    procs = max(1, min(procs, total // 8))
    per = max(8, total // procs // 8 * 8)
    jobs = [(w, stage, k * per, per, warmup, steps) for k in range(procs)]
    ctx = mp.get_context("spawn")
    if procs == 1:
        res = [_oracle_slice(jobs[0])]
    else:
        barrier = ctx.Manager().Barrier(procs)
        with ctx.Pool(procs, initializer=_slice_init, initargs=(barrier,)) as pool:
            res = pool.map(_oracle_slice, jobs, chunksize=1)
    elems = sum(n for n, _ in res)
    worst = max(dt for _, dt in res)
    return elems * steps / worst, worst / steps, elems


def cpu_baseline(w, steps: int = 2, stage: int = 2) -> dict:
    """The oracle, as it stands, on a bounded sample of the workload: the
    first transformer layer's elements (50,358,272 params for the 1.2B list),
    the same N and bucket size, ``steps`` literal steps of the bench's stage
    -- on one core, and split over every usable core."""
    k = w.layer_id.count(0)
    total = int(sum(w.numel[:k])) // 8 * 8
    one, one_s, _ = oracle_parallel(w, stage, total, 0, steps, 1)
    cores = usable_cores()
    allc, all_s, elems = oracle_parallel(w, stage, total, 1, steps, cores)
    return {"value": allc, "unit": "params/s", "cores": cores, "kind": "oracle",
            "sample": f"first layer of the workload ({elems} params, N={w.n_ranks}) split into {cores} "
                      f"contiguous slices, one spawned process per usable core, {steps} literal "
                      f"ZeRO-{stage} steps each after one warm-up, timed together; C+numpy oracle, "
                      f"input generation untimed",
            "single_core": {"value": one, "unit": "params/s", "cores": 1, "seconds_per_step": one_s,
                            "sample": f"the same {total} params in one process, {steps} steps"}}


# -------------------------------------------------------------------- ours ----

def run_ours(args, world, rank, local):
    import torch

    import synth
    import zero_sharded_optimizer_sm_b200 as z
    from synth import workloads as W

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    w = workload()
    stream = torch.cuda.current_stream(dev)
    s = stream.cuda_stream
    stage = bench_stage()
    opt = z.ZeroOptimizer(w.numel, w.layer_id, w.n_ranks, stage, bucket_elems=w.bucket_elems,
                          hparams=z.AdamHParams(**w.hyper.__dict__), keep_grad_shards=args.clip > 0,
                          replica_pad=args.replica_pad, blocks_per_sm=args.blocks_per_sm,
                          kernel={"auto": 0, "register": 1, "tma": 2, "bulk": 3}[args.kernel], pipeline=True,
                          tma_tile=args.tile, tma_warps=args.warps, tma_stages=args.ring,
                          dtype=z.ZERO_DTYPE_F16 if args.dtype == "f16" else z.ZERO_DTYPE_BF16, device=dev)
    if args.dtype == "f16":
        opt.set_loss_scale(1024.0)
        w.grad_dist = synth.Dist(w.grad_dist.kind, w.grad_dist.width * 1024.0, w.grad_dist.zero_mod)
    fill16 = synth.dev_f16 if args.dtype == "f16" else synth.dev_bf16
    if args.clip > 0:
        opt.set_clip(args.clip, True)
    offsets = opt.offsets()
    mv = opt.view(z.ZERO_VIEW_MASTER)
    b = W.master_base(w)
    for off, n in zip(offsets, w.numel):
        synth.dev_f32(b, off, n, W.MASTER_DIST, mv.data_ptr() + 4 * off, s)
    opt.load_master(None)
    # the step's inputs: N full gradient replicas resident in HBM (19.3 GB)
    reps = torch.empty((w.n_ranks, opt.psi_pad), dtype=torch.int16, device=dev)
    for r in range(w.n_ranks):
        gb = W.grad_base(w, 1, r)
        for off, n in zip(offsets, w.numel):
            fill16(gb, off, n, w.grad_dist, reps[r].data_ptr() + 2 * off, s)
    rep_list = list(reps)
    opt.set_pdl(not args.no_pdl)
    opt.set_layered(not args.no_layered)
    torch.cuda.synchronize(dev)
    # model bytes of one step's fused launches, from the library's own record
    opt.set_timing(True)
    opt.kernel_timing()
    opt.step_resident(rep_list)
    torch.cuda.synchronize(dev)
    rec = opt.kernel_timing()
    model_bytes_per_step, per_step_launches = rec["model_bytes"], rec["launches"]
    opt.set_timing(False)
    for _ in range(args.warmup):
        opt.step_resident(rep_list)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(nvsmi_index(local))
    sampler.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(dist)
    torch.cuda.synchronize(dev)
    n0 = opt.launch_count()
    e0.record(stream)
    for _ in range(args.steps):
        opt.step_resident(rep_list)
    e1.record(stream)
    region_launches = opt.launch_count() - n0
    torch.cuda.synchronize(dev)
    barrier(dist)
    clocks = sampler.stop()
    ms_local = e0.elapsed_time(e1)
    ms = max_over_ranks(ms_local, dist, dev)
    stats = opt.read_stats()
    value = world * w.psi * args.steps / (ms / 1e3)
    # The fused kernels run back to back on this stream (with programmatic
    # dependent launch each starts as the one before finishes); beside them a
    # step runs only the two one-thread kernels that form and commit its
    # device-held counter and scalars (a few microseconds in a step of
    # milliseconds).  The fused kernel's average launch duration is taken as
    # the region's time over the fused launches, which charges it those two.
    intervals = len(opt.buckets()) if stage != 3 else len(opt.layers())
    launches = args.steps * per_step_launches
    kernel_ms = ms_local / launches
    achieved = model_bytes_per_step * args.steps / (ms_local / 1e3) / 1e9
    # the same kernel timed launch by launch (CUDA events around each launch,
    # which also turns programmatic dependent launch off)
    iso_steps = 20
    opt.set_timing(True)
    opt.kernel_timing()
    for _ in range(iso_steps):
        opt.step_resident(rep_list)
    torch.cuda.synchronize(dev)
    kt = opt.kernel_timing()
    opt.set_timing(False)
    kernel_ms_isolated = kt["ms"] / kt["launches"] if kt["launches"] else None
    peak, peak_kind = measured_peaks()
    pattern = pattern_ceiling(opt, rep_list, stream, model_bytes_per_step, args) if args.clip <= 0 else None
    copy_gbs = same_box_copy(dev)
    elems_per_launch = w.psi / intervals
    fc = opt.fused_config()
    ckey = f"stage{stage}_N{w.n_ranks}_{fc['kernel']}" + (f"_g{fc['groups']}_s{fc['stages']}" if fc["kernel"] == "tma" else
                                                          f"_t{fc['tile']}_w{fc['groups']}_s{fc['stages']}"
                                                          if fc["kernel"] == "bulk" else "")
    traffic = traffic_for_current_kernel(fc["kernel"], ckey, elems_per_launch) if args.clip <= 0 else None

    # end to end through the C ABI: every bucket's N gradient slices copied
    # from pinned host memory into the fixed-size buffer, then the fused
    # launch; the step's statistics read back to the host.
    e2e = None
    if not args.no_e2e:
        max_bucket = max(hi - lo for lo, hi in opt.buckets())
        if stage == 3:
            max_bucket = max(hi - lo for _, lo, hi in opt.layers())
        host = torch.empty((w.n_ranks, max_bucket), dtype=torch.int16, pin_memory=True)
        host.copy_(reps[:, :max_bucket])
        h2d = 0

        def grad_fn(t, lo, hi, bufs, stream_):
            nonlocal h2d
            with torch.cuda.stream(torch.cuda.ExternalStream(stream_) if stream_ else stream):
                for r, ptr in enumerate(bufs):
                    dst = opt._tensor_at(ptr, hi - lo, torch.int16)
                    dst.copy_(host[r, : hi - lo], non_blocking=True)
                    h2d += 2 * (hi - lo)
            return 0

        del reps, rep_list
        torch.cuda.empty_cache()
        opt.step(grad_fn, stats=True)  # warm-up of the host path
        h2d = 0
        barrier(dist)
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        for _ in range(args.e2e_steps):
            opt.step(grad_fn, stats=True)
        e2e_s = time.perf_counter() - t0
        barrier(dist)
        e2e_s = max_over_ranks(e2e_s, dist, dev)
        e2e = {"value": world * w.psi * args.e2e_steps / e2e_s, "unit": "params/s",
               "h2d_bytes_per_step": h2d // args.e2e_steps, "d2h_bytes_per_step": 16,
               "steps": args.e2e_steps,
               "how": "zero_step through the C ABI with ZERO_OPT_PIPELINE; grad_fn copies each "
                      "bucket's N gradient slices from pinned host memory into one of the two "
                      "200M-element buffers, one bucket ahead of the fused kernel; only the step's "
                      "16-byte statistics (sum of squares, non-finite count) come back to the host "
                      "each step -- the updated parameters stay on the device for the next forward"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, stage=stage)
    out = {
        "metric": METRIC,
        "value": value,
        "unit": "params/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp32",
        "data": "synthetic (seeded counter-hash gradients and weights, no dataset)",
        "config": {"workload": w.name, "params": w.psi, "n_ranks": w.n_ranks, "stage": stage,
                   "step": (f"two-pass (clip at {args.clip}, overflow skip)" if args.clip > 0 else "fused"),
                   "bucket_elems": w.bucket_elems, "buckets": len(opt.buckets()), "launches_per_step": intervals,
                   "storage": ("binary16 grads/params (loss scale 1024)" if args.dtype == "f16" else "bf16 grads/params")
                              + ", fp32 master/m/v",
                   "l2": f"inputs larger than L2: {(4 * w.n_ranks + 24) * w.psi / 1e9:.1f} GB moved "
                         f"per step vs 126 MB L2",
                   "parallelism": f"{w.n_ranks} logical ranks per GPU x {world} GPU replicas",
                   "kernel": args.kernel, "fused_config": fc, "pdl": not args.no_pdl,
                   "layered": args.stage == 3 and not args.no_layered},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": (achieved / peak) if achieved else None, "traffic": traffic,
                     "peak_kind": f"{peak_kind} copy peak",
                     "kernel": (fused_kernel_name(fc, w.n_ranks, args.stage == 3 and not args.no_layered)
                                if args.clip <= 0
                                else "reduce_kernel + adam_bcast_kernel (two-pass step)"),
                     "kernel_config": ckey,
                     "kernel_ms_per_launch": kernel_ms, "launches": launches,
                     "model_bytes_per_launch": model_bytes_per_step / per_step_launches,
                     "achieved_how": "model bytes of the timed launches / CUDA-event time of the timed "
                                     "region (the fused launches back to back"
                                     + ("" if args.no_pdl else ", programmatic dependent launch")
                                     + "; the region also holds two one-thread step-state kernels a step)",
                     "kernel_ms_per_launch_isolated": kernel_ms_isolated,
                     "achieved_isolated": (kt["model_bytes"] / kt["launches"] / (kernel_ms_isolated / 1e3) / 1e9
                                           if kernel_ms_isolated else None),
                     "frac_of_nominal_8tbs": (achieved / NOMINAL_HBM_GBS) if achieved else None,
                     "pattern_peak": pattern["GBps"] if pattern else None,
                     "frac_of_pattern": (achieved / pattern["GBps"]) if pattern else None,
                     "pattern_how": pattern["how"] if pattern else None,
                     "pattern_by_config": pattern["by_config"] if pattern else None,
                     "copy_same_box": copy_gbs,
                     "frac_of_copy_same_box": (achieved / copy_gbs) if copy_gbs else None},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": region_launches,
        "clocks": clocks,
        "grad_norm_last_step": stats["grad_norm"],
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    opt.close()
    if dist is not None:
        dist.destroy_process_group()


def pattern_ceiling(opt, rep_list, stream, model_bytes_per_step, args, steps=None):
    """The step's own traffic pattern with no arithmetic: the movement-only
    twin of the bulk-store kernel (zero_probe_pattern) over the same
    intervals, in the same launch chaining, timed like the step, in the
    step's configuration and in four others (tiles of 1024 and 2048
    elements, 8 or 16 consumer warps, 2-4 stages).  The twin's pace depends
    on its configuration -- without arithmetic its copies bunch up -- so the
    ceiling is the fastest of them.  GB/s of the step's byte model over the
    twin's time; None where no twin exists."""
    import torch

    import zero_sharded_optimizer_sm_b200 as z

    steps = steps or max(20, min(args.steps, 60))
    fc = opt.fused_config()
    own = (fc["tile"], fc["groups"], fc["stages"]) if fc["kernel"] == "bulk" else None
    configs = [own] if own else []
    configs += [c for c in ((1024, 8, 3), (1024, 8, 4), (2048, 8, 2), (2048, 16, 2)) if c != own]
    results = {}
    for cfg in configs:
        try:
            opt.set_staged(*cfg)
            for _ in range(3):
                opt.probe_pattern(rep_list)
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(steps):
                opt.probe_pattern(rep_list)
            e1.record(stream)
            torch.cuda.synchronize()
        except z.ZeroError:
            continue
        results["x".join(map(str, cfg))] = model_bytes_per_step / (e0.elapsed_time(e1) / steps / 1e3) / 1e9
    opt.set_staged(args.tile, args.warps, args.ring)  # the step's own configuration again
    if not results:
        return None
    best = max(results, key=results.get)
    return {"GBps": results[best], "by_config": results, "best_config": best,
            "own_config": "x".join(map(str, own)) if own else None,
            "how": "zero_probe_pattern: the bulk-store kernel's movement-only twin (same bulk loads, shared-memory "
                   "traffic and bulk stores, no reduction or Adam) over the step's intervals with the same launch "
                   "chaining, in the step's configuration and four others (tile x consumer warps x stages); the "
                   "fastest, as the step's byte model over its CUDA-event time"}


def same_box_copy(dev, gib: int = 4, reps: int = 20):
    """Device-to-device copy of a 4 GiB buffer on this GPU (torch's copy
    kernel), read + write bytes over CUDA-event time: the plain-copy ceiling
    of the box the step ran on."""
    import torch

    try:
        a = torch.empty(gib << 30, dtype=torch.uint8, device=dev)
        b = torch.empty_like(a)
    except RuntimeError:
        return None
    for _ in range(3):
        b.copy_(a)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        b.copy_(a)
    e1.record()
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / reps
    del a, b
    torch.cuda.empty_cache()
    return 2 * (gib << 30) / (ms / 1e3) / 1e9


# ------------------------------------------------------------------- sweep ----

def run_sweep(args):
    """Flat-buffer ZeRO-2 sweep: for each (E, N) cell, the fused step (the
    library's kernel choice) and the unfused reduce-scatter -> Adam ->
    all-gather sequence over the same resident replicas, timed with CUDA
    events over enough repetitions for ~50 ms.  GB/s are reported against the
    (4N+24) B/element model of the fused step; the unfused path's own
    (4N+32) B/element traffic is reported beside it.  Cells whose working set
    fits in L2 (126 MB) measure L2 and launch latency, and are labelled so."""
    import torch

    import synth
    import zero_sharded_optimizer_sm_b200 as z
    from synth import workloads as W

    torch.cuda.set_device(0)
    s = torch.cuda.current_stream().cuda_stream
    for n_ranks in W.SWEEP_RANKS:
        for elems in W.SWEEP_ELEMS:
            resident = (4 * n_ranks + 14) * elems  # replicas in, params out, states, grad shard
            cell = {"sweep": "flat-zero2", "elems": elems, "n_ranks": n_ranks}
            if resident > args.sweep_max_gb * 1e9:
                cell["skipped"] = f"exceeds HBM budget ({resident / 1e9:.0f} GB)"
                print(json.dumps(cell), flush=True)
                continue
            w = W.flat_sweep(elems, n_ranks)
            reps = None
            for name in ("fused", "unfused"):
                # the fused step keeps the reduced gradient in registers (the
                # 4N+24 model); the unfused path needs the shard arena
                opt = z.ZeroOptimizer(w.numel, w.layer_id, n_ranks, z.ZERO_STAGE_2,
                                      keep_grad_shards=(name == "unfused"), grad_buffers=False,
                                      kernel={"auto": 0, "register": 1, "tma": 2, "bulk": 3}[args.kernel])
                mv = opt.view(z.ZERO_VIEW_MASTER)
                synth.dev_f32(W.master_base(w), 0, elems, W.MASTER_DIST, mv.data_ptr(), s)
                opt.load_master(None)
                if reps is None:
                    reps = torch.empty((n_ranks, opt.psi_pad), dtype=torch.int16, device="cuda")
                    for r in range(n_ranks):
                        synth.dev_bf16(W.grad_base(w, 1, r), 0, elems, w.grad_dist, reps[r].data_ptr(), s)
                rl = list(reps)
                ptrs = [t.data_ptr() for t in rl]
                psi_pad = opt.psi_pad
                model = (4 * n_ranks + 24) * psi_pad
                reps_n = int(min(2000, max(3, 5e-2 / max(model / 6.0e12, 3e-6))))
                if name == "fused":
                    cell["fused_config"] = opt.fused_config()

                    def fn(opt=opt, rl=rl):
                        opt.step_resident(rl)
                else:
                    def fn(opt=opt, ptrs=ptrs, t=[0]):
                        t[0] += 1
                        opt.reduce_scatter(0, opt.psi_pad, ptrs)
                        opt.adam_shard(-1, t[0])
                        opt.all_gather(0, opt.psi_pad)
                for _ in range(3):
                    fn()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize()
                e0.record()
                for _ in range(reps_n):
                    fn()
                e1.record()
                torch.cuda.synchronize()
                ms = e0.elapsed_time(e1) / reps_n
                cell[f"{name}_us"] = ms * 1e3
                cell[f"{name}_gbs_model_4n24"] = model / (ms / 1e3) / 1e9
                opt.close()
                del opt, mv, fn
                torch.cuda.empty_cache()
            cell["unfused_gbs_own_4n32"] = (4 * n_ranks + 32) * psi_pad / (cell["unfused_us"] / 1e6) / 1e9
            cell["fused_speedup"] = cell["unfused_us"] / cell["fused_us"]
            cell["regime"] = "L2-resident / launch-bound" if model < 126e6 * 2 else "HBM"
            cell["reps"] = reps_n
            print(json.dumps(cell), flush=True)
            del reps, rl
            torch.cuda.empty_cache()


# ------------------------------------------------------------------ stages ----

def run_stages(args):
    """Fused-step throughput per ZeRO stage.  Byte models per element: ZeRO-1
    6N+24 (the all-reduce result is written back to the N replicas), ZeRO-2
    4N+24, ZeRO-3 4N+26 (the parameter shard besides the N temporary layer
    buffers).  Where the N full replicas fit in HBM they are resident and the
    step is timed with CUDA events; the 6.4B / N = 64 ZeRO-3 workload keeps one
    layer's 64 replicas live (filled between launches by the generator), so
    only the library's kernels are timed there (ZERO_OPT_TIMING)."""
    import torch

    import synth
    import zero_sharded_optimizer_sm_b200 as z
    from synth import workloads as W

    torch.cuda.set_device(0)
    s = torch.cuda.current_stream().cuda_stream
    kern = {"auto": 0, "register": 1, "tma": 2, "bulk": 3}[args.kernel]

    def master_fill(opt, w):
        mv = opt.view(z.ZERO_VIEW_MASTER)
        for off, n in zip(opt.offsets(), w.numel):
            synth.dev_f32(W.master_base(w), off, n, W.MASTER_DIST, mv.data_ptr() + 4 * off, s)
        opt.load_master(None)

    for w in (W.gpt_1p2b_n8(), W.gpt_85m_n8()):
        reps = None
        for stage in (1, 2, 3):
            opt = z.ZeroOptimizer(w.numel, w.layer_id, w.n_ranks, stage,
                                  bucket_elems=w.bucket_elems or 200_000_000, hparams=z.AdamHParams(),
                                  keep_grad_shards=False, grad_buffers=False, kernel=kern)
            master_fill(opt, w)
            if reps is None:
                reps = torch.empty((w.n_ranks, opt.psi_pad), dtype=torch.int16, device="cuda")
                for r in range(w.n_ranks):
                    for off, n in zip(opt.offsets(), w.numel):
                        synth.dev_bf16(W.grad_base(w, 1, r), off, n, w.grad_dist, reps[r].data_ptr() + 2 * off, s)
            rl = list(reps)
            opt.set_pdl(not args.no_pdl)
            opt.set_layered(not args.no_layered)
            for _ in range(3):
                opt.step_resident(rl)
            steps = max(5, int(2e9 / ((4 * w.n_ranks + 24) * w.psi)) + 5)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record()
            for _ in range(steps):
                opt.step_resident(rl)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / steps
            # the kernels launch by launch (events around each: no programmatic launch)
            opt.set_timing(True)
            opt.kernel_timing()
            for _ in range(steps):
                opt.step_resident(rl)
            torch.cuda.synchronize()
            kt = opt.kernel_timing()
            opt.set_timing(False)
            per = {1: 6 * w.n_ranks + 24, 2: 4 * w.n_ranks + 24, 3: 4 * w.n_ranks + 26}[stage]
            print(json.dumps({"stages": w.name, "stage": stage, "n_ranks": w.n_ranks, "params": w.psi,
                              "ms_per_step": ms, "params_per_s": w.psi / (ms / 1e3),
                              "bytes_per_elem_model": per,
                              "step_gbs_model": per * w.psi / (ms / 1e3) / 1e9,
                              "kernel_gbs_model_isolated": kt["model_bytes"] / (kt["ms"] / 1e3) / 1e9,
                              "pdl": not args.no_pdl, "layered": stage == 3 and not args.no_layered,
                              "launches_per_step": kt["launches"] // steps,
                              "fused_config": opt.fused_config(), "steps": steps}), flush=True)
            opt.close()
            del opt
            torch.cuda.empty_cache()
        del reps, rl
        torch.cuda.empty_cache()

    w = W.gpt_6p4b_n64()
    free, _ = torch.cuda.mem_get_info()
    need = 12 * w.psi + 2 * w.psi + 4 * 64 * 201_379_840
    if free < need + (4 << 30):
        print(json.dumps({"stages": w.name, "skipped": f"needs {need / 1e9:.0f} GB"}), flush=True)
        return
    opt = z.ZeroOptimizer(w.numel, w.layer_id, w.n_ranks, 3, hparams=z.AdamHParams(), keep_grad_shards=False,
                          kernel=kern)
    master_fill(opt, w)
    offsets = opt.offsets()

    def gfn(t, lo, hi, bufs, stream):
        for r, ptr in enumerate(bufs):
            gb = W.grad_base(w, 1, r)
            for off, n in zip(offsets, w.numel):
                a, b = max(lo, off), min(hi, off + n)
                if a < b:
                    synth.dev_bf16(gb, a, b - a, w.grad_dist, ptr + 2 * (a - lo), stream)
        return 0

    opt.step(gfn)
    opt.set_timing(True)
    opt.kernel_timing()
    steps = 2
    for _ in range(steps):
        opt.step(gfn)
    kt = opt.kernel_timing()
    per = 4 * w.n_ranks + 26
    kms = kt["ms"] / steps
    print(json.dumps({"stages": w.name, "stage": 3, "n_ranks": w.n_ranks, "params": w.psi,
                      "kernel_ms_per_step": kms, "params_per_s_kernels": w.psi / (kms / 1e3),
                      "bytes_per_elem_model": per, "kernel_gbs_model": kt["model_bytes"] / (kt["ms"] / 1e3) / 1e9,
                      "launches_per_step": kt["launches"] // steps, "fused_config": opt.fused_config(),
                      "note": "one layer's 64 replicas live; gradients generated between launches (untimed)"}),
          flush=True)
    opt.close()


# --------------------------------------------------------------- reference ----

def run_reference(args, world, rank, local):
    """The CPU oracle timed on this machine's host cores, same metric and unit:
    each step a bounded sample of the workload (leading elements of its first
    layer), split over every usable core."""
    if rank != 0:
        return
    w = workload()
    procs = usable_cores()
    k = w.layer_id.count(0)
    layer_elems = int(sum(w.numel[:k])) // 8 * 8
    if args.ref_sample_elems > 0:
        total = args.ref_sample_elems
    else:  # about a minute of oracle work per core for the whole run
        per_core = max(8192 * w.n_ranks, int(5e8 / max(1, args.steps + args.warmup)))
        total = min(layer_elems, procs * per_core)
    total = max(8, total // 8 * 8)
    value, s_per_step, elems = oracle_parallel(w, args.stage, total, args.warmup, args.steps, procs)
    cores = max(1, min(procs, total // 8))
    sample = (f"leading {elems} params of the first layer of {w.name} (N={w.n_ranks}) per step, split into "
              f"{cores} contiguous slices in as many spawned processes; literal ZeRO-{args.stage} steps of "
              f"the C+numpy oracle, input generation untimed")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "params/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": s_per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32",
        "data": "synthetic", "config": {"workload": w.name, "params": w.psi, "n_ranks": w.n_ranks,
                                        "stage": args.stage, "bucket_elems": w.bucket_elems},
        "cpu_baseline": {"value": value, "unit": "params/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "params/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_rank_per_gpu(args, world, rank, local):
    """ZeRO-2 with one logical rank per GPU on the workload's layout (N = the
    number of GPUs, not the workload's logical N): every step each rank
    reduces its shard from the N gradient replicas (peers' over NVLink),
    updates it and writes the result into every rank's parameter replica
    (arm "fused"), or does the same with NCCL reduce-scatter and all-gather
    around the library's shard update (arm "nccl").  Time = the max over
    ranks of the CUDA-event time of the timed steps (host barriers between
    the ranks inside the fused arm's steps are part of it)."""
    import datetime

    import torch
    import torch.distributed as tdist

    import synth
    import zero_sharded_optimizer_sm_b200 as z
    from synth import workloads as W

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist = init_dist(world, "nccl")
    else:  # a one-rank group for the library's host protocol
        import socket

        with socket.socket() as so:
            so.bind(("127.0.0.1", 0))
            port = so.getsockname()[1]
        tdist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                 timeout=datetime.timedelta(seconds=120))
        dist = None
    w = workload()
    opt = z.ZeroDist(w.numel, w.layer_id, bench_stage(), z.AdamHParams(**w.hyper.__dict__), device=dev)
    stream = torch.cuda.current_stream(dev)
    s = stream.cuda_stream
    offs = opt.offsets()
    master = torch.zeros(opt.psi_pad, dtype=torch.float32, device=dev)
    for off, n in zip(offs, w.numel):
        synth.dev_f32(W.master_base(w), off, n, W.MASTER_DIST, master.data_ptr() + 4 * off, s)
    opt.load_master(master)
    del master
    grads = opt.view(z.ZERO_VIEW_GRAD_BUF)
    for off, n in zip(offs, w.numel):
        synth.dev_bf16(W.grad_base(w, 1, rank), off, n, w.grad_dist, grads.data_ptr() + 2 * off, s)
    torch.cuda.synchronize(dev)
    nccl = args.arm == "nccl" and world > 1
    if nccl:
        shard = torch.empty(opt.shard, dtype=torch.bfloat16, device=dev)
        gin = grads.view(torch.bfloat16)
        pout = opt.view(z.ZERO_VIEW_PARAM).view(torch.bfloat16)
        mine = pout[rank * opt.shard:(rank + 1) * opt.shard]

        def one():
            tdist.reduce_scatter_tensor(shard, gin, op=tdist.ReduceOp.AVG)
            opt.adam_shard(shard)
            tdist.all_gather_into_tensor(pout, mine)
    else:
        def one():
            opt.step()
    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize(dev)
    barrier(dist if world > 1 else None)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        one()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_local = e0.elapsed_time(e1)
    ms = max_over_ranks(ms_local, dist if world > 1 else None, dev)
    S, N = opt.shard, world
    nvlink_bytes = 2 * 2 * S * (N - 1)  # per rank per step: peers' gradient slices in, its result out
    hbm_bytes = (4 * N + 24) * S        # per rank per step, every access counted once where it lands
    out = {"metric": METRIC + " -- one logical rank per GPU", "value": w.psi * args.steps / (ms / 1e3),
           "unit": "params/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
           "dtype": "fp32", "data": "synthetic (seeded counter-hash gradients and weights, no dataset)",
           "config": {"workload": w.name, "params": w.psi, "n_ranks": N, "stage": bench_stage(),
                      "arm": args.arm if world > 1 else "fused", "parallelism": f"dp{N}, one rank per GPU",
                      "shard": S},
           "per_rank": {"nvlink_bytes_per_step": nvlink_bytes, "hbm_bytes_per_step": hbm_bytes,
                        "nvlink_GBps": nvlink_bytes / (ms / args.steps / 1e3) / 1e9,
                        "hbm_GBps": hbm_bytes / (ms / args.steps / 1e3) / 1e9}}
    if rank == 0:
        print(json.dumps(out), flush=True)
    opt.close()
    tdist.destroy_process_group()


def run_overlap(args):
    """Overlap of the caller's backward with the step (ZERO_OPT_PIPELINE).
    grad_fn stands in for the backward: it draws each rank's gradients of the
    interval with the seeded generator (one launch per rank; an integer-hash
    kernel, so it competes with the HBM-bound step for issue slots rather than
    for bandwidth).  Per cell: the step time in order (grad_fn, then the
    interval's kernel, on one stream) and pipelined (grad_fn one interval
    ahead on the context's own stream), both CUDA events on the caller's
    stream around whole steps; the generator alone and the step's kernels
    alone (from runs in order) bound what overlap can reach: in order costs
    about their sum, perfect overlap their maximum."""
    import torch

    import synth
    import zero_sharded_optimizer_sm_b200 as z
    from synth import workloads as W

    torch.cuda.set_device(0)
    s = torch.cuda.current_stream().cuda_stream
    kern = {"auto": 0, "register": 1, "tma": 2, "bulk": 3}[args.kernel]
    cells = [(W.gpt_1p2b_n8(), 3, None), (W.gpt_1p2b_n8(), 2, 200_000_000), (W.gpt_85m_n8(), 3, None),
             (W.gpt_85m_n8(), 2, 20_000_000)]
    for w, stage, bucket in cells:
        res = {}
        for pipe in (0, 1, 2):
            opt = z.ZeroOptimizer(w.numel, w.layer_id, w.n_ranks, stage, bucket_elems=bucket,
                                  hparams=z.AdamHParams(), keep_grad_shards=False, kernel=kern, pipeline=pipe)
            assert opt.psi_pad == w.psi and all(o + n == e for o, n, e in
                                                zip(opt.offsets(), w.numel, opt.offsets()[1:] + [w.psi]))
            mv = opt.view(z.ZERO_VIEW_MASTER)
            synth.dev_f32(W.master_base(w), 0, w.psi, W.MASTER_DIST, mv.data_ptr(), s)
            opt.load_master(None)

            def gfn(t, lo, hi, bufs, stream):  # no pads in these layouts: one range per rank
                for r, ptr in enumerate(bufs):
                    synth.dev_bf16(W.grad_base(w, 1, r), lo, hi - lo, w.grad_dist, ptr, stream)
                return 0

            for _ in range(3):
                opt.step(gfn)
            steps = 5
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            opt.set_timing(not pipe)
            opt.kernel_timing()
            torch.cuda.synchronize()
            e0.record()
            for _ in range(steps):
                opt.step(gfn)
            e1.record()
            torch.cuda.synchronize()
            res[("in_order", "pipelined", "pipelined_priority")[pipe]] = e0.elapsed_time(e1) / steps
            if not pipe:
                kt = opt.kernel_timing()
                res["kernels_alone"] = kt["ms"] / steps
                iv = opt.buckets() if stage != 3 else [(lo, hi) for _, lo, hi in reversed(opt.layers())]
                bufs = [opt.view(z.ZERO_VIEW_GRAD_BUF, r).data_ptr() for r in range(w.n_ranks)]
                torch.cuda.synchronize()
                e0.record()
                for _ in range(steps):
                    for lo, hi in iv:
                        gfn(1, lo, hi, bufs, s)
                e1.record()
                torch.cuda.synchronize()
                res["grad_fn_alone"] = e0.elapsed_time(e1) / steps
                res["intervals"] = len(iv)
            opt.close()
            del opt, mv
            torch.cuda.empty_cache()
        lower = max(res["kernels_alone"], res["grad_fn_alone"])
        hidden = (res["in_order"] - res["pipelined"]) / min(res["kernels_alone"], res["grad_fn_alone"])
        print(json.dumps({"overlap": w.name, "stage": stage, "n_ranks": w.n_ranks, "params": w.psi,
                          "intervals": res["intervals"], "bucket_elems": bucket,
                          "ms_in_order": res["in_order"], "ms_pipelined": res["pipelined"],
                          "ms_pipelined_priority": res["pipelined_priority"],
                          "speedup_priority": res["in_order"] / res["pipelined_priority"],
                          "ms_kernels_alone": res["kernels_alone"], "ms_grad_fn_alone": res["grad_fn_alone"],
                          "ms_perfect_overlap": lower, "speedup": res["in_order"] / res["pipelined"],
                          "fraction_of_shorter_phase_hidden": hidden, "steps": steps}), flush=True)


def main(argv=None):
    global _ARGS
    args = parse_args(argv)
    _ARGS = args
    world, rank, local = dist_env()
    if args.gpus != world and world > 1:
        print(f"--gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, world, rank, local)
    elif args.sweep:
        run_sweep(args)
    elif args.stages:
        run_stages(args)
    elif args.overlap:
        run_overlap(args)
    elif args.rank_per_gpu:
        run_rank_per_gpu(args, world, rank, local)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
