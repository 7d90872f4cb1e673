"""bench.py's multi-process plumbing on CPU: two ranks over gloo, as
torch.distributed.run would launch them.  The timing taken is the maximum
over ranks, every rank makes the same collective calls, and only rank 0
prints the JSON line (the reference arm runs on rank 0 alone).  Also its
host helpers: the clock sampler's GPU match and the kernel name the
roofline reports."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, os, sys
sys.path.insert(0, {root!r})
import bench
world, rank, local = bench.dist_env()
d = bench.init_dist(world, "gloo")
m = bench.max_over_ranks(float(10 * rank + 1), d, "cpu")
bench.barrier(d)
m2 = bench.max_over_ranks(float(100 - rank), d, "cpu")
print(json.dumps({{"rank": rank, "max": m, "max2": m2}}))
d.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _launch(code_or_args, world=2, timeout=120):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(world),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        cmd = [sys.executable] + (["-c", code_or_args] if isinstance(code_or_args, str) else code_or_args)
        procs.append(subprocess.Popen(cmd, env=env, cwd=ROOT, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=timeout)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
        outs.append((p.returncode, o, e))
    return outs


def test_max_over_ranks_two_gloo_ranks():
    outs = _launch(CHILD.format(root=ROOT))
    for rc, o, e in outs:
        assert rc == 0, e
    got = [json.loads(o.strip().splitlines()[-1]) for _, o, _ in outs]
    assert all(g["max"] == 11.0 and g["max2"] == 100.0 for g in got)


def test_reference_arm_prints_once_on_rank_zero():
    outs = _launch(["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "1",
                    "--ref-sample-elems", "65536"], timeout=300)
    assert all(rc == 0 for rc, _, _ in outs), [e for _, _, e in outs]
    lines0 = [l for l in outs[0][1].splitlines() if l.startswith("{")]
    lines1 = [l for l in outs[1][1].splitlines() if l.startswith("{")]
    assert len(lines0) == 1 and not lines1
    d = json.loads(lines0[0])
    assert d["impl"] == "reference" and d["unit"] == "params/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["cores"] >= 1 and d["n_gpus"] == 2


def test_clock_sampler_matches_the_gpu_by_pci_bus_id(monkeypatch):
    """nvidia-smi numbers GPUs by PCI order, CUDA by what CUDA_VISIBLE_DEVICES
    leaves: the sampler's index is the nvidia-smi row with the CUDA device's
    PCI domain/bus/device, else the CUDA index."""
    import types

    import torch

    sys.path.insert(0, ROOT)
    import bench

    props = types.SimpleNamespace(pci_domain_id=0, pci_bus_id=0x9C, pci_device_id=0)
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda i: props)
    rows = "0, 00000000:1B:00.0\n1, 00000000:43:00.0\n2, 00000000:9C:00.0\n"
    monkeypatch.setattr(bench.subprocess, "run",
                        lambda *a, **k: types.SimpleNamespace(stdout=rows, returncode=0))
    assert bench.nvsmi_index(0) == 2
    props.pci_bus_id = 0x55  # no such row: the CUDA index
    assert bench.nvsmi_index(1) == 1

    def no_smi(*a, **k):
        raise FileNotFoundError("nvidia-smi")

    monkeypatch.setattr(bench.subprocess, "run", no_smi)
    assert bench.nvsmi_index(3) == 3


def test_fused_kernel_name_follows_the_context_configuration():
    """The roofline's kernel name (the one the ncu launch list shows) from a
    context's fused configuration: the bulk-store kernel, its rank-chunked
    form above 16 ranks, its layered stage-3 launch, and the older kernels."""
    import bench

    bulk = {"kernel": "bulk", "groups": 8, "stages": 4, "tile": 1024}
    assert bench.fused_kernel_name(bulk, 8) == "fused_bulk_kernel"
    assert bench.fused_kernel_name(bulk, 8, layered=True) == "fused_bulk_layered_kernel"
    assert bench.fused_kernel_name(bulk, 64) == "fused_bulk_chunked_kernel"
    assert bench.fused_kernel_name(bulk, 64, layered=True) == "fused_bulk_chunked_kernel"
    assert bench.fused_kernel_name({"kernel": "register", "groups": 0}, 8) == "fused_step_kernel"
    assert bench.fused_kernel_name({"kernel": "tma", "groups": 1}, 8) == "fused_step_tma_kernel"
    assert bench.fused_kernel_name({"kernel": "tma", "groups": 3}, 8) == "fused_step_tma_wide_kernel"
    assert bench.fused_kernel_name({"kernel": "tma", "groups": 1}, 17) == "fused_step_chunked_kernel"
