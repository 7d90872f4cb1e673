"""NVTX ranges of the library (ZERO_OPT_NVTX) on the GPU, seen through the
test recorder (tests/nvtx_recorder.c) loaded as the process's NVTX tool: a
child process runs steps with the ranges on and off, and the recorded
domain "zero_sm" holds, in order, one range per step with one nested range
per launch naming its bucket or layer and its [lo, hi) -- the intervals of
the step's schedule --, the clipped step's reduce (one launch over the
resident replicas) / decision / update ranges, the stage-3 step's single range when its layers run as one launch,
a range per unfused call, and nothing while the option is off."""
import json
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")

from test_nvtx_recorder import build_recorder  # noqa: E402

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, sys
sys.path.insert(0, {root!r})
import torch
import zero_sharded_optimizer_sm_b200 as z
torch.cuda.set_device(0)
N = 4
numel, layer = [70_000, 50_000, 30_001, 9], [0, 1, 2, 2]
out = {{}}
for stage in (2, 3):
    opt = z.ZeroOptimizer(numel, layer, N, stage, bucket_elems=40_000, hparams=z.AdamHParams(lr=1e-3))
    g = torch.Generator(device="cuda").manual_seed(stage)
    opt.load_master(torch.randn(opt.psi_pad, device="cuda", generator=g) * 0.1)
    reps = (torch.randn(N, opt.psi_pad, device="cuda", generator=g) * 1e-2).to(torch.bfloat16).view(torch.int16)
    rl = list(reps)
    opt.set_layered(False)
    opt.set_nvtx(True)
    opt.step_resident(rl)
    opt.set_clip(1e-3, True)
    opt.step_resident(rl)
    opt.set_clip(0.0, False)
    if stage == 3:
        opt.set_layered(True)
        opt.step_resident(rl)
    lo, hi = (opt.buckets()[0] if stage == 2 else opt.layers()[-1][1:])
    opt.reduce_scatter(lo, hi, [int(t.data_ptr()) + 2 * lo for t in rl])
    opt.adam_shard(-1, 3)
    opt.all_gather(lo, hi)
    opt.set_nvtx(False)
    opt.step_resident(rl)
    torch.cuda.synchronize()
    out[stage] = dict(buckets=[list(b) for b in opt.buckets()], layers=[list(l) for l in opt.layers()],
                      psi_pad=opt.psi_pad, unfused=[lo, hi])
    opt.close()
print(json.dumps(out))
"""


def _expected(stage, info):
    lines = []
    if stage == 2:
        sched = [("bucket", k, lo, hi) for k, (lo, hi) in enumerate(info["buckets"])]
    else:
        sched = [("layer", lid, lo, hi) for lid, lo, hi in reversed(info["layers"])]
    lines.append(f"push zero_sm step 1 (stage {stage}, N = 4)")
    for kind, k, lo, hi in sched:
        lines += [f"push zero_sm {kind} {k} [{lo}, {hi})", "pop zero_sm"]
    lines.append("pop zero_sm")
    lines.append(f"push zero_sm step 2 (stage {stage}, N = 4)")
    # the resident replicas' first pass: one launch over the flat space
    lines += [f"push zero_sm reduce all 0 [0, {info['psi_pad']})", "pop zero_sm"]
    lines += ["push zero_sm clip decision", "pop zero_sm"]
    if stage == 2:
        lines += [f"push zero_sm update all 0 [0, {info['psi_pad']})", "pop zero_sm"]
    else:
        for kind, k, lo, hi in sched:
            lines += [f"push zero_sm update layer {k} [{lo}, {hi})", "pop zero_sm"]
    lines.append("pop zero_sm")
    if stage == 3:  # the stage-3 step as one layered launch
        layers = info["layers"]
        lines += [f"push zero_sm step 3 (stage 3, N = 4)",
                  f"push zero_sm layers x {len(layers)} [{layers[0][1]}, {layers[-1][2]}) in one launch",
                  "pop zero_sm", "pop zero_sm"]
    lo, hi = info["unfused"]
    lines += [f"push zero_sm reduce-scatter [{lo}, {hi})", "pop zero_sm", "push zero_sm adam shard -1", "pop zero_sm",
              f"push zero_sm all-gather [{lo}, {hi})", "pop zero_sm"]
    return lines


def test_ranges_name_every_launch_of_the_schedule(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib = build_recorder(str(tmp_path))
    rec = tmp_path / "rec.txt"
    env = dict(os.environ, NVTX_INJECTION64_PATH=lib, NVTX_RECORD_FILE=str(rec))
    res = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], env=env, cwd=ROOT, capture_output=True,
                         text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-3000:]
    info = json.loads(res.stdout.strip().splitlines()[-1])
    got = [ln for ln in rec.read_text().splitlines() if ln.split()[:2] in (["push", "zero_sm"], ["pop", "zero_sm"])]
    assert "domain zero_sm" in rec.read_text().splitlines()
    want = _expected(2, info["2"]) + _expected(3, info["3"])
    assert got == want
