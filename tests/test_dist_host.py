"""Host side of the one-rank-per-GPU step, on CPU over gloo (2 and 3 ranks,
launched as torch.distributed.run would): the exchange of the ranks' IPC
records arrives complete and in rank order on every rank, the global norm is
the rank-ordered binary64 sum of the partials (the same bits on every rank),
and the cross-rank order of a step holds -- no rank launches before every
rank's pending work is done, and no rank goes on before every rank's launch
has finished.  Argument checks of zero_dist_* that need no device."""
import ctypes
import json
import math
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import datetime, json, os, sys, time
sys.path.insert(0, {root!r})
import torch.distributed as dist
import zero_sharded_optimizer_sm_b200 as z
world, rank = int(os.environ["WORLD_SIZE"]), int(os.environ["RANK"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
rec = bytes([(rank * 37 + k) % 256 for k in range(z.ZERO_DIST_HANDLE_BYTES)])
recs = z.exchange_records(dist, rec)
ok_records = [r == bytes([(q * 37 + k) % 256 for k in range(z.ZERO_DIST_HANDLE_BYTES)]) for q, r in enumerate(recs)]
partial = [0.1 * (q + 1) ** 3 + 1e-17 * q for q in range(world)]
norm, nf = z.rank_ordered_norm(dist, partial[rank], rank + 2)
events = []
def sync():
    time.sleep(0.05 * (world - rank))  # ranks finish their pending work at different times
    events.append(("sync", time.monotonic_ns()))
def launch():
    events.append(("launch0", time.monotonic_ns()))
    time.sleep(0.05 * (rank + 1))
    events.append(("launch1", time.monotonic_ns()))
for _ in range(2):
    z.ordered_step(dist, sync, launch)
events.append(("after", time.monotonic_ns()))
bad = None
try:
    z.exchange_records(dist, b"short")
except ValueError:
    bad = "refused"
dist.barrier()
print(json.dumps({{"rank": rank, "records": ok_records, "norm": norm.hex(), "nf": nf, "events": events,
                  "bad": bad}}))
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _launch(code, world, timeout=120):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(world),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env, cwd=ROOT, stdout=subprocess.PIPE,
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


@pytest.mark.parametrize("world", [2, 3])
def test_records_norm_and_step_order_over_gloo(world):
    outs = _launch(CHILD.format(root=ROOT), world)
    for rc, _, e in outs:
        assert rc == 0, e
    got = [json.loads(o.strip().splitlines()[-1]) for _, o, _ in outs]
    partial = [0.1 * (q + 1) ** 3 + 1e-17 * q for q in range(world)]
    total = 0.0
    for x in partial:  # rank order, binary64
        total += x
    for g in got:
        assert all(g["records"]) and len(g["records"]) == world
        assert g["norm"] == math.sqrt(total).hex()
        assert g["nf"] == sum(q + 2 for q in range(world))
        assert g["bad"] == "refused"
    # two steps: each launch starts after every rank's sync before it, and
    # every rank's work after a step starts after every rank's launch ended
    for k in range(2):
        syncs = [[t for n, t in g["events"] if n == "sync"] for g in got]
        l0 = [[t for n, t in g["events"] if n == "launch0"][k] for g in got]
        l1 = [[t for n, t in g["events"] if n == "launch1"][k] for g in got]
        before = max(s[2 * k] for s in syncs)
        assert before <= min(l0)
        nxt = [s[2 * k + 2] if len(s) > 2 * k + 2 else [t for n, t in g["events"] if n == "after"][0]
               for s, g in zip(syncs, got)]
        assert max(l1) <= min(nxt)


def test_dist_argument_checks_need_no_device():
    import zero_sharded_optimizer_sm_b200 as z

    numel = (ctypes.c_int64 * 2)(100, 28)
    layer = (ctypes.c_int32 * 2)(0, 1)
    lay = z.zero_layout(2, numel, layer)
    ctx = ctypes.c_void_p()
    assert z.zero_dist_init(ctypes.byref(lay), 0, 0, 2, ctypes.byref(ctx)) == z.ZERO_EINVAL
    assert z.zero_dist_init(ctypes.byref(lay), 4, 4, 2, ctypes.byref(ctx)) == z.ZERO_EINVAL
    assert z.zero_dist_init(ctypes.byref(lay), 4, 1, 0, ctypes.byref(ctx)) == z.ZERO_ENOTIMPL  # plain DP
    assert b"oracle" in z.zero_dist_last_error(None)
    assert z.zero_dist_init(ctypes.byref(lay), 4, 1, 5, ctypes.byref(ctx)) == z.ZERO_EINVAL
    # stage 3: one layer's gradient, the parameter shard, one gathered layer
    assert z.zero_dist_init(ctypes.byref(lay), 4, 1, 3, ctypes.byref(ctx)) == z.ZERO_OK
    try:
        ab = (ctypes.c_int64 * z.ZERO_DIST_NUM_ARENAS)()
        assert z.zero_dist_sizes(ctx, None, ab) == z.ZERO_OK
        assert ab[z.ZERO_DIST_ARENA_GRAD] >= 2 * 104 and ab[z.ZERO_DIST_ARENA_GATHER] >= 2 * 104  # largest layer
        assert 2 * 40 <= ab[z.ZERO_DIST_ARENA_PARAM] < 2 * 160                                     # the shard
        assert z.zero_dist_step_layer(ctx, 0, 1, None) == z.ZERO_ESTATE  # not bound
    finally:
        z.zero_dist_destroy(ctx)
    assert z.zero_dist_init(None, 4, 1, 2, ctypes.byref(ctx)) == z.ZERO_EINVAL
    assert z.zero_dist_init(ctypes.byref(lay), 4, 1, 2, ctypes.byref(ctx)) == z.ZERO_OK
    try:
        plan = (ctypes.c_int64 * 3)()
        ab = (ctypes.c_int64 * z.ZERO_DIST_NUM_ARENAS)()
        assert z.zero_dist_sizes(ctx, plan, ab) == z.ZERO_OK
        # 100 -> 104, + 28 -> 132, padded to a multiple of 8 x 4 ranks = 160
        assert tuple(plan) == (128, 160, 40)
        assert ab[z.ZERO_DIST_ARENA_GRAD] >= 2 * 160 and ab[z.ZERO_DIST_ARENA_PARAM] >= 2 * 160
        assert ab[z.ZERO_DIST_ARENA_STATES] >= 12 * 40
        assert ab[z.ZERO_DIST_ARENA_GATHER] == 0  # stage 3 only
        offs = (ctypes.c_int64 * 2)()
        assert z.zero_dist_tensor_offsets(ctx, offs, 2) == z.ZERO_OK and list(offs) == [0, 104]
        # calls out of order fail cleanly before any device work
        assert z.zero_dist_step(ctx, None) == z.ZERO_ESTATE
        assert z.zero_dist_load_master(ctx, None, None) == z.ZERO_ESTATE
        rec = ctypes.create_string_buffer(z.ZERO_DIST_HANDLE_BYTES)
        assert z.zero_dist_export(ctx, rec) == z.ZERO_ESTATE
        assert z.zero_dist_open_peers(ctx, rec) == z.ZERO_ESTATE
        assert z.zero_dist_bind(ctx, None) == z.ZERO_EINVAL
    finally:
        z.zero_dist_destroy(ctx)
    # the norm combination is host code: rank order, binary64
    sq = (ctypes.c_double * 3)(1e16, 1.0, -1e16)
    nf = (ctypes.c_int64 * 3)(1, 0, 2)
    norm, tot = ctypes.c_double(), ctypes.c_int64()
    assert z.zero_dist_combine_partials(3, sq, nf, ctypes.byref(norm), ctypes.byref(tot)) == z.ZERO_OK
    assert norm.value == 0.0 and tot.value == 3  # (1e16 + 1) rounds to 1e16 first
