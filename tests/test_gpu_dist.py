"""GPU parity of ZeRO with one logical rank per GPU (zero_dist_*), against
the oracle's literal per-rank run, bit for bit.

Only one GPU is available to this suite, so the ranks are processes that
share it: each maps the others' replicas through CUDA IPC exactly as on
several GPUs (same code path; the peer mapping is then same-device memory).
The ranks' kernels never wait on one another -- the order between them is
host barriers over gloo -- so ranks time-sliced on one device are safe.
Each rank saves its shard's master / m / v and its replicas; the parent
compares them with the oracle (N = world)."""
import datetime
import gc
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402
from synth import workloads as W  # noqa: E402

pytestmark = pytest.mark.gpu

STAGE_OF = {1: oracle.STAGE_Z1, 2: oracle.STAGE_Z2, 3: oracle.STAGE_Z3}
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _workload(world, stage, steps=3):
    numel, layer = W.transformer_layers(2, 64, 256)
    numel = list(numel) + [1001]  # a ragged tail
    layer = list(layer) + [layer[-1] + 1]
    return W.Workload("dist", numel, layer, world, (stage,), 0, synth.Dist(synth.NORMAL, 1e-2, zero_mod=13),
                      W.MASTER_DIST, steps, W.Hyper(lr=1e-2, weight_decay=0.05), 0xD150 + 8 * world + stage)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, stage, outdir, nccl_style):
    """One rank: ZeroDist on cuda:0, its own seeded gradients each step."""
    import sys

    sys.path.insert(0, ROOT)
    import torch as t
    import torch.distributed as dist

    import synth as sy
    import zero_sharded_optimizer_sm_b200 as z
    from synth import workloads as WW

    t.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=90))
    w = _workload(world, stage)
    opt = z.ZeroDist(w.numel, w.layer_id, stage, z.AdamHParams(**w.hyper.__dict__), device="cuda:0")
    s = t.cuda.current_stream().cuda_stream
    offs = opt.offsets()
    master = t.zeros(opt.psi_pad, dtype=t.float32, device="cuda:0")
    for off, n in zip(offs, w.numel):
        sy.dev_f32(WW.master_base(w), off, n, WW.MASTER_DIST, master.data_ptr() + 4 * off, s)
    opt.load_master(master)
    grads = opt.view(z.ZERO_VIEW_GRAD_BUF)
    stats = []
    gathered = []
    if stage == 3:
        # layer by layer from the last: this rank's gradient of the layer, then
        # the layer's step on every rank; the gathered layer is kept on the last step
        import oracle as o

        p = o.plan(w.numel, w.layer_id, world, 1 << 40)
        for step in range(1, w.steps + 1):
            order = list(reversed(range(len(p.layers))))
            for k, li in enumerate(order):
                _, l_lo, l_hi = p.layers[li]
                grads.zero_()
                for off, n in zip(offs, w.numel):
                    if l_lo <= off < l_hi and n:
                        sy.dev_bf16(WW.grad_base(w, step, rank), off, n, w.grad_dist,
                                    grads.data_ptr() + 2 * (off - l_lo), s)
                st = opt.step_layer(li, k == len(order) - 1, stats=True)
                if step == w.steps:
                    g = opt.view(z.ZERO_VIEW_GATHER)[: l_hi - l_lo].cpu().numpy().view(np.uint16).copy()
                    gathered.append((li, g))
                if st is not None:
                    stats.append(st)
        t.cuda.synchronize()
        np.savez(os.path.join(outdir, f"rank{rank}.npz"),
                 master=opt.view(z.ZERO_VIEW_MASTER).cpu().numpy(), m=opt.view(z.ZERO_VIEW_EXP_AVG).cpu().numpy(),
                 v=opt.view(z.ZERO_VIEW_EXP_AVG_SQ).cpu().numpy(),
                 params=opt.view(z.ZERO_VIEW_PARAM).cpu().numpy().view(np.uint16),
                 grads=np.zeros(1, np.uint16),
                 gathered_ids=np.array([li for li, _ in gathered], dtype=np.int64),
                 **{f"gathered{li}": g for li, g in gathered},
                 norms=np.array([x["grad_norm"] for x in stats], dtype=np.float64),
                 nfs=np.array([x["nonfinite"] for x in stats], dtype=np.int64),
                 steps=np.array([x["step"] for x in stats], dtype=np.int64))
        opt.close()
        dist.destroy_process_group()
        return
    for step in range(1, w.steps + 1):
        grads.zero_()
        for off, n in zip(offs, w.numel):
            sy.dev_bf16(WW.grad_base(w, step, rank), off, n, w.grad_dist, grads.data_ptr() + 2 * off, s)
        if nccl_style:
            # the update alone, from a reduced shard formed by the oracle on
            # the host (the building block of an NCCL reduce-scatter arm)
            import oracle as o

            t.cuda.synchronize()
            dist.barrier()
            all_g = [None] * world
            dist.all_gather_object(all_g, grads.cpu().numpy().view(np.uint16).copy())
            lo, hi = rank * opt.shard, (rank + 1) * opt.shard
            red = o.reduce_mean([g[lo:hi] for g in all_g])
            opt.adam_shard(t.from_numpy(red.view(np.int16)).cuda())
            t.cuda.synchronize()
            dist.barrier()
        else:
            stats.append(opt.step(stats=True))
    t.cuda.synchronize()
    np.savez(os.path.join(outdir, f"rank{rank}.npz"),
             master=opt.view(z.ZERO_VIEW_MASTER).cpu().numpy(), m=opt.view(z.ZERO_VIEW_EXP_AVG).cpu().numpy(),
             v=opt.view(z.ZERO_VIEW_EXP_AVG_SQ).cpu().numpy(),
             params=opt.view(z.ZERO_VIEW_PARAM).cpu().numpy().view(np.uint16),
             grads=opt.view(z.ZERO_VIEW_GRAD_BUF).cpu().numpy().view(np.uint16),
             norms=np.array([x["grad_norm"] for x in stats], dtype=np.float64),
             nfs=np.array([x["nonfinite"] for x in stats], dtype=np.int64),
             steps=np.array([x["step"] for x in stats], dtype=np.int64))
    opt.close()
    dist.destroy_process_group()


def _run(world, stage, tmp_path, nccl_style=False):
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, stage, str(tmp_path), nccl_style))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    for p in procs:
        if p.is_alive():
            p.kill()
            p.join()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    return [np.load(os.path.join(tmp_path, f"rank{r}.npz")) for r in range(world)]


def _oracle(w, stage):
    p = oracle.plan(w.numel, w.layer_id, w.n_ranks, 1 << 40)
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)

    def g(t, r):
        return W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, t, r), w.grad_dist)

    ranks, reps = oracle.run(p, STAGE_OF[stage], m0, g, w.steps, oracle.AdamHP(**w.hyper.__dict__))
    return p, ranks, reps, oracle.full_view(p, STAGE_OF[stage], ranks)


def _compare(got, w, stage, p, ranks, reps, ref, with_stats=True):
    S = p.shard
    for r, d in enumerate(got):
        lo, hi = r * S, (r + 1) * S
        for k in ("master", "m", "v"):
            assert np.array_equal(d[k].view(np.uint32), ref[k][lo:hi].view(np.uint32)), (r, k)
        if stage == 3:
            assert np.array_equal(d["params"], ref["params"][lo:hi]), f"rank {r} parameter shard"
            # every layer of the last step, gathered on every rank: the oracle's temporary buffers
            want = {lid: tmp for (lid, _, _), tmp in zip(reversed(p.layers), reps[-1].gathered)}
            for li in d["gathered_ids"]:
                lid = p.layers[int(li)][0]
                assert np.array_equal(d[f"gathered{int(li)}"], want[lid][r]), f"rank {r} gathered layer {lid}"
        else:
            assert np.array_equal(d["params"], ref["params"]), f"rank {r} parameter replica"
        if stage == 1:
            assert np.array_equal(d["grads"], ranks[r].grads), f"rank {r} all-reduced gradient"
        if with_stats:
            assert list(d["steps"]) == list(range(1, w.steps + 1))
            for k in range(w.steps):
                assert d["nfs"][k] == reps[k].nonfinite
                n = p.psi_pad
                assert abs(d["norms"][k] - reps[k].grad_norm) <= (2 * n * 2.0**-53 + 1e-15) * reps[k].grad_norm
    # every rank reports the same norm bits
    if with_stats:
        assert all(np.array_equal(d["norms"], got[0]["norms"]) for d in got)


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("stage", [1, 2, 3])
def test_ranks_as_processes_against_the_oracle(world, stage, tmp_path):
    w = _workload(world, stage)
    p, ranks, reps, ref = _oracle(w, stage)
    got = _run(world, stage, tmp_path)
    _compare(got, w, stage, p, ranks, reps, ref)


def test_update_from_a_reduced_shard_equals_the_fused_step(tmp_path):
    """zero_dist_adam_shard from an externally reduced shard (what an NCCL
    reduce-scatter would deliver; here the oracle's mean) updates the shard
    and this rank's own replica range exactly as the fused step does."""
    world, stage = 2, 2
    w = _workload(world, stage)
    p, ranks, reps, ref = _oracle(w, stage)
    got = _run(world, stage, tmp_path, nccl_style=True)
    S = p.shard
    for r, d in enumerate(got):
        lo, hi = r * S, (r + 1) * S
        for k in ("master", "m", "v"):
            assert np.array_equal(d[k].view(np.uint32), ref[k][lo:hi].view(np.uint32)), (r, k)
        assert np.array_equal(d["params"][lo:hi], ref["params"][lo:hi])


def test_single_rank_in_process(tmp_path):
    """world = 1: no peers to open; the step is the N = 1 step."""
    import datetime as dt

    import torch.distributed as dist

    import zero_sharded_optimizer_sm_b200 as z

    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=dt.timedelta(seconds=60))
    try:
        w = _workload(1, 2)
        p, ranks, reps, ref = _oracle(w, 2)
        opt = z.ZeroDist(w.numel, w.layer_id, 2, z.AdamHParams(**w.hyper.__dict__), device="cuda:0")
        s = torch.cuda.current_stream().cuda_stream
        master = torch.zeros(opt.psi_pad, dtype=torch.float32, device="cuda:0")
        for off, n in zip(opt.offsets(), w.numel):
            synth.dev_f32(W.master_base(w), off, n, W.MASTER_DIST, master.data_ptr() + 4 * off, s)
        opt.load_master(master)
        grads = opt.view(z.ZERO_VIEW_GRAD_BUF)
        for step in range(1, w.steps + 1):
            grads.zero_()
            for off, n in zip(opt.offsets(), w.numel):
                synth.dev_bf16(W.grad_base(w, step, 0), off, n, w.grad_dist, grads.data_ptr() + 2 * off, s)
            st = opt.step(stats=True)
            assert st["step"] == step and st["nonfinite"] == reps[step - 1].nonfinite
        for k, v in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
            assert np.array_equal(opt.view(v).cpu().numpy().view(np.uint32), ref[k].view(np.uint32)), k
        assert np.array_equal(opt.view(z.ZERO_VIEW_PARAM).cpu().numpy().view(np.uint16), ref["params"])
        opt.close()
    finally:
        dist.destroy_process_group()
