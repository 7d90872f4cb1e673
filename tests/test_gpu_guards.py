"""Guard bytes of the bound arenas (ZERO_OPT_GUARD) on the GPU, the library's
stand-in for a bounds-checking sanitizer.

The guard bytes are worked out here from the public views: each row of an
arena (a replica, master / m / v, a gradient or layer buffer, either slot
set) ends where its view ends, and the next row starts where the next view
starts; the last 256 bytes of every arena are its tail.  Checked:
* after zero_load_master every one of those bytes holds 0xA5;
* steps at every stage and with every kernel, plain, padded and pipelined,
  and clipped (two passes), leave them all untouched (mode 2 checks after
  each step) and equal the oracle bit for bit;
* a byte planted in any row's guard or any tail is reported with its arena
  and offset, written back, and a later check is clean;
* with mode 2 the step after a planted byte fails with ZERO_EGUARD.
"""
import gc

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402
from synth import workloads as W  # noqa: E402

from harness import DeviceFill, assert_bits_equal, to_np  # noqa: E402

pytestmark = pytest.mark.gpu

STAGE_OF = {1: oracle.STAGE_Z1, 2: oracle.STAGE_Z2, 3: oracle.STAGE_Z3}
GUARD_BYTE = 0xA5
TAIL = 256
# a zero-size tensor, sizes that are not multiples of 8, three layers; the
# padded length (220,096 at N = 8) makes every 16-bit row end 128 bytes short
# of its 256-byte pitch, so the rows have guard bytes even without a pad
NUMEL, LAYER = [150_000, 0, 7, 70_001, 77], [0, 0, 1, 1, 2]
BUCKET = 65_536


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _z():
    import zero_sharded_optimizer_sm_b200 as z
    return z


def _workload(stage, n_ranks=8, steps=2):
    return W.Workload("guards", NUMEL, LAYER, n_ranks, (stage,), BUCKET,
                      synth.Dist(synth.NORMAL, 1e-2, zero_mod=13), W.MASTER_DIST, steps,
                      W.Hyper(lr=1e-2, weight_decay=0.05), 0x6A0 + stage)


def _make(w, stage, guard=2, **kw):
    z = _z()
    opt = z.ZeroOptimizer(w.numel, w.layer_id, w.n_ranks, stage, bucket_elems=BUCKET,
                          hparams=z.AdamHParams(**w.hyper.__dict__), guard=guard, **kw)
    fill = DeviceFill(w, opt.offsets(), opt.psi_pad)
    mv = opt.view(z.ZERO_VIEW_MASTER)
    fill.master_into(mv.data_ptr(), mv, torch.cuda.current_stream().cuda_stream)
    opt.load_master(None)
    return opt, fill


def _gfn(opt, fill):
    def gfn(t, lo, hi, bufs, stream):
        for r, ptr in enumerate(bufs):
            fill.grads_into(t, r, lo, hi, ptr, opt._tensor_at(ptr, hi - lo, torch.int16), stream)
        return 0
    return gfn


def _guard_spans(opt):
    """{arena: [(lo, hi), ...]}: the guard bytes of each arena, from the views."""
    z = _z()
    n = opt.n_ranks
    slots = 2 if opt.pipeline and opt.stage != 1 else 1
    rows = {z.ZERO_ARENA_STATES: [(z.ZERO_VIEW_MASTER, 0), (z.ZERO_VIEW_EXP_AVG, 0), (z.ZERO_VIEW_EXP_AVG_SQ, 0)],
            z.ZERO_ARENA_PARAMS: [(z.ZERO_VIEW_PARAM, r) for r in range(1 if opt.stage == 3 else n)],
            z.ZERO_ARENA_GRADS: [(z.ZERO_VIEW_GRAD_BUF, r) for r in range(n * slots)],
            z.ZERO_ARENA_GRAD_SHARDS: [(z.ZERO_VIEW_GRAD_SHARD, 0)],
            z.ZERO_ARENA_GATHER: [(z.ZERO_VIEW_GATHER, r) for r in range(n * slots)] if opt.stage == 3 else [],
            z.ZERO_ARENA_SCRATCH: []}
    spans = {}
    for k, views in rows.items():
        arena = opt.arenas[k]
        if arena is None:
            continue
        base, size = arena.data_ptr(), arena.numel()
        starts = []
        for what, r in views:
            v = opt.view(what, r)
            starts.append((v.data_ptr() - base, v.data_ptr() - base + v.numel() * v.element_size()))
        out = []
        for i, (lo, end) in enumerate(starts):
            nxt = starts[i + 1][0] if i + 1 < len(starts) else size - TAIL
            assert lo < end <= nxt, (k, i)
            if nxt > end:
                out.append((end, nxt))
        out.append((size - TAIL, size))
        spans[k] = out
    return spans


def _oracle_ref(w, stage, clip=0.0):
    p = oracle.plan(w.numel, w.layer_id, w.n_ranks, BUCKET)
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)

    def g(t, r):
        return W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, t, r), w.grad_dist)

    ranks, reps = oracle.run(p, STAGE_OF[stage], m0, g, w.steps, oracle.AdamHP(**w.hyper.__dict__),
                             clip_norm=clip, skip_nonfinite=clip > 0)
    return oracle.full_view(p, STAGE_OF[stage], ranks)


VARIANTS = {
    "plain": {},
    "pad-pipeline": dict(replica_pad=512, pipeline=1),
    "clipped": {},
}


@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("kernel", [1, 2, 3])
@pytest.mark.parametrize("stage", [1, 2, 3])
def test_steps_leave_every_guard_byte_and_match_the_oracle(stage, kernel, variant):
    z = _z()
    w = _workload(stage)
    opt, fill = _make(w, stage, kernel=kernel, **VARIANTS[variant])
    clip = 0.0
    if variant == "clipped":
        clip = 0.05  # the norm of these gradients is above it: the coefficient applies
        opt.set_clip(clip, True)
    spans = _guard_spans(opt)
    assert spans[z.ZERO_ARENA_PARAMS][0][1] - spans[z.ZERO_ARENA_PARAMS][0][0] >= 128  # rows do have guards
    torch.cuda.synchronize()
    for k, sp in spans.items():  # armed by the load
        host = opt.arenas[k].cpu().numpy()
        for lo, hi in sp:
            assert (host[lo:hi] == GUARD_BYTE).all(), (k, lo, hi)
    gfn = _gfn(opt, fill)
    for _ in range(w.steps):
        opt.step(gfn)  # mode 2: checked after each step
    res = opt.check_guards()
    assert res == dict(changed=0, arena=-1, offset=-1)
    ref = _oracle_ref(w, stage, clip)
    for key, view in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert_bits_equal(to_np(opt.view(view)), ref[key], f"stage {stage} kernel {kernel} {variant} {key}")
    for r in ((0,) if stage == 3 else (0, w.n_ranks - 1)):
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM, r)), ref["params"], f"stage {stage} params {r}")
    opt.close()


@pytest.mark.parametrize("stage", [1, 2, 3])
def test_unfused_calls_leave_every_guard_byte(stage):
    """reduce-scatter (all-reduce at stage 1) per interval through the
    context's gradient buffers, Adam on every shard, all-gather per interval."""
    z = _z()
    w = _workload(stage, steps=1)
    opt, fill = _make(w, stage, guard=1, kernel=1)
    gfn = _gfn(opt, fill)
    s = torch.cuda.current_stream().cuda_stream
    intervals = opt.buckets() if stage != 3 else [(lo, hi) for _, lo, hi in reversed(opt.layers())]
    for lo, hi in intervals:
        off = 2 * lo if stage == 1 else 0
        gfn(1, lo, hi, [opt.view(z.ZERO_VIEW_GRAD_BUF, r).data_ptr() + off for r in range(w.n_ranks)], s)
        if stage == 1:
            opt.all_reduce(lo, hi)
        else:
            opt.reduce_scatter(lo, hi)
    opt.adam_shard(-1, 1)
    for lo, hi in intervals:
        opt.all_gather(lo, hi)
    assert opt.check_guards() == dict(changed=0, arena=-1, offset=-1)
    opt.close()


@pytest.mark.parametrize("stage", [1, 2, 3])
def test_a_planted_byte_is_reported_with_its_place_and_written_back(stage):
    z = _z()
    w = _workload(stage, steps=1)
    opt, fill = _make(w, stage, guard=1, replica_pad=256)
    gfn = _gfn(opt, fill)
    opt.step(gfn)
    assert opt.check_guards()["changed"] == 0
    spans = _guard_spans(opt)
    planted = 0
    for k, sp in spans.items():
        for lo, hi in sp:
            for off in sorted({lo, hi - 1}):
                opt.arenas[k][off] = 0x5A
                res = opt.check_guards()
                assert (res["changed"], res["arena"], res["offset"]) == (1, k, off), (k, lo, hi, res)
                assert f"arena {k}" in res["message"]
                assert opt.arenas[k][off].item() == GUARD_BYTE  # written back
                assert opt.check_guards()["changed"] == 0
                planted += 1
    assert planted >= 2 * len(spans)
    # several at once: the count, and the lowest (arena, offset) first
    k = z.ZERO_ARENA_STATES
    (lo0, _), (lo1, _) = spans[k][0], spans[k][1]
    opt.arenas[k][lo1] = 0
    opt.arenas[k][lo0 + 3] = 0
    opt.arenas[z.ZERO_ARENA_SCRATCH][-1] = 0
    res = opt.check_guards()
    assert (res["changed"], res["arena"], res["offset"]) == (3, k, lo0 + 3)
    # mode 2: the step after a planted byte reports it
    opt.set_guard(2)
    opt.arenas[z.ZERO_ARENA_PARAMS][spans[z.ZERO_ARENA_PARAMS][0][0]] = 1
    with pytest.raises(z.ZeroError) as err:
        opt.step(gfn)
    assert err.value.status == z.ZERO_EGUARD and f"arena {z.ZERO_ARENA_PARAMS}" in str(err.value)
    opt.step(gfn)  # written back by that check
    assert np.isfinite(to_np(opt.view(z.ZERO_VIEW_MASTER)).view(np.float32)).all()
    opt.close()
