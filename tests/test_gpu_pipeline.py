"""GPU tests of ZERO_OPT_PIPELINE: the callbacks (the caller's backward,
grad_fn, and its use of each gathered layer, gather_fn) run on the
context's own stream one interval ahead of the step's kernels, with two
alternating gradient / gather slot sets.  The values must not change: every
element against the oracle, and bit for bit against the same steps without
the option, in the fused and the two-pass (clip / skip) step, with callback
gradients and with resident replicas; a callback that fails mid-pipeline
leaves the context usable."""
import gc
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402
from synth import workloads as W  # noqa: E402

from harness import DeviceFill, assert_bits_equal, to_np  # noqa: E402

pytestmark = pytest.mark.gpu

STAGE_OF = {1: oracle.STAGE_Z1, 2: oracle.STAGE_Z2, 3: oracle.STAGE_Z3}


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


def _on(stream):
    return torch.cuda.stream(torch.cuda.ExternalStream(stream) if stream else torch.cuda.default_stream())


def make_opt(w, stage, bucket, pipeline, **kw):
    z = _z()
    opt = z.ZeroOptimizer(w.numel, w.layer_id, w.n_ranks, stage, bucket_elems=bucket,
                          hparams=z.AdamHParams(**w.hyper.__dict__), pipeline=pipeline, **kw)
    fill = DeviceFill(w, opt.offsets(), opt.psi_pad)
    mv = opt.view(z.ZERO_VIEW_MASTER)
    fill.master_into(mv.data_ptr(), mv, torch.cuda.current_stream().cuda_stream)
    opt.load_master(None)
    return opt, fill


def grad_fn_for(opt, fill, seen=None):
    def fn(t, lo, hi, bufs, stream):
        if seen is not None:
            seen.append(("grad", lo, hi, tuple(bufs), stream))
        for r, p in enumerate(bufs):
            fill.grads_into(t, r, lo, hi, p, opt._tensor_at(p, hi - lo, torch.int16), stream)
        return 0
    return fn


def gather_recorder(opt, out, seen=None):
    """Copies every gathered layer on the callback's stream (the buffers are
    reused two layers later)."""
    def fn(layer, lo, hi, bufs, stream):
        if seen is not None:
            seen.append(("gather", lo, hi, tuple(bufs), stream))
        with _on(stream):
            out.append((layer, lo, hi, [opt._tensor_at(b, hi - lo, torch.int16).clone() for b in bufs]))
        return 0
    return fn


def _oracle(w, stage, bucket, **kw):
    p = oracle.plan(w.numel, w.layer_id, w.n_ranks, bucket)
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)

    def g(t, r):
        return W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, t, r), w.grad_dist)

    return p, *oracle.run(p, STAGE_OF[stage], m0, g, w.steps, oracle.AdamHP(**w.hyper.__dict__), **kw)


def _check_state(opt, p, stage, ranks, what):
    z = _z()
    ref = oracle.full_view(p, STAGE_OF[stage], ranks)
    for name, v in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert_bits_equal(to_np(opt.view(v)), ref[name], f"{what} {name}")
    for r in (range(p.n_ranks) if stage != 3 else [0]):
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM, r)), ref["params"], f"{what} params {r}")
    if stage != 1:
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GRAD_SHARD)), ref["grad"], f"{what} grad shards")
    return ref


LAYOUTS = [([33, 1, 2, 17], [0, 1, 1, 2]), ([16, 0, 24, 0], [0, 1, 2, 3]), ([3000, 1, 4100], [0, 1, 2])]


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("layout", LAYOUTS)
def test_pipeline_every_element_against_the_oracle(layout, mode):
    """N = 1, 2, 5, 8; stages 1-3; buckets 8 and all; 3 steps; the callbacks
    see the side stream and alternating slot sets, every gathered layer and
    every statistic match the oracle (the empty layers of the second layout
    come first in reverse order at N = 1 and 5)."""
    z = _z()
    numel, layer = layout
    for n_ranks in (1, 2, 5, 8):
        p0 = oracle.plan(numel, layer, n_ranks, 8)
        for bucket in sorted({8, p0.psi_pad}):
            for stage in (1, 2, 3):
                w = W.Workload("pipe", numel, layer, n_ranks, (stage,), bucket,
                               synth.Dist(synth.NORMAL, 1e-2, zero_mod=7), W.MASTER_DIST, 3,
                               W.Hyper(lr=1e-2, weight_decay=0.1), 0x300 + n_ranks)
                p, ranks, reps = _oracle(w, stage, bucket)
                opt, fill = make_opt(w, stage, bucket, mode)
                caller = torch.cuda.current_stream().cuda_stream
                for t in range(1, w.steps + 1):
                    seen, gathered = [], []
                    st = opt.step(grad_fn_for(opt, fill, seen), gather_recorder(opt, gathered, seen) if stage == 3
                                  else None, stats=True)
                    rep = reps[t - 1]
                    assert st["step"] == t and st["nonfinite"] == rep.nonfinite
                    assert st["grad_norm"] == rep.grad_norm or math.isclose(
                        st["grad_norm"], rep.grad_norm, rel_tol=2 * p.psi_pad * 2.0**-53 + 1e-15)
                    assert all(s_ != caller for *_, s_ in seen)  # the context's own stream
                    grads = [e for e in seen if e[0] == "grad"]
                    if stage != 1 and len(grads) > 1:
                        assert grads[0][3] != grads[1][3]       # alternating slot sets
                        assert grads[0][3] == grads[2][3] if len(grads) > 2 else True
                torch.cuda.synchronize()
                ref = _check_state(opt, p, stage, ranks, f"pipeline N={n_ranks} b={bucket} stage {stage}")
                if stage == 3:
                    want = reps[-1].gathered
                    assert len(gathered) == len(want) == len(p.layers)
                    for (lid, lo, hi, bufs), (plid, plo, phi), tmp in zip(gathered, reversed(p.layers), want):
                        assert (lid, lo, hi) == (plid, plo, phi)
                        for r in range(n_ranks):
                            assert_bits_equal(to_np(bufs[r]), tmp[r], f"gathered layer {lid} rank {r}")
                opt.close()


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("stage", [1, 2, 3])
@pytest.mark.parametrize("two_pass", [False, True])
def test_pipeline_equals_in_order_step(stage, two_pass, mode):
    """2 layers, hidden 768 (14.2M params), N = 8, 3M-element buckets, 4
    steps: with and without the pipeline the same bits everywhere, also in
    the two-pass step (clip at a norm the gradients exceed, overflow skip on)."""
    z = _z()
    numel, layer = W.transformer_layers(2, 768, 3072)
    w = W.Workload("pipe-h768", numel, layer, 8, (stage,), 3_000_000, synth.Dist(synth.NORMAL, 1e-2, zero_mod=100),
                   W.MASTER_DIST, 4, W.Hyper(weight_decay=0.01), W.SEED0 + 30)
    a, fa = make_opt(w, stage, 3_000_000, 0)
    b, fb = make_opt(w, stage, 3_000_000, mode)
    if two_pass:
        a.set_clip(0.5, True)
        b.set_clip(0.5, True)
    ga, gb = [], []
    for t in range(1, w.steps + 1):
        sa = a.step(grad_fn_for(a, fa), gather_recorder(a, ga) if stage == 3 else None, stats=True)
        sb = b.step(grad_fn_for(b, fb), gather_recorder(b, gb) if stage == 3 else None, stats=True)
        assert sa == sb
    for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ):
        assert torch.equal(a.view(what), b.view(what))
    for r in range(8 if stage != 3 else 1):
        assert torch.equal(a.view(z.ZERO_VIEW_PARAM, r), b.view(z.ZERO_VIEW_PARAM, r))
    if stage != 1:
        assert torch.equal(a.view(z.ZERO_VIEW_GRAD_SHARD), b.view(z.ZERO_VIEW_GRAD_SHARD))
    assert len(ga) == len(gb)
    for (la, loa, hia, ba), (lb, lob, hib, bb) in zip(ga, gb):
        assert (la, loa, hia) == (lb, lob, hib)
        for x, y in zip(ba, bb):
            assert torch.equal(x, y)
    a.close()
    b.close()


@pytest.mark.parametrize("mode", [1, 2])
def test_pipeline_resident_stage3_gathers(mode):
    z = _z()
    numel, layer = W.transformer_layers(4, 128, 512)
    w = W.Workload("pipe-res", numel, layer, 4, (3,), None, synth.Dist(synth.NORMAL, 1e-2), W.MASTER_DIST, 2,
                   W.Hyper(), 0x340)
    a, fa = make_opt(w, 3, None, 0)
    b, fb = make_opt(w, 3, None, mode)
    s = torch.cuda.current_stream().cuda_stream
    ga, gb = [], []
    for t in (1, 2):
        reps = [torch.empty(a.psi_pad, dtype=torch.int16, device="cuda") for _ in range(4)]
        for r in range(4):
            fa.grads_into(t, r, 0, a.psi_pad, reps[r].data_ptr(), reps[r], s)
        a.step_resident(reps, gather_recorder(a, ga))
        b.step_resident(reps, gather_recorder(b, gb))
    torch.cuda.synchronize()
    for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ, z.ZERO_VIEW_PARAM):
        assert torch.equal(a.view(what), b.view(what))
    assert len(ga) == len(gb) == 2 * len(a.layers())
    for (la, _, _, ba), (lb, _, _, bb) in zip(ga, gb):
        assert la == lb and all(torch.equal(x, y) for x, y in zip(ba, bb))
    a.close()
    b.close()


def test_pipeline_callback_failure_leaves_the_context_usable():
    z = _z()
    numel, layer = W.transformer_layers(3, 64, 256)
    w = W.Workload("pipe-fail", numel, layer, 4, (3,), None, synth.Dist(synth.NORMAL, 1e-2), W.MASTER_DIST, 1,
                   W.Hyper(), 0x350)
    ref, fr = make_opt(w, 3, None, 0)
    opt, fill = make_opt(w, 3, None, 2)
    good = grad_fn_for(opt, fill)
    calls = [0]

    def bad(t, lo, hi, bufs, stream):
        calls[0] += 1
        return 5 if calls[0] == 2 else good(t, lo, hi, bufs, stream)

    with pytest.raises(z.ZeroError) as ei:
        opt.step(bad)
    assert ei.value.status == z.ZERO_EINVAL and opt.t == 0
    # the aborted step already updated the layers before the failure; re-import
    # the reference's state and step both once more
    torch.cuda.synchronize()
    opt.import_state(ref.export_state())
    st_ref = ref.step(grad_fn_for(ref, fr), stats=True)
    st = opt.step(good, stats=True)
    assert st == st_ref
    for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ, z.ZERO_VIEW_PARAM):
        assert torch.equal(ref.view(what), opt.view(what))
    ref.close()
    opt.close()


@pytest.mark.parametrize("mode", [1, 2])
def test_pipeline_pinned_copies_on_the_callback_stream_outlive_the_context(mode):
    """The callbacks copy from pinned host memory on the stream they are
    given; torch remembers that stream for the pinned block and records an
    event on it when the block is freed -- here after the optimizer is closed.
    The binding hands the library torch's own pooled streams, which stay
    valid, so the free is harmless; the values equal the in-order step's."""
    z = _z()
    numel, layer = W.transformer_layers(2, 64, 256)
    w = W.Workload("pinned", numel, layer, 4, (2,), 16384, synth.Dist(synth.NORMAL, 1e-2), W.MASTER_DIST, 2,
                   W.Hyper(), 0x360)
    ref, fr = make_opt(w, 2, 16384, 0)
    opt, _ = make_opt(w, 2, 16384, mode)
    p = oracle.plan(numel, layer, 4, 16384)
    host = torch.empty((4, p.psi_pad), dtype=torch.int16, pin_memory=True)
    for r in range(4):
        host[r].copy_(torch.from_numpy(W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, 1, r),
                                                     w.grad_dist).view(np.int16)))

    def gfn(t, lo, hi, bufs, stream):
        with _on(stream):
            for r, ptr in enumerate(bufs):
                opt._tensor_at(ptr, hi - lo, torch.int16).copy_(host[r, lo:hi], non_blocking=True)
        return 0

    st = opt.step(gfn, stats=True)
    st_ref = ref.step(lambda t, lo, hi, bufs, s: grad_fn_for(ref, fr)(1, lo, hi, bufs, s), stats=True)
    assert st == st_ref
    assert torch.equal(opt.view(z.ZERO_VIEW_MASTER), ref.view(z.ZERO_VIEW_MASTER))
    opt.close()
    ref.close()
    del host
    gc.collect()
    torch.cuda.synchronize()
    x = torch.empty(1 << 20, dtype=torch.int16, pin_memory=True)  # the host allocator runs again
    del x
    torch.cuda.synchronize()


def test_pipeline_streams_are_fixed_after_the_first_pipelined_step():
    z = _z()
    numel, layer = W.transformer_layers(2, 32, 128)
    w = W.Workload("streams", numel, layer, 2, (2,), 4096, synth.Dist(synth.NORMAL, 1e-2), W.MASTER_DIST, 1,
                   W.Hyper(), 0x370)
    opt, fill = make_opt(w, 2, 4096, 1)
    opt.step(grad_fn_for(opt, fill))
    other = torch.cuda.Stream()
    assert z.zero_set_pipeline_streams(opt.ctx, other.cuda_stream, None) == z.ZERO_ESTATE
    opt.close()


@pytest.mark.parametrize("mode", [1, 2])
def test_clipped_pipelined_stage3_repeated_equals_in_order(mode):
    """A clipped ZeRO-3 step with the callbacks (and a gather consumer) on the
    side stream, repeated: the staged Adam-broadcast pass must not see a stage
    refilled while its shared-memory reads are still in flight -- the
    producer's proxy fence orders them (without it this case differed in
    scattered elements in every repetition on B200)."""
    z = _z()
    numel, layer = W.transformer_layers(2, 768, 3072)
    w = W.Workload("pipe-race", numel, layer, 8, (3,), 3_000_000, synth.Dist(synth.NORMAL, 1e-2, zero_mod=100),
                   W.MASTER_DIST, 3, W.Hyper(weight_decay=0.01), W.SEED0 + 31)
    for _ in range(4):
        a, fa = make_opt(w, 3, 3_000_000, 0)
        b, fb = make_opt(w, 3, 3_000_000, mode)
        a.set_clip(0.5, True)
        b.set_clip(0.5, True)
        ga, gb = [], []
        for t in range(1, w.steps + 1):
            ga.clear()
            gb.clear()
            a.step(grad_fn_for(a, fa), gather_recorder(a, ga), stats=True)
            b.step(grad_fn_for(b, fb), gather_recorder(b, gb), stats=True)
            for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ, z.ZERO_VIEW_PARAM):
                assert torch.equal(a.view(what), b.view(what)), (t, what)
            for (_, _, _, x), (_, _, _, y) in zip(ga, gb):
                assert all(torch.equal(u, v) for u, v in zip(x, y))
        a.close()
        b.close()
