"""GPU parity of the bulk-store staged kernel (ZERO_KERNEL_BULK) against the
CPU oracle, bit for bit, in every built (tile, consumer warps) configuration,
ring depth, stage, 16-bit format and launch mode; and the contract of the
movement-only pass (zero_probe_pattern): it leaves the optimizer state, the
parameters and the step counter as the step left them."""
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
BULK = 3  # ZERO_KERNEL_BULK
CONFIGS = [(2048, 8), (2048, 16), (1024, 4), (1024, 8), (1024, 16)]
CHUNKED_CONFIGS = [(2048, 8), (1024, 8)]  # N > 16: the rank-chunked form
# ragged layout: a zero-size tensor, tensors that are not multiples of 8, and
# 220,000 elements in all (over a hundred 1024-element tiles, a ragged last
# tile, several tiles per CTA at the small bucket)
RAGGED = ([150_000, 0, 7, 70_001, 13], [0, 0, 1, 1, 2])


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


def _workload(numel, layer, n_ranks, stage, bucket, steps=3, f16_scale=0.0, seed=0xB0):
    scale = f16_scale if f16_scale else 1.0
    return W.Workload("bulk", numel, layer, n_ranks, (stage,), bucket,
                      synth.Dist(synth.NORMAL, 1e-2 * scale, zero_mod=11), W.MASTER_DIST, steps,
                      W.Hyper(lr=1e-2, weight_decay=0.05), seed + 16 * n_ranks + stage)


def _oracle(w, stage, bucket, f16_scale=0.0):
    p = oracle.plan(w.numel, w.layer_id, w.n_ranks, bucket)
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)
    f16 = f16_scale > 0

    def g(t, r):
        return W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, t, r), w.grad_dist, f16=f16)

    ranks, reps = oracle.run(p, STAGE_OF[stage], m0, g, w.steps, oracle.AdamHP(**w.hyper.__dict__),
                             fmt=oracle.F16 if f16 else oracle.BF16, loss_scale=f16_scale or 1.0)
    return p, ranks, reps, oracle.full_view(p, STAGE_OF[stage], ranks)


def _make(w, stage, bucket, keep, tile, warps, stages=0, f16_scale=0.0, **kw):
    z = _z()
    opt = z.ZeroOptimizer(w.numel, w.layer_id, w.n_ranks, stage, bucket_elems=bucket,
                          hparams=z.AdamHParams(**w.hyper.__dict__), keep_grad_shards=keep, kernel=BULK,
                          tma_tile=tile, tma_warps=warps, tma_stages=stages,
                          dtype=z.ZERO_DTYPE_F16 if f16_scale else z.ZERO_DTYPE_BF16, **kw)
    if f16_scale:
        opt.set_loss_scale(f16_scale)
    fill = DeviceFill(w, opt.offsets(), opt.psi_pad, f16=f16_scale > 0)
    mv = opt.view(z.ZERO_VIEW_MASTER)
    fill.master_into(mv.data_ptr(), mv, torch.cuda.current_stream().cuda_stream)
    opt.load_master(None)
    return opt, fill


def _grad_fn(opt, fill):
    def fn(t, lo, hi, bufs, stream):
        for r, ptr in enumerate(bufs):
            fill.grads_into(t, r, lo, hi, ptr, opt._tensor_at(ptr, hi - lo, torch.int16), stream)
        return 0
    return fn


def _compare(opt, w, stage, p, ranks, reps, ref, keep, tag):
    z = _z()
    fc = opt.fused_config()
    assert fc["kernel"] == "bulk", (tag, fc)
    for k, view in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert_bits_equal(to_np(opt.view(view)), ref[k], f"{tag} {k}")
    if stage in (1, 2):
        for r in range(w.n_ranks):
            assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM, r)), ref["params"], f"{tag} params replica {r}")
    else:
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM)), ref["params"], f"{tag} param shards")
    if stage == 1:
        for r in range(w.n_ranks):
            assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GRAD_BUF, r)), ranks[r].grads, f"{tag} all-reduced grads {r}")
    elif keep:
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GRAD_SHARD)), ref["grad"], f"{tag} grad shards")


def _run_steps(opt, fill, w, stage, p, reps, tag, gathered=None):
    gfn = _grad_fn(opt, fill)

    def gather(layer, lo, hi, bufs, stream):
        gathered.append((layer, lo, hi, [to_np(opt._tensor_at(b, hi - lo, torch.int16)) for b in bufs]))
        return 0

    for t in range(1, w.steps + 1):
        if gathered is not None:
            gathered.clear()
        st = opt.step(gfn, gather if (stage == 3 and gathered is not None) else None, stats=True)
        assert st["step"] == t, tag
        assert st["nonfinite"] == reps[t - 1].nonfinite, tag
        n = p.psi_pad
        assert abs(st["grad_norm"] - reps[t - 1].grad_norm) <= (2 * n * 2.0**-53 + 1e-15) * reps[t - 1].grad_norm, tag


@pytest.mark.parametrize("n_ranks", [1, 3, 8, 16, 17, 33])
@pytest.mark.parametrize("stage", [1, 2, 3])
@pytest.mark.parametrize("small_bucket", [False, True])
def test_every_bulk_configuration_against_the_oracle(n_ranks, stage, small_bucket):
    """Every built (tile, warps) pair, with and without the reduced-gradient
    shards, on a ragged 220K-element layout: one bucket, or 8192-element
    buckets (many intervals shorter than a tile); ZeRO-3 also checks every
    gathered layer buffer of the last step.  Above 16 ranks the rank-chunked
    form (8 ranks a chunk; 33 ranks end on a chunk of one)."""
    numel, layer = RAGGED
    p_all = oracle.plan(numel, layer, n_ranks, 1 << 40)
    bucket = 8192 if small_bucket else p_all.psi_pad
    w = _workload(numel, layer, n_ranks, stage, bucket)
    p, ranks, reps, ref = _oracle(w, stage, bucket)
    for tile, warps in (CONFIGS if n_ranks <= 16 else CHUNKED_CONFIGS):
        for keep in (True, False):
            tag = f"N={n_ranks} stage {stage} bucket {bucket} tile {tile} warps {warps} keep {keep}"
            opt, fill = _make(w, stage, bucket, keep, tile, warps)
            assert opt.offsets() == p.offset and opt.buckets() == p.buckets
            gathered = [] if stage == 3 else None
            _run_steps(opt, fill, w, stage, p, reps, tag, gathered)
            _compare(opt, w, stage, p, ranks, reps, ref, keep, tag)
            if stage == 3:
                want = reps[-1].gathered
                assert len(gathered) == len(want) == len(p.layers), tag
                for (lid, lo, hi, bufs), (wl, wlo, whi), tmp in zip(gathered, reversed(p.layers), want):
                    assert (lid, lo, hi) == (wl, wlo, whi), tag
                    for r in range(n_ranks):
                        assert_bits_equal(bufs[r], tmp[r], f"{tag} gathered layer {lid} rank {r}")
            opt.close()


@pytest.mark.parametrize("tile,stages", [(1024, 2), (1024, 3), (1024, 5), (1024, 8), (2048, 2), (2048, 3),
                                         (2048, 4)])
def test_ring_depths_against_the_oracle(tile, stages):
    """Ring depths from two stages to the most that fit, N = 8, ZeRO-2 without
    gradient shards (the benchmark's arrangement) and ZeRO-1 (which also
    stages the averaged gradient), every element."""
    numel, layer = RAGGED
    for stage in (2, 1):
        p_all = oracle.plan(numel, layer, 8, 1 << 40)
        w = _workload(numel, layer, 8, stage, p_all.psi_pad, steps=2)
        p, ranks, reps, ref = _oracle(w, stage, p_all.psi_pad)
        opt, fill = _make(w, stage, p_all.psi_pad, False, tile, 8, stages=stages)
        got = opt.fused_config()["stages"]
        assert got <= stages and got >= 2
        _run_steps(opt, fill, w, stage, p, reps, f"tile {tile} stages {stages}")
        _compare(opt, w, stage, p, ranks, reps, ref, False, f"tile {tile} stages {stages} stage {stage}")
        opt.close()


@pytest.mark.parametrize("stage", [1, 2, 3])
def test_binary16_with_loss_scale(stage):
    """IEEE binary16 storage with loss scale 512, N = 5: the bulk kernel's F16
    instantiation against the oracle's binary16 run."""
    numel, layer = RAGGED
    p_all = oracle.plan(numel, layer, 5, 1 << 40)
    w = _workload(numel, layer, 5, stage, 16384, f16_scale=512.0)
    p, ranks, reps, ref = _oracle(w, stage, 16384, f16_scale=512.0)
    for tile, warps in ((1024, 8), (2048, 16)):
        opt, fill = _make(w, stage, 16384, True, tile, warps, f16_scale=512.0)
        _run_steps(opt, fill, w, stage, p, reps, f"f16 stage {stage}")
        _compare(opt, w, stage, p, ranks, reps, ref, True, f"f16 stage {stage} tile {tile}")
        opt.close()
    assert p_all.psi_pad >= 16384


@pytest.mark.parametrize("stage", [1, 2, 3])
@pytest.mark.parametrize("pdl", [True, False])
def test_resident_steps_chained_launches(stage, pdl):
    """zero_step_resident over 27 intervals, launches chained with
    programmatic dependent launch or plain, 3 steps: every element against the
    oracle."""
    z = _z()
    numel, layer = W.transformer_layers(3, 96, 384)
    w = _workload(numel, layer, 8, stage, 4096)
    p, ranks, reps, ref = _oracle(w, stage, 4096)
    opt, fill = _make(w, stage, 4096, True, 1024, 8)
    opt.set_pdl(pdl)
    s = torch.cuda.current_stream().cuda_stream
    for t in range(1, w.steps + 1):
        reps_t = torch.empty((w.n_ranks, opt.psi_pad), dtype=torch.int16, device="cuda")
        for r in range(w.n_ranks):
            fill.grads_into(t, r, 0, opt.psi_pad, reps_t[r].data_ptr(), reps_t[r], s)
        opt.step_resident(list(reps_t))
        torch.cuda.synchronize()
        if stage == 1 and t == w.steps:
            for r in range(w.n_ranks):
                assert_bits_equal(to_np(reps_t[r]), ranks[r].grads, f"resident all-reduce rank {r}")
    st = opt.read_stats()
    assert st["step"] == w.steps and st["nonfinite"] == reps[-1].nonfinite
    for k, view in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert_bits_equal(to_np(opt.view(view)), ref[k], f"resident {k}")
    if stage != 3:
        for r in range(w.n_ranks):
            assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM, r)), ref["params"], f"resident params {r}")
    else:
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM)), ref["params"], "resident param shards")
    opt.close()


@pytest.mark.parametrize("stage", [1, 2, 3])
@pytest.mark.parametrize("n_ranks", [4, 17])
def test_probe_pattern_leaves_the_state(stage, n_ranks):
    """The movement-only pass between two steps changes no bit of master, m,
    v or the parameters and does not move the step counter: the second step
    still equals the oracle's second step (one-stage and rank-chunked twins)."""
    z = _z()
    numel, layer = RAGGED
    w = _workload(numel, layer, n_ranks, stage, 16384, steps=2)
    p, ranks, reps, ref = _oracle(w, stage, 16384)
    opt, fill = _make(w, stage, 16384, True, 1024, 8)
    gfn = _grad_fn(opt, fill)
    opt.step(gfn, stats=True)
    before = {v: opt.view(v).clone() for v in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ)}
    params = [opt.view(z.ZERO_VIEW_PARAM, r).clone() for r in range(n_ranks if stage != 3 else 1)]
    reps_t = torch.zeros((n_ranks, opt.psi_pad), dtype=torch.int16, device="cuda")
    for _ in range(3):
        opt.probe_pattern(list(reps_t))
    torch.cuda.synchronize()
    for v, t0 in before.items():
        assert torch.equal(opt.view(v), t0)
    for r, t0 in enumerate(params):
        assert torch.equal(opt.view(z.ZERO_VIEW_PARAM, r), t0)
    assert opt.read_stats()["step"] == 1
    st = opt.step(gfn, stats=True)
    assert st["step"] == 2 and st["nonfinite"] == reps[-1].nonfinite
    _compare(opt, w, stage, p, ranks, reps, ref, True, f"after probe, stage {stage}")
    opt.close()


def test_probe_pattern_refuses_a_configuration_that_is_not_built():
    """Four consumer warps exist for the one-stage kernel only: at 17 ranks
    the probe refuses them (ZERO_ENOTIMPL) and a step fails at launch."""
    z = _z()
    numel, layer = [4096], [0]
    w = _workload(numel, layer, 17, 2, 1 << 20, steps=1)
    opt, _ = _make(w, 2, None, True, 1024, 4)
    reps_t = torch.zeros((17, opt.psi_pad), dtype=torch.int16, device="cuda")
    with pytest.raises(z.ZeroError) as e:
        opt.probe_pattern(list(reps_t))
    assert e.value.status == z.ZERO_ENOTIMPL
    with pytest.raises(z.ZeroError) as e:
        opt.step_resident(list(reps_t))
    assert e.value.status == z.ZERO_ECUDA
    opt.close()


# stage-3 layer lengths in flat order (the schedule runs from the last
# layer to the first), chosen for what the launches leave in the shared layer
# buffers: only the last launch ("last-longest"); the longest layer
# mid-schedule leaves its tail, the launches before it nothing ("mixed");
# every launch leaves a part ("falling")
UNEQUAL_LAYERS = {
    "last-longest": [3_000_000, 1_000_000, 2_000_000, 500_000],
    "mixed": [1_000_000, 3_000_000, 500_000, 2_000_000],
    "falling": [300_008, 700_000, 1_500_000, 2_500_000],
}
_UNEQUAL_REF = {}


@pytest.mark.parametrize("layout", list(UNEQUAL_LAYERS))
@pytest.mark.parametrize("kernel,layered", [(1, False), (2, False), (3, False), (3, True)])
def test_zero3_chained_launches_leave_each_buffer_byte_of_its_last_writer(layout, kernel, layered):
    """Stage-3 steps of unequal layers into the one set of shared layer
    buffers: chained launches (programmatic and plain) in every kernel
    family, and the bulk-store kernel's single layered launch (every layer in
    one cooperative launch, each layer's buffer stores after every CTA's
    stores of the layers before).  Every byte of every rank's buffer after
    the step must hold the parameter of the layer scheduled last among those
    that write it (the serialised step's result), against the oracle."""
    z = _z()
    sizes = UNEQUAL_LAYERS[layout]
    numel, layer = list(sizes), list(range(len(sizes)))
    n_ranks = 8
    w = _workload(numel, layer, n_ranks, 3, 1 << 30, steps=2)
    if layout not in _UNEQUAL_REF:  # one oracle run per layout, shared by the kernels
        _UNEQUAL_REF[layout] = _oracle(w, 3, 1 << 30)[3]
    ref = _UNEQUAL_REF[layout]
    s = torch.cuda.current_stream().cuda_stream
    opts = []
    for pdl in (True, False):
        opt = z.ZeroOptimizer(w.numel, w.layer_id, n_ranks, 3, bucket_elems=1 << 30,
                              hparams=z.AdamHParams(**w.hyper.__dict__), kernel=kernel)
        fill = DeviceFill(w, opt.offsets(), opt.psi_pad)
        mv = opt.view(z.ZERO_VIEW_MASTER)
        fill.master_into(mv.data_ptr(), mv, s)
        opt.load_master(None)
        opt.set_pdl(pdl)
        opt.set_layered(layered)
        opts.append((opt, fill))
    launches = []
    for t in range(1, w.steps + 1):
        for opt, fill in opts:
            reps_t = torch.empty((n_ranks, opt.psi_pad), dtype=torch.int16, device="cuda")
            for r in range(n_ranks):
                fill.grads_into(t, r, 0, opt.psi_pad, reps_t[r].data_ptr(), reps_t[r], s)
            before = opt.launch_count()
            opt.step_resident(list(reps_t))
            launches.append(opt.launch_count() - before)
        torch.cuda.synchronize()
    # begin + commit around the fused launches: one when layered, one per layer otherwise
    assert set(launches) == {2 + (1 if layered else len(sizes))}, launches
    (a, _), (b, _) = opts
    layers = a.layers()
    width = max(hi - lo for _, lo, hi in layers)
    # the byte each position ends with: the last launch of the schedule (the
    # first layer in flat order) long enough to write it
    want = np.zeros(width, dtype=ref["params"].dtype)
    done = np.zeros(width, dtype=bool)
    for _, lo, hi in layers:  # flat order = the schedule's last launch first
        fresh = ~done[: hi - lo]
        want[: hi - lo][fresh] = ref["params"][lo:hi][fresh]
        done[: hi - lo] = True
    assert done.all()
    for key, view in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert_bits_equal(to_np(a.view(view)), ref[key], f"{layout} kernel {kernel} {key}")
    assert_bits_equal(to_np(a.view(z.ZERO_VIEW_PARAM)), ref["params"], f"{layout} param shards")
    for r in range(n_ranks):
        for opt, tag in ((a, "chained"), (b, "plain")):
            assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GATHER, r))[:width], want, f"{layout} {tag} buffer {r}")
    a.close()
    b.close()


@pytest.mark.parametrize("n_ranks", [4, 8])
def test_zero3_chained_layers_order_their_shared_buffer_stores(n_ranks):
    """ZeRO-3 resident steps with chained launches.  Every layer writes the
    same temporary layer buffers, so a launch's stores wait until the launch
    before has finished; its loads and arithmetic may start earlier.  The
    test uses three layers of about 3.1M elements (more than 16 tiles per
    CTA).  It compares them with the same steps launched plainly, on every
    view and every rank's layer buffer.  It also compares them with the
    oracle: states, parameter shards, and the last gathered layer (the first
    layer, which ends in the buffers)."""
    z = _z()
    numel, layer = W.transformer_layers(3, 512, 2048)
    w = _workload(numel, layer, n_ranks, 3, 1 << 30, steps=2)
    p, ranks, reps, ref = _oracle(w, 3, 1 << 30)
    s = torch.cuda.current_stream().cuda_stream
    opts = []
    for pdl in (True, False):
        opt, fill = _make(w, 3, None, True, 1024, 8)
        opt.set_pdl(pdl)
        opts.append((opt, fill))
    for t in range(1, w.steps + 1):
        for opt, fill in opts:
            reps_t = torch.empty((n_ranks, opt.psi_pad), dtype=torch.int16, device="cuda")
            for r in range(n_ranks):
                fill.grads_into(t, r, 0, opt.psi_pad, reps_t[r].data_ptr(), reps_t[r], s)
            opt.step_resident(list(reps_t))
        torch.cuda.synchronize()
    (a, _), (b, _) = opts
    assert len(a.layers()) == 3 and all(hi - lo > 16 * 148 * 1024 for _, lo, hi in a.layers())
    for k, view in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert torch.equal(a.view(view), b.view(view))
        assert_bits_equal(to_np(a.view(view)), ref[k], f"chained ZeRO-3 {k}")
    assert torch.equal(a.view(z.ZERO_VIEW_PARAM), b.view(z.ZERO_VIEW_PARAM))
    assert_bits_equal(to_np(a.view(z.ZERO_VIEW_PARAM)), ref["params"], "chained ZeRO-3 param shards")
    _, lo0, hi0 = a.layers()[0]
    for r in range(n_ranks):
        assert torch.equal(a.view(z.ZERO_VIEW_GATHER, r), b.view(z.ZERO_VIEW_GATHER, r)), r
        assert_bits_equal(to_np(a.view(z.ZERO_VIEW_GATHER, r))[: hi0 - lo0], ref["params"][lo0:hi0],
                          f"chained ZeRO-3 last gathered layer, rank {r}")
    a.close()
    b.close()


@pytest.mark.parametrize("clipped", [False, True])
def test_layered_buffers_equal_per_layer_launches_step_after_step(clipped):
    """Ordering stress for the layered stage-3 launches: layer lengths that
    fall along the schedule, so every layer leaves a part of the layer
    buffers and a store landing out of layer order would change bytes that
    survive the step.  Twelve steps, every rank's layer buffers, the states
    and the parameter shards compared bit for bit after each step between the
    layered launch and one launch per layer (the fused step, and the clipped
    step's update pass)."""
    z = _z()
    numel, layer = [300_008, 700_000, 1_500_000, 2_500_000], [0, 1, 2, 3]
    n_ranks = 8
    w = _workload(numel, layer, n_ranks, 3, 1 << 30, steps=12)
    s = torch.cuda.current_stream().cuda_stream
    opts = []
    for layered in (True, False):
        opt = z.ZeroOptimizer(w.numel, w.layer_id, n_ranks, 3, bucket_elems=1 << 30,
                              hparams=z.AdamHParams(**w.hyper.__dict__), kernel=BULK)
        fill = DeviceFill(w, opt.offsets(), opt.psi_pad)
        mv = opt.view(z.ZERO_VIEW_MASTER)
        fill.master_into(mv.data_ptr(), mv, s)
        opt.load_master(None)
        opt.set_layered(layered)
        if clipped:
            opt.set_clip(0.05, True)
        opts.append((opt, fill))
    (a, fa), (b, _) = opts
    rp = torch.empty((n_ranks, a.psi_pad), dtype=torch.int16, device="cuda")
    for t in range(1, w.steps + 1):
        for r in range(n_ranks):
            fa.grads_into(t, r, 0, a.psi_pad, rp[r].data_ptr(), rp[r], s)
        sa = a.step_resident(list(rp), stats=True)
        sb = b.step_resident(list(rp), stats=True)
        assert sa["step"] == sb["step"] == t and sa["clip_coef"] == sb["clip_coef"]
        for r in range(n_ranks):
            assert torch.equal(a.view(z.ZERO_VIEW_GATHER, r), b.view(z.ZERO_VIEW_GATHER, r)), (t, r)
        for view in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ, z.ZERO_VIEW_PARAM):
            assert torch.equal(a.view(view), b.view(view)), (t, view)
    a.close()
    b.close()
