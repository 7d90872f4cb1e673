"""The staged kernels' failure path on the GPU, made to run without stalling
anything: with ZERO_OPT_WAIT_LIMIT_NS = 0 every ring wait is one
non-blocking test, so the first wait whose bulk copies are still in flight
runs out.  The kernel records the error word, drains the copies it issued
(those waits keep their 2 s limit: every copy lands) and ends; the next
synchronising call returns ZERO_ECUDA and clears the word; the context stays
usable, and after the state is restored (zero_import_state) the next step
equals the oracle bit for bit.  Each staged family: one and two producer /
consumer groups, the sixteen-warp group, the rank-chunked kernel (N > 16),
the bulk-store kernel, and the two passes of a clipped step (the second pass
with per-lane stores and with bulk stores)."""
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
TMA, BULK = 2, 3
FAMILIES = {
    "tma-1-group": (8, dict(kernel=TMA, tma_groups=1), False),
    "tma-2-groups": (8, dict(kernel=TMA, tma_groups=2), False),
    "tma-16-warps": (8, dict(kernel=TMA, tma_groups=3), False),
    "rank-chunked": (17, dict(kernel=TMA), False),
    "bulk-store": (8, dict(kernel=BULK), False),
    "two-pass": (8, dict(kernel=TMA), True),
    "two-pass-bulk-store": (8, dict(kernel=BULK), True),
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    gc.collect()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("family", list(FAMILIES))
@pytest.mark.parametrize("stage", [1, 2, 3])
def test_expired_ring_wait_reports_and_the_context_recovers(family, stage):
    import zero_sharded_optimizer_sm_b200 as z

    n_ranks, kw, clipped = FAMILIES[family]
    numel, layer = W.transformer_layers(2, 128, 512)  # 396,800 params: ~200 tiles of 2048
    w = W.Workload("failure", numel, layer, n_ranks, (stage,), 65536, synth.Dist(synth.NORMAL, 1e-2, zero_mod=17),
                   W.MASTER_DIST, 2, W.Hyper(weight_decay=0.01), 0xFA0 + 8 * stage + n_ranks)
    p = oracle.plan(w.numel, w.layer_id, n_ranks, 65536)
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)

    def g(t, r):
        return W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, t, r), w.grad_dist)

    clip = 1e9 if clipped else 0.0  # a clip that never applies: the two-pass step, same values
    ranks, reps = oracle.run(p, STAGE_OF[stage], m0, g, 2, oracle.AdamHP(**w.hyper.__dict__), clip_norm=clip,
                             skip_nonfinite=clipped)
    ref = oracle.full_view(p, STAGE_OF[stage], ranks)

    opt = z.ZeroOptimizer(w.numel, w.layer_id, n_ranks, stage, bucket_elems=65536,
                          hparams=z.AdamHParams(**w.hyper.__dict__), **kw)
    if clipped:
        opt.set_clip(clip, True)
    fill = DeviceFill(w, opt.offsets(), opt.psi_pad)
    mv = opt.view(z.ZERO_VIEW_MASTER)
    fill.master_into(mv.data_ptr(), mv, torch.cuda.current_stream().cuda_stream)
    opt.load_master(None)

    def gfn(t, lo, hi, bufs, stream):
        for r, ptr in enumerate(bufs):
            fill.grads_into(t, r, lo, hi, ptr, opt._tensor_at(ptr, hi - lo, torch.int16), stream)
        return 0

    assert opt.step(gfn, stats=True)["step"] == 1
    saved = opt.export_state()
    opt.set_wait_limit(0)
    with pytest.raises(z.ZeroError) as err:
        opt.step(gfn, stats=True)
    assert err.value.status == z.ZERO_ECUDA
    assert "bounded wait" in str(err.value)
    opt.set_wait_limit(2_000_000_000)
    # the error word was cleared: a synchronising read succeeds
    opt.read_stats()
    # restore the state of step 1 and run step 2 again
    opt.import_state(saved)
    assert opt.t == 1
    st = opt.step(gfn, stats=True)
    assert st["step"] == 2 and st["nonfinite"] == reps[1].nonfinite
    for k, view in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert_bits_equal(to_np(opt.view(view)), ref[k], f"{family} stage {stage} {k} after recovery")
    if stage != 3:
        for r in (0, n_ranks - 1):
            assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM, r)), ref["params"], f"{family} params {r}")
    else:
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM)), ref["params"], f"{family} param shards")
    opt.close()
    assert np.isfinite(reps[1].grad_norm)


@pytest.mark.parametrize("n_ranks", [4, 8])
def test_layered_launch_wait_runs_out_and_the_context_recovers(n_ranks):
    """The stage-3 step as one layered launch (resident gradients, no
    callbacks): with ZERO_OPT_WAIT_LIMIT_NS = 0 a ring wait or a storer's
    wait for the other CTAs' layer stores runs out.  The CTA aborts, still
    arrives for the layers it has left (so the other CTAs' waits end), and
    the next synchronising call returns ZERO_ECUDA.  After the state is
    restored, the next step equals the oracle bit for bit, layer buffers
    included."""
    import zero_sharded_optimizer_sm_b200 as z

    numel, layer = W.transformer_layers(3, 128, 512)
    w = W.Workload("failure-layered", numel, layer, n_ranks, (3,), 65536, synth.Dist(synth.NORMAL, 1e-2, zero_mod=17),
                   W.MASTER_DIST, 2, W.Hyper(weight_decay=0.01), 0xFB0 + n_ranks)
    p = oracle.plan(w.numel, w.layer_id, n_ranks, 65536)
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)

    def g(t, r):
        return W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, t, r), w.grad_dist)

    ranks, reps = oracle.run(p, oracle.STAGE_Z3, m0, g, 2, oracle.AdamHP(**w.hyper.__dict__))
    ref = oracle.full_view(p, oracle.STAGE_Z3, ranks)
    opt = z.ZeroOptimizer(w.numel, w.layer_id, n_ranks, 3, bucket_elems=65536,
                          hparams=z.AdamHParams(**w.hyper.__dict__), kernel=BULK)
    fill = DeviceFill(w, opt.offsets(), opt.psi_pad)
    mv = opt.view(z.ZERO_VIEW_MASTER)
    s = torch.cuda.current_stream().cuda_stream
    fill.master_into(mv.data_ptr(), mv, s)
    opt.load_master(None)

    def grads(t):
        rp = torch.empty((n_ranks, opt.psi_pad), dtype=torch.int16, device="cuda")
        for r in range(n_ranks):
            fill.grads_into(t, r, 0, opt.psi_pad, rp[r].data_ptr(), rp[r], s)
        return list(rp)

    before = opt.launch_count()
    assert opt.step_resident(grads(1), stats=True)["step"] == 1
    assert opt.launch_count() - before == 3  # step begin, one layered launch, step commit
    saved = opt.export_state()
    g2 = grads(2)
    opt.set_wait_limit(0)
    with pytest.raises(z.ZeroError) as err:
        opt.step_resident(g2, stats=True)
    assert err.value.status == z.ZERO_ECUDA and "bounded wait" in str(err.value)
    opt.set_wait_limit(2_000_000_000)
    opt.read_stats()
    opt.import_state(saved)
    st = opt.step_resident(g2, stats=True)
    assert st["step"] == 2 and st["nonfinite"] == reps[1].nonfinite
    for k, view in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert_bits_equal(to_np(opt.view(view)), ref[k], f"layered N={n_ranks} {k} after recovery")
    assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM)), ref["params"], "layered param shards")
    _, lo0, hi0 = opt.layers()[0]
    for r in range(n_ranks):
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GATHER, r))[: hi0 - lo0], ref["params"][lo0:hi0],
                          f"layered last gathered layer, rank {r}")
    opt.close()
