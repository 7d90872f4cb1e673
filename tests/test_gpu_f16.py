"""GPU parity of the IEEE binary16 storage format (fp16 gradient replicas,
reduced shards and parameters, with a loss scale): the CUDA path, called
through the C ABI, against the oracle's fp16 run on the same seeded inputs.

The pages account the 16-bit copies as 2 bytes per parameter and leave the
format open; fp16 with a loss scale is the mixed-precision recipe they build
on.  Same bar as bf16: reduced shards and parameters bit-exact, fp32 state
bit-exact (within 2 ulp is the stated tolerance; the design computes the
oracle's operations in its order).
"""
import gc
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402
from synth import workloads as W  # noqa: E402

from harness import DeviceFill, assert_bits_equal, assert_f32_close, to_np  # noqa: E402

pytestmark = pytest.mark.gpu

STAGE_OF = {1: oracle.STAGE_Z1, 2: oracle.STAGE_Z2, 3: oracle.STAGE_Z3}
REG, TMA = 1, 2
VARIANTS = {"reg": dict(kernel=REG), "tma1": dict(kernel=TMA, tma_groups=1),
            "tma2": dict(kernel=TMA, tma_groups=2), "tmaw": dict(kernel=TMA, tma_groups=3),
            "tmac": dict(kernel=TMA)}


def kernels_for(n_ranks):
    return ("reg", "tma1", "tma2", "tmaw") if n_ranks <= 16 else ("reg", "tmac")


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


def norm_tol(n):
    return 2 * n * 2.0**-53 + 1e-15


def make_opt(w, stage, bucket, loss_scale, variant=None, **kw):
    z = _z()
    if variant is not None:
        kw.update(VARIANTS[variant])
    opt = z.ZeroOptimizer(w.numel, w.layer_id, w.n_ranks, stage, bucket_elems=bucket,
                          hparams=z.AdamHParams(**w.hyper.__dict__), dtype=z.ZERO_DTYPE_F16, **kw)
    if loss_scale != 1.0:
        opt.set_loss_scale(loss_scale)
    fill = DeviceFill(w, opt.offsets(), opt.psi_pad, f16=True)
    stream = torch.cuda.current_stream().cuda_stream
    mv = opt.view(z.ZERO_VIEW_MASTER)
    fill.master_into(mv.data_ptr(), mv, stream)
    opt.load_master(None)
    return opt, fill


def grad_fn_for(opt, fill):
    def fn(t, lo, hi, bufs, stream):
        for r, p in enumerate(bufs):
            fill.grads_into(t, r, lo, hi, p, opt._tensor_at(p, hi - lo, torch.int16), stream)
        return 0
    return fn


def oracle_run(w, stage, bucket, loss_scale, **kw):
    p = oracle.plan(w.numel, w.layer_id, w.n_ranks, bucket)
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)

    def g(t, r):
        return W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, t, r), w.grad_dist, f16=True)

    ranks, reps = oracle.run(p, STAGE_OF[stage], m0, g, w.steps, oracle.AdamHP(**w.hyper.__dict__),
                             fmt=oracle.F16, loss_scale=loss_scale, **kw)
    return p, ranks, reps


def check_state(opt, p, stage, ranks, what):
    z = _z()
    ref = oracle.full_view(p, STAGE_OF[stage], ranks)
    for name, v in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        got = to_np(opt.view(v))
        assert_f32_close(got, ref[name], f"{what} {name}")
        assert_bits_equal(got, ref[name], f"{what} {name}")
    for r in (range(p.n_ranks) if stage != 3 else [0]):
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM, r)), ref["params"], f"{what} params {r}")
    if stage == 1:
        for r in range(p.n_ranks):
            assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GRAD_BUF, r)), ranks[r].grads, f"{what} all-reduced {r}")
    else:
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GRAD_SHARD)), ref["grad"], f"{what} grad shards")


def check_variant(w, stage, bucket, loss_scale, variant, oracle_result):
    p, ranks, reps = oracle_result
    opt, fill = make_opt(w, stage, bucket, loss_scale, variant)
    assert opt.offsets() == p.offset
    gfn = grad_fn_for(opt, fill)
    for t in range(1, w.steps + 1):
        st = opt.step(gfn, stats=True)
        rep = reps[t - 1]
        assert st["step"] == t and st["nonfinite"] == rep.nonfinite
        assert st["grad_norm"] == rep.grad_norm or math.isclose(st["grad_norm"], rep.grad_norm,
                                                                rel_tol=norm_tol(p.psi_pad))
    check_state(opt, p, stage, ranks, f"fp16 S={loss_scale} stage {stage} {variant}")
    opt.close()


# -------------------------------------------------------------- generator ----

def test_device_f16_generator_matches_host_bitwise():
    s = torch.cuda.current_stream().cuda_stream
    for dist in (synth.Dist(synth.NORMAL, 1e-2, zero_mod=100), synth.Dist(synth.UNIFORM, 7e4),
                 synth.Dist(synth.NORMAL, 1e-6)):
        b = synth.base(0x5EED0002, synth.STREAM_GRAD, 3, 5)
        n, idx0 = 1_000_003, 987_654_321
        dev = torch.empty(n, dtype=torch.int16, device="cuda")
        synth.dev_f16(b, idx0, n, dist, dev.data_ptr(), s)
        assert np.array_equal(to_np(dev), synth.host_f16(b, idx0, n, dist))


# ------------------------------------------------------ every element, tiny ----

TINY = [([5, 3], [0, 1]), ([33, 1, 2, 17], [0, 1, 1, 2]), ([3000, 1, 4100], [0, 1, 2])]


@pytest.mark.parametrize("layout", TINY)
@pytest.mark.parametrize("loss_scale", [1.0, 1024.0])
def test_f16_tiny_layouts_every_kernel(layout, loss_scale):
    """N = 1..4, 8, 9, 16, 17; buckets 8 and all; stages 1-3; 3 steps; every
    fused-kernel variant for that N; loss-scaled gradients N(0, (1e-2 S)^2)."""
    numel, layer = layout
    for n_ranks in (1, 2, 3, 4, 8, 9, 16, 17):
        p0 = oracle.plan(numel, layer, n_ranks, 8)
        for bucket in sorted({8, p0.psi_pad}):
            for stage in (1, 2, 3):
                w = W.Workload("tiny-f16", numel, layer, n_ranks, (stage,), bucket,
                               synth.Dist(synth.NORMAL, 1e-2 * loss_scale, zero_mod=7), W.MASTER_DIST, 3,
                               W.Hyper(lr=1e-2, weight_decay=0.1), 0x160 + n_ranks)
                res = oracle_run(w, stage, bucket, loss_scale)
                for variant in kernels_for(n_ranks):
                    check_variant(w, stage, bucket, loss_scale, variant, res)


def test_f16_two_layer_h768_n8_all_stages_every_kernel():
    """2 layers, hidden 768 (14.2M params), N = 8, loss scale 4096, 1% zero
    grads, AdamW wd 0.01, 3 steps: every element, every stage and variant."""
    numel, layer = W.transformer_layers(2, 768, 3072)
    S = 4096.0
    w = W.Workload("transformer-2L-h768-N8-f16", numel, layer, 8, (1, 2, 3), 3_000_000,
                   synth.Dist(synth.NORMAL, 1e-2 * S, zero_mod=100), W.MASTER_DIST, 3,
                   W.Hyper(weight_decay=0.01), W.SEED0 + 16)
    for stage in (1, 2, 3):
        res = oracle_run(w, stage, 3_000_000, S)
        for variant in kernels_for(8):
            check_variant(w, stage, 3_000_000, S, variant, res)


def test_f16_n64_chunked_kernel():
    numel, layer = [40000, 8, 24000], [0, 1, 1]
    w = W.Workload("n64-f16", numel, layer, 64, (2,), None, synth.Dist(synth.NORMAL, 8.0), W.MASTER_DIST, 2,
                   W.Hyper(), 0x1640)
    bucket = oracle.plan(numel, layer, 64, 1 << 40).psi_pad
    for stage in (2, 3):
        res = oracle_run(w, stage, bucket, 512.0)
        for variant in kernels_for(64):
            check_variant(w, stage, bucket, 512.0, variant, res)


# ------------------------------------------------------------ unfused calls ----

@pytest.mark.parametrize("stage", [1, 2, 3])
def test_f16_unfused_calls_equal_fused_step(stage):
    z = _z()
    numel, layer = W.transformer_layers(3, 64, 256)
    S = 128.0
    w = W.Workload("unfused-f16", numel, layer, 6, (stage,), 4096, synth.Dist(synth.NORMAL, 1.0, zero_mod=9),
                   W.MASTER_DIST, 3, W.Hyper(weight_decay=0.01), 0x170 + stage)
    fused, ff = make_opt(w, stage, 4096, S)
    split, sf = make_opt(w, stage, 4096, S)
    gf, gs = grad_fn_for(fused, ff), grad_fn_for(split, sf)
    intervals = split.buckets() if stage != 3 else [(lo, hi) for _, lo, hi in reversed(split.layers())]
    stream = torch.cuda.current_stream().cuda_stream
    for t in range(1, w.steps + 1):
        a = fused.step(gf, stats=True)
        for lo, hi in intervals:
            if stage == 1:
                gs(t, lo, hi, [split.view(z.ZERO_VIEW_GRAD_BUF, r).data_ptr() + 2 * lo for r in range(6)], stream)
                split.all_reduce(lo, hi)
            else:
                gs(t, lo, hi, [split.view(z.ZERO_VIEW_GRAD_BUF, r).data_ptr() for r in range(6)], stream)
                split.reduce_scatter(lo, hi)
        split.adam_shard(-1, t)
        for lo, hi in intervals:
            split.all_gather(lo, hi)
        split.t = t
        b = split.read_stats()
        assert math.isclose(a["grad_norm"], b["grad_norm"], rel_tol=1e-12) and a["nonfinite"] == b["nonfinite"]
    for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ):
        assert torch.equal(fused.view(what), split.view(what))
    for r in range(6 if stage != 3 else 1):
        assert torch.equal(fused.view(z.ZERO_VIEW_PARAM, r), split.view(z.ZERO_VIEW_PARAM, r))
    fused.close()
    split.close()


# ----------------------------------------------------- clip / overflow skip ----

@pytest.mark.parametrize("stage", [1, 2, 3])
def test_f16_clip_and_overflow_skip(stage):
    """Loss scale 256, clip at a norm the unscaled gradients exceed, and a
    binary16 overflow in call 2 (one element of rank 1 is +Inf, 0x7C00): that
    call is skipped and t does not advance.  In call 3 two ranks hold 65504 at
    one element: their sum is beyond binary16's range, but it is taken in
    fp32 and the mean (about 32760) is not, so call 3 runs, heavily clipped."""
    z = _z()
    numel, layer = W.transformer_layers(2, 64, 256)
    n_ranks, bucket, clip, S = 4, 8192, 0.05, 256.0
    dist = synth.Dist(synth.NORMAL, 1e-2 * S, zero_mod=11)
    w = W.Workload("clip-f16", numel, layer, n_ranks, (stage,), bucket, dist, W.MASTER_DIST, 3,
                   W.Hyper(weight_decay=0.01), 0x180 + stage)
    p = oracle.plan(numel, layer, n_ranks, bucket)
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)

    def host_grad(k, r):
        g = W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, k, r), dist, f16=True)
        if k == 2 and r == 1:
            g[7] = 0x7C00
        if k == 3 and r in (2, 3):
            g[9] = 0x7BFF  # 65504 twice: the fp32 sum is finite and the mean 32752 fits binary16
        return g

    ranks, reps = oracle.run(p, STAGE_OF[stage], m0, host_grad, 3, oracle.AdamHP(**w.hyper.__dict__),
                             clip_norm=clip, skip_nonfinite=True, fmt=oracle.F16, loss_scale=S)
    assert [r.skipped for r in reps] == [False, True, False] and reps[0].coef < 1.0 and reps[2].nonfinite == 0
    opt = z.ZeroOptimizer(numel, layer, n_ranks, stage, bucket_elems=bucket,
                          hparams=z.AdamHParams(**w.hyper.__dict__), dtype=z.ZERO_DTYPE_F16)
    opt.load_master(torch.from_numpy(m0).cuda())
    opt.set_loss_scale(S)
    opt.set_clip(clip, True)
    call = [0]

    def gfn(t, lo, hi, bufs, stream):
        for r, ptr in enumerate(bufs):
            opt._tensor_at(ptr, hi - lo, torch.int16).copy_(
                torch.from_numpy(host_grad(call[0], r)[lo:hi].view(np.int16)))
        return 0

    for k in range(1, 4):
        call[0] = k
        st = opt.step(gfn, stats=True)
        rep = reps[k - 1]
        assert st["skipped"] == rep.skipped and st["nonfinite"] == rep.nonfinite
        assert st["clip_coef"] == (rep.coef if not rep.skipped else 1.0)
        assert st["grad_norm"] == rep.grad_norm or math.isclose(st["grad_norm"], rep.grad_norm,
                                                                rel_tol=norm_tol(p.psi_pad))
    assert opt.t == 2
    ref = oracle.full_view(p, STAGE_OF[stage], ranks)
    for name, what in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert_bits_equal(to_np(opt.view(what)), ref[name], f"fp16 clip stage {stage} {name}")
    for r in (range(n_ranks) if stage != 3 else [0]):
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM, r)), ref["params"], f"fp16 clip stage {stage} params {r}")
    opt.close()


@pytest.mark.parametrize("stage", [2, 3])
def test_f16_resident_step_equals_callback_step(stage):
    """step_resident on fp16 replicas (the bench's path) equals the callback
    step; at stage 3 the resident step is the layered launch (every layer in
    one launch) and the callback step one launch per layer, layer buffers
    included."""
    z = _z()
    numel, layer = [65536, 4096, 30_000], [0, 1, 2]
    w = W.Workload("resident-f16", numel, layer, 8, (stage,), None, synth.Dist(synth.NORMAL, 4.0), W.MASTER_DIST, 2,
                   W.Hyper(), 0x190 + stage)
    bucket = oracle.plan(numel, layer, 8, 1 << 40).psi_pad
    a, fa = make_opt(w, stage, bucket, 1024.0)
    b, fb = make_opt(w, stage, bucket, 1024.0)
    ga = grad_fn_for(a, fa)
    stream = torch.cuda.current_stream().cuda_stream
    for t in (1, 2):
        a.step(ga)
        reps = [torch.empty(b.psi_pad, dtype=torch.int16, device="cuda") for _ in range(8)]
        for r in range(8):
            fb.grads_into(t, r, 0, b.psi_pad, reps[r].data_ptr(), reps[r], stream)
        b.step_resident(reps)
    for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ):
        assert torch.equal(a.view(what), b.view(what))
    if stage == 3:
        assert torch.equal(a.view(z.ZERO_VIEW_PARAM), b.view(z.ZERO_VIEW_PARAM))
        for r in range(8):
            assert torch.equal(a.view(z.ZERO_VIEW_GATHER, r), b.view(z.ZERO_VIEW_GATHER, r))
    else:
        for r in range(8):
            assert torch.equal(a.view(z.ZERO_VIEW_PARAM, r), b.view(z.ZERO_VIEW_PARAM, r))
    a.close()
    b.close()
