"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle
on the same seeded inputs.

Tolerances (stated for the method): reduced gradients and all indexing
bit-exact; fp32 master/m/v within 2 ulp (relative 2.4e-7); bf16 parameters
within 1 bf16 ulp.  The design computes the same IEEE operations in the same
order as the oracle, so most checks below also assert bit equality.
"""
import gc
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402
from synth import workloads as W  # noqa: E402

from harness import (DeviceFill, assert_bf16_close, assert_bits_equal, assert_f32_close,  # noqa: E402
                     oracle_sampled, sample_indices, to_np)

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


def _hp(w):
    z = _z()
    return z.AdamHParams(**w.hyper.__dict__)


REG, TMA, BULK = 1, 2, 3  # ZERO_KERNEL_REGISTER, ZERO_KERNEL_TMA, ZERO_KERNEL_BULK
# fused-kernel variants: the register path, the staged path with one and two
# groups, one wide group, the rank-chunked form; the bulk-store staged kernel
VARIANTS = {"reg": dict(kernel=REG), "tma1": dict(kernel=TMA, tma_groups=1),
            "tma2": dict(kernel=TMA, tma_groups=2), "tmaw": dict(kernel=TMA, tma_groups=3),
            "tmac": dict(kernel=TMA), "blk": dict(kernel=BULK),
            "blk2k16": dict(kernel=BULK, tma_tile=2048, tma_warps=16)}


def kernels_for(n_ranks):
    """Fused-kernel variants at this N: register, the staged kernel with one
    group, two groups and one wide group, and the bulk-store kernel in two
    configurations (N <= 16); register and the rank-chunked staged kernel
    (N > 16)."""
    return ("reg", "tma1", "tma2", "tmaw", "blk", "blk2k16") if n_ranks <= 16 else ("reg", "tmac")


def make_opt(w, stage, bucket=None, keep=True, variant=None, **kw):
    z = _z()
    if variant is not None:
        kw.update(VARIANTS[variant])
    opt = z.ZeroOptimizer(w.numel, w.layer_id, w.n_ranks, stage, bucket_elems=bucket, hparams=_hp(w),
                          keep_grad_shards=keep, **kw)
    fill = DeviceFill(w, opt.offsets(), opt.psi_pad)
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


def norm_tol(n):
    # both sides sum n exactly-squared terms in binary64 in different orders
    return 2 * n * 2.0**-53 + 1e-15


# -------------------------------------------------------------- generator ----

def test_device_generator_matches_host_bitwise():
    s = torch.cuda.current_stream().cuda_stream
    for dist in (synth.Dist(synth.NORMAL, 1e-2, zero_mod=100), synth.Dist(synth.UNIFORM, 1e-2),
                 synth.Dist(synth.NORMAL, 0.02)):
        b = synth.base(0x5EED0002, synth.STREAM_GRAD, 3, 5)
        n, idx0 = 1_000_003, 987_654_321
        dev = torch.empty(n, dtype=torch.int16, device="cuda")
        synth.dev_bf16(b, idx0, n, dist, dev.data_ptr(), s)
        assert np.array_equal(to_np(dev), synth.host_bf16(b, idx0, n, dist))
        devf = torch.empty(n, dtype=torch.float32, device="cuda")
        synth.dev_f32(b, idx0, n, dist, devf.data_ptr(), s)
        assert np.array_equal(to_np(devf).view(np.uint32), synth.host_f32(b, idx0, n, dist).view(np.uint32))


# ------------------------------------------------------ oracle literal runs ----

def _oracle_run(w, stage, bucket):
    p = oracle.plan(w.numel, w.layer_id, w.n_ranks, bucket)
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)

    def g(t, r):
        return W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, t, r), w.grad_dist)

    ranks, reps = oracle.run(p, stage, m0, g, w.steps, oracle.AdamHP(**w.hyper.__dict__))
    return p, ranks, reps


def _check_against_oracle(w, stage, bucket, exact=True, kernels=None):
    if bucket is None:  # one bucket spanning the padded flat space
        bucket = oracle.plan(w.numel, w.layer_id, w.n_ranks, 1 << 40).psi_pad
    p, ranks, reps = _oracle_run(w, STAGE_OF[stage], bucket)
    for variant in (kernels or kernels_for(w.n_ranks)):
        _check_kernel_against_oracle(w, stage, bucket, p, ranks, reps, variant, exact)


def _check_kernel_against_oracle(w, stage, bucket, p, ranks, reps, variant, exact):
    z = _z()
    ref = oracle.full_view(p, STAGE_OF[stage], ranks)
    opt, fill = make_opt(w, stage, bucket=bucket, keep=True, variant=variant)
    assert opt.offsets() == p.offset and opt.buckets() == p.buckets
    gathered = []

    def gather(layer, lo, hi, bufs, stream):
        gathered.append((layer, lo, hi, [to_np(opt._tensor_at(b, hi - lo, torch.int16)) for b in bufs]))
        return 0

    gfn = grad_fn_for(opt, fill)
    for t in range(1, w.steps + 1):
        gathered.clear()
        st = opt.step(gfn, gather if stage == 3 else None, stats=True)
        assert st["step"] == t
        rep = reps[t - 1]
        assert st["nonfinite"] == rep.nonfinite
        assert math.isclose(st["grad_norm"], rep.grad_norm, rel_tol=norm_tol(p.psi_pad))
    got = dict(master=to_np(opt.view(z.ZERO_VIEW_MASTER)), m=to_np(opt.view(z.ZERO_VIEW_EXP_AVG)),
               v=to_np(opt.view(z.ZERO_VIEW_EXP_AVG_SQ)))
    for k in ("master", "m", "v"):
        assert_f32_close(got[k], ref[k], f"stage {stage} {k}")
        if exact:
            assert_bits_equal(got[k], ref[k], f"stage {stage} {k}")
    if stage in (1, 2):
        for r in range(w.n_ranks):
            pr = to_np(opt.view(z.ZERO_VIEW_PARAM, r))
            assert_bf16_close(pr, ref["params"], f"stage {stage} params replica {r}")
            if exact:
                assert_bits_equal(pr, ref["params"], f"stage {stage} params replica {r}")
    else:
        ps = to_np(opt.view(z.ZERO_VIEW_PARAM))
        assert_bf16_close(ps, ref["params"], "stage 3 param shards")
        if exact:
            assert_bits_equal(ps, ref["params"], "stage 3 param shards")
        want = reps[-1].gathered
        assert len(gathered) == len(want) == len(p.layers)
        for (layer, lo, hi, bufs), (lid, llo, lhi), tmp in zip(gathered, reversed(p.layers), want):
            assert (layer, lo, hi) == (lid, llo, lhi)
            for r in range(w.n_ranks):
                assert_bits_equal(bufs[r], tmp[r], f"stage 3 gathered layer {layer} rank {r}")
    if stage == 1:
        for r in range(w.n_ranks):
            assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GRAD_BUF, r)), ranks[r].grads,
                              f"stage 1 all-reduced grads rank {r}")
    else:
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GRAD_SHARD)), ref["grad"], f"stage {stage} grad shards")
    opt.close()


def test_flat_1m_n4_zero2_every_element():
    """1,048,576 params (4 x 512x512), N = 4, ZeRO-2, one bucket, 3 steps."""
    w = W.flat_1m_n4()
    _check_against_oracle(w, 2, None)


TINY = [([1], [0]), ([5, 3], [0, 1]), ([8, 16, 9], [0, 0, 1]), ([33, 1, 2, 17], [0, 1, 1, 2]),
        ([7, 0, 11, 13, 2], [0, 0, 1, 2, 2]), ([3000, 1, 4100], [0, 1, 2]),
        ([16, 0, 24, 0], [0, 1, 2, 3])]  # empty layers; at N = 1 and 5 the first in reverse order


@pytest.mark.parametrize("layout", TINY)
def test_tiny_layouts_all_ranks_buckets_stages(layout):
    """Brute force: N = 1..9 and 16, bucket sizes 8/16/24/all, stages 1-3, 3
    steps each, every element against the oracle's literal per-rank run."""
    numel, layer = layout
    for n_ranks in list(range(1, 10)) + [16, 17]:
        p0 = oracle.plan(numel, layer, n_ranks, 8)
        for bucket in sorted({8, 16, 24, p0.psi_pad}):
            for stage in (1, 2, 3):
                w = W.Workload("tiny", numel, layer, n_ranks, (stage,), bucket,
                               synth.Dist(synth.NORMAL, 1e-2, zero_mod=7), W.MASTER_DIST, 3,
                               W.Hyper(lr=1e-2, weight_decay=0.1), 0xA0 + n_ranks)
                _check_against_oracle(w, stage, bucket)


def test_max_ranks_128():
    numel, layer = [1000, 24], [0, 1]
    w = W.Workload("tiny-N128", numel, layer, 128, (2,), 512, synth.Dist(synth.NORMAL, 1e-2),
                   W.MASTER_DIST, 2, W.Hyper(), 0xC0)
    for stage in (1, 2, 3):
        _check_against_oracle(w, stage, 512)


def test_two_layer_h768_n8_all_stages_every_element():
    """Reduced transformer list (2 layers, hidden 768, 14.2M params), N = 8,
    1% zero grads, AdamW wd 0.01, 5 steps: every element of every stage."""
    numel, layer = W.transformer_layers(2, 768, 3072)
    w = W.Workload("transformer-2L-h768-N8", numel, layer, 8, (1, 2, 3), 3_000_000,
                   synth.Dist(synth.NORMAL, 1e-2, zero_mod=100), W.MASTER_DIST, 5,
                   W.Hyper(weight_decay=0.01), W.SEED0 + 2)
    for stage in (1, 2, 3):
        _check_against_oracle(w, stage, 3_000_000)


# ------------------------------------------------------------ unfused path ----

@pytest.mark.parametrize("stage", [1, 2, 3])
def test_unfused_calls_equal_fused_step(stage):
    """reduce-scatter (or all-reduce) per interval, Adam on every shard,
    all-gather: the same bits as the fused step."""
    z = _z()
    numel, layer = W.transformer_layers(3, 64, 256)
    w = W.Workload("unfused", numel, layer, 6, (stage,), 4096, synth.Dist(synth.NORMAL, 1e-2, zero_mod=9),
                   W.MASTER_DIST, 3, W.Hyper(weight_decay=0.01), 0xD0 + stage)
    fused, ff = make_opt(w, stage, bucket=w.bucket_elems)
    split, sf = make_opt(w, stage, bucket=w.bucket_elems)
    gf = grad_fn_for(fused, ff)
    gs = grad_fn_for(split, sf)
    intervals = split.buckets() if stage != 3 else [(lo, hi) for _, lo, hi in reversed(split.layers())]
    for t in range(1, w.steps + 1):
        sf_ = fused.step(gf, stats=True)
        for lo, hi in intervals:
            if stage == 1:
                bufs = [split.view(z.ZERO_VIEW_GRAD_BUF, r).data_ptr() + 2 * lo for r in range(w.n_ranks)]
                gs(t, lo, hi, bufs, torch.cuda.current_stream().cuda_stream)
                split.all_reduce(lo, hi)
            else:
                bufs = [split.view(z.ZERO_VIEW_GRAD_BUF, r).data_ptr() for r in range(w.n_ranks)]
                gs(t, lo, hi, bufs, torch.cuda.current_stream().cuda_stream)
                split.reduce_scatter(lo, hi)
        split.adam_shard(-1, t)
        for lo, hi in intervals:
            split.all_gather(lo, hi)
        split.t = t
        ss = split.read_stats()
        assert ss["grad_norm"] == sf_["grad_norm"] or math.isclose(ss["grad_norm"], sf_["grad_norm"], rel_tol=1e-12)
        assert ss["nonfinite"] == sf_["nonfinite"]
    for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ):
        assert torch.equal(fused.view(what), split.view(what))
    for r in range(w.n_ranks if stage != 3 else 1):
        assert torch.equal(fused.view(z.ZERO_VIEW_PARAM, r), split.view(z.ZERO_VIEW_PARAM, r))
    if stage == 3:
        # the last all-gather left the first layer in the temporary buffers
        lo, hi = intervals[-1]
        for r in range(w.n_ranks):
            assert torch.equal(fused.view(z.ZERO_VIEW_GATHER, r)[: hi - lo], split.view(z.ZERO_VIEW_GATHER, r)[: hi - lo])
    fused.close()
    split.close()


@pytest.mark.parametrize("stage", [1, 2, 3])
def test_adam_shard_step_counter_mixed_with_fused_steps(stage):
    """Unfused steps that take the context's step counter (t = 0, every
    shard) advance it, so a fused step after two of them is step 3; explicit
    steps t = 1, 2 leave it, and zero_set_step(2) puts it in line.  Both
    mixes end bit for bit on the oracle's three steps."""
    z = _z()
    numel, layer = W.transformer_layers(2, 64, 256)
    w = W.Workload("mixed-t", numel, layer, 4, (stage,), 8192, synth.Dist(synth.NORMAL, 1e-2, zero_mod=9),
                   W.MASTER_DIST, 3, W.Hyper(weight_decay=0.01), 0x7A0 + stage)
    p, ranks, reps = _oracle_run(w, stage, 8192)
    ref = oracle.full_view(p, STAGE_OF[stage], ranks)
    s = torch.cuda.current_stream().cuda_stream
    for explicit in (False, True):
        opt, fill = make_opt(w, stage, bucket=8192)
        gfn = grad_fn_for(opt, fill)
        intervals = opt.buckets() if stage != 3 else [(lo, hi) for _, lo, hi in reversed(opt.layers())]
        for t in (1, 2):
            for lo, hi in intervals:
                if stage == 1:
                    bufs = [opt.view(z.ZERO_VIEW_GRAD_BUF, r).data_ptr() + 2 * lo for r in range(w.n_ranks)]
                    gfn(t, lo, hi, bufs, s)
                    opt.all_reduce(lo, hi)
                else:
                    bufs = [opt.view(z.ZERO_VIEW_GRAD_BUF, r).data_ptr() for r in range(w.n_ranks)]
                    gfn(t, lo, hi, bufs, s)
                    opt.reduce_scatter(lo, hi)
            opt.adam_shard(-1, t if explicit else 0)
            for lo, hi in intervals:
                opt.all_gather(lo, hi)
            assert opt.t == (0 if explicit else t)
        if explicit:
            opt.t = 2
        st = opt.step(gfn, stats=True)
        assert st["step"] == 3 and st["nonfinite"] == reps[2].nonfinite
        for k, view in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
            assert_bits_equal(to_np(opt.view(view)), ref[k], f"stage {stage} explicit {explicit} {k}")
        opt.close()


def test_adam_shard_per_rank_equals_all_ranks():
    z = _z()
    numel, layer = [4096, 2048], [0, 1]
    w = W.Workload("per-rank", numel, layer, 4, (2,), 8192, synth.Dist(synth.NORMAL, 1e-2), W.MASTER_DIST,
                   1, W.Hyper(), 0xE0)
    a, fa = make_opt(w, 2, bucket=8192)
    b, fb = make_opt(w, 2, bucket=8192)
    for o, f in ((a, fa), (b, fb)):
        bufs = [o.view(z.ZERO_VIEW_GRAD_BUF, r).data_ptr() for r in range(4)]
        grad_fn_for(o, f)(1, 0, o.psi_pad, bufs, torch.cuda.current_stream().cuda_stream)
        o.reduce_scatter(0, o.psi_pad)
    a.adam_shard(-1, 1)
    for r in range(4):
        b.adam_shard(r, 1)
    for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ):
        assert torch.equal(a.view(what), b.view(what))
    for r in range(4):
        assert torch.equal(a.view(z.ZERO_VIEW_PARAM, r), b.view(z.ZERO_VIEW_PARAM, r))
    a.close()
    b.close()


@pytest.mark.parametrize("stage", [1, 2, 3])
@pytest.mark.parametrize("clip", [0.0, 0.5])
def test_launch_count_is_the_timed_launches_plus_the_step_kernels(stage, clip):
    """zero_launch_count advances by exactly the launches zero_kernel_timing
    records plus the two one-thread step kernels, per step, plain and clipped;
    a plain stage-3 step is one layered launch, or one launch per layer with
    ZERO_OPT_LAYERED off; a clipped step's first pass over resident replicas
    is one launch."""
    numel, layer = W.transformer_layers(3, 64, 256)
    w = W.Workload("count", numel, layer, 4, (stage,), 16_000, synth.Dist(synth.NORMAL, 1e-2), W.MASTER_DIST, 2,
                   W.Hyper(), 0x600 + stage)
    opt, fill = make_opt(w, stage, bucket=16_000)
    p = oracle.plan(w.numel, w.layer_id, w.n_ranks, 16_000)
    if clip > 0:
        opt.set_clip(clip, True)
    dev = [torch.from_numpy(W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, 1, r),
                                          w.grad_dist).view(np.int16)).cuda() for r in range(w.n_ranks)]
    opt.set_timing(True)
    opt.kernel_timing()
    assert opt.fused_config()["kernel"] == "bulk"  # AUTO's kernel at N = 4
    for layered in ((True, False) if stage == 3 else (True,)):
        opt.set_layered(layered)
        for _ in range(2):
            n0 = opt.launch_count()
            opt.step_resident(dev)
            torch.cuda.synchronize()
            timed = opt.kernel_timing()["launches"]
            intervals = len(opt.buckets()) if stage != 3 else len(opt.layers())
            if clip == 0:
                expect = 1 if stage == 3 and layered else intervals
            else:  # pass 1 over the resident replicas in one launch; pass 2 per layer at stage 3 unless layered
                expect = 1 + (1 if stage != 3 or layered else intervals)
            assert timed == expect, (layered, timed, expect)
            assert opt.launch_count() - n0 == timed + 2
    opt.set_timing(False)
    opt.close()


@pytest.mark.parametrize("stage", [1, 2, 3])
def test_pdl_resident_steps_equal_plain_launches(stage):
    """Resident steps with ZERO_OPT_PDL launch their fused kernels with
    programmatic dependent launch (at stage 1/2 each later launch streams its
    interval while the one before finishes).  Against the same steps launched
    plainly:
    the same bits, for every kernel variant, N = 4, 8, 16 and 17, eight or
    more intervals per step, 3 steps, and against the oracle."""
    z = _z()
    numel, layer = W.transformer_layers(4, 96, 384)
    for n_ranks in (4, 8, 16, 17):
        w = W.Workload("pdl", numel, layer, n_ranks, (stage,), 40_000, synth.Dist(synth.NORMAL, 1e-2, zero_mod=13),
                       W.MASTER_DIST, 3, W.Hyper(weight_decay=0.01), 0x400 + n_ranks)
        p, ranks, reps = _oracle_run(w, STAGE_OF[stage], 40_000)
        ref = oracle.full_view(p, STAGE_OF[stage], ranks)
        host = {t: [W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, t, r), w.grad_dist)
                    for r in range(n_ranks)] for t in range(1, 4)}
        for variant in kernels_for(n_ranks):
            a, _ = make_opt(w, stage, bucket=40_000, variant=variant)
            b, _ = make_opt(w, stage, bucket=40_000, variant=variant)
            a.set_pdl(True)
            b.set_pdl(False)
            assert len(a.buckets() if stage != 3 else a.layers()) >= 4
            for t in range(1, 4):
                dev = [torch.from_numpy(h.view(np.int16)).cuda() for h in host[t]]
                devb = [x.clone() for x in dev]
                sa = a.step_resident(dev, stats=True)
                sb = b.step_resident(devb, stats=True)
                assert sa == sb
                assert math.isclose(sa["grad_norm"], reps[t - 1].grad_norm, rel_tol=norm_tol(p.psi_pad))
                if stage == 1:
                    for r in range(n_ranks):
                        assert torch.equal(dev[r], devb[r])
            for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ):
                assert torch.equal(a.view(what), b.view(what))
            for name, what in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
                assert_bits_equal(to_np(a.view(what)), ref[name], f"pdl {variant} N={n_ranks} {name}")
            for r in range(n_ranks if stage != 3 else 1):
                assert torch.equal(a.view(z.ZERO_VIEW_PARAM, r), b.view(z.ZERO_VIEW_PARAM, r))
                assert_bits_equal(to_np(a.view(z.ZERO_VIEW_PARAM, r)), ref["params"], f"pdl {variant} params {r}")
            if stage == 3:
                assert torch.equal(a.view(z.ZERO_VIEW_GATHER, 0), b.view(z.ZERO_VIEW_GATHER, 0))
            a.close()
            b.close()


# ------------------------------------------------------------- edge cases ----

def test_nonfinite_gradients_are_counted_and_propagate_like_the_oracle():
    z = _z()
    numel, layer = [4096, 1024], [0, 1]
    w = W.Workload("nonfinite", numel, layer, 4, (2,), 8192, synth.Dist(synth.NORMAL, 1e-2), W.MASTER_DIST,
                   1, W.Hyper(), 0xF0)
    opt, fill = make_opt(w, 2, bucket=8192)
    p = oracle.plan(numel, layer, 4, 8192)
    host = [W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, 1, r), w.grad_dist) for r in range(4)]
    host[1][[5, 77, 4100]] = [0x7F80, 0xFFC0, 0xFF80]  # +inf, NaN, -inf in rank 1
    host[3][77] = 0x7F80
    dev = [torch.from_numpy(h.view(np.int16)).cuda() for h in host]
    st = opt.step_resident(dev, stats=True)
    ranks = oracle.init_states(p, oracle.STAGE_Z2, W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w),
                                                                 W.MASTER_DIST, as_f32=True))
    rep = oracle.step(p, oracle.STAGE_Z2, ranks, lambda t, r: host[r], 1, oracle.AdamHP())
    assert st["nonfinite"] == rep.nonfinite == 3
    assert math.isnan(st["grad_norm"]) and math.isnan(rep.grad_norm)
    ref = oracle.full_view(p, oracle.STAGE_Z2, ranks)
    got = to_np(opt.view(z.ZERO_VIEW_MASTER))
    assert np.array_equal(np.isnan(got), np.isnan(ref["master"]))
    assert_f32_close(got, ref["master"], "master with nonfinite grads")
    opt.close()


def test_grad_fn_failure_aborts_the_step_with_einval():
    z = _z()
    w = W.Workload("abort", [1024], [0], 2, (2,), 1024, synth.Dist(synth.NORMAL, 1e-2), W.MASTER_DIST, 1,
                   W.Hyper(), 1)
    opt, _ = make_opt(w, 2)
    with pytest.raises(z.ZeroError) as ei:
        opt.step(lambda t, lo, hi, bufs, s: 7)
    assert ei.value.status == z.ZERO_EINVAL
    assert opt.t == 0
    with pytest.raises(z.ZeroError):
        opt.reduce_scatter(0, 12)  # not a multiple of 8
    with pytest.raises(z.ZeroError):
        opt.all_gather(0, opt.psi_pad + 8)
    opt.close()


# ------------------------------------------- full-size workloads, sampled ----

def _sampled_check(opt, w, steps, stage, idx, ref):
    z = _z()
    it = torch.from_numpy(idx).cuda()
    for name, what in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        got = to_np(opt.view(what)[it])
        assert_f32_close(got, ref[name], f"{w.name} stage {stage} {name}")
        assert_bits_equal(got, ref[name], f"{w.name} stage {stage} {name}")
    if stage == 3:
        got = to_np(opt.view(z.ZERO_VIEW_PARAM)[it])
        assert_bits_equal(got, ref["params"], f"{w.name} param shards")
    else:
        for r in sorted({0, w.n_ranks // 2, w.n_ranks - 1}):
            got = to_np(opt.view(z.ZERO_VIEW_PARAM, r)[it])
            assert_bf16_close(got, ref["params"], f"{w.name} params replica {r}")
            assert_bits_equal(got, ref["params"], f"{w.name} params replica {r}")
    if stage in (2, 3):
        got = to_np(opt.view(z.ZERO_VIEW_GRAD_SHARD)[it])
        assert_bits_equal(got, ref["grad"], f"{w.name} grad shards")


def test_transformer_85m_n8_stages_agree_and_match_dp():
    """12 layers, hidden 768 (85,054,464 params), N = 8, ZeRO-1/2/3 from the
    same seed, 5 steps: the three stages agree bit for bit on the device, and
    sampled elements match the oracle's plain-DP result."""
    z = _z()
    w = W.gpt_85m_n8()
    opts = {}
    for stage in (1, 2, 3, "tma1-1", "tma1-2", "tma1-3", "tma2-1", "tma2-2", "tma2-3", "tmaw-1", "tmaw-2",
                  "tmaw-3"):
        variant = stage.split("-")[0] if isinstance(stage, str) else "reg"
        st_ = int(str(stage)[-1])
        opt, fill = make_opt(w, st_, bucket=20_000_000, variant=variant)
        gathered_ok = []

        def gather(layer, lo, hi, bufs, stream, opt=opt):
            shard = opt.view(z.ZERO_VIEW_PARAM)[lo:hi]
            gathered_ok.append(all(torch.equal(opt._tensor_at(b, hi - lo, torch.int16), shard) for b in bufs))
            return 0

        gfn = grad_fn_for(opt, fill)
        for t in range(1, w.steps + 1):
            opt.step(gfn, gather if st_ == 3 else None)
        if st_ == 3:
            assert len(gathered_ok) == 12 * w.steps and all(gathered_ok)
        else:
            for r in range(1, w.n_ranks):
                assert torch.equal(opt.view(z.ZERO_VIEW_PARAM, 0), opt.view(z.ZERO_VIEW_PARAM, r))
        opts[stage] = opt
    # the staged kernel computes the same bits as the register kernel
    for st_, v in [(x, y) for x in (1, 2, 3) for y in ("tma1", "tma2", "tmaw")]:
        a, b = opts[st_], opts[f"{v}-{st_}"]
        for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ, z.ZERO_VIEW_PARAM):
            assert torch.equal(a.view(what), b.view(what)), (st_, what)
        if st_ == 1:
            for r in range(w.n_ranks):
                assert torch.equal(a.view(z.ZERO_VIEW_GRAD_BUF, r), b.view(z.ZERO_VIEW_GRAD_BUF, r))
        else:
            assert torch.equal(a.view(z.ZERO_VIEW_GRAD_SHARD), b.view(z.ZERO_VIEW_GRAD_SHARD))
        b.close()
    for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ):
        assert torch.equal(opts[1].view(what), opts[2].view(what))
        assert torch.equal(opts[1].view(what), opts[3].view(what))
    assert torch.equal(opts[1].view(z.ZERO_VIEW_PARAM, 0), opts[3].view(z.ZERO_VIEW_PARAM))
    assert torch.equal(opts[2].view(z.ZERO_VIEW_GRAD_SHARD), opts[3].view(z.ZERO_VIEW_GRAD_SHARD))
    o = opts[2]
    idx = sample_indices(o.offsets(), w.numel, o.psi_pad, o.shard, w.n_ranks, 60_000, intervals=o.buckets())
    ref = oracle_sampled(w, idx, w.steps)
    for stage in (1, 2, 3):
        _sampled_check(opts[stage], w, w.steps, stage, idx, ref)
    # stage 1 keeps the all-reduced gradient in every replica
    it = torch.from_numpy(idx).cuda()
    for r in (0, 7):
        assert_bits_equal(to_np(opts[1].view(z.ZERO_VIEW_GRAD_BUF, r)[it]), ref["grad"], "stage 1 grads")
    for o in opts.values():
        o.close()


def test_transformer_1p2b_n8_zero2_bucket200m():
    """24 layers, hidden 2048 (1,208,598,528 params), N = 8, ZeRO-2 through
    the fixed 200M-element buffer, 3 steps: sampled elements against the
    oracle, and the resident-replica step (the bench's launch configuration)
    equal bit for bit on the device."""
    z = _z()
    w = W.gpt_1p2b_n8()
    opt, fill = make_opt(w, 2, bucket=w.bucket_elems)
    assert len(opt.buckets()) == 7
    gfn = grad_fn_for(opt, fill)
    norms = []
    for t in range(1, w.steps + 1):
        norms.append(opt.step(gfn, stats=True))
    idx = sample_indices(opt.offsets(), w.numel, opt.psi_pad, opt.shard, w.n_ranks, 40_000,
                         intervals=opt.buckets())
    ref = oracle_sampled(w, idx, w.steps)
    _sampled_check(opt, w, w.steps, 2, idx, ref)
    keep = {what: opt.view(what).clone() for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ)}
    keep["p0"] = opt.view(z.ZERO_VIEW_PARAM, 0).clone()
    opt.close()
    del opt
    gc.collect()
    torch.cuda.empty_cache()
    # resident replicas, no keep of the grad shard: the bench configuration
    res, rfill = make_opt(w, 2, bucket=w.bucket_elems, keep=False)
    reps = torch.empty((w.n_ranks, res.psi_pad), dtype=torch.int16, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    for t in range(1, w.steps + 1):
        for r in range(w.n_ranks):
            rfill.grads_into(t, r, 0, res.psi_pad, reps[r].data_ptr(), reps[r], s)
        st = res.step_resident(list(reps), stats=True)
        assert st["grad_norm"] == norms[t - 1]["grad_norm"] or math.isclose(
            st["grad_norm"], norms[t - 1]["grad_norm"], rel_tol=1e-12)
    for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ):
        assert torch.equal(res.view(what), keep[what])
    for r in range(w.n_ranks):
        assert torch.equal(res.view(z.ZERO_VIEW_PARAM, r), keep["p0"])
    res.close()
    del res
    gc.collect()
    torch.cuda.empty_cache()
    # the staged kernel (one and two groups), resident replicas: the same bits
    for variant in ("tma1", "tma2", "tmaw"):
        tma, tfill = make_opt(w, 2, bucket=w.bucket_elems, keep=False, variant=variant)
        for t in range(1, w.steps + 1):
            for r in range(w.n_ranks):
                tfill.grads_into(t, r, 0, tma.psi_pad, reps[r].data_ptr(), reps[r], s)
            tma.step_resident(list(reps), stats=True)
        for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ):
            assert torch.equal(tma.view(what), keep[what]), variant
        for r in range(w.n_ranks):
            assert torch.equal(tma.view(z.ZERO_VIEW_PARAM, r), keep["p0"]), variant
        tma.set_timing(True)
        tma.step_resident(list(reps))
        kt = tma.kernel_timing()  # also reads the device error word
        assert kt["launches"] == 7 and kt["model_bytes"] == 56 * tma.psi_pad
        tma.close()
        del tma
        gc.collect()
        torch.cuda.empty_cache()
    del reps, keep
    gc.collect()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("variant", ["reg", "tmac"])
def test_transformer_6p4b_n64_zero3_one_layer_live(variant):
    """32 layers, hidden 4096 (6,444,154,880 params), N = 64, ZeRO-3 with one
    layer's 64 gradient replicas and 64 temporary gathered layers live, 2
    steps: every gathered layer equals the updated shards on every rank, and
    sampled elements match the oracle."""
    z = _z()
    w = W.gpt_6p4b_n64()
    free, _ = torch.cuda.mem_get_info()
    opt_need = 12 * 6_444_154_880 + 2 * 6_444_154_880 + 4 * 64 * 201_379_840
    if free < opt_need + (4 << 30):
        pytest.skip(f"needs {opt_need / 1e9:.0f} GB free, have {free / 1e9:.0f} GB")
    opt, fill = make_opt(w, 3, keep=False, variant=variant)
    assert opt.sizes.max_layer == 201_379_840
    ok = []

    def gather(layer, lo, hi, bufs, stream):
        shard = opt.view(z.ZERO_VIEW_PARAM)[lo:hi]
        ok.append(all(torch.equal(opt._tensor_at(b, hi - lo, torch.int16), shard) for b in bufs))
        return 0

    gfn = grad_fn_for(opt, fill)
    for t in range(1, w.steps + 1):
        opt.step(gfn, gather)
    assert len(ok) == 32 * w.steps and all(ok)
    idx = sample_indices(opt.offsets(), w.numel, opt.psi_pad, opt.shard, w.n_ranks, 20_000,
                         intervals=[(lo, hi) for _, lo, hi in opt.layers()])
    ref = oracle_sampled(w, idx, w.steps)
    it = torch.from_numpy(idx).cuda()
    for name, what in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert_bits_equal(to_np(opt.view(what)[it]), ref[name], f"6.4B {name}")
    assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM)[it]), ref["params"], "6.4B param shards")
    opt.close()
    del opt
    gc.collect()
    torch.cuda.empty_cache()


SWEEP_SMALL = [(e, n) for e in (1024, 16384, 262144) for n in W.SWEEP_RANKS]


@pytest.mark.parametrize("elems,n_ranks", SWEEP_SMALL)
def test_flat_sweep_cells_every_element(elems, n_ranks):
    """Flat-buffer sweep cells (U(-1e-2, 1e-2) grads, one bucket), every element."""
    w = W.flat_sweep(elems, n_ranks)
    _check_against_oracle(w, 2, None)


@pytest.mark.parametrize("elems,n_ranks", [(1 << 30, 2), (1 << 28, 16), (1 << 26, 64), (1 << 24, 8)])
def test_flat_sweep_large_cells_fused_equals_unfused_and_oracle_samples(elems, n_ranks):
    z = _z()
    w = W.flat_sweep(elems, n_ranks)
    fused, ff = make_opt(w, 2, keep=False, variant=kernels_for(n_ranks)[-1])
    s = torch.cuda.current_stream().cuda_stream
    reps = torch.empty((n_ranks, fused.psi_pad), dtype=torch.int16, device="cuda")
    for r in range(n_ranks):
        ff.grads_into(1, r, 0, fused.psi_pad, reps[r].data_ptr(), reps[r], s)
    fused.step_resident(list(reps))
    idx = sample_indices(fused.offsets(), w.numel, fused.psi_pad, fused.shard, n_ranks, 20_000)
    ref = oracle_sampled(w, idx, 1)
    it = torch.from_numpy(idx).cuda()
    assert_bits_equal(to_np(fused.view(z.ZERO_VIEW_MASTER)[it]), ref["master"], "sweep master")
    assert_bits_equal(to_np(fused.view(z.ZERO_VIEW_PARAM, n_ranks - 1)[it]), ref["params"], "sweep params")
    keep = fused.view(z.ZERO_VIEW_MASTER).clone()
    p_last = fused.view(z.ZERO_VIEW_PARAM, n_ranks - 1).clone()
    fused.close()
    del fused
    split, sf = make_opt(w, 2, keep=True)
    split.reduce_scatter(0, split.psi_pad, [reps[r].data_ptr() for r in range(n_ranks)])
    split.adam_shard(-1, 1)
    split.all_gather(0, split.psi_pad)
    assert torch.equal(split.view(z.ZERO_VIEW_MASTER), keep)
    assert torch.equal(split.view(z.ZERO_VIEW_PARAM, n_ranks - 1), p_last)
    split.close()
    del split, reps, keep, p_last
    gc.collect()
    torch.cuda.empty_cache()


# ------------------------------------------------------ checkpoint / re-shard ----

def test_checkpoint_resume_and_reshard():
    """3 ZeRO-2 steps over 8 ranks, export the flat state, import it into a
    ZeRO-3 context over 4 ranks, 2 more steps: every element equals the
    oracle's plain-DP trajectory (8 ranks averaged for steps 1-3, 4 for steps
    4-5).  Resuming at the same N equals the uninterrupted run bit for bit."""
    z = _z()
    numel, layer = W.transformer_layers(2, 128, 512)
    dist = synth.Dist(synth.NORMAL, 1e-2, zero_mod=40)
    hp = W.Hyper(weight_decay=0.01)
    w8 = W.Workload("ckpt-N8", numel, layer, 8, (2,), 65536, dist, W.MASTER_DIST, 3, hp, 0xC4)
    w4 = W.Workload("ckpt-N4", numel, layer, 4, (3,), None, dist, W.MASTER_DIST, 2, hp, 0xC4)
    a, fa = make_opt(w8, 2, bucket=65536)
    ga = grad_fn_for(a, fa)
    for t in range(1, 4):
        a.step(ga)
    state = a.export_state()
    assert state["t"] == 3
    # re-shard: N = 8, stage 2  ->  N = 4, stage 3
    b, fb = make_opt(w4, 3)
    b.import_state(state)
    assert b.t == 3
    gb = grad_fn_for(b, fb)
    for t in range(4, 6):
        st = b.step(gb, stats=True)
        assert st["step"] == t
    # oracle: every real element
    idx = np.concatenate([np.arange(o, o + n) for o, n in zip(b.offsets(), numel)]).astype(np.int64)
    m0 = synth.host_f32_at(W.master_base(w8), idx, W.MASTER_DIST)
    per_step = [np.stack([synth.host_bf16_at(W.grad_base(w8, t, r), idx, dist) for r in range(8)]) for t in (1, 2, 3)]
    per_step += [np.stack([synth.host_bf16_at(W.grad_base(w4, t, r), idx, dist) for r in range(4)]) for t in (4, 5)]
    ref = oracle.trajectory_at(m0, per_step, oracle.AdamHP(**hp.__dict__))
    it = torch.from_numpy(idx).cuda()
    for name, what in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert_bits_equal(to_np(b.view(what)[it]), ref[name], f"re-shard {name}")
    assert_bits_equal(to_np(b.view(z.ZERO_VIEW_PARAM)[it]), ref["params"], "re-shard param shards")
    # same N: resume == uninterrupted
    c, fc = make_opt(w8, 2, bucket=65536)
    c.import_state(state)
    gc_ = grad_fn_for(c, fc)
    for t in (4, 5):
        a.step(ga)
        c.step(gc_)
    for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ):
        assert torch.equal(a.view(what), c.view(what))
    for r in range(8):
        assert torch.equal(a.view(z.ZERO_VIEW_PARAM, r), c.view(z.ZERO_VIEW_PARAM, r))
    for o in (a, b, c):
        o.close()


# ------------------------------------------------------------- clip / skip ----

@pytest.mark.parametrize("stage", [1, 2, 3])
def test_clip_and_overflow_skip_against_oracle(stage):
    """Two-pass step: clip at a norm the gradients exceed, and skip a step
    whose gradients hold an Inf (planted in call 2, rank 1).  Every element,
    every step's statistics, and the step counter against the oracle."""
    z = _z()
    numel, layer = W.transformer_layers(2, 64, 256)
    n_ranks, bucket, clip = 4, 8192, 0.05
    dist = synth.Dist(synth.NORMAL, 1e-2, zero_mod=11)
    hp = W.Hyper(weight_decay=0.01)
    w = W.Workload("clip", numel, layer, n_ranks, (stage,), bucket, dist, W.MASTER_DIST, 3, hp, 0xC1 + stage)
    p = oracle.plan(numel, layer, n_ranks, bucket)
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)

    def host_grad(k, r):
        g = W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, k, r), dist)
        if k == 2 and r == 1:
            g[7] = 0x7F80
        return g

    ranks, reps = oracle.run(p, STAGE_OF[stage], m0, host_grad, 3, oracle.AdamHP(**hp.__dict__),
                             clip_norm=clip, skip_nonfinite=True)
    assert [r.skipped for r in reps] == [False, True, False] and reps[0].coef < 1.0
    opt = z.ZeroOptimizer(numel, layer, n_ranks, stage, bucket_elems=bucket, hparams=_hp(w))
    opt.load_master(torch.from_numpy(m0).cuda())
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
        assert st["grad_norm"] == rep.grad_norm or math.isclose(
            st["grad_norm"], rep.grad_norm, rel_tol=norm_tol(p.psi_pad))
    assert opt.t == 2
    ref = oracle.full_view(p, STAGE_OF[stage], ranks)
    for name, what in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert_bits_equal(to_np(opt.view(what)), ref[name], f"clip stage {stage} {name}")
    for r in (range(n_ranks) if stage != 3 else [0]):
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM, r)), ref["params"], f"clip stage {stage} params {r}")
    if stage == 3:  # the update pass's layers in one launch: the buffers end with the first layer
        _, lo0, hi0 = opt.layers()[0]
        for r in range(n_ranks):
            assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GATHER, r))[: hi0 - lo0], ref["params"][lo0:hi0],
                              f"clip stage 3 last gathered layer, rank {r}")
    opt.close()


@pytest.mark.parametrize("layered", [True, False])
def test_clipped_zero3_update_pass_layered_equals_per_layer(layered):
    """The clipped stage-3 step's update pass, every layer in one cooperative
    launch (layered) or one launch per layer, on unequal layers: states,
    parameter shards and every rank's layer buffers against the oracle, bit
    for bit, over two steps whose norms are clipped."""
    z = _z()
    numel, layer = [1_000_000, 3_000_000, 500_000, 2_000_000], [0, 1, 2, 3]
    n_ranks, clip = 8, 0.05
    w = W.Workload("clip-layered", numel, layer, n_ranks, (3,), 1 << 30, synth.Dist(synth.NORMAL, 1e-2, zero_mod=7),
                   W.MASTER_DIST, 2, W.Hyper(weight_decay=0.01), 0xC7)
    p = oracle.plan(numel, layer, n_ranks, 1 << 30)
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)

    def g(t, r):
        return W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, t, r), w.grad_dist)

    ranks, reps = oracle.run(p, oracle.STAGE_Z3, m0, g, 2, oracle.AdamHP(**w.hyper.__dict__), clip_norm=clip,
                             skip_nonfinite=True)
    assert all(r.coef < 1.0 for r in reps)
    ref = oracle.full_view(p, oracle.STAGE_Z3, ranks)
    opt, fill = make_opt(w, 3, bucket=1 << 30)
    opt.set_clip(clip, True)
    opt.set_layered(layered)
    s = torch.cuda.current_stream().cuda_stream
    for t in (1, 2):
        rp = torch.empty((n_ranks, opt.psi_pad), dtype=torch.int16, device="cuda")
        for r in range(n_ranks):
            fill.grads_into(t, r, 0, opt.psi_pad, rp[r].data_ptr(), rp[r], s)
        before = opt.launch_count()
        st = opt.step_resident(list(rp), stats=True)
        # begin, pass 1 (one launch), decision, pass 2 (one or four launches)
        assert opt.launch_count() - before == 3 + (1 if layered else len(numel))
        assert st["clip_coef"] == reps[t - 1].coef
    for name, what in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert_bits_equal(to_np(opt.view(what)), ref[name], f"clipped layered={layered} {name}")
    assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM)), ref["params"], f"clipped layered={layered} shards")
    width = max(hi - lo for _, lo, hi in opt.layers())
    want = np.zeros(width, dtype=ref["params"].dtype)
    done = np.zeros(width, dtype=bool)
    for _, lo, hi in opt.layers():  # flat order = the schedule's last launch first
        fresh = ~done[: hi - lo]
        want[: hi - lo][fresh] = ref["params"][lo:hi][fresh]
        done[: hi - lo] = True
    for r in range(n_ranks):
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GATHER, r))[:width], want, f"clipped layered={layered} buffer {r}")
    opt.close()


@pytest.mark.parametrize("stage", [1, 2, 3])
def test_two_pass_staged_kernels_equal_register_kernels(stage):
    """The clipped step's two passes run staged through shared memory (the
    reduce in chunks of 8 ranks above 16) and on the register path when that
    is asked for: the same bits.
    Small layouts make the shards 8-64 elements long, so a 2048-element tile
    reads the reduced gradient from many owners (stage 1: one copy per owner);
    ragged tails; clip active; 3 steps; both 16-bit formats."""
    z = _z()
    for numel, layer in (([3000, 1, 4100], [0, 1, 2]), ([40, 8, 24], [0, 0, 1]), ([70000], [0])):
        for n_ranks in (1, 2, 3, 5, 8, 16, 17, 40):  # above 16 the reduce streams rank chunks
            for dtype in (z.ZERO_DTYPE_BF16, z.ZERO_DTYPE_F16):
                w = W.Workload("two-pass", numel, layer, n_ranks, (stage,), 16384,
                               synth.Dist(synth.NORMAL, 1e-2, zero_mod=7), W.MASTER_DIST, 3, W.Hyper(weight_decay=0.01),
                               0x500 + n_ranks)
                opts = []
                for kernel in (TMA, REG, BULK):  # BULK: pass 2 with bulk stores
                    o, f = make_opt(w, stage, bucket=16384, kernel=kernel, dtype=dtype)
                    o.set_clip(0.01, True)
                    opts.append((o, f))
                for t in range(1, 4):
                    sts = [o.step(grad_fn_for(o, f), stats=True) for o, f in opts]
                    assert sts[0]["clip_coef"] < 1.0
                    for other in sts[1:]:
                        assert sts[0]["nonfinite"] == other["nonfinite"]
                        assert math.isclose(sts[0]["grad_norm"], other["grad_norm"], rel_tol=1e-12)
                (b, _) = opts[1]
                for a, _ in (opts[0], opts[2]):
                    for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ):
                        assert torch.equal(a.view(what), b.view(what)), (numel, n_ranks, stage, what)
                    for r in range(n_ranks if stage != 3 else 1):
                        assert torch.equal(a.view(z.ZERO_VIEW_PARAM, r), b.view(z.ZERO_VIEW_PARAM, r))
                if stage == 1:
                    for r in range(n_ranks):
                        assert torch.equal(a.view(z.ZERO_VIEW_GRAD_BUF, r), b.view(z.ZERO_VIEW_GRAD_BUF, r))
                else:
                    assert torch.equal(a.view(z.ZERO_VIEW_GRAD_SHARD), b.view(z.ZERO_VIEW_GRAD_SHARD))
                for o, _ in opts:
                    o.close()


@pytest.mark.parametrize("stage", [1, 2, 3])
def test_clipped_steps_back_to_back_without_statistics(stage):
    """The clipped step's decision is taken on the device, so steps issued
    back to back without reading statistics never wait on the host; the state,
    the step count (a skipped step, call 2, does not advance it) and the last
    statistics equal those of steps read one at a time."""
    z = _z()
    numel, layer = W.transformer_layers(2, 64, 256)
    n_ranks, bucket = 4, 8192
    dist = synth.Dist(synth.NORMAL, 1e-2, zero_mod=11)
    w = W.Workload("clip-async", numel, layer, n_ranks, (stage,), bucket, dist, W.MASTER_DIST, 4,
                   W.Hyper(weight_decay=0.01), 0xCA + stage)
    p = oracle.plan(numel, layer, n_ranks, bucket)

    def host_grad(k, r):
        g = W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, k, r), dist)
        if k == 2 and r == 1:
            g[7] = 0x7F80
        return g

    dev = {k: [torch.from_numpy(host_grad(k, r).view(np.int16)).cuda() for r in range(n_ranks)] for k in range(1, 5)}
    opts = []
    for _ in range(2):
        o, _f = make_opt(w, stage, bucket=bucket)
        o.set_clip(0.05, True)
        opts.append(o)
    a, b = opts
    for k in range(1, 5):
        sa = a.step_resident([x.clone() for x in dev[k]], stats=True)
        b.step_resident([x.clone() for x in dev[k]])           # no statistics: nothing waits
        if k == 2:
            assert sa["skipped"] == 1
    assert b.t == a.t == 3
    assert b.read_stats() == a.read_stats()
    for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ):
        assert torch.equal(a.view(what), b.view(what))
    for r in range(n_ranks if stage != 3 else 1):
        assert torch.equal(a.view(z.ZERO_VIEW_PARAM, r), b.view(z.ZERO_VIEW_PARAM, r))
    a.close()
    b.close()


@pytest.mark.parametrize("stage", [2, 3])
@pytest.mark.parametrize("clip", [False, True])
def test_resident_step_captured_in_a_cuda_graph(stage, clip):
    """A step enqueues only kernels (its scalars come from the device step
    counter), so it can be captured once in a CUDA graph and replayed: four
    replays equal four eager steps bit for bit -- the fused step and the
    clipped two-pass step -- and the device step counter advances with each."""
    z = _z()
    numel, layer = W.transformer_layers(3, 64, 256)
    w = W.Workload("graph", numel, layer, 4, (stage,), 16384, synth.Dist(synth.NORMAL, 1e-2), W.MASTER_DIST, 1,
                   W.Hyper(weight_decay=0.01), 0xD7 + stage)
    p = oracle.plan(numel, layer, 4, 16384)
    host = [W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, 1, r), w.grad_dist) for r in range(4)]
    a, _ = make_opt(w, stage, bucket=16384)
    b, _ = make_opt(w, stage, bucket=16384)
    if clip:
        a.set_clip(0.05, True)
        b.set_clip(0.05, True)
    ga = [torch.from_numpy(h.view(np.int16)).cuda() for h in host]
    gb = [x.clone() for x in ga]
    torch.cuda.synchronize()
    for _ in range(4):
        a.step_resident(ga)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        b.step_resident(gb)
    assert b.t == 0  # capturing runs nothing
    for _ in range(4):
        g.replay()
    torch.cuda.synchronize()
    assert a.t == b.t == 4
    assert a.read_stats() == b.read_stats()
    for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ):
        assert torch.equal(a.view(what), b.view(what))
    for r in range(4 if stage != 3 else 1):
        assert torch.equal(a.view(z.ZERO_VIEW_PARAM, r), b.view(z.ZERO_VIEW_PARAM, r))
    del g
    a.close()
    b.close()


def test_inactive_clip_two_pass_equals_fused_step():
    z = _z()
    numel, layer = W.transformer_layers(2, 64, 256)
    w = W.Workload("clip-off", numel, layer, 8, (2,), 16384, synth.Dist(synth.NORMAL, 1e-2), W.MASTER_DIST, 3,
                   W.Hyper(), 0xC9)
    a, fa = make_opt(w, 2, bucket=16384)
    b, fb = make_opt(w, 2, bucket=16384)
    b.set_clip(1e9, True)
    ga, gb = grad_fn_for(a, fa), grad_fn_for(b, fb)
    for _ in range(3):
        sa = a.step(ga, stats=True)
        sb = b.step(gb, stats=True)
        assert sb["clip_coef"] == 1.0 and not sb["skipped"]
        assert math.isclose(sa["grad_norm"], sb["grad_norm"], rel_tol=1e-12)
    for what in (z.ZERO_VIEW_MASTER, z.ZERO_VIEW_EXP_AVG, z.ZERO_VIEW_EXP_AVG_SQ):
        assert torch.equal(a.view(what), b.view(what))
    for r in range(8):
        assert torch.equal(a.view(z.ZERO_VIEW_PARAM, r), b.view(z.ZERO_VIEW_PARAM, r))
    a.close()
    b.close()
