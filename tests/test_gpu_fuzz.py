"""Randomized GPU parity: seeded random combinations of the layout (tensor
sizes including zero-size tensors, layer grouping), N, stage, bucket, 16-bit
format and loss scale, clipping with the overflow skip, the callback
pipeline, programmatic dependent launch and the kernel family, each run for
two steps through the C ABI -- through the gradient callback and from
resident replicas -- and compared with the oracle's literal per-rank run:
fp32 states, parameters and reduced gradients bit for bit, statistics
exactly (the norm within its summation bound)."""
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
N_CASES = 30


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _case(k):
    rng = np.random.default_rng(0xF022 + k)
    n_t = int(rng.integers(1, 7))
    numel = [int(x) if rng.random() > 0.15 else 0 for x in rng.integers(1, 5000, size=n_t)]
    if sum(numel) == 0:
        numel[0] = 8
    layer = np.cumsum(rng.random(n_t) < 0.5).tolist()
    layer = [int(x) - int(layer[0]) for x in layer]
    n_ranks = int(rng.choice([1, 2, 3, 4, 5, 7, 8, 9, 12, 16, 17, 24, 33]))
    stage = int(rng.integers(1, 4))
    p_all = oracle.plan(numel, layer, n_ranks, 1 << 40)
    bucket = int(rng.choice([8, 64, 1000, p_all.psi_pad]))
    f16 = bool(rng.random() < 0.4)
    scale = float(rng.choice([1.0, 256.0])) if f16 else 1.0
    clip = float(rng.choice([0.0, 0.0, 0.02, 1e9]))
    c = dict(numel=numel, layer=layer, n_ranks=n_ranks, stage=stage, bucket=bucket, f16=f16, scale=scale,
             clip=clip, pipeline=int(rng.integers(0, 3)), pdl=bool(rng.random() < 0.5),
             kernel=int(rng.choice([0, 0, 1])), seed=0xF100 + k, tile=0, warps=0)
    # drawn last, so that the fields above stay those of the seed
    if rng.random() < 0.4:
        c["kernel"] = 3  # the bulk-store staged kernel, in one of its built configurations
        pick = int(rng.integers(0, 5))
        if n_ranks <= 16:
            c["tile"], c["warps"] = [(2048, 8), (2048, 16), (1024, 4), (1024, 8), (1024, 16)][pick]
        else:  # the rank-chunked form's configurations
            c["tile"], c["warps"] = [(2048, 8), (1024, 8)][pick % 2]
    return c


@pytest.mark.parametrize("k", range(N_CASES))
def test_random_configuration_against_the_oracle(k):
    import zero_sharded_optimizer_sm_b200 as z

    c = _case(k)
    dist = synth.Dist(synth.NORMAL, 1e-2 * c["scale"], zero_mod=9)
    w = W.Workload("fuzz", c["numel"], c["layer"], c["n_ranks"], (c["stage"],), c["bucket"], dist, W.MASTER_DIST, 2,
                   W.Hyper(lr=1e-2, weight_decay=0.05), c["seed"])
    p = oracle.plan(w.numel, w.layer_id, w.n_ranks, c["bucket"])
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)

    def g(t, r):
        return W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, t, r), dist, f16=c["f16"])

    fmt = oracle.F16 if c["f16"] else oracle.BF16
    ranks, reps = oracle.run(p, STAGE_OF[c["stage"]], m0, g, 2, oracle.AdamHP(**w.hyper.__dict__),
                             clip_norm=c["clip"], skip_nonfinite=c["clip"] > 0, fmt=fmt, loss_scale=c["scale"])
    ref = oracle.full_view(p, STAGE_OF[c["stage"]], ranks)

    opt = z.ZeroOptimizer(w.numel, w.layer_id, w.n_ranks, c["stage"], bucket_elems=c["bucket"],
                          hparams=z.AdamHParams(**w.hyper.__dict__), kernel=c["kernel"], pipeline=c["pipeline"],
                          tma_tile=c["tile"], tma_warps=c["warps"],
                          dtype=z.ZERO_DTYPE_F16 if c["f16"] else z.ZERO_DTYPE_BF16)
    opt.set_pdl(c["pdl"])
    if c["scale"] != 1.0:
        opt.set_loss_scale(c["scale"])
    if c["clip"] > 0:
        opt.set_clip(c["clip"], True)
    fill = DeviceFill(w, opt.offsets(), opt.psi_pad, f16=c["f16"])
    mv = opt.view(z.ZERO_VIEW_MASTER)
    fill.master_into(mv.data_ptr(), mv, torch.cuda.current_stream().cuda_stream)
    opt.load_master(None)

    def gfn(t, lo, hi, bufs, stream):
        for r, ptr in enumerate(bufs):
            fill.grads_into(t, r, lo, hi, ptr, opt._tensor_at(ptr, hi - lo, torch.int16), stream)
        return 0

    for t in (1, 2):
        st = opt.step(gfn, stats=True)
        rep = reps[t - 1]
        assert st["nonfinite"] == rep.nonfinite and st["skipped"] == rep.skipped, c
        if c["clip"] > 0 and not rep.skipped:
            assert st["clip_coef"] == rep.coef, c
        assert st["grad_norm"] == rep.grad_norm or math.isclose(
            st["grad_norm"], rep.grad_norm, rel_tol=2 * p.psi_pad * 2.0**-53 + 1e-15), c
    torch.cuda.synchronize()
    what = f"case {k} {c}"
    for name, v in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert_bits_equal(to_np(opt.view(v)), ref[name], f"{what} {name}")
    for r in (range(w.n_ranks) if c["stage"] != 3 else [0]):
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM, r)), ref["params"], f"{what} params {r}")
    if c["stage"] != 1:
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GRAD_SHARD)), ref["grad"], f"{what} grad shards")
    else:
        for r in range(w.n_ranks):
            assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GRAD_BUF, r)), ranks[r].grads, f"{what} all-reduced {r}")
    opt.close()


@pytest.mark.parametrize("k", range(N_CASES))
def test_random_configuration_resident_against_the_oracle(k):
    """The same seeded configurations stepped from resident replicas
    (zero_step_resident): a stage-3 step on the bulk-store kernel runs as
    one layered launch, a clipped step's first pass as one launch over the
    flat space.  States, parameters and reduced gradients bit for bit, and
    at stage 3 every rank's layer buffers: each byte the parameter of the
    last layer in the schedule long enough to write it."""
    import zero_sharded_optimizer_sm_b200 as z

    c = _case(k)
    dist = synth.Dist(synth.NORMAL, 1e-2 * c["scale"], zero_mod=9)
    w = W.Workload("fuzz", c["numel"], c["layer"], c["n_ranks"], (c["stage"],), c["bucket"], dist, W.MASTER_DIST, 2,
                   W.Hyper(lr=1e-2, weight_decay=0.05), c["seed"])
    p = oracle.plan(w.numel, w.layer_id, w.n_ranks, c["bucket"])
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)

    def g(t, r):
        return W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, t, r), dist, f16=c["f16"])

    fmt = oracle.F16 if c["f16"] else oracle.BF16
    ranks, reps = oracle.run(p, STAGE_OF[c["stage"]], m0, g, 2, oracle.AdamHP(**w.hyper.__dict__),
                             clip_norm=c["clip"], skip_nonfinite=c["clip"] > 0, fmt=fmt, loss_scale=c["scale"])
    ref = oracle.full_view(p, STAGE_OF[c["stage"]], ranks)

    opt = z.ZeroOptimizer(w.numel, w.layer_id, w.n_ranks, c["stage"], bucket_elems=c["bucket"],
                          hparams=z.AdamHParams(**w.hyper.__dict__), kernel=c["kernel"], pipeline=c["pipeline"],
                          tma_tile=c["tile"], tma_warps=c["warps"],
                          dtype=z.ZERO_DTYPE_F16 if c["f16"] else z.ZERO_DTYPE_BF16)
    opt.set_pdl(c["pdl"])
    if c["scale"] != 1.0:
        opt.set_loss_scale(c["scale"])
    if c["clip"] > 0:
        opt.set_clip(c["clip"], True)
    fill = DeviceFill(w, opt.offsets(), opt.psi_pad, f16=c["f16"])
    s = torch.cuda.current_stream().cuda_stream
    mv = opt.view(z.ZERO_VIEW_MASTER)
    fill.master_into(mv.data_ptr(), mv, s)
    opt.load_master(None)
    for t in (1, 2):
        rp = torch.empty((w.n_ranks, opt.psi_pad), dtype=torch.int16, device="cuda")
        for r in range(w.n_ranks):
            fill.grads_into(t, r, 0, opt.psi_pad, rp[r].data_ptr(), rp[r], s)
        st = opt.step_resident(list(rp), stats=True)
        rep = reps[t - 1]
        assert st["nonfinite"] == rep.nonfinite and st["skipped"] == rep.skipped, c
        if c["clip"] > 0 and not rep.skipped:
            assert st["clip_coef"] == rep.coef, c
        assert st["grad_norm"] == rep.grad_norm or math.isclose(
            st["grad_norm"], rep.grad_norm, rel_tol=2 * p.psi_pad * 2.0**-53 + 1e-15), c
    torch.cuda.synchronize()
    what = f"resident case {k} {c}"
    for name, v in (("master", z.ZERO_VIEW_MASTER), ("m", z.ZERO_VIEW_EXP_AVG), ("v", z.ZERO_VIEW_EXP_AVG_SQ)):
        assert_bits_equal(to_np(opt.view(v)), ref[name], f"{what} {name}")
    for r in (range(w.n_ranks) if c["stage"] != 3 else [0]):
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_PARAM, r)), ref["params"], f"{what} params {r}")
    if c["stage"] != 1:
        assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GRAD_SHARD)), ref["grad"], f"{what} grad shards")
    else:  # the all-reduce written back into the resident replicas
        for r in range(w.n_ranks):
            assert_bits_equal(to_np(rp[r]), ranks[r].grads, f"{what} all-reduced {r}")
    if c["stage"] == 3:
        layers = [(lo, hi) for _, lo, hi in opt.layers() if hi > lo]
        width = max(hi - lo for lo, hi in layers)
        want = np.zeros(width, dtype=ref["params"].dtype)
        done = np.zeros(width, dtype=bool)
        for lo, hi in layers:  # flat order = the schedule's last launch first
            fresh = ~done[: hi - lo]
            want[: hi - lo][fresh] = ref["params"][lo:hi][fresh]
            done[: hi - lo] = True
        for r in range(w.n_ranks):
            assert_bits_equal(to_np(opt.view(z.ZERO_VIEW_GATHER, r))[:width], want, f"{what} layer buffer {r}")
    opt.close()
