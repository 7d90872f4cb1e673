"""zero_fused_step_static: the one entry point that allocates nothing.

It is for callers that cannot allocate device memory when they run the step
(their device memory is owned by another allocator, or a cudaMalloc's
possible device synchronisation is not acceptable where they run, or they
keep no context to hold a scratch arena).  Its scratch is a fixed array in the
library's own device memory.  These tests call it through the C ABI and check
it, on two calls in a row, against the context-based fused step
(zero_step_resident of a stage-2 context with one bucket) within the
tolerances the parity tests use, and against the CPU oracle's literal ZeRO-2
run bit for bit: at N = 1, 3, 8, 17 and 64 on an interval that is not a
multiple of a CTA's 2048 elements, with and without statistics; on an
interval larger than one pass of the capped grid (the kernel's grid-stride
loop); and with planted infinities and NaNs (the exact non-finite count).
The file name makes pytest collect it last.
"""
import ctypes
import gc
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from harness import assert_bf16_close, assert_f32_close, to_np  # noqa: E402

import oracle  # noqa: E402
import synth  # noqa: E402
from synth import workloads as W  # noqa: E402

pytestmark = pytest.mark.gpu


def _ptrs(ptr_list):
    arr = (ctypes.c_void_p * len(ptr_list))()
    for i, p in enumerate(ptr_list):
        arr[i] = int(p)
    return arr


@pytest.mark.parametrize("n_ranks", [8, 12])
def test_static_scratch_step_matches_context_step_twice(n_ranks):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import zero_sharded_optimizer_sm_b200 as z

    torch.cuda.set_device(0)
    numel, layer = W.transformer_layers(2, 256, 1024)  # 1,584,640 params
    w = W.Workload("no-alloc", numel, layer, n_ranks, (2,), None, synth.Dist(synth.NORMAL, 1e-2, zero_mod=50),
                   W.MASTER_DIST, 2, W.Hyper(weight_decay=0.01), 0xAB0 + n_ranks)
    hp = z.AdamHParams(**w.hyper.__dict__)
    s = torch.cuda.current_stream().cuda_stream
    ref = z.ZeroOptimizer(numel, layer, n_ranks, z.ZERO_STAGE_2, hparams=hp, keep_grad_shards=False,
                          kernel=z.ZERO_KERNEL_REGISTER)
    P = ref.psi_pad
    offs = ref.offsets()
    master0 = torch.zeros(P, dtype=torch.float32, device="cuda")
    for off, n in zip(offs, numel):
        synth.dev_f32(W.master_base(w), off, n, W.MASTER_DIST, master0.data_ptr() + 4 * off, s)
    ref.load_master(master0)
    # the caller's own buffers for the allocation-free entry point
    master = master0.clone()
    m = torch.zeros_like(master)
    v = torch.zeros_like(master)
    params = torch.empty((n_ranks, P), dtype=torch.int16, device="cuda")
    stats = torch.zeros(2, dtype=torch.float64, device="cuda")
    grads = torch.zeros((n_ranks, P), dtype=torch.int16, device="cuda")
    h = z.zero_adam_hparams(hp.lr, hp.beta1, hp.beta2, hp.eps, hp.weight_decay)
    for t in (1, 2):
        for r in range(n_ranks):
            for off, n in zip(offs, numel):
                synth.dev_bf16(W.grad_base(w, t, r), off, n, w.grad_dist, grads[r].data_ptr() + 2 * off, s)
        want = ref.step_resident(list(grads), stats=True)
        st = z.zero_fused_step_static(n_ranks, P, _ptrs([g.data_ptr() for g in grads]), master.data_ptr(),
                                      m.data_ptr(), v.data_ptr(), _ptrs([p.data_ptr() for p in params]),
                                      ctypes.byref(h), t, stats.data_ptr(), s)
        assert st == z.ZERO_OK, z.STATUS_NAMES.get(st, st)
        torch.cuda.synchronize()
        assert_f32_close(to_np(master), to_np(ref.view(z.ZERO_VIEW_MASTER)), f"master, call {t}")
        assert_f32_close(to_np(m), to_np(ref.view(z.ZERO_VIEW_EXP_AVG)), f"m, call {t}")
        assert_f32_close(to_np(v), to_np(ref.view(z.ZERO_VIEW_EXP_AVG_SQ)), f"v, call {t}")
        for r in (0, n_ranks - 1):
            assert_bf16_close(to_np(params[r]), to_np(ref.view(z.ZERO_VIEW_PARAM, r)), f"params {r}, call {t}")
        sq = float(stats[0].item())
        nf = int(stats[1:].view(torch.int64).item())
        assert nf == want["nonfinite"]
        assert math.isclose(math.sqrt(sq), want["grad_norm"], rel_tol=1e-12)
    ref.close()
    del ref, master, m, v, params, grads, stats, master0
    gc.collect()
    torch.cuda.empty_cache()


def test_static_scratch_step_rejects_bad_arguments():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import zero_sharded_optimizer_sm_b200 as z

    buf = torch.zeros(64, dtype=torch.float32, device="cuda")
    g = torch.zeros(64, dtype=torch.int16, device="cuda")
    h = z.zero_adam_hparams(1e-3, 0.9, 0.999, 1e-8, 0.0)
    one = _ptrs([g.data_ptr()])
    s = torch.cuda.current_stream().cuda_stream
    call = lambda n, t=1, hp=h, nr=1: z.zero_fused_step_static(nr, n, one, buf.data_ptr(), buf.data_ptr(),
                                                               buf.data_ptr(), one, ctypes.byref(hp), t, None, s)
    assert call(12) == z.ZERO_EINVAL                  # not a multiple of 8
    assert call(8, t=0) == z.ZERO_EINVAL              # step numbers start at 1
    assert call(8, nr=0) == z.ZERO_EINVAL
    bad = z.zero_adam_hparams(1e-3, 1.5, 0.999, 1e-8, 0.0)
    assert call(8, hp=bad) == z.ZERO_EINVAL
    assert call(0) == z.ZERO_OK                       # an empty interval is a no-op
    torch.cuda.synchronize()


def _bits_or_both_nan(got, ref, what):
    """Equal bit patterns, except that two NaNs match whatever their payloads
    (a NaN's payload is not part of the method's result)."""
    g = np.ascontiguousarray(got)
    r = np.ascontiguousarray(ref)
    if g.dtype == np.float32:
        gn, rn = np.isnan(g), np.isnan(r)
        gb, rb = g.view(np.uint32), r.view(np.uint32)
    else:
        gb, rb = g.view(np.uint16), r.view(np.uint16)
        gn = ((gb & 0x7F80) == 0x7F80) & ((gb & 0x7F) != 0)
        rn = ((rb & 0x7F80) == 0x7F80) & ((rb & 0x7F) != 0)
    ok = (gb == rb) | (gn & rn)
    if not np.all(ok):
        i = int(np.flatnonzero(~ok)[0])
        raise AssertionError(f"{what}: {int((~ok).sum())} elements differ; first at {i}: "
                             f"got {hex(int(gb[i]))} ref {hex(int(rb[i]))}")


def _oracle_and_static(n_ranks, n, seed, plant=None, stats_on=(True, False)):
    """Two calls (t = 1, 2) of the allocation-free step on the caller's own
    buffers, and the oracle's literal ZeRO-2 run of the same flat interval;
    `plant(t, r, host_grad)` may overwrite gradient values on the host."""
    import zero_sharded_optimizer_sm_b200 as z

    w = W.Workload("no-alloc-oracle", [n], [0], n_ranks, (2,), None, synth.Dist(synth.NORMAL, 1e-2, zero_mod=37),
                   W.MASTER_DIST, 2, W.Hyper(lr=2e-3, weight_decay=0.02), seed)
    p = oracle.plan(w.numel, w.layer_id, n_ranks, 1 << 40)
    m0 = W.host_padded(p.offset, p.numel, p.psi_pad, W.master_base(w), W.MASTER_DIST, as_f32=True)

    def g(t, r):
        x = W.host_padded(p.offset, p.numel, p.psi_pad, W.grad_base(w, t, r), w.grad_dist)
        if plant is not None:
            plant(t, r, x)
        return x

    ranks, reps = oracle.run(p, oracle.STAGE_Z2, m0, g, 2, oracle.AdamHP(**w.hyper.__dict__))
    ref = oracle.full_view(p, oracle.STAGE_Z2, ranks)

    hp = z.zero_adam_hparams(w.hyper.lr, w.hyper.beta1, w.hyper.beta2, w.hyper.eps, w.hyper.weight_decay)
    s = torch.cuda.current_stream().cuda_stream
    master = torch.from_numpy(m0[:n].copy()).cuda()
    m = torch.zeros_like(master)
    v = torch.zeros_like(master)
    params = torch.full((n_ranks, n), 0x5555, dtype=torch.int16, device="cuda")
    grads = torch.empty((n_ranks, n), dtype=torch.int16, device="cuda")
    stats = torch.full((2,), float("nan"), dtype=torch.float64, device="cuda")
    got_stats = []
    for t in (1, 2):
        for r in range(n_ranks):
            grads[r].copy_(torch.from_numpy(g(t, r)[:n].view(np.int16)))
        with_stats = stats_on[t - 1]
        st = z.zero_fused_step_static(n_ranks, n, _ptrs([x.data_ptr() for x in grads]), master.data_ptr(),
                                      m.data_ptr(), v.data_ptr(), _ptrs([x.data_ptr() for x in params]),
                                      ctypes.byref(hp), t, stats.data_ptr() if with_stats else None, s)
        assert st == z.ZERO_OK, z.STATUS_NAMES.get(st, st)
        torch.cuda.synchronize()
        if with_stats:
            got_stats.append((float(stats[0].item()), int(stats[1:].view(torch.int64).item())))
        else:
            got_stats.append(None)
    for key, dev in (("master", master), ("m", m), ("v", v)):
        _bits_or_both_nan(to_np(dev), ref[key][:n], f"N={n_ranks} {key}")
    for r in range(n_ranks):
        _bits_or_both_nan(to_np(params[r]).view(np.uint16), ref["params"][:n], f"N={n_ranks} params {r}")
    for t, gs in zip((1, 2), got_stats):
        if gs is None:
            continue
        sq, nf = gs
        assert nf == reps[t - 1].nonfinite, (t, nf, reps[t - 1].nonfinite)
        if nf == 0:
            tol = 2 * p.psi_pad * 2.0**-53 + 1e-15
            assert abs(math.sqrt(sq) - reps[t - 1].grad_norm) <= tol * reps[t - 1].grad_norm
    del master, m, v, params, grads, stats
    return reps


@pytest.mark.parametrize("n_ranks", [1, 3, 8, 17, 64])
def test_static_step_equals_the_oracle_bit_for_bit(n_ranks):
    """10,264 elements (five 2048-element CTA spans and a ragged 24), two calls
    in a row, statistics on the first call and stats_out = NULL on the
    second: master, m, v and every rank's parameters bit for bit."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    _oracle_and_static(n_ranks, 5 * 2048 + 24, 0xAC0 + n_ranks, stats_on=(True, False))


def test_static_step_grid_stride_over_a_long_interval():
    """16,777,216 elements at N = 2: more than the capped grid covers in one
    pass (148 SMs x resident CTAs x 2048 elements), so every CTA loops;
    bit for bit against the oracle, statistics on both calls."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    _oracle_and_static(2, 1 << 24, 0xAD0, stats_on=(True, True))


def test_static_step_counts_planted_nonfinite_values():
    """Infinities, NaNs, opposite infinities in one element and a sum that
    overflows bf16 planted in the ranks' gradients: the exact non-finite
    count of the averaged gradient, and the states (NaN where the oracle's are
    NaN) bit for bit."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)

    def plant(t, r, x):
        if t != 2:
            return
        if r == 1:
            x[100] = 0x7F80           # +inf
        if r == 2:
            x[2000] = 0x7FC1          # NaN
        if r == 0:
            x[5000] = 0x7F80          # +inf ...
        if r == 3:
            x[5000] = 0xFF80          # ... and -inf in the same element: NaN
        x[7000] = 0x7F7F              # the largest finite bf16 on every rank: the sum overflows

    reps = _oracle_and_static(4, 65536, 0xAE0, plant=plant, stats_on=(True, True))
    assert reps[1].nonfinite == 4 and reps[0].nonfinite == 0
