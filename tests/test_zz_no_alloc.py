"""zero_fused_step_static: the one entry point that allocates nothing.

It is for callers that cannot allocate device memory when they run the step
(their device memory is owned by another allocator, or a cudaMalloc's
possible device synchronisation is not acceptable where they run, or they
keep no context to hold a scratch arena).  Its scratch is a fixed array in the
library's own device memory.  This test calls it through the C ABI and checks
its results against the context-based fused step (zero_step_resident of a
stage-2 context with one bucket) on two calls in a row, within the
tolerances the parity tests use.  The file name makes pytest collect it last.
"""
import ctypes
import gc
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from harness import assert_bf16_close, assert_f32_close, to_np  # noqa: E402

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
