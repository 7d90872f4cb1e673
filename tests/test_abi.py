"""CPU tests of the C-ABI library: it loads, exports every function the
header declares, and its host-side planning and validation agree with the
oracle's independently written plan.  No call here needs a GPU."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
from synth import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zero_sm.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[a-z_][\w\s\*]*?\b(zero_\w+)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if not n.endswith("_fn")))


def test_library_loads_and_exports_every_declared_symbol():
    import zero_sharded_optimizer_sm_b200 as z

    declared = _declared_functions()
    assert len(declared) >= 20, declared
    lib = ctypes.CDLL(z.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in zero_sm.h but not exported"
    assert z.zero_version() == 3
    # and the binding exposes the same names
    for name in declared:
        assert callable(getattr(z, name)), name


def test_exported_symbols_are_exactly_the_header():
    import zero_sharded_optimizer_sm_b200 as z

    out = subprocess.run(["nm", "-D", "--defined-only", z.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = sorted(set(re.findall(r"\bT (zero_\w+)$", out, flags=re.M)))
    assert exported == _declared_functions()


def _init(numel, layer, n_ranks, stage, bucket):
    import zero_sharded_optimizer_sm_b200 as z

    n = len(numel)
    lay = z.zero_layout(n, (ctypes.c_int64 * n)(*numel), (ctypes.c_int32 * n)(*layer))
    ctx = ctypes.c_void_p()
    st = z.zero_init(ctypes.byref(lay), n_ranks, stage, bucket, ctypes.byref(ctx))
    return st, ctx


def _plan_of(ctx):
    import zero_sharded_optimizer_sm_b200 as z

    sizes = z.zero_sizes()
    assert z.zero_buffer_sizes(ctx, ctypes.byref(sizes)) == 0
    n = ctypes.c_int32()
    z.zero_buckets(ctx, None, 0, ctypes.byref(n))
    bk = (ctypes.c_int64 * (2 * n.value))()
    assert z.zero_buckets(ctx, bk, n.value, ctypes.byref(n)) == 0
    z.zero_layers(ctx, None, 0, ctypes.byref(n))
    ly = (ctypes.c_int64 * (3 * n.value))()
    assert z.zero_layers(ctx, ly, n.value, ctypes.byref(n)) == 0
    return sizes, [(bk[2 * k], bk[2 * k + 1]) for k in range(len(bk) // 2)], \
        [(int(ly[3 * k]), ly[3 * k + 1], ly[3 * k + 2]) for k in range(len(ly) // 3)]


LAYOUTS = [
    ([1], [0]),
    ([5, 3], [0, 1]),
    ([33, 1, 2, 17], [0, 1, 1, 2]),
    ([7, 0, 11, 13, 2], [0, 0, 1, 2, 2]),
    W.transformer_layers(3, 24, 96),
    ([100], [0]),
    ([16, 0, 24, 0], [0, 1, 2, 3]),  # empty layers (all-zero tensors), first in reverse order at N = 1, 5
]


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("n_ranks", [1, 2, 3, 4, 8, 9, 64, 128])
@pytest.mark.parametrize("bucket", [8, 16, 24, 200, 1 << 20])
def test_planner_matches_oracle_plan(layout, n_ranks, bucket):
    import zero_sharded_optimizer_sm_b200 as z

    numel, layer = layout
    for stage in (1, 2, 3):
        st, ctx = _init(numel, layer, n_ranks, stage, bucket)
        assert st == 0
        try:
            sizes, buckets, layers = _plan_of(ctx)
            p = oracle.plan(numel, layer, n_ranks, bucket)
            assert (sizes.psi, sizes.psi_pad, sizes.shard) == (p.psi, p.psi_pad, p.shard)
            assert buckets == p.buckets
            assert layers == p.layers
            offs = (ctypes.c_int64 * len(numel))()
            assert z.zero_tensor_offsets(ctx, offs, len(numel)) == 0
            assert list(offs) == p.offset
            for r in (0, n_ranks - 1):
                got = (ctypes.c_int64 * 3)()
                assert z.zero_state_bytes(ctx, r, got) == 0
                assert tuple(got) == oracle.state_bytes(p, stage)
            ce = (ctypes.c_int64 * 3)()
            assert z.zero_comm_elems(ctx, ce) == 0
            want = oracle.comm_elems(p, stage)
            assert tuple(ce) == (want["all_reduce"], want["reduce_scatter"], want["all_gather"])
            # arena sizes cover what each stage keeps
            ab = list(sizes.arena_bytes)
            assert ab[z.ZERO_ARENA_STATES] >= 12 * p.psi_pad
            assert ab[z.ZERO_ARENA_SCRATCH] > 0
            if stage in (1, 2):
                assert ab[z.ZERO_ARENA_PARAMS] >= 2 * p.psi_pad * n_ranks
            else:
                assert ab[z.ZERO_ARENA_PARAMS] >= 2 * p.psi_pad
                assert ab[z.ZERO_ARENA_GATHER] >= 2 * n_ranks * max(hi - lo for _, lo, hi in p.layers)
            if stage == 2:
                assert ab[z.ZERO_ARENA_GRADS] >= 2 * n_ranks * max(hi - lo for lo, hi in p.buckets)
            if all(a % 256 == 0 for a in ab):
                pass
        finally:
            z.zero_destroy(ctx)


@pytest.mark.parametrize("stage", [1, 2, 3])
def test_pipeline_option_doubles_only_the_slot_arenas(stage):
    """ZERO_OPT_PIPELINE (set before binding): a second gradient slot set at
    stage 2/3 and a second gather slot set at stage 3; stage 1 and every other
    arena unchanged."""
    import zero_sharded_optimizer_sm_b200 as z

    numel, layer = W.transformer_layers(3, 24, 96)
    sizes = []
    for pipe in (0, 1):
        st, ctx = _init(numel, layer, 4, stage, 4096)
        assert st == 0
        try:
            assert z.zero_set_option(ctx, z.ZERO_OPT_PIPELINE, pipe) == 0
            zs = z.zero_sizes()
            assert z.zero_buffer_sizes(ctx, ctypes.byref(zs)) == 0
            sizes.append(list(zs.arena_bytes))
        finally:
            z.zero_destroy(ctx)
    off, on = sizes
    for k in range(z.ZERO_NUM_ARENAS):
        doubled = (k == z.ZERO_ARENA_GRADS and stage != 1) or (k == z.ZERO_ARENA_GATHER and stage == 3)
        assert on[k] == (2 * off[k] if doubled else off[k]), (k, off[k], on[k])


@pytest.mark.parametrize("stage", [1, 2, 3])
@pytest.mark.parametrize("extra", [{}, {"pipe": 1, "pad": 512}, {"keep": 0}])
def test_guard_option_adds_a_tail_to_every_arena_in_use(stage, extra):
    """ZERO_OPT_GUARD (before binding) grows every arena in use by its
    256-byte tail and leaves the rows' pitches alone; unused arenas stay 0."""
    import zero_sharded_optimizer_sm_b200 as z

    numel, layer = W.transformer_layers(3, 24, 96)
    got = []
    for guard in (0, 1, 2):
        st, ctx = _init(numel, layer, 4, stage, 4096)
        assert st == 0
        try:
            if "pipe" in extra:
                assert z.zero_set_option(ctx, z.ZERO_OPT_PIPELINE, extra["pipe"]) == 0
            if "pad" in extra:
                assert z.zero_set_option(ctx, z.ZERO_OPT_REPLICA_PAD, extra["pad"]) == 0
            if "keep" in extra:
                assert z.zero_set_option(ctx, z.ZERO_OPT_KEEP_GRAD_SHARDS, extra["keep"]) == 0
            assert z.zero_set_option(ctx, z.ZERO_OPT_GUARD, guard) == 0
            zs = z.zero_sizes()
            assert z.zero_buffer_sizes(ctx, ctypes.byref(zs)) == 0
            got.append((list(zs.arena_bytes), zs.replica_pitch))
        finally:
            z.zero_destroy(ctx)
    (off, pitch0), (on1, pitch1), (on2, pitch2) = got
    assert pitch0 == pitch1 == pitch2
    assert on1 == on2
    for k in range(z.ZERO_NUM_ARENAS):
        assert on1[k] == (off[k] + 256 if off[k] else 0), (k, off[k], on1[k])


def test_guard_and_nvtx_option_values_and_the_check_without_a_device():
    """ZERO_OPT_GUARD takes 0, 1 or 2 and ZERO_OPT_NVTX any value at any
    time; zero_check_guards refuses a context without guard bytes or not yet
    bound, before any device work, and leaves {0, -1, -1}."""
    import zero_sharded_optimizer_sm_b200 as z

    st, ctx = _init([100, 28], [0, 1], 2, 2, 64)
    assert st == 0
    try:
        out = (ctypes.c_int64 * 3)(7, 7, 7)
        assert z.zero_check_guards(ctx, None, out) == z.ZERO_ESTATE and list(out) == [0, -1, -1]
        assert b"ZERO_OPT_GUARD" in z.zero_last_error(ctx)
        assert z.zero_set_option(ctx, z.ZERO_OPT_GUARD, 3) == z.ZERO_EINVAL
        assert z.zero_set_option(ctx, z.ZERO_OPT_GUARD, -1) == z.ZERO_EINVAL
        assert z.zero_set_option(ctx, z.ZERO_OPT_GUARD, 2) == z.ZERO_OK
        assert z.zero_check_guards(ctx, None, out) == z.ZERO_ESTATE  # not bound
        assert b"armed" in z.zero_last_error(ctx)
        assert z.zero_check_guards(ctx, None, None) == z.ZERO_ESTATE
        for v in (1, 0, 5):
            assert z.zero_set_option(ctx, z.ZERO_OPT_NVTX, v) == z.ZERO_OK
    finally:
        z.zero_destroy(ctx)
    assert z.zero_check_guards(None, None, None) == z.ZERO_EINVAL


def test_pipeline_streams_and_option_values_on_the_host():
    """zero_set_pipeline_streams needs no GPU before the first pipelined step
    (it only records the handles); ZERO_OPT_PIPELINE takes 0, 1 or 2."""
    import zero_sharded_optimizer_sm_b200 as z

    st, ctx = _init([64, 64], [0, 1], 2, 3, 64)
    assert st == 0
    try:
        assert z.zero_set_pipeline_streams(ctx, None, None) == z.ZERO_OK
        assert z.zero_set_pipeline_streams(ctx, 0x1000, None) == z.ZERO_OK
        assert z.zero_set_pipeline_streams(None, None, None) == z.ZERO_EINVAL
        for v in (0, 1, 2):
            assert z.zero_set_option(ctx, z.ZERO_OPT_PIPELINE, v) == z.ZERO_OK
        assert z.zero_set_option(ctx, z.ZERO_OPT_PIPELINE, 3) == z.ZERO_EINVAL
        assert z.zero_set_option(ctx, z.ZERO_OPT_PDL, 0) == z.ZERO_OK
    finally:
        z.zero_destroy(ctx)


def test_launch_count_starts_at_zero_and_refused_calls_launch_nothing():
    """zero_launch_count is a host counter: 0 after zero_init, unchanged by
    calls that are refused before any launch, EINVAL for NULL arguments."""
    import zero_sharded_optimizer_sm_b200 as z

    st, ctx = _init([64, 64], [0, 1], 4, 2, 64)
    assert st == 0
    try:
        n = ctypes.c_int64(-1)
        assert z.zero_launch_count(ctx, ctypes.byref(n)) == z.ZERO_OK and n.value == 0
        assert z.zero_reduce_scatter(ctx, 0, 64, None, None) == z.ZERO_ESTATE
        assert z.zero_adam_shard(ctx, -1, 1, None) == z.ZERO_ESTATE
        assert z.zero_launch_count(ctx, ctypes.byref(n)) == z.ZERO_OK and n.value == 0
        assert z.zero_launch_count(ctx, None) == z.ZERO_EINVAL
        assert z.zero_launch_count(None, ctypes.byref(n)) == z.ZERO_EINVAL
    finally:
        z.zero_destroy(ctx)


def test_init_rejects_bad_arguments():
    import zero_sharded_optimizer_sm_b200 as z

    assert _init([8], [0], 0, 2, 8)[0] == z.ZERO_EINVAL            # no ranks
    assert _init([8], [0], 129, 2, 8)[0] == z.ZERO_EINVAL          # beyond the rank limit
    assert _init([8], [0], 2, 4, 8)[0] == z.ZERO_EINVAL            # no such stage
    assert _init([8], [0], 2, 0, 8)[0] == z.ZERO_ENOTIMPL          # plain DP is oracle-only
    assert _init([8], [0], 2, 2, 12)[0] == z.ZERO_EINVAL           # bucket not a multiple of 8
    assert _init([8], [0], 2, 2, -8)[0] == z.ZERO_EINVAL           # negative bucket (0 = one bucket)
    assert _init([8, 8], [1, 0], 2, 2, 8)[0] == z.ZERO_EINVAL      # decreasing layer ids
    assert b"non-decreasing" in z.zero_last_error(None)
    assert _init([8, -1], [0, 0], 2, 2, 8)[0] == z.ZERO_EINVAL     # negative size
    assert b"negative" in z.zero_last_error(None)
    ctx = ctypes.c_void_p()
    assert z.zero_init(None, 2, 2, 8, ctypes.byref(ctx)) == z.ZERO_EINVAL
    assert z.zero_init(None, 2, 2, 8, None) == z.ZERO_EINVAL


def test_calls_out_of_order_and_bad_pointers_fail_cleanly():
    import zero_sharded_optimizer_sm_b200 as z

    st, ctx = _init([64, 64], [0, 1], 4, 2, 64)
    assert st == 0
    try:
        # nothing bound: every device call refuses with ZERO_ESTATE
        assert z.zero_reduce_scatter(ctx, 0, 64, None, None) == z.ZERO_ESTATE
        assert z.zero_adam_shard(ctx, -1, 1, None) == z.ZERO_ESTATE
        assert z.zero_all_gather(ctx, 0, 64, None, None) == z.ZERO_ESTATE
        assert z.zero_step(ctx, z.zero_grad_fn(), None, z.zero_gather_fn(), None, None, None) == z.ZERO_ESTATE
        assert z.zero_load_master(ctx, None, None) == z.ZERO_ESTATE
        assert b"not bound" in z.zero_last_error(ctx)
        # options are validated
        assert z.zero_set_option(ctx, z.ZERO_OPT_REPLICA_PAD, 100) == z.ZERO_EINVAL
        assert z.zero_set_option(ctx, 99, 1) == z.ZERO_EINVAL
        assert z.zero_set_option(ctx, z.ZERO_OPT_REPLICA_PAD, 512) == 0
        # bind validates the pointers before touching the device
        arenas = (ctypes.c_void_p * z.ZERO_NUM_ARENAS)(*([0x1000] * z.ZERO_NUM_ARENAS))
        arenas[z.ZERO_ARENA_STATES] = 0x1010  # not 256-byte aligned
        assert z.zero_bind(ctx, arenas) == z.ZERO_EINVAL
        arenas[z.ZERO_ARENA_STATES] = None
        assert z.zero_bind(ctx, arenas) == z.ZERO_EINVAL
        assert z.zero_bind(ctx, None) == z.ZERO_EINVAL
        hp = z.zero_adam_hparams(1e-3, 1.0, 0.999, 1e-8, 0.0)  # beta1 = 1 is out of range
        assert z.zero_set_hparams(ctx, ctypes.byref(hp)) == z.ZERO_EINVAL
        hp = z.zero_adam_hparams(1e-3, 0.9, 0.999, 1e-8, 0.0)
        assert z.zero_set_hparams(ctx, ctypes.byref(hp)) == 0
        v = ctypes.c_void_p()
        n = ctypes.c_int64()
        assert z.zero_view(ctx, z.ZERO_VIEW_MASTER, 0, ctypes.byref(v), ctypes.byref(n)) == z.ZERO_ESTATE
        assert z.zero_state_bytes(ctx, 4, (ctypes.c_int64 * 3)()) == z.ZERO_EINVAL
    finally:
        z.zero_destroy(ctx)
    z.zero_destroy(None)


def test_planner_matches_oracle_plan_on_random_layouts():
    """Seeded random parameter lists (1-12 tensors, zero-size ones included,
    random layer grouping), N in 1..128 and any bucket that is a multiple of
    8: the library's flat offsets, padding, shard size, layer spans and
    bucket schedule equal the oracle's."""
    from hypothesis import given, settings
    from hypothesis import strategies as st

    import zero_sharded_optimizer_sm_b200 as z

    @st.composite
    def layouts(draw):
        n = draw(st.integers(1, 12))
        numel = draw(st.lists(st.one_of(st.just(0), st.integers(1, 5000)), min_size=n, max_size=n))
        if sum(numel) == 0:
            numel[0] = draw(st.integers(1, 64))
        steps = draw(st.lists(st.booleans(), min_size=n, max_size=n))
        layer, cur = [], 0
        for k in range(n):
            cur += 1 if (k and steps[k]) else 0
            layer.append(cur)
        return numel, layer

    @settings(max_examples=300, deadline=None, derandomize=True)
    @given(layouts(), st.integers(1, 128), st.integers(1, 2500).map(lambda b: 8 * b), st.integers(1, 3))
    def check(layout, n_ranks, bucket, stage):
        numel, layer = layout
        status, ctx = _init(numel, layer, n_ranks, stage, bucket)
        assert status == 0
        try:
            sizes, buckets, layers = _plan_of(ctx)
            p = oracle.plan(numel, layer, n_ranks, bucket)
            assert (sizes.psi, sizes.psi_pad, sizes.shard) == (p.psi, p.psi_pad, p.shard)
            assert buckets == p.buckets and layers == p.layers
            offs = (ctypes.c_int64 * len(numel))()
            assert z.zero_tensor_offsets(ctx, offs, len(numel)) == 0
            assert list(offs) == p.offset
        finally:
            z.zero_destroy(ctx)

    check()


@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("n_ranks", [1, 3, 8, 64])
def test_bucket_zero_is_one_bucket_over_the_padded_space(layout, n_ranks):
    """bucket_elems = 0 asks the library for one bucket spanning the padded
    flat space: the same plan as the oracle's with a bucket of psi_pad
    elements (the binding passes 0 when no bucket is given)."""
    import zero_sharded_optimizer_sm_b200 as z

    numel, layer = layout
    for stage in (1, 2, 3):
        st, ctx = _init(numel, layer, n_ranks, stage, 0)
        assert st == 0
        try:
            sizes, buckets, layers = _plan_of(ctx)
            p_any = oracle.plan(numel, layer, n_ranks, 8)
            p = oracle.plan(numel, layer, n_ranks, p_any.psi_pad)
            assert buckets == p.buckets
            assert len(buckets) == 1 and buckets[0][1] - buckets[0][0] <= p.psi_pad
            assert layers == p.layers and sizes.psi_pad == p.psi_pad
            if stage == 2:
                assert sizes.arena_bytes[z.ZERO_ARENA_GRADS] >= 2 * p.psi_pad * n_ranks
        finally:
            z.zero_destroy(ctx)
