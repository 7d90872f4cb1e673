"""Pins for the oracle's partition, collectives and step flows:
 * the ownership partition covers the flat vector exactly once;
 * all-gather inverts the partition; reduce-scatter equals all-reduce then slicing;
 * plain DP keeps every replica identical without a post-update sync;
 * ZeRO-1, ZeRO-2 and ZeRO-3 reproduce plain-DP Adam bit for bit;
 * the bucket size changes the schedule only, never a value;
 * brute force over tiny parameter lists, rank counts and bucket sizes."""
import itertools

import numpy as np
import pytest

import oracle
import synth
from synth import workloads as W

STAGES = (oracle.STAGE_DP, oracle.STAGE_Z1, oracle.STAGE_Z2, oracle.STAGE_Z3)


def _grad_fn(p, seed, dist):
    def fn(t, r):
        return W.host_padded(p.offset, p.numel, p.psi_pad, synth.base(seed, synth.STREAM_GRAD, t, r),
                             dist)
    return fn


def _master0(p, seed):
    return W.host_padded(p.offset, p.numel, p.psi_pad, synth.base(seed, synth.STREAM_MASTER, 0, 0),
                         W.MASTER_DIST, as_f32=True)


def _run_all(p, seed, dist, steps, hp):
    out = {}
    for s in STAGES:
        ranks, reps = oracle.run(p, s, _master0(p, seed), _grad_fn(p, seed, dist), steps, hp)
        out[s] = (ranks, reps)
    return out


def _assert_equivalent(p, res):
    ref = oracle.full_view(p, oracle.STAGE_DP, res[oracle.STAGE_DP][0])
    for s in (oracle.STAGE_Z1, oracle.STAGE_Z2, oracle.STAGE_Z3):
        got = oracle.full_view(p, s, res[s][0])
        for k in ("master", "m", "v", "params", "grad"):
            assert np.array_equal(got[k].view(np.uint8), ref[k].view(np.uint8)), (s, k)
        for a, b in zip(res[s][1], res[oracle.STAGE_DP][1]):
            assert a.nonfinite == b.nonfinite
            assert a.grad_norm == b.grad_norm or (np.isnan(a.grad_norm) and np.isnan(b.grad_norm))
    # ZeRO-1/2: every rank's full parameter replica equals the DP result
    for s in (oracle.STAGE_Z1, oracle.STAGE_Z2):
        for st in res[s][0]:
            assert np.array_equal(st.params, ref["params"])
    # ZeRO-3: every rank's temporary gathered layer equals DP's params there
    reps = res[oracle.STAGE_Z3][1]
    for (lid, lo, hi), tmp in zip(reversed(p.layers), reps[-1].gathered):
        for buf in tmp:
            assert np.array_equal(buf, ref["params"][lo:hi]), lid


def _check_plan(p):
    assert p.psi_pad % (8 * p.n_ranks) == 0 and p.psi_pad >= p.psi
    assert p.shard * p.n_ranks == p.psi_pad
    own = np.full(p.psi_pad, -1)
    for r in range(p.n_ranks):
        lo, hi = p.owned(r)
        assert np.all(own[lo:hi] == -1)
        own[lo:hi] = r
    assert np.all(own >= 0)
    assert all(p.owner(i) == own[i] for i in range(0, p.psi_pad, max(1, p.psi_pad // 97)))
    prev_end = 0
    for off, n, end in zip(p.offset, p.numel, p.slot_end):
        assert off % 8 == 0 and off >= prev_end and off + n <= end and end % 8 == 0
        prev_end = end
    assert p.slot_end[-1] == p.psi_pad
    # buckets: disjoint, in descending order, cover [0, psi_pad), within size
    cover = np.zeros(p.psi_pad, dtype=int)
    last_lo = p.psi_pad
    for lo, hi in p.buckets:
        assert lo % 8 == 0 and hi % 8 == 0 and 0 < hi - lo <= p.bucket_elems
        assert hi <= last_lo
        last_lo = lo
        cover[lo:hi] += 1
    assert np.all(cover == 1)
    # layers are contiguous, in order, and cover everything
    assert p.layers[0][1] == 0 and p.layers[-1][2] == p.psi_pad
    assert all(a[2] == b[1] for a, b in zip(p.layers, p.layers[1:]))


def test_bucket_schedule_worked_example():
    """Hand-worked: tensors of 10, 20, 30, 5 elements on 8-element slots
    [0,16) [16,40) [40,72) [72,80) with N = 2 (psi_pad 80), buffer 32:
    reverse walk -> [72,80) + [40,72) would be 40 > 32 so flush [72,80);
    [40,72) (32) fits alone; [16,40) (24) cannot join it -> flush; [0,16)
    joins [16,40) -> [0,40) is 40 > 32 -> flush [16,40), then [0,16)."""
    p = oracle.plan([10, 20, 30, 5], [0, 0, 1, 1], 2, 32)
    assert p.offset == [0, 16, 40, 72] and p.psi_pad == 80
    assert p.buckets == [(72, 80), (40, 72), (16, 40), (0, 16)]
    # a tensor larger than the buffer is cut into chunks from its end
    q = oracle.plan([100], [0], 1, 32)
    assert q.psi_pad == 104 and q.buckets == [(72, 104), (40, 72), (8, 40), (0, 8)]
    # everything in one buffer
    r = oracle.plan([10, 20, 30, 5], [0, 0, 1, 1], 2, 80)
    assert r.buckets == [(0, 80)]


def test_all_gather_inverts_partition_and_rs_equals_ar_slice():
    rng = np.random.default_rng(21)
    for n_ranks in (1, 2, 3, 4, 7, 8):
        p = oracle.plan([37, 5, 64, 1], [0, 0, 1, 2], n_ranks, 16)
        x = rng.integers(0, 1 << 16, size=p.psi_pad, dtype=np.uint16)
        shards = [x[slice(*p.owned(r))].copy() for r in range(n_ranks)]
        outs = [np.zeros(p.psi_pad, np.uint16) for _ in range(n_ranks)]
        oracle.all_gather(shards, p, 0, p.psi_pad, outs)
        assert all(np.array_equal(o, x) for o in outs)
        grads = [rng.integers(0, 0x3F00, size=p.psi_pad, dtype=np.uint16) for _ in range(n_ranks)]
        rs = [np.zeros(p.shard, np.uint16) for _ in range(n_ranks)]
        for lo, hi in p.buckets:
            oracle.reduce_scatter(grads, p, lo, hi, rs)
        ar = [g.copy() for g in grads]
        oracle.all_reduce(ar, 0, p.psi_pad)
        assert all(np.array_equal(a, ar[0]) for a in ar)
        for r in range(n_ranks):
            assert np.array_equal(rs[r], ar[0][slice(*p.owned(r))])


TINY_LISTS = [
    ([1], [0]),
    ([5, 3], [0, 1]),
    ([8, 16, 9], [0, 0, 1]),
    ([33, 1, 2, 17], [0, 1, 1, 2]),
    ([64], [0]),
    ([7, 0, 11, 13, 2], [0, 0, 1, 2, 2]),
]


@pytest.mark.parametrize("layout", TINY_LISTS)
def test_brute_force_tiny(layout):
    numel, layer = layout
    hp = oracle.AdamHP(lr=1e-2, weight_decay=0.1)
    dist = synth.Dist(synth.NORMAL, 1e-2, zero_mod=7)
    for n_ranks in range(1, 10):
        base_plan = oracle.plan(numel, layer, n_ranks, 8)
        for bucket in sorted({8, 16, 24, base_plan.psi_pad}):
            p = oracle.plan(numel, layer, n_ranks, bucket)
            _check_plan(p)
            res = _run_all(p, 0xB0 + n_ranks, dist, 3, hp)
            _assert_equivalent(p, res)
            # pad elements stay exactly zero in every state
            view = oracle.full_view(p, oracle.STAGE_Z2, res[oracle.STAGE_Z2][0])
            pad = ~p.real_mask()
            for k in ("master", "m", "v", "params", "grad"):
                assert not view[k][pad].any()


def test_bucket_size_changes_no_value():
    numel, layer = W.transformer_layers(2, 16, 64)
    hp = oracle.AdamHP(weight_decay=0.01)
    dist = synth.Dist(synth.NORMAL, 1e-2, zero_mod=100)
    views = []
    for bucket in (8, 16, 24, 200, 1024, 10**6):
        p = oracle.plan(numel, layer, 4, bucket)
        ranks, _ = oracle.run(p, oracle.STAGE_Z2, _master0(p, 77), _grad_fn(p, 77, dist), 3, hp)
        views.append(oracle.full_view(p, oracle.STAGE_Z2, ranks))
    for v in views[1:]:
        for k in v:
            assert np.array_equal(v[k], views[0][k])


def test_dp_replicas_stay_identical_without_sync():
    p = oracle.plan([1000, 24], [0, 1], 5, 64)
    ranks, _ = oracle.run(p, oracle.STAGE_DP, _master0(p, 5), _grad_fn(p, 5, W.Dist(0, 1e-2)), 3,
                          oracle.AdamHP())
    for st in ranks[1:]:
        for k in ("master", "m", "v", "params", "grads"):
            assert np.array_equal(getattr(st, k), getattr(ranks[0], k))


def test_stage_equivalence_flat_1m():
    """The 1,048,576-parameter, N = 4 workload: all four flows agree bitwise."""
    w = W.flat_1m_n4()
    hp = oracle.AdamHP(**w.hyper.__dict__)
    p = oracle.plan(w.numel, w.layer_id, w.n_ranks, 1 << 20)
    res = _run_all(p, w.seed, w.grad_dist, w.steps, hp)
    _assert_equivalent(p, res)


def test_trajectory_at_matches_full_run():
    """Sampled per-element evaluation equals the full literal run."""
    numel, layer = W.transformer_layers(1, 32, 128)
    p = oracle.plan(numel, layer, 3, 256)
    seed, dist, hp = 99, synth.Dist(synth.NORMAL, 1e-2, zero_mod=50), oracle.AdamHP(weight_decay=0.01)
    ranks, _ = oracle.run(p, oracle.STAGE_Z2, _master0(p, seed), _grad_fn(p, seed, dist), 4, hp)
    full = oracle.full_view(p, oracle.STAGE_Z2, ranks)
    idx = np.array(sorted(set(np.random.default_rng(3).integers(0, p.psi_pad, 300).tolist())))
    m0 = _master0(p, seed)[idx]
    gfn = _grad_fn(p, seed, dist)
    per_step = [np.stack([gfn(t, r)[idx] for r in range(p.n_ranks)]) for t in range(1, 5)]
    got = oracle.trajectory_at(m0, per_step, hp)
    for k in ("master", "m", "v", "params", "grad"):
        assert np.array_equal(got[k], full[k][idx]), k
