"""Pins for the oracle's prefix-cache simulator (transcript cues 11, 13, 35)."""
import numpy as np
import pytest

from conftest import read_golden


def _run(oracle_mod, cap, accesses, L=1, E=8):
    """accesses: list of (layer, expert, depth, batch)."""
    a = np.array(accesses, dtype=np.int64)
    return oracle_mod.cache_sim_prefix(L, E, cap, a[:, 0], a[:, 1], a[:, 2], a[:, 3])


def test_golden_topup_and_no_io(oracle_mod):
    for r, b, read, after in read_golden("cache_trace_examples.txt"):
        r, b, after = int(r), int(b), int(after)
        expect_read = [] if read == "-" else [int(p) for p in read.split(",")]
        before, log, fetched = _run(oracle_mod, 64, [(0, 0, r, 0), (0, 0, b, 1)])
        assert before[1] == r
        assert fetched - r == len(expect_read)
        # planes read are r+1..b (1-based), exactly the missing suffix
        assert list(range(r + 1, max(r, b) + 1)) == expect_read
        _, _, f2 = _run(oracle_mod, 64, [(0, 0, r, 0), (0, 0, b, 1), (0, 0, after, 2)])
        assert f2 == fetched  # resident depth after the access is `after`
        assert len(log) == 0


def test_eviction_takes_deepest_planes_first(oracle_mod):
    # A at 3 bits, B at 2 bits fill 5 planes; C needs 2 more -> A's planes 2 and 1 go
    before, log, fetched = _run(oracle_mod, 5, [(0, 0, 3, 0), (0, 1, 2, 1), (0, 2, 2, 2)])
    assert list(log) == [0 * 8 + 2, 0 * 8 + 1]
    assert fetched == 7


def test_refresh_covers_only_the_requested_prefix(oracle_mod):
    # A at 4 (t=0), B at 2 (t=1), A again at 2 (t=2): A's planes 0-1 are refreshed, 2-3 keep t=0
    acc = [(0, 0, 4, 0), (0, 1, 2, 1), (0, 0, 2, 2), (0, 2, 3, 3)]
    before, log, fetched = _run(oracle_mod, 7, acc)
    assert list(before) == [0, 0, 4, 0]
    assert list(log) == [3, 2]          # A's deepest planes age out before B's
    # now A is back at depth 2; a request for 3 tops up one plane only
    before2, _, fetched2 = _run(oracle_mod, 7, acc + [(0, 0, 3, 4)])
    assert before2[-1] == 2


def test_current_batch_is_not_evicted(oracle_mod):
    # capacity 4: A(2) and B(2) in the same batch; C(2) in that batch cannot fit
    with pytest.raises(ValueError):
        _run(oracle_mod, 4, [(0, 0, 2, 0), (0, 1, 2, 0), (0, 2, 2, 0)])
    before, log, _ = _run(oracle_mod, 4, [(0, 0, 2, 0), (0, 1, 2, 0), (0, 2, 2, 1)])
    assert list(log) == [1, 0]


def test_invariants_on_random_trace(oracle_mod):
    rng = np.random.default_rng(0)
    L, E, n = 4, 32, 3000
    lay = rng.integers(0, L, n)
    exp_ = rng.integers(0, E, n)
    dep = rng.integers(1, 9, n)
    bat = np.arange(n)
    cap = 200
    before, log, fetched = oracle_mod.cache_sim_prefix(L, E, cap, lay, exp_, dep, bat)
    # every fetch is the missing suffix: planes fetched = sum max(0, b - r)
    assert fetched == int(np.maximum(0, dep - before.astype(int)).sum())
    # replay resident depths from the log and check capacity and prefix shape
    depth = np.zeros(L * E, int)
    ev = iter(log)
    for a in range(n):
        x = lay[a] * E + exp_[a]
        assert depth[x] == before[a]
        need = max(0, dep[a] - depth[x])
        while depth.sum() + need > cap:
            v = next(ev)
            ent, plane = divmod(int(v), 8)
            assert plane == depth[ent] - 1       # only an entry's deepest plane leaves
            depth[ent] -= 1
        depth[x] = max(depth[x], dep[a])
        assert depth.sum() <= cap


def test_independent_objects_hit_only_exact_precision(oracle_mod):
    acc = np.array([(0, 0, 2, 0), (0, 0, 4, 1), (0, 0, 2, 2), (0, 0, 3, 3)])
    hit, fetched = oracle_mod.cache_sim_independent(1, 4, 64, acc[:, 0], acc[:, 1], acc[:, 2], acc[:, 3])
    assert list(hit) == [0, 0, 1, 0]
    assert fetched == 2 + 4 + 3
    # the prefix cache serves the same trace with 4 planes fetched in total
    _, _, fp = oracle_mod.cache_sim_prefix(1, 4, 64, acc[:, 0], acc[:, 1], acc[:, 2], acc[:, 3])
    assert fp == 4


# Independent objects with downward reuse (transcript cue 51: a resident higher-precision copy
# serves lower-bit requests and is promoted when a request needs more).

def _down(oracle_mod, cap, accesses, L=1, E=8):
    a = np.array(accesses, dtype=np.int64)
    return oracle_mod.cache_sim_independent_down(L, E, cap, a[:, 0], a[:, 1], a[:, 2], a[:, 3])


def test_downward_reuse_hand_traces(oracle_mod):
    # 6 resident, 3 requested: served by the deeper copy (an exact-object cache misses here)
    hit, fetched = _down(oracle_mod, 64, [(0, 1, 6, 0), (0, 1, 3, 1)])
    assert list(hit) == [0, 1] and fetched == 6
    hit_i, fetched_i = oracle_mod.cache_sim_independent(1, 8, 64, [0, 0], [1, 1], [6, 3], [0, 1])
    assert list(hit_i) == [0, 0] and fetched_i == 9
    # 3 resident, 5 requested: promoted by loading a whole 5-plane copy (a prefix cache reads 2)
    hit, fetched = _down(oracle_mod, 64, [(0, 1, 3, 0), (0, 1, 5, 1)])
    assert list(hit) == [0, 0] and fetched == 8
    _, _, fetched_p = oracle_mod.cache_sim_prefix(1, 8, 64, [0, 0], [1, 1], [3, 5], [0, 1])
    assert fetched_p == 5


def test_downward_reuse_evicts_whole_lru_objects(oracle_mod):
    # capacity 6: A(3) then B(2); C(3) needs room -> A (least recent) goes entirely
    hit, fetched = _down(oracle_mod, 6, [(0, 0, 3, 0), (0, 1, 2, 1), (0, 2, 3, 2), (0, 0, 1, 3)])
    assert list(hit) == [0, 0, 0, 0] and fetched == 3 + 2 + 3 + 1
    # a promotion frees its own old copy first: A(2) -> A(5) fits in 5 planes
    hit, fetched = _down(oracle_mod, 5, [(0, 0, 2, 0), (0, 0, 5, 1)])
    assert list(hit) == [0, 0] and fetched == 7
    # entries of the current batch are not evicted
    with pytest.raises(ValueError):
        _down(oracle_mod, 4, [(0, 0, 2, 0), (0, 1, 2, 0), (0, 2, 2, 0)])


def test_downward_reuse_without_capacity_pressure_is_running_max(oracle_mod):
    rng = np.random.default_rng(3)
    L, E, n = 2, 16, 2000
    lay = rng.integers(0, L, n)
    exp_ = rng.integers(0, E, n)
    dep = rng.integers(1, 9, n)
    bat = np.arange(n)
    hit, fetched = oracle_mod.cache_sim_independent_down(L, E, L * E * 8, lay, exp_, dep, bat)
    best = {}
    exp_hit, exp_fetched = [], 0
    for l, e, b in zip(lay, exp_, dep):
        r = best.get((l, e), 0)
        exp_hit.append(1 if r >= b else 0)
        if r < b:
            exp_fetched += b
            best[(l, e)] = b
    assert list(hit) == exp_hit and fetched == exp_fetched
    # exact-object hits are a subset of downward hits; a prefix cache fetches the least
    hit_i, fetched_i = oracle_mod.cache_sim_independent(L, E, L * E * 8 * 8, lay, exp_, dep, bat)
    assert np.all(hit >= hit_i)
    _, _, fetched_p = oracle_mod.cache_sim_prefix(L, E, L * E * 8, lay, exp_, dep, bat)
    assert fetched_p <= fetched <= fetched_i
