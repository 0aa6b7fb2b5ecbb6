"""The library's prefix-cache manager and independent-precision simulator
against the oracle's simulators (host only, no GPU): same hits, same
resident depths, same evictions in the same order, same bytes.

Pages: PagedMoE podcast transcript, cues 11, 13 and 35; arxivlens Abstract."""
import numpy as np
import pytest

import bitplane_mixed_precision_b200 as pm
from conftest import read_golden


def _trace(seed, L, E, tokens, k, zipf=False):
    """Token-major accesses: per token and layer, k distinct experts with depths 1..8."""
    rng = np.random.default_rng(seed)
    lay, exp_, dep, bat = [], [], [], []
    w = None
    if zipf:
        w = 1.0 / np.arange(1, E + 1) ** 1.1
        w /= w.sum()
    for t in range(tokens):
        for l in range(L):
            ids = rng.choice(E, size=k, replace=False, p=w)
            for e in ids:
                lay.append(l)
                exp_.append(int(e))
                dep.append(int(rng.integers(1, 9)))
                bat.append(t)
    return (np.array(lay, np.int32), np.array(exp_, np.int32), np.array(dep, np.uint8),
            np.array(bat, np.int32))


def _run_product(L, E, cap, lay, exp_, dep, bat, per_call):
    """Feeds the trace to a host-only cache, per_call accesses of one (layer, batch) per call."""
    c = pm.Cache(L, E, cap, 4, keep_log=True)
    before = np.zeros(len(lay), np.uint8)
    i = 0
    while i < len(lay):
        j = i + 1
        while j < len(lay) and j - i < per_call and lay[j] == lay[i] and bat[j] == bat[i]:
            j += 1
        rb = np.zeros(j - i, np.uint8)
        c.extend(int(lay[i]), exp_[i:j], dep[i:j], int(bat[i]), resident_before=rb)
        before[i:j] = rb
        i = j
    st = c.stats()
    log = c.eviction_log()
    c.close()
    return before, log, st


@pytest.mark.parametrize("seed,L,E,tokens,k,cap_frac,zipf,per_call", [
    (0, 2, 16, 60, 4, 0.3, False, 4),
    (1, 4, 32, 40, 6, 0.25, True, 6),
    (2, 3, 64, 50, 8, 0.4, True, 1),
    (3, 1, 8, 200, 3, 0.5, False, 3),
])
def test_manager_matches_oracle_simulator(oracle_mod, seed, L, E, tokens, k, cap_frac, zipf, per_call):
    lay, exp_, dep, bat = _trace(seed, L, E, tokens, k, zipf)
    cap = max(int(cap_frac * L * E * 8), 8 * k)
    before_o, log_o, fetched_o = oracle_mod.cache_sim_prefix(L, E, cap, lay, exp_, dep, bat)
    before_p, log_p, st = _run_product(L, E, cap, lay, exp_, dep, bat, per_call)
    assert np.array_equal(before_p, before_o)
    assert np.array_equal(log_p, log_o)
    assert st.planes_fetched == fetched_o
    assert st.requests == len(lay)
    assert st.hits == int(np.sum(before_o >= dep))
    assert st.planes_evicted == len(log_o)
    assert st.bytes_fetched == fetched_o * 16
    assert len(log_o) > 0  # the trace exercised eviction


def test_golden_topup_reads_only_missing_planes():
    # transcript cues 13 and 35: resident r, requested b -> planes r+1..b read (1-based)
    for r, b, read, after in read_golden("cache_trace_examples.txt"):
        r, b, after = int(r), int(b), int(after)
        expect = 0 if read == "-" else len(read.split(","))
        c = pm.Cache(1, 4, 64, 4)
        c.extend(0, [1], [r], 0)
        f0 = c.stats().planes_fetched
        rb = np.zeros(1, np.uint8)
        st = c.extend(0, [1], [b], 1, resident_before=rb)
        assert rb[0] == r
        assert st.planes_fetched - f0 == expect
        assert int(c.resident_depth(0)[1]) == after


def test_pinned_batch_and_out_of_slots(oracle_mod):
    # capacity 4: two 2-plane entries of batch 0 fill it; a third in batch 0 cannot fit
    c = pm.Cache(1, 8, 4, 4, keep_log=True)
    c.extend(0, [0, 1], [2, 2], 0)
    with pytest.raises(pm.PmoeError) as ei:
        c.extend(0, [2], [2], 0)
    assert ei.value.code == 3
    with pytest.raises(ValueError):
        oracle_mod.cache_sim_prefix(1, 8, 4, [0, 0, 0], [0, 1, 2], [2, 2, 2], [0, 0, 0])
    # in the next batch the oldest deepest planes go: expert 1's plane 1 was stamped last... both at
    # depth 2; expert 0 (older) loses plane 1 first, then plane 0
    c2 = pm.Cache(1, 8, 4, 4, keep_log=True)
    c2.extend(0, [0, 1], [2, 2], 0)
    c2.extend(0, [2], [2], 1)
    _, log_o, _ = oracle_mod.cache_sim_prefix(1, 8, 4, [0, 0, 0], [0, 1, 2], [2, 2, 2], [0, 0, 1])
    assert list(c2.eviction_log()) == list(log_o) == [1, 0]


def test_invalid_accesses_change_nothing():
    c = pm.Cache(2, 8, 16, 4)
    c.extend(0, [3], [2], 0)
    for layer, e, b in [(2, 0, 1), (-1, 0, 1), (0, 8, 1), (0, -1, 1), (0, 0, 0), (0, 0, 9)]:
        with pytest.raises(pm.PmoeError) as ei:
            c.extend(layer, [1, e], [1, b], 1)
        assert ei.value.code == 1
    assert c.stats().requests == 1
    assert list(c.resident_depth(0)) == [0, 0, 0, 2, 0, 0, 0, 0]
    with pytest.raises(pm.PmoeError):
        pm.Cache(0, 8, 16, 4)
    with pytest.raises(pm.PmoeError):
        pm.Cache(1, 8, 16, 6)  # slot_words % 4


def test_log_needs_keep_log():
    c = pm.Cache(1, 8, 16, 4)
    with pytest.raises(pm.PmoeError) as ei:
        c.eviction_log()
    assert ei.value.code == 7


@pytest.mark.parametrize("seed,cap_frac", [(0, 0.3), (1, 0.15), (2, 0.5)])
def test_independent_simulator_matches_oracle(oracle_mod, seed, cap_frac):
    L, E = 3, 32
    lay, exp_, dep, bat = _trace(seed + 10, L, E, 60, 6, zipf=True)
    cap = max(int(cap_frac * L * E * 8), 48)
    hit_o, fetched_o = oracle_mod.cache_sim_independent(L, E, cap, lay, exp_, dep, bat)
    hit_p, fetched_p = pm.cache_sim_independent(L, E, cap, lay, exp_, dep, bat)
    assert np.array_equal(hit_p, hit_o)
    assert fetched_p == fetched_o


def test_prefix_sharing_beats_independent_objects(oracle_mod):
    # the same experts asked at varying depths: one shared prefix serves every shallower request
    L, E = 2, 16
    lay, exp_, dep, bat = _trace(5, L, E, 100, 4, zipf=True)
    cap = int(0.4 * L * E * 8)
    _, _, st = _run_product(L, E, cap, lay, exp_, dep, bat, 4)
    hit_i, fetched_i = pm.cache_sim_independent(L, E, cap, lay, exp_, dep, bat)
    assert st.hits > int(hit_i.sum())
    assert st.planes_fetched < fetched_i


def test_route_host_matches_oracle(oracle_mod, synth_mod):
    E, k, T = 512, 10, 16
    logits = np.stack([synth_mod.router_logits(3, t, 0, E) for t in range(T)]).astype(np.float32)
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    pm.route_host(logits, T, E, k, ids, w)
    ids_o, w_o = oracle_mod.route(logits, k)
    assert np.array_equal(ids, ids_o)
    assert np.array_equal(w, w_o)
    # ties go to the lower id
    tied = np.zeros((1, 8), np.float32)
    tied[0, [2, 5, 6]] = 1.0
    ids1 = np.zeros((1, 3), np.int32)
    w1 = np.zeros((1, 3), np.float32)
    pm.route_host(tied, 1, 8, 3, ids1, w1)
    assert list(ids1[0]) == [2, 5, 6]


@pytest.mark.parametrize("seed,cap_frac", [(0, 0.3), (1, 0.12), (2, 0.5)])
def test_downward_reuse_simulator_matches_oracle(oracle_mod, seed, cap_frac):
    L, E = 3, 32
    lay, exp_, dep, bat = _trace(seed + 20, L, E, 60, 6, zipf=True)
    cap = max(int(cap_frac * L * E * 8), 8 * 6 * L)  # a token pins up to L layers x 6 experts x 8 planes
    hit_o, fetched_o = oracle_mod.cache_sim_independent_down(L, E, cap, lay, exp_, dep, bat)
    hit_p, fetched_p = pm.cache_sim_independent_down(L, E, cap, lay, exp_, dep, bat)
    assert np.array_equal(hit_p, hit_o)
    assert fetched_p == fetched_o


def test_prefix_cache_bounds_downward_reuse(oracle_mod):
    # with ample capacity: exact-object hits <= downward-reuse hits <= prefix hits, and the
    # prefix cache fetches the fewest planes
    L, E = 2, 16
    lay, exp_, dep, bat = _trace(7, L, E, 80, 4, zipf=True)
    cap = L * E * 8 * 8
    _, _, st = _run_product(L, E, L * E * 8, lay, exp_, dep, bat, 4)
    hit_d, fetched_d = pm.cache_sim_independent_down(L, E, cap, lay, exp_, dep, bat)
    hit_i, fetched_i = pm.cache_sim_independent(L, E, cap, lay, exp_, dep, bat)
    assert int(hit_i.sum()) <= int(hit_d.sum()) <= st.hits
    assert st.planes_fetched <= fetched_d <= fetched_i
