"""Randomised checks of the library's host-side routing, allocation and cache manager against
the oracle: hypothesis draws the shapes, budgets and values, ties and extreme budgets included.
Everything is compared exactly (PagedMoE transcript cues 4, 11, 13, 29, 31, 35, 61)."""
import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import bitplane_mixed_precision_b200 as pm

FUZZ = settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.function_scoped_fixture])


def _ids(rng, T, E, k):
    return np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)


def _weights(rng, T, k, ties):
    w = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    if ties:
        w[:] = np.float32(1.0 / k)  # every slot equal: ties decide every step
    elif k > 1 and rng.random() < 0.3:
        w[:, rng.integers(0, k)] = 0.0  # a routing weight that underflowed to zero
    return w


@st.composite
def routing_cases(draw):
    E = draw(st.integers(1, 600))
    k = draw(st.integers(1, min(32, E)))
    T = draw(st.integers(1, 6))
    rng = np.random.default_rng(draw(st.integers(0, 2**32 - 1)))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    if draw(st.booleans()):
        logits = (np.round(logits * 2) / 2).astype(np.float32)  # many equal logits
    return logits, k


@FUZZ
@given(routing_cases())
def test_route_host_matches_oracle(oracle_mod, case):
    logits, k = case
    T, E = logits.shape
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    pm.route_host(logits, T, E, k, ids, w)
    ids_o, w_o = oracle_mod.route(logits, k)
    assert np.array_equal(ids, ids_o)
    assert np.array_equal(w, w_o)


@st.composite
def select_cases(draw):
    k = draw(st.integers(1, 12))
    T = draw(st.integers(1, 5))
    E = draw(st.integers(k, 64))
    avg = draw(st.sampled_from([1.0, 1.5, 2.0, 2.5, 3.0, 4.0, 7.9, 8.0]) | st.floats(1.0, 8.0, width=32))
    rng = np.random.default_rng(draw(st.integers(0, 2**32 - 1)))
    ties = draw(st.booleans())
    w = _weights(rng, T, k, ties)
    sens = np.exp(0.5 * rng.standard_normal(E)).astype(np.float32)
    if draw(st.booleans()):
        sens[:] = np.float32(1.0)
    return w, _ids(rng, T, E, k), sens, float(avg), rng


@FUZZ
@given(select_cases())
def test_host_select_matches_oracle(oracle_mod, case):
    w, ids, sens, avg, _ = case
    T, k = w.shape
    dep = np.zeros((T, k), np.uint8)
    pm.select_prefix(w, ids, sens, T, k, avg, dep, on_device=False)
    assert np.array_equal(dep, oracle_mod.select(w, ids, sens, avg))
    assert np.all(dep.astype(int).sum(axis=1) == oracle_mod.budget(k, avg))


@FUZZ
@given(select_cases(), st.integers(0, 64))
def test_host_cache_aware_select_matches_oracle(oracle_mod, case, fetch_draw):
    w, ids, sens, _, rng = case
    T, k = w.shape
    resident = rng.integers(0, 9, size=(T, k)).astype(np.uint8)
    fetch = fetch_draw % (8 * k + 1)
    dep = np.zeros((T, k), np.uint8)
    pm.select_prefix_cache_aware(w, ids, sens, resident, T, k, fetch, dep)
    assert np.array_equal(dep, oracle_mod.select_cache_aware(w, ids, sens, resident, fetch))


@FUZZ
@given(select_cases(), st.booleans())
def test_host_table_select_matches_oracle(oracle_mod, case, convex):
    w, ids, sens, avg, rng = case
    T, k = w.shape
    E = sens.shape[0]
    if convex:
        table = (sens[:, None].astype(np.float64) ** 2 * 4.0 ** -np.arange(1, 9)).astype(np.float32)
    else:
        table = np.sort(rng.random((E, 8)), axis=1)[:, ::-1].astype(np.float32)
        table[:, 7] = 0.0
    table = np.ascontiguousarray(table)
    dep = np.zeros((T, k), np.uint8)
    pm.select_prefix_table(w, ids, table, T, k, avg, dep, on_device=False)
    assert np.array_equal(dep, oracle_mod.select_table(w, ids, table, avg))


@st.composite
def cache_traces(draw):
    L = draw(st.integers(1, 3))
    E = draw(st.integers(2, 16))
    k = draw(st.integers(1, min(4, E)))
    n_tok = draw(st.integers(1, 30))
    rng = np.random.default_rng(draw(st.integers(0, 2**32 - 1)))
    lay, exp_, dep, bat = [], [], [], []
    for t in range(n_tok):
        for l in range(L):
            for e in rng.choice(E, size=k, replace=False):
                lay.append(l)
                exp_.append(int(e))
                dep.append(int(rng.integers(1, 9)))
                bat.append(t)
    # room for one batch (token) pinned across all its layers, up to everything resident
    cap = draw(st.integers(8 * k * L, max(8 * k * L, L * E * 8)))
    return (L, E, cap, np.array(lay, np.int32), np.array(exp_, np.int32), np.array(dep, np.uint8),
            np.array(bat, np.int32))


@FUZZ
@given(cache_traces(), st.integers(1, 4))
def test_cache_manager_matches_oracle_simulator(oracle_mod, trace, per_call):
    L, E, cap, lay, exp_, dep, bat = trace
    before_o, log_o, fetched_o = oracle_mod.cache_sim_prefix(L, E, cap, lay, exp_, dep, bat)
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
    st_ = c.stats()
    log = c.eviction_log()
    c.close()
    assert np.array_equal(before, before_o)
    assert np.array_equal(log, log_o)
    assert st_.planes_fetched == fetched_o
    hit_o, fetched_i_o = oracle_mod.cache_sim_independent(L, E, cap, lay, exp_, dep, bat)
    hit_p, fetched_i_p = pm.cache_sim_independent(L, E, cap, lay, exp_, dep, bat)
    assert np.array_equal(hit_p, hit_o) and fetched_i_p == fetched_i_o
    hit_od, fetched_d_o = oracle_mod.cache_sim_independent_down(L, E, cap, lay, exp_, dep, bat)
    hit_pd, fetched_d_p = pm.cache_sim_independent_down(L, E, cap, lay, exp_, dep, bat)
    assert np.array_equal(hit_pd, hit_od) and fetched_d_p == fetched_d_o


@FUZZ
@given(st.integers(1, 8), st.integers(1, 8), st.integers(1, 8), st.integers(0, 2**32 - 1))
def test_host_pack_matches_oracle(oracle_mod, n16, k128, depth, seed):
    N, K = 16 * n16, 128 * k128
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    stride = N * K // 32
    out = np.zeros(stride * depth, dtype=np.uint32)
    pm.pack_bitplanes(codes, N, K, depth, out, stride, on_device=False)
    ref = oracle_mod.pack(codes, depth)
    for p in range(depth):
        assert np.array_equal(out[p * stride:(p + 1) * stride], ref[p])
