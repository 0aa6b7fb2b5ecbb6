"""Pins for the oracle's prefix GEMV, routing, prefix selection and MoE layer."""
import itertools
import math

import numpy as np
import pytest

from conftest import read_golden


def _dequant(oracle_mod, codes, scales, cb, G, b, bf16=False):
    lv = oracle_mod.level(cb.astype(np.float32), b)
    s = np.repeat(scales, G, axis=1)
    if bf16:
        v = (s * lv[codes >> (8 - b)]).astype(np.float32)  # float product, then bf16 rounding
        u = v.view(np.uint32).astype(np.uint64)
        u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
        return u.astype(np.uint32).view(np.float32).astype(np.float64)
    return s.astype(np.float64) * lv[codes >> (8 - b)].astype(np.float64)


@pytest.mark.parametrize("b", range(1, 9))
def test_gemv_against_numpy_dequant_matmul(oracle_mod, synth_mod, b):
    w = synth_mod.expert_weights(5, 0, 0, 0, 128, 256)
    scales, codes = oracle_mod.quantize(w, 64)
    cb = oracle_mod.tree_codebook_f32()
    x = synth_mod.activation_f32(5, 0, 0, 256).astype(np.float64)
    y = oracle_mod.gemv(codes, scales, cb, 64, b, x)
    ref = _dequant(oracle_mod, codes, scales, cb, 64, b) @ x
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)
    yb = oracle_mod.gemv(codes, scales, cb, 64, b, x, bf16_weights=True)
    refb = _dequant(oracle_mod, codes, scales, cb, 64, b, bf16=True) @ x
    np.testing.assert_allclose(yb, refb, rtol=1e-12, atol=1e-15)


def test_gemv_unit_vectors(oracle_mod):
    """x = e_k returns column k of the dequantised matrix: scale * C[b][code >> (8-b)]."""
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 256, size=(16, 128), dtype=np.uint8)
    scales = rng.uniform(0.5, 2.0, size=(16, 2)).astype(np.float32)
    cb = oracle_mod.tree_codebook_f32()
    for k in (0, 63, 64, 127):
        x = np.zeros(128)
        x[k] = 1.0
        for b in (1, 3, 8):
            y = oracle_mod.gemv(codes, scales, cb, 64, b, x)
            lv = oracle_mod.level(cb, b)
            expect = scales[:, k // 64].astype(np.float64) * lv[codes[:, k] >> (8 - b)]
            np.testing.assert_array_equal(y, expect)


def test_route_hand_examples(oracle_mod):
    logits = np.array([[0.5, 2.0, 2.0, -1.0, 1.0, 2.0],
                       [0.0, 0.0, 0.0, 0.0, 0.0, 0.0]], dtype=np.float32)
    ids, w = oracle_mod.route(logits, 3)
    np.testing.assert_array_equal(ids[0], [1, 2, 5])      # ties go to the lower id
    np.testing.assert_array_equal(ids[1], [0, 1, 2])
    np.testing.assert_allclose(w[0], [1 / 3] * 3, rtol=1e-7)
    np.testing.assert_allclose(w[1], [1 / 3] * 3, rtol=1e-7)


def test_route_against_sort_and_softmax(oracle_mod, synth_mod):
    E, k = 512, 10
    logits = np.stack([synth_mod.router_logits(9, t, 0, E) for t in range(64)])
    ids, w = oracle_mod.route(logits, k)
    for t in range(64):
        order = sorted(range(E), key=lambda e: (-float(logits[t, e]), e))[:k]
        np.testing.assert_array_equal(ids[t], order)
        sel = logits[t, order].astype(np.float64)
        ref = np.exp(sel - sel.max()) / np.exp(sel - sel.max()).sum()
        np.testing.assert_allclose(w[t], ref, rtol=1e-7)
        assert abs(float(w[t].astype(np.float64).sum()) - 1.0) < 1e-6


def _objective(w, s, b):
    return sum(float(wi) ** 2 * float(si) ** 2 * 4.0 ** (-int(bi)) for wi, si, bi in zip(w, s, b))


@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_select_is_brute_force_optimum(oracle_mod, k):
    """Greedy on w^2 s^2 4^-b equals the exhaustive minimum under sum b = B (cue 29)."""
    rng = np.random.default_rng(k)
    for trial in range(40):
        w = rng.dirichlet(np.ones(k)).astype(np.float32)[None, :]
        ids = np.arange(k, dtype=np.int32)[None, :]
        sens = np.exp(0.5 * rng.standard_normal(k)).astype(np.float32)
        avg = float(rng.choice([1.0, 1.5, 2.5, 3.25, 5.0, 8.0]))
        B = oracle_mod.budget(k, avg)
        d = oracle_mod.select(w, ids, sens, avg)[0]
        assert int(d.sum()) == B
        best = math.inf
        for cand in itertools.product(range(1, 9), repeat=k):
            if sum(cand) == B:
                best = min(best, _objective(w[0], sens, cand))
        got = _objective(w[0], sens, d)
        assert got == pytest.approx(best, rel=1e-12)


def test_select_equals_offset_rule(oracle_mod, synth_mod):
    """b_i = clamp(ceil(c + log2(w_i s_i / geomean)), 1, 8), c set so that mean b = 2.5."""
    E, k = 512, 10
    sens = synth_mod.sensitivities(2, 0, E)
    logits = np.stack([synth_mod.router_logits(2, t, 0, E) for t in range(200)])
    ids, w = oracle_mod.route(logits, k)
    depth = oracle_mod.select(w, ids, sens, 2.5)
    for t in range(200):
        v = (w[t] * sens[ids[t]]).astype(np.float32).astype(np.float64)
        lg = np.log2(v) - np.log2(v).mean()
        # breakpoints of the step function c -> sum clamp(ceil(c + lg), 1, 8)
        bps = sorted({n - x for x in lg for n in range(-20, 30)})
        ok = None
        for lo, hi in zip(bps[:-1], bps[1:]):
            c = 0.5 * (lo + hi)
            b = np.clip(np.ceil(c + lg), 1, 8)
            if b.sum() == 25:
                ok = b
                break
        assert ok is not None
        np.testing.assert_array_equal(depth[t], ok.astype(np.uint8))
        assert depth[t].mean() == 2.5


def test_select_budget_and_candidates(oracle_mod):
    rows = read_golden("allocator_candidates.txt")
    k, first, last, cand = map(int, rows[0])
    assert k * (last - first) == cand          # 10 experts x 7 upgrades = 70 (cue 29)
    assert oracle_mod.budget(10, 2.5) == 25
    assert oracle_mod.budget(8, 2.5) == 20
    assert oracle_mod.budget(10, 0.1) == 10     # clamped to one bit each
    assert oracle_mod.budget(10, 9.0) == 80     # clamped to eight bits each
    w = np.full((1, 10), 0.1, np.float32)
    ids = np.arange(10, dtype=np.int32)[None, :]
    d = oracle_mod.select(w, ids, np.ones(10, np.float32), 8.0)
    assert np.all(d == 8)
    d = oracle_mod.select(w, ids, np.ones(10, np.float32), 2.5)
    # all priorities equal: upgrades cycle through the slots in order
    np.testing.assert_array_equal(d[0], [3, 3, 3, 3, 3, 2, 2, 2, 2, 2])


def test_moe_layer_against_numpy(oracle_mod, synth_mod):
    E, k, H, I, G, T = 8, 3, 256, 128, 64, 3
    cb = oracle_mod.tree_codebook_f32()
    experts = {}
    deq = {}
    for e in range(E):
        codes, scales = [], []
        for m, (n, kk) in enumerate(((I, H), (I, H), (H, I))):
            s, c = oracle_mod.quantize(synth_mod.expert_weights(4, 0, e, m, n, kk), G)
            codes.append(c)
            scales.append(s)
        experts[e] = oracle_mod.Expert(codes, scales, [cb, cb, cb])
    logits = np.stack([synth_mod.router_logits(4, t, 0, E) for t in range(T)])
    ids, w = oracle_mod.route(logits, k)
    sens = synth_mod.sensitivities(4, 0, E)
    depth = oracle_mod.select(w, ids, sens, 2.5)
    x = np.stack([synth_mod.bf16_to_f32(synth_mod.activation_bf16(4, t, 0, H)) for t in range(T)])
    y = oracle_mod.moe_layer(experts, E, H, I, G, ids, w, depth, x.astype(np.float64))
    for t in range(T):
        ref = np.zeros(H)
        for i in range(k):
            e, b = int(ids[t, i]), int(depth[t, i])
            ex = experts[e]
            Wg = _dequant(oracle_mod, ex.codes[0], ex.scales[0], cb, G, b)
            Wu = _dequant(oracle_mod, ex.codes[1], ex.scales[1], cb, G, b)
            Wd = _dequant(oracle_mod, ex.codes[2], ex.scales[2], cb, G, b)
            g = Wg @ x[t]
            u = Wu @ x[t]
            h = g / (1 + np.exp(-g)) * u
            ref += float(w[t, i]) * (Wd @ h)
        np.testing.assert_allclose(y[t], ref, rtol=1e-10, atol=1e-13)


@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_cache_aware_select_is_brute_force_optimum(oracle_mod, k):
    """Under a budget of fetched planes (resident planes free, every expert at least one plane),
    the greedy reaches the exhaustive minimum of sum w^2 s^2 4^-b (transcript cue 61)."""
    rng = np.random.default_rng(100 + k)
    for trial in range(40):
        w = rng.dirichlet(np.ones(k)).astype(np.float32)[None, :]
        ids = np.arange(k, dtype=np.int32)[None, :]
        sens = np.exp(0.5 * rng.standard_normal(k)).astype(np.float32)
        res = rng.integers(0, 9, k).astype(np.uint8)
        fetch = int(rng.integers(0, 3 * k + 1))
        d = oracle_mod.select_cache_aware(w, ids, sens, res[None, :], fetch)[0]

        def fetched(b):
            return sum(max(0, int(bi) - int(ri)) for bi, ri in zip(b, res))
        need = sum(1 for r in res if r == 0)
        cap = max(fetch, need)
        assert fetched(d) <= cap
        assert all(int(bi) >= max(1, int(ri)) for bi, ri in zip(d, res))
        best = math.inf
        for cand in itertools.product(range(1, 9), repeat=k):
            if fetched(cand) <= cap:
                best = min(best, _objective(w[0], sens, cand))
        assert _objective(w[0], sens, d) == pytest.approx(best, rel=1e-12)


def test_cache_aware_select_special_cases(oracle_mod):
    w = np.array([[0.5, 0.3, 0.2]], np.float32)
    ids = np.array([[0, 1, 2]], np.int32)
    sens = np.ones(3, np.float32)
    # nothing resident: with a budget of k*B-style fetches it is the cache-oblivious greedy
    d = oracle_mod.select_cache_aware(w, ids, sens, np.zeros((1, 3), np.uint8), 8)
    assert np.array_equal(d, oracle_mod.select(w, ids, sens, 8 / 3))
    # everything resident deeply, no fetch budget: all resident planes are used, nothing fetched
    d = oracle_mod.select_cache_aware(w, ids, sens, np.array([[6, 3, 8]], np.uint8), 0)
    assert list(d[0]) == [6, 3, 8]
    # a zero budget still gives an absent expert its first plane
    d = oracle_mod.select_cache_aware(w, ids, sens, np.array([[0, 2, 0]], np.uint8), 0)
    assert list(d[0]) == [1, 2, 1]


# Profile-driven allocation (transcript cues 29-31): isotonic repair of error profiles and
# greedy selection from a per-expert table.

def test_isotonic_matches_library_regression(oracle_mod):
    from sklearn.isotonic import IsotonicRegression
    rng = np.random.default_rng(4)
    for trial in range(50):
        g = rng.standard_normal(7) * rng.choice([0.1, 1.0, 10.0])
        got = oracle_mod.isotonic_nonincreasing(g)
        ref = IsotonicRegression(increasing=False).fit_transform(np.arange(7), g)
        assert np.allclose(got, ref, rtol=0, atol=1e-12)
    assert list(oracle_mod.isotonic_nonincreasing([3.0, 1.0, 2.0])) == [3.0, 1.5, 1.5]


def test_profile_repair_keeps_valid_profiles_and_fixes_others(oracle_mod):
    good = np.array([[0.7, 0.35, 0.15, 0.06, 0.024, 0.0096, 0.0028, 0.0]])
    assert np.allclose(oracle_mod.profile_repair(good), good, rtol=0, atol=1e-15)
    bad = np.array([[0.7, 0.6, 0.15, 0.14, 0.02, 0.0096, 0.0028, 0.0]])  # gains 0.1 < 0.45: not convex
    rep = oracle_mod.profile_repair(bad)[0]
    gains = rep[:-1] - rep[1:]
    assert np.all(np.diff(gains) <= 1e-15) and np.all(gains >= 0)
    assert rep[7] == bad[0, 7] and rep[0] == pytest.approx(bad[0, 0])  # total drop is preserved


def test_select_table_reduces_to_closed_form_profiles(oracle_mod, synth_mod):
    # E_e(b) = s_e^2 4^-b gives the same depths as the closed-form allocator
    E, k, T = 64, 8, 200
    sens = synth_mod.sensitivities(9, 0, E)
    table = (sens.astype(np.float64)[:, None] ** 2 * 4.0 ** -np.arange(1, 9)[None, :]).astype(np.float32)
    logits = np.stack([synth_mod.router_logits(9, t, 0, E) for t in range(T)])
    ids, w = oracle_mod.route(logits, k)
    assert np.array_equal(oracle_mod.select_table(w, ids, table, 2.5), oracle_mod.select(w, ids, sens, 2.5))


@pytest.mark.parametrize("k", [2, 3, 4])
def test_select_table_is_brute_force_optimum(oracle_mod, k):
    rng = np.random.default_rng(200 + k)
    for trial in range(30):
        w = rng.dirichlet(np.ones(k)).astype(np.float32)[None, :]
        ids = np.arange(k, dtype=np.int32)[None, :]
        gains = np.sort(rng.random((k, 7)))[:, ::-1] * rng.random((k, 1))  # non-increasing gains
        table = np.concatenate([np.cumsum(gains[:, ::-1], axis=1)[:, ::-1], np.zeros((k, 1))], axis=1)
        table = table.astype(np.float32)
        avg = float(rng.choice([1.5, 2.5, 4.0]))
        B = oracle_mod.budget(k, avg)
        d = oracle_mod.select_table(w, ids, table, avg)[0]
        assert int(d.sum()) == B
        obj = lambda b: sum(float(w[0, i]) ** 2 * float(table[i, b[i] - 1]) for i in range(k))
        best = min(obj(c) for c in itertools.product(range(1, 9), repeat=k) if sum(c) == B)
        assert obj(d) == pytest.approx(best, rel=1e-5, abs=1e-12)


def test_expert_profile_shape(oracle_mod, synth_mod):
    # the full expert's relative output error: zero at 8 bits, falling with depth, and a few times
    # the squared relative weight error sqrt(D_b) of one matrix (three quantised matrices compound)
    H, I, G, E = 1024, 256, 128, 4
    cb = oracle_mod.tree_codebook_f32()
    codes, scales = [], []
    for m, (n, kk) in enumerate(((I, H), (I, H), (H, I))):
        s, c = oracle_mod.quantize(synth_mod.expert_weights(5, 0, 1, m, n, kk), G)
        codes.append(c)
        scales.append(s)
    ex = oracle_mod.Expert(codes, scales, [cb] * 3)
    xs = np.random.default_rng(0).standard_normal((10, H))
    prof = oracle_mod.expert_profile(ex, E, H, I, G, xs)
    assert prof[7] == 0.0 and np.all(np.diff(prof) < 0)
    D = np.array([0.603, 0.373, 0.234, 0.149, 0.096, 0.063, 0.041]) ** 2
    assert np.all(prof[:7] / D > 1.0) and np.all(prof[:7] / D < 4.0)


# The layer's composition (gate/up -> SwiGLU -> down -> weighted combine), pinned by cases whose
# result follows from the definition by hand, not by re-running its formula: PagedMoE transcript
# cue 4 (top-k experts combined with routing weights that sum to one) and the SwiGLU expert FFN.

def _const_expert(oracle_mod, H, I, G, cb, codes_gud, scales_gud):
    """An expert whose three matrices have one code and one scale each (all weights equal)."""
    codes = [np.full(shape, c, np.uint8) for shape, c in zip(((I, H), (I, H), (H, I)), codes_gud)]
    scales = [np.full((n, kk // G), s, np.float32)
              for (n, kk), s in zip(((I, H), (I, H), (H, I)), scales_gud)]
    return oracle_mod.Expert(codes, scales, [cb] * 3)


def _ident_codebook():
    """A 510-entry table whose every depth maps index 0 to 0.0 and the all-ones index to 1.0
    (any other entry 0.5): code 0 reads as 0 and code 255 as 1 at every depth."""
    cb = np.full(510, 0.5, np.float32)
    for d in range(1, 9):
        cb[(1 << d) - 2] = 0.0
        cb[(1 << d) - 2 + (1 << d) - 1] = 1.0
    return cb


@pytest.mark.parametrize("b", [1, 3, 8])
def test_layer_negative_gate_silences_the_expert(oracle_mod, b):
    """Gate weights all at the most negative tree node, up weights all at the most positive one,
    x > 0: g is a large negative number, silu(g) ~ 0, so the expert adds (almost) nothing.
    With gate and up swapped (silu(u) * g) the output would be of order -u*g*H instead."""
    H, I, G = 128, 128, 64
    cb = oracle_mod.tree_codebook_f32()
    ex = _const_expert(oracle_mod, H, I, G, cb, (0, 255, 255), (1.0, 1.0, 1.0))
    x = np.full((1, H), 0.5)
    y = oracle_mod.moe_layer({0: ex}, 1, H, I, G, np.zeros((1, 1), np.int32), np.ones((1, 1), np.float32),
                             np.full((1, 1), b, np.uint8), x)
    c_lo, c_hi = float(oracle_mod.level(cb, b)[0]), float(oracle_mod.level(cb, b)[-1])
    g, u = c_lo * 0.5 * H, c_hi * 0.5 * H   # every row of Wg x and Wu x
    assert g < -40 and u > 40
    bound = abs(g) * math.exp(g) * u * c_hi * I * 1.01  # |silu(g)| <= |g| e^g for g < 0
    assert np.all(np.abs(y) <= bound)
    assert bound < 1e-10
    swapped = (u / (1 + math.exp(-u))) * g * c_hi * I
    assert abs(swapped) > 1e3


def test_layer_identity_down_returns_swiglu(oracle_mod):
    """Wg = a*I, Wu = c*I, Wd = I (codes 255 on the diagonal, 0 elsewhere, a table with 0 and 1
    at its ends): y = w * silu(a x) * (c x) element by element, with a != c so that a swapped
    gate/up gives another value. silu(z) = z * sigmoid(z) is checked at points with known values."""
    H = I = 128
    G = 64
    cb = _ident_codebook()
    a, c, wt = 1.5, -0.75, 0.625
    eye = np.where(np.eye(H, dtype=bool), 255, 0).astype(np.uint8)
    codes = [eye, eye, eye]
    scales = [np.full((I, H // G), a, np.float32), np.full((I, H // G), c, np.float32),
              np.full((H, I // G), 1.0, np.float32)]
    ex = oracle_mod.Expert(codes, scales, [cb] * 3)
    x = np.linspace(-3.0, 3.0, H)[None, :]
    for b in (1, 2, 5, 8):
        y = oracle_mod.moe_layer({0: ex}, 1, H, I, G, np.zeros((1, 1), np.int32),
                                 np.full((1, 1), wt, np.float32), np.full((1, 1), b, np.uint8), x)[0]
        g, u = a * x[0], c * x[0]
        # sigmoid from tanh: sigma(z) = (1 + tanh(z/2)) / 2, another route to the same function
        want = wt * g * (0.5 * (1.0 + np.tanh(0.5 * g))) * u
        np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-15)
        swapped = wt * u * (0.5 * (1.0 + np.tanh(0.5 * u))) * g
        assert np.max(np.abs(swapped - want)) > 0.1
    # silu at points with closed-form values: silu(0) = 0 and silu(2 ln 3) = ln 3 * 3/2 ... via x
    x0 = np.zeros((1, H))
    y0 = oracle_mod.moe_layer({0: ex}, 1, H, I, G, np.zeros((1, 1), np.int32), np.ones((1, 1), np.float32),
                              np.full((1, 1), 8, np.uint8), x0)
    assert np.all(y0 == 0.0)


def test_layer_is_linear_in_routing_weights(oracle_mod, synth_mod):
    """y = sum_i w_i * expert_i(x): splitting the weights into one-hot vectors and summing the
    results reproduces the output (a weight applied before gate/up, where silu is not linear,
    would break this)."""
    E, k, H, I, G = 6, 3, 256, 128, 64
    cb = oracle_mod.tree_codebook_f32()
    experts = {}
    for e in range(E):
        codes, scales = [], []
        for m, (n, kk) in enumerate(((I, H), (I, H), (H, I))):
            s, cc = oracle_mod.quantize(synth_mod.expert_weights(8, 0, e, m, n, kk), G)
            codes.append(cc)
            scales.append(s)
        experts[e] = oracle_mod.Expert(codes, scales, [cb] * 3)
    ids = np.array([[4, 1, 3]], np.int32)
    depth = np.array([[2, 5, 1]], np.uint8)
    x = 3.0 * synth_mod.activation_f32(8, 0, 0, H).astype(np.float64)[None, :]
    w = np.array([[0.5, 0.3, 0.2]], np.float32)
    y = oracle_mod.moe_layer(experts, E, H, I, G, ids, w, depth, x)[0]
    parts = [oracle_mod.moe_layer(experts, E, H, I, G, ids, np.eye(k, dtype=np.float32)[i:i + 1], depth, x)[0]
             for i in range(k)]
    np.testing.assert_allclose(y, sum(float(w[0, i]) * parts[i] for i in range(k)), rtol=1e-12, atol=1e-14)
    y2 = oracle_mod.moe_layer(experts, E, H, I, G, ids, 2 * w, depth, x)[0]
    np.testing.assert_allclose(y2, 2 * y, rtol=1e-12, atol=1e-14)
    # the expert itself is not linear in x (SwiGLU): doubling x does not double y
    y3 = oracle_mod.moe_layer(experts, E, H, I, G, ids, w, depth, 2 * x)[0]
    assert np.linalg.norm(y3 - 2 * y) > 0.05 * np.linalg.norm(2 * y)
