"""The C-ABI library without a GPU: it loads, exports every declared symbol,
and its host-side paths agree with the oracle bit for bit."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def pm():
    import __graft_entry__
    __graft_entry__._library_builder().build()
    import bitplane_mixed_precision_b200 as pm
    return pm


def declared_symbols():
    names = []
    with open(os.path.join(ROOT, "include", "pmoe.h")) as f:
        text = f.read()
    for m in re.finditer(r"PMOE_API\s+[\w\s\*]+?\b(pmoe_\w+)\s*\(", text):
        names.append(m.group(1))
    return sorted(set(names))


def test_library_exports_every_declared_symbol(pm):
    lib = ctypes.CDLL(pm.LIB_PATH)
    names = declared_symbols()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    # the binding wraps exactly the declared entry points
    assert sorted(pm.exported_symbols()) == names


def test_codebook_matches_oracle(pm, oracle_mod):
    cb = np.empty(510, np.float32)
    pm.tree_codebook(cb)
    np.testing.assert_array_equal(cb, oracle_mod.tree_codebook_f32())


@pytest.mark.parametrize("N,K,depth", [(16, 128, 8), (48, 384, 3), (32, 256, 1), (64, 640, 5)])
def test_host_pack_matches_oracle(pm, oracle_mod, N, K, depth):
    rng = np.random.default_rng(N + K + depth)
    codes = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    ref = oracle_mod.pack(codes, depth)
    stride = N * K // 32 + 64  # planes spaced wider than needed
    out = np.full(stride * depth, 0xDEADBEEF, dtype=np.uint32)
    pm.pack_bitplanes(codes, N, K, depth, out, stride, on_device=False)
    for p in range(depth):
        np.testing.assert_array_equal(out[p * stride: p * stride + N * K // 32], ref[p])
        assert np.all(out[p * stride + N * K // 32: (p + 1) * stride] == 0xDEADBEEF)


@pytest.mark.parametrize("k,avg", [(10, 2.5), (8, 2.5), (4, 3.25), (16, 1.0), (3, 8.0)])
def test_host_select_matches_oracle(pm, oracle_mod, synth_mod, k, avg):
    E, T = 512, 300
    sens = synth_mod.sensitivities(5, 0, E)
    logits = np.stack([synth_mod.router_logits(5, t, 0, E) for t in range(T)])
    ids, w = oracle_mod.route(logits, k)
    ref = oracle_mod.select(w, ids, sens, avg)
    out = np.empty((T, k), np.uint8)
    pm.select_prefix(w, ids, sens, T, k, avg, out, on_device=False)
    np.testing.assert_array_equal(out, ref)


def test_invalid_arguments_are_rejected_on_the_host(pm):
    codes = np.zeros((15, 128), np.uint8)
    out = np.zeros(64 * 8, np.uint32)
    with pytest.raises(pm.PmoeError) as ei:
        pm.pack_bitplanes(codes, 15, 128, 8, out, 60, on_device=False)
    assert ei.value.code == 1
    with pytest.raises(pm.PmoeError):
        pm.tree_codebook(None)
    w = np.zeros((1, 40), np.float32)
    with pytest.raises(pm.PmoeError):
        pm.select_prefix(w, np.zeros((1, 40), np.int32), np.ones(8, np.float32), 1, 40, 2.5,
                         np.zeros(40, np.uint8), on_device=False)


def test_tensor_core_settings_are_checked_on_the_host(pm):
    """The tensor-core threshold takes 0 (off) or >= 8 (units are sized for at least 8 pairs); the
    operand self-check refuses shapes outside N in {16, 32, 48, 64}, K in {32, 64, 96, 128} before
    touching the device."""
    for bad in (-1, 1, 7):
        with pytest.raises(pm.PmoeError) as ei:
            pm.set_tc_min_tokens(bad)
        assert ei.value.code == 1
    for good in (0, 12, 16, 8):
        pm.set_tc_min_tokens(good)
    a = np.zeros((128, 128), np.int16)
    d = np.zeros((128, 64), np.float32)
    for N, K in ((8, 64), (24, 64), (80, 64), (32, 16), (32, 160), (32, 48)):
        with pytest.raises(pm.PmoeError) as ei:
            pm.tc_selfcheck(a, a, d, N, K)
        assert ei.value.code == 1


def test_workspace_queries(pm):
    a = pm.layer_workspace_bytes(1, 10, 512, 4096, 1024)
    b = pm.layer_workspace_bytes(32, 10, 512, 4096, 1024)
    assert 0 < a < b
    # batches of 8 tokens or more carry the tensor-core operand rows (3 x pairs rows of H and I
    # halves) and the gate/up rows of tensor-core pairs
    c7, c8 = pm.layer_workspace_bytes(7, 10, 512, 4096, 1024), pm.layer_workspace_bytes(8, 10, 512, 4096, 1024)
    assert c8 - c7 > 80 * (4096 + 1024) * 2
    m = pm.materialise_workspace_bytes(1, 10, 512, 4096, 1024)
    assert m >= 10 * 3 * 4096 * 1024 * 2  # bf16 copies of the ten selected experts


def test_host_buffer_decode_step_is_checked_on_the_host(pm):
    """The host-buffer decode step's workspace is the layer workspace plus 256-byte-padded room for
    the tokens' logits, x and y; null buffers and a short workspace are refused before any copy
    (the layer record only has to look valid: nothing is read from it on these paths)."""
    T, k, E, H, I = 3, 10, 512, 4096, 1024
    al = lambda n: (n + 255) // 256 * 256
    lb = pm.layer_workspace_bytes(T, k, E, H, I)
    assert pm.decode_host_workspace_bytes(T, k, E, H, I) == lb + al(T * E * 4) + al(T * H * 2) + al(T * H * 4)
    assert pm.decode_host_workspace_bytes(T, 0, E, H, I) == 0
    L = pm.Layer(E=E, H=H, I=I, G=128, pool=0x100000, slot_words=3 * H * I // 32, slot_of=0x200000,
                 scales=0x300000, codebooks=0x400000)
    host = np.zeros(T * H, np.float32)
    need = pm.decode_host_workspace_bytes(T, k, E, H, I)
    args = dict(logits=host, sens=0x500000, x=host, y=host, ws=0x600000)
    for missing in ("logits", "sens", "x", "y", "ws"):
        a = dict(args, **{missing: None})
        with pytest.raises(pm.PmoeError) as ei:
            pm.moe_decode_step_host(L, a["logits"], a["sens"], a["x"], T, k, 2.5, a["y"], a["ws"], need)
        assert ei.value.code == 1, missing
    with pytest.raises(pm.PmoeError) as ei:
        pm.moe_decode_step_host(L, host, 0x500000, host, T, k, 2.5, host, 0x600000, need - 256)
    assert ei.value.code == 5
    # zero tokens: nothing to do, no buffer is touched (all may be null)
    pm.moe_decode_step_host(L, None, None, None, 0, k, 2.5, None, None, 0)


def test_cache_aware_select_matches_oracle(pm, oracle_mod):
    rng = np.random.default_rng(11)
    T, k, E = 64, 10, 512
    w = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    sens = np.exp(0.5 * rng.standard_normal(E)).astype(np.float32)
    res = rng.integers(0, 9, (T, k)).astype(np.uint8)
    for fetch in (0, 3, 10, 25, 80):
        got = np.zeros((T, k), np.uint8)
        pm.select_prefix_cache_aware(w, ids, sens, res, T, k, fetch, got)
        assert np.array_equal(got, oracle_mod.select_cache_aware(w, ids, sens, res, fetch))


def test_profile_repair_and_table_select_match_oracle(pm, oracle_mod):
    rng = np.random.default_rng(12)
    n = 64
    raw = np.sort(rng.random((n, 8)) * rng.random((n, 1)), axis=1)[:, ::-1].copy()
    raw[:, 7] = 0.0
    raw[::3, 2] = raw[::3, 1]  # some profiles with a flat step (not convex)
    raw = raw.astype(np.float32)
    table = np.zeros_like(raw)
    pm.profile_repair(raw, n, table)
    ref = oracle_mod.profile_repair(raw.astype(np.float64))
    assert np.allclose(table, ref, rtol=1e-6, atol=1e-9)
    T, k = 100, 10
    w = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    ids = np.stack([rng.choice(n, k, replace=False) for _ in range(T)]).astype(np.int32)
    got = np.zeros((T, k), np.uint8)
    pm.select_prefix_table(w, ids, table, T, k, 2.5, got, on_device=False)
    assert np.array_equal(got, oracle_mod.select_table(w, ids, table, 2.5))


def test_cache_aware_matched_against_oracle():
    """pmoe_select_prefix_cache_aware_matched = the oracle's cache-aware selection with the fetch
    budget of the oracle's plain depths, and its surrogate sums; with nothing resident it is the
    plain allocator."""
    import oracle
    import synth
    import bitplane_mixed_precision_b200 as pm
    E, k, T = 512, 10, 64
    sens = synth.sensitivities(77, 0, E)
    logits = np.stack([synth.router_logits(77, t, 0, E) for t in range(T)])
    ids, w = oracle.route(logits, k)
    rng = np.random.default_rng(5)
    res = rng.integers(0, 9, (T, k)).astype(np.uint8)
    res[::3] = 0
    dep = np.empty((T, k), np.uint8)
    sur = np.zeros(2)
    pm.select_prefix_cache_aware_matched(w, ids, sens, res, T, k, 2.5, dep, sur)
    plain = oracle.select(w, ids, sens, 2.5)
    want_sur = np.zeros(2)
    for t in range(T):
        fetch = int(np.maximum(plain[t].astype(int) - res[t].astype(int), 0).sum())
        ref = oracle.select_cache_aware(w[t:t + 1], ids[t:t + 1], sens, res[t:t + 1], fetch)[0]
        np.testing.assert_array_equal(dep[t], ref)
        v2 = (w[t].astype(np.float64) * sens[ids[t]].astype(np.float64)) ** 2
        want_sur += [np.sum(v2 * 4.0 ** -plain[t].astype(float)), np.sum(v2 * 4.0 ** -ref.astype(float))]
    np.testing.assert_allclose(sur, want_sur, rtol=1e-12)
    assert sur[1] <= sur[0]
    zero = np.zeros((T, k), np.uint8)
    pm.select_prefix_cache_aware_matched(w, ids, sens, zero, T, k, 2.5, dep, None)
    np.testing.assert_array_equal(dep, plain)
