"""Parity at the workloads' own shapes, against the oracle.

* The large layer: 512 experts, top-10, hidden 4096, expert intermediate 1024,
  group 128, batch-1 decode steps at an average of 2.5 bits (routing, selection
  and grouping on the device), and a uniform 4-bit call on the same layer.
* The batch over it: 32 tokens whose router logits carry a Zipf(1.1) popularity
  bias, one decode step, (token, expert) pairs grouped per expert.
* 16 stacked layers of that shape decoded through the HBM prefix cache with a
  slot pool small enough to evict: outputs bit-identical to the same layers
  fully resident, the cache's decisions equal to the oracle simulator's, and
  layers checked against the oracle with their own inputs (teacher forcing).
PagedMoE transcript cues 4, 13, 29, 35; the model shape of cue 4.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from bitplane_mixed_precision_b200.store import ResidentLayer
from gpu_common import OracleExperts, assert_close, device_fill, tokens

pytestmark = pytest.mark.gpu

E, H, I, G, K, AVG = 512, 4096, 1024, 128, 10, 2.5
SEED = 2027


@pytest.fixture(scope="module")
def pm():
    import bitplane_mixed_precision_b200 as pm
    return pm


@pytest.fixture(scope="module")
def big():
    R = ResidentLayer(E, H, I, G, device_fill(SEED))
    O = OracleExperts(SEED, H, I, G)
    torch.cuda.synchronize()
    return R, O


def _decode(pm, R, logits, xb, sens, T):
    y = torch.empty(T * H, dtype=torch.float32, device="cuda")
    ids = torch.empty(T * K, dtype=torch.int32, device="cuda")
    w = torch.empty(T * K, dtype=torch.float32, device="cuda")
    dep = torch.empty(T * K, dtype=torch.uint8, device="cuda")
    nb = pm.layer_workspace_bytes(T, K, E, H, I)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    pm.moe_decode_step(R.layer, torch.from_numpy(logits).cuda(), torch.from_numpy(sens).cuda(),
                       torch.from_numpy(xb.view(np.int16)).cuda(), T, K, AVG, y, ids, w, dep, ws, nb)
    torch.cuda.synchronize()
    assert pm.layer_error(ws) == (0, 0)
    return (y.cpu().numpy().reshape(T, H), ids.cpu().numpy().reshape(T, K), w.cpu().numpy().reshape(T, K),
            dep.cpu().numpy().reshape(T, K))


def _check_routing(logits, sens, ids, w, dep):
    ids_ref, w_ref = oracle.route(logits, K)
    np.testing.assert_array_equal(ids, ids_ref)
    np.testing.assert_array_equal(w, w_ref)
    np.testing.assert_array_equal(dep, oracle.select(w_ref, ids_ref, sens, AVG))


def test_large_layer_batch1_decode_steps(pm, big):
    """Four fresh batch-1 tokens through the whole decode step at the headline shape."""
    R, O = big
    sens = synth.sensitivities(SEED, 0, E)
    for t in range(4):
        logits, xb = tokens(SEED, 1, E, H, token0=100 + t)
        y, ids, w, dep = _decode(pm, R, logits, xb, sens, 1)
        _check_routing(logits, sens, ids, w, dep)
        assert dep.sum() == 25
        ref = O.run(E, ids, w, dep, synth.bf16_to_f32(xb).astype(np.float64))
        assert_close(y[0], ref[0], msg=f"token {t}")


def test_large_layer_uniform_4_bits(pm, big):
    R, O = big
    logits, xb = tokens(SEED, 2, E, H, token0=200)
    ids, w = oracle.route(logits, K)
    dep = np.full((2, K), 4, np.uint8)
    y = torch.empty(2 * H, dtype=torch.float32, device="cuda")
    nb = pm.layer_workspace_bytes(2, K, E, H, I)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    pm.moe_layer_fwd(R.layer, torch.from_numpy(xb.view(np.int16)).cuda(), torch.from_numpy(ids).cuda(),
                     torch.from_numpy(w).cuda(), torch.from_numpy(dep).cuda(), 2, K, y, ws, nb)
    torch.cuda.synchronize()
    assert pm.layer_error(ws) == (0, 0)
    ref = O.run(E, ids, w, dep, synth.bf16_to_f32(xb).astype(np.float64))
    got = y.cpu().numpy().reshape(2, H)
    for t in range(2):
        assert_close(got[t], ref[t], msg=f"token {t}")


def test_large_layer_zipf_batch_of_32(pm, big):
    """32 tokens in one step, Zipf(1.1)-biased routing: popular experts carry many pairs at mixed
    depths, rare ones one or two."""
    R, O = big
    sens = synth.sensitivities(SEED, 0, E)
    bias = synth.zipf_bias(SEED, E)
    logits, xb = tokens(SEED, 32, E, H, token0=300, bias=bias)
    y, ids, w, dep = _decode(pm, R, logits, xb, sens, 32)
    _check_routing(logits, sens, ids, w, dep)
    counts = np.bincount(ids.reshape(-1), minlength=E)
    assert counts.max() >= 8  # some experts are hit by many tokens
    ref = O.run(E, ids, w, dep, synth.bf16_to_f32(xb).astype(np.float64))
    for t in range(32):
        assert_close(y[t], ref[t], msg=f"token {t}")


@pytest.mark.parametrize("T", [64, 128])
def test_large_layer_zipf_batches_of_64_and_128(pm, big, T):
    """Larger Zipf(1.1)-biased batches: the popular experts go to the tensor-core units (one
    accumulator per tree level, up to 64 pairs each); routing and selection bit-exact, a sample of
    tokens (those with the most tensor-core pairs and a few others) element-wise against the oracle."""
    R, O = big
    sens = synth.sensitivities(SEED, 0, E)
    bias = synth.zipf_bias(SEED, E)
    logits, xb = tokens(SEED, T, E, H, token0=1000 + T, bias=bias)
    y, ids, w, dep = _decode(pm, R, logits, xb, sens, T)
    _check_routing(logits, sens, ids, w, dep)
    shallow = np.bincount(ids[dep <= 4], minlength=E)
    hot = shallow >= 8
    assert hot.sum() >= 4
    n_tc = (hot[ids] & (dep <= 4)).sum(axis=1)
    sample = sorted(set(np.argsort(-n_tc, kind="stable")[:6].tolist()) | {0, T // 2, T - 1})
    ref = O.run(E, ids[sample], w[sample], dep[sample], synth.bf16_to_f32(xb[sample]).astype(np.float64))
    for j, t in enumerate(sample):
        assert_close(y[t], ref[j], msg=f"token {t}")


L_STACK = 16


def _backing(b):
    st = torch.cuda.current_stream()

    def fill(e, m, w):
        synth.expert_weights_device(SEED + 1, b, e, m, w.numel(), w.data_ptr(), st.cuda_stream)
    return ResidentLayer(E, H, I, G, fill)


def test_cached_16_layer_decode_with_evictions(pm):
    """16 layers of the large shape through the prefix cache (layer l backed by the planes of
    backing l % 2), 3 tokens of AR(1)-correlated routing, 700 plane slots so that later tokens
    evict: outputs equal the resident layers bit for bit, the evictions and fetches equal the
    oracle simulator's, and three layers of the last token match the oracle."""
    from bitplane_mixed_precision_b200.cached import CachedStack
    synth.build()
    dev = torch.device("cuda", 0)
    backs = [_backing(b) for b in range(2)]
    sens = [synth.sensitivities(SEED + 1, b, E) for b in range(2)]
    torch.cuda.synchronize()
    slots, ntok = 700, 3
    S = CachedStack(L_STACK, E, H, I, G, K, AVG, slots, backs, sens, device=dev, keep_log=True)
    logits = np.stack([synth.ar1_logits(SEED + 1, l, ntok, E) for l in range(L_STACK)], axis=1)
    r = torch.empty(H, dtype=torch.float32, device=dev)
    x = torch.empty(H, dtype=torch.int16, device=dev)
    y = torch.empty(H, dtype=torch.float32, device=dev)
    rr, xr, yr = torch.empty_like(r), torch.empty_like(x), torch.empty_like(y)
    ws = torch.empty(pm.layer_workspace_bytes(1, K, E, H, I), dtype=torch.uint8, device=dev)
    last = None
    for t in range(ntok):
        r.copy_(torch.from_numpy(synth.activation_f32(SEED + 1, t, 99, H)))
        pm.residual_norm(r, None, 1, H, x)
        rr.copy_(r)
        xr.copy_(x)
        y_out = torch.empty(L_STACK, H, dtype=torch.float32, device=dev)
        s = S.decode_token(logits[t], r, x, y, t, y_out=y_out)
        ids, w, dep = S.routing(s)
        xs = []
        for l in range(L_STACK):
            xs.append(xr.clone())
            pm.moe_layer_fwd(backs[l % 2].layer, xr, torch.from_numpy(ids[l]).to(dev),
                             torch.from_numpy(w[l]).to(dev), torch.from_numpy(dep[l]).to(dev), 1, K, yr, ws,
                             ws.numel())
            assert torch.equal(y_out[l], yr), f"token {t} layer {l}"
            pm.residual_norm(rr, yr, 1, H, xr)
        torch.cuda.synchronize()
        assert S.check_errors() == (0, 0)
        assert pm.layer_error(ws) == (0, 0)
        for l in range(L_STACK):
            ids_o, w_o = oracle.route(logits[t][l][None, :], K)
            assert np.array_equal(ids[l], ids_o[0]) and np.array_equal(w[l], w_o[0])
            assert np.array_equal(dep[l], oracle.select(w_o, ids_o, sens[l % 2], AVG)[0])
        last = (ids, w, dep, [xx.cpu().numpy().view(np.uint16) for xx in xs], y_out.cpu().numpy())
    st = S.cache.stats()
    assert st.planes_evicted > 0 and st.hits > 0
    lay, exp_, dp, bat = S.trace_arrays()
    _, log_o, fetched_o = oracle.cache_sim_prefix(L_STACK, E, slots, lay.astype(np.int32), exp_.astype(np.int32),
                                                  dp.astype(np.uint8), bat.astype(np.int32))
    assert np.array_equal(S.cache.eviction_log(), log_o)
    assert st.planes_fetched == fetched_o
    S.close()
    ids, w, dep, xs, youts = last
    oe = [OracleExperts(SEED + 1, H, I, G, layer=b) for b in range(2)]
    for l in (0, 7, 15):
        x64 = synth.bf16_to_f32(xs[l]).astype(np.float64)[None, :]
        ref = oe[l % 2].run(E, ids[l][None, :], w[l][None, :], dep[l][None, :], x64)
        assert_close(youts[l], ref[0], msg=f"layer {l}")
