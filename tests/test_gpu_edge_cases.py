"""Edge cases of the method on the GPU, against the oracle.

* A skewed, heavy-tailed tree codebook built from sorted leaves with frequencies
  (PagedMoE transcript cues 19 and 21: parents are frequency-weighted means), so
  the table is not antisymmetric: the general depth-1 path and per-depth
  fixed-point exponents of a wide table are exercised at every depth.
* Heavy-tailed activations: channels at 100x and 1000x the rest, and Student-t
  values, through the single-matrix GEMV and the layer.
* Routing ties between -0 and +0 logits on the device (they are equal numbers:
  the lower expert id wins).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from bitplane_mixed_precision_b200.store import ResidentLayer
from gpu_common import OracleExperts, assert_close, device_fill, tokens

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pm():
    import bitplane_mixed_precision_b200 as pm
    return pm


def f32_to_bf16(v):
    """Round-to-nearest-even float32 -> bf16 bit patterns (uint16)."""
    u = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def skewed_table(pm, seed):
    leaves, freq = synth.tree_leaves(seed)
    cb = np.empty(510, np.float32)
    pm.tree_codebook_from_leaves(leaves, freq, cb)
    ref = oracle.tree_from_leaves(leaves, freq.astype(np.float64)).astype(np.float32)
    assert np.array_equal(cb, ref)
    assert cb[0] != -cb[1]  # not antisymmetric at depth 1
    return cb


def heavy_x(seed, n, kind):
    z = synth.activation_f32(seed, 0, 0, n).astype(np.float64)
    if kind == "outliers":
        z[[5, 300 % n, n - 7]] *= np.array([100.0, 1000.0, -1000.0])
        z[(n // 2) + 1] *= 100.0
    elif kind == "student_t":
        c = synth.normal_f64(seed, synth.stream_id(synth.K_X, 7, 1), 3 * n).reshape(3, n)
        z = z / np.sqrt((c ** 2).sum(axis=0) / 3.0)
    return z.astype(np.float32)


def _matrix(pm, seed, N, K, G, cb):
    w = synth.expert_weights(seed, 0, 0, 0, N, K)
    s_ref, c_ref = oracle.quantize(w, G)
    s = torch.empty(N * (K // G), dtype=torch.float32, device="cuda")
    c = torch.empty(N * K, dtype=torch.uint8, device="cuda")
    pm.quantize(torch.from_numpy(w).cuda(), N, K, G, s, c)
    planes = torch.empty(8 * N * K // 32, dtype=torch.int32, device="cuda")
    pm.pack_bitplanes(c, N, K, 8, planes, N * K // 32, on_device=True)
    cbd = torch.from_numpy(cb).cuda()
    torch.cuda.synchronize()
    assert np.array_equal(c.cpu().numpy().reshape(N, K), c_ref)
    return pm.make_matrix(planes, N * K // 32, s, cbd, N, K, G), (planes, s, cbd), (c_ref, s_ref)


@pytest.mark.parametrize("b", range(1, 9))
def test_gemv_skewed_codebook(pm, b):
    N, K, G = 256, 1024, 128
    cb = skewed_table(pm, 11)
    m, keep, (c_ref, s_ref) = _matrix(pm, 12, N, K, G, cb)
    x = synth.activation_f32(12, 0, 0, K)
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    pm.expert_gemv(m, b, torch.from_numpy(x).cuda(), False, y)
    torch.cuda.synchronize()
    ref = oracle.gemv(c_ref, s_ref, cb, G, b, x.astype(np.float64))
    assert_close(y.cpu().numpy(), ref, msg=f"skewed table b={b}")


@pytest.mark.parametrize("kind", ["outliers", "student_t"])
@pytest.mark.parametrize("b", [1, 2, 3, 4, 6, 8])
def test_gemv_heavy_tailed_activations(pm, kind, b):
    N, K, G = 128, 4096, 128
    cb = oracle.tree_codebook_f32()
    m, keep, (c_ref, s_ref) = _matrix(pm, 13, N, K, G, cb)
    x = heavy_x(14, K, kind)
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    pm.expert_gemv(m, b, torch.from_numpy(x).cuda(), False, y)
    torch.cuda.synchronize()
    ref = oracle.gemv(c_ref, s_ref, cb, G, b, x.astype(np.float64))
    assert_close(y.cpu().numpy(), ref, msg=f"{kind} b={b}")


def _oracle_run(O, E, ids, w, dep, x64, tables=None):
    need = {}
    for e in np.unique(ids):
        codes, scales = [], []
        for m, (n, k) in enumerate(((O.I, O.H), (O.I, O.H), (O.H, O.I))):
            wt = synth.expert_weights(O.seed, O.layer, int(e), m, n, k)
            s, c = oracle.quantize(wt, O.G)
            codes.append(c)
            scales.append(s)
        cbs = tables if tables is not None else [oracle.tree_codebook_f32()] * 3
        need[int(e)] = oracle.Expert(codes, scales, cbs)
    return oracle.moe_layer(need, E, O.H, O.I, O.G, ids, w, dep, x64)


def _run_layer(pm, R, xb, ids, w, dep):
    T, k = ids.shape
    y = torch.empty(T * R.H, dtype=torch.float32, device="cuda")
    nbytes = pm.layer_workspace_bytes(T, k, R.E, R.H, R.I)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    pm.moe_layer_fwd(R.layer, torch.from_numpy(xb.view(np.int16)).cuda(), torch.from_numpy(ids).cuda(),
                     torch.from_numpy(w).cuda(), torch.from_numpy(dep).cuda(), T, k, y, ws, nbytes)
    torch.cuda.synchronize()
    assert pm.layer_error(ws) == (0, 0)
    return y.cpu().numpy().reshape(T, R.H)


@pytest.mark.parametrize("T", [1, 3])
def test_layer_skewed_tables_every_depth(pm, T):
    """Gate, up and down decode with three different skewed tables; the k experts of each token
    are set to depths 1..8 in turn, so every depth runs through the layer."""
    seed, E, H, I, G, k = 15, 16, 4096, 1024, 128, 8
    tables = [skewed_table(pm, 20 + m) for m in range(3)]
    R = ResidentLayer(E, H, I, G, device_fill(seed))
    R.codebooks.copy_(torch.from_numpy(np.concatenate([np.concatenate(tables)] * E)))
    O = OracleExperts(seed, H, I, G)
    logits, xb = tokens(seed, T, E, H)
    ids, w = oracle.route(logits, k)
    dep = np.stack([np.roll(np.arange(1, 9, dtype=np.uint8), t) for t in range(T)])
    got = _run_layer(pm, R, xb, ids, w, dep)
    ref = _oracle_run(O, E, ids, w, dep, synth.bf16_to_f32(xb).astype(np.float64), tables)
    for t in range(T):
        assert_close(got[t], ref[t], msg=f"token {t}")


@pytest.mark.parametrize("kind", ["outliers", "student_t"])
def test_layer_heavy_tailed_activations(pm, kind):
    seed, E, H, I, G, k, T = 16, 16, 4096, 1024, 128, 10, 2
    R = ResidentLayer(E, H, I, G, device_fill(seed))
    O = OracleExperts(seed, H, I, G)
    logits, _ = tokens(seed, T, E, H)
    xb = np.stack([f32_to_bf16(heavy_x(30 + t, H, kind)) for t in range(T)])
    ids, w = oracle.route(logits, k)
    dep = oracle.select(w, ids, synth.sensitivities(seed, 0, E), 2.5)
    got = _run_layer(pm, R, xb, ids, w, dep)
    ref = O.run(E, ids, w, dep, synth.bf16_to_f32(xb).astype(np.float64))
    for t in range(T):
        assert_close(got[t], ref[t], msg=f"{kind} token {t}")


def test_route_signed_zero_ties_on_device(pm):
    """-0 and +0 are the same logit value: ties, broken toward the lower expert id, on the
    device as in the oracle; the softmax weights of tied zeros are equal."""
    E, k = 64, 6
    logits = np.full((3, E), -1.0, np.float32)
    logits[0, [9, 3, 40, 17]] = [-0.0, 0.0, -0.0, 0.0]          # four tied zeros, k > 4
    logits[1, [5, 6, 7, 8, 9, 10, 11]] = [0.0, -0.0, 0.0, -0.0, 0.0, -0.0, 0.0]  # boundary inside the ties
    logits[2, [33, 2]] = [-0.0, 0.0]
    logits[2, 50] = 0.5
    ids_ref, w_ref = oracle.route(logits, k)
    d = torch.from_numpy(logits).cuda()
    ids = torch.empty(3 * k, dtype=torch.int32, device="cuda")
    w = torch.empty(3 * k, dtype=torch.float32, device="cuda")
    pm.route(d, 3, E, k, ids, w)
    torch.cuda.synchronize()
    ids_d = ids.cpu().numpy().reshape(3, k)
    np.testing.assert_array_equal(ids_d, ids_ref)
    np.testing.assert_array_equal(w.cpu().numpy().reshape(3, k), w_ref)
    np.testing.assert_array_equal(ids_d[0][:4], [3, 9, 17, 40])
    np.testing.assert_array_equal(ids_d[1], [5, 6, 7, 8, 9, 10])
    np.testing.assert_array_equal(ids_d[2][:3], [50, 2, 33])
    # the decode step routes the same way (batch-1 tokens, one at a time)
    R = ResidentLayer(E, 1024, 256, 128, device_fill(3), experts=[])
    sens = synth.sensitivities(3, 0, E)
    for t in range(3):
        y = torch.empty(1024, dtype=torch.float32, device="cuda")
        i1 = torch.empty(k, dtype=torch.int32, device="cuda")
        w1 = torch.empty(k, dtype=torch.float32, device="cuda")
        d1 = torch.empty(k, dtype=torch.uint8, device="cuda")
        nb = pm.layer_workspace_bytes(1, k, E, 1024, 256)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        pm.moe_decode_step(R.layer, torch.from_numpy(logits[t]).cuda(), torch.from_numpy(sens).cuda(),
                           torch.zeros(1024, dtype=torch.int16, device="cuda"), 1, k, 2.5, y, i1, w1, d1,
                           ws, nb)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(i1.cpu().numpy(), ids_ref[t])
        np.testing.assert_array_equal(w1.cpu().numpy(), w_ref[t])
