"""The batched layer's tensor-core path (experts hit by many tokens of a batch), against the oracle.

* The operand path itself: D = A * B^T through the tcgen05 MMA with the kernel's shared-memory
  layout, descriptors and tensor-memory loads, against a float64 matmul of the same f16 values.
* Layers whose popular experts are hit by 8 or more pairs at depths 1..4 (they go to the tensor
  cores, one accumulator per tree level) next to deeper pairs of the same experts and rare experts
  (they stay with the persistent kernel): every token's output against the oracle's dequantise-then-
  multiply, at the workloads' tolerance. Batches of 24 and 128 tokens; the 128-token batch gives an
  expert more pairs than one unit holds (64), so its pairs are split between two units.
PagedMoE transcript cues 13, 29, 35 (pairs grouped per expert, tokens at different depths sharing the
planes they have in common).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from bitplane_mixed_precision_b200.store import ResidentLayer
from gpu_common import OracleExperts, assert_close, device_fill

pytestmark = pytest.mark.gpu

E, H, I, G = 16, 1024, 256, 128
SEED = 2031
TC_DEFAULT = 8  # the library's default threshold (pairs per expert)


@pytest.fixture(scope="module")
def pm():
    import bitplane_mixed_precision_b200 as pm
    return pm


@pytest.fixture(scope="module")
def mid():
    R = ResidentLayer(E, H, I, G, device_fill(SEED))
    O = OracleExperts(SEED, H, I, G)
    torch.cuda.synchronize()
    return R, O


@pytest.mark.parametrize("N,K", [(16, 32), (32, 64), (48, 96), (64, 128)])
def test_operand_path_matches_matmul(pm, N, K):
    g = torch.Generator().manual_seed(1000 * N + K)
    A = torch.randn(128, K, generator=g).half()
    B = torch.randn(N, K, generator=g).half()
    D = torch.full((128, N), float("nan"), device="cuda")
    pm.tc_selfcheck(A.cuda().view(torch.int16), B.cuda().view(torch.int16), D, N, K)
    torch.cuda.synchronize()
    ref = A.double() @ B.double().T
    err = float((D.cpu().double() - ref).abs().max() / ref.abs().max())
    assert err < 1e-5, err


def test_operand_path_rejects_other_shapes(pm):
    A = torch.zeros(128, 64, dtype=torch.int16, device="cuda")
    D = torch.zeros(128, 64, device="cuda")
    for N, K in ((8, 64), (24, 64), (80, 64), (32, 16), (32, 160)):
        with pytest.raises(RuntimeError):
            pm.tc_selfcheck(A, A, D, N, K)


def _batch(T, k, rng):
    """Experts 0..2 are hit by every token (0: depths 1..4; 1: depths 1..6, the deeper ones staying with
    the persistent kernel; 2: depth 4), the last slot goes to a rare expert."""
    ids = np.zeros((T, k), np.int32)
    dep = np.zeros((T, k), np.uint8)
    for t in range(T):
        ids[t] = [0, 1, 2] + [3 + (t + j) % (E - 3) for j in range(k - 3)]
        dep[t] = [1 + t % 4, 1 + t % 6, 4] + [1 + (t + j) % 8 for j in range(k - 3)]
    z = rng.standard_normal((T, k))
    w = np.exp(z - z.max(axis=1, keepdims=True))
    w = (w / w.sum(axis=1, keepdims=True)).astype(np.float32)
    x = np.stack([synth.activation_bf16(SEED, 50 + t, 0, H) for t in range(T)])
    return ids, w, dep, x


@pytest.mark.parametrize("T,tc_min", [(24, 8), (128, 8), (128, 12)])
def test_layer_with_tensor_core_units(pm, mid, T, tc_min):
    """The rule at the default threshold (8 pairs, the smallest the workspace allows) and at 12."""
    R, O = mid
    k = 4
    ids, w, dep, x = _batch(T, k, np.random.default_rng(T))
    y = torch.empty(T * H, dtype=torch.float32, device="cuda")
    nb = pm.layer_workspace_bytes(T, k, E, H, I)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    pm.set_tc_min_tokens(tc_min)
    try:
        pm.moe_layer_fwd(R.layer, torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(ids).cuda(),
                         torch.from_numpy(w).cuda(), torch.from_numpy(dep).cuda(), T, k, y, ws, nb)
        torch.cuda.synchronize()
    finally:
        pm.set_tc_min_tokens(TC_DEFAULT)
    assert pm.layer_error(ws) == (0, 0)
    blocks, units, tcu, rows = pm.layer_counts(ws)
    # every expert with at least tc_min pairs at depth <= 4 gives them to units of at most 64 pairs
    shallow = np.bincount(ids[dep <= 4], minlength=E)
    expect = sum((int(n) + 63) // 64 for n in shallow if n >= tc_min)
    assert tcu == expect >= 3, (tcu, expect)
    assert rows >= int(shallow[shallow >= tc_min].sum()) and rows % 16 == 0
    ref = O.run(E, ids, w, dep, synth.bf16_to_f32(x).astype(np.float64))
    got = y.cpu().numpy().reshape(T, H)
    for t in range(T):
        assert_close(got[t], ref[t], msg=f"token {t}")


@pytest.mark.parametrize("Gs", [64, 32])
def test_tensor_core_units_with_smaller_scale_groups(pm, Gs):
    """Scale groups of 64 and 32 columns: the epilogue applies two or four group scales per 128-column
    tile of the tensor-core accumulators; every token against the oracle."""
    R = ResidentLayer(E, H, I, Gs, device_fill(SEED + Gs))
    O = OracleExperts(SEED + Gs, H, I, Gs)
    T, k = 24, 4
    ids, w, dep, x = _batch(T, k, np.random.default_rng(T))
    y = torch.empty(T * H, dtype=torch.float32, device="cuda")
    nb = pm.layer_workspace_bytes(T, k, E, H, I)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    pm.moe_layer_fwd(R.layer, torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(ids).cuda(),
                     torch.from_numpy(w).cuda(), torch.from_numpy(dep).cuda(), T, k, y, ws, nb)
    torch.cuda.synchronize()
    assert pm.layer_error(ws) == (0, 0)
    assert pm.layer_counts(ws)[2] >= 3  # tensor-core units were formed
    ref = O.run(E, ids, w, dep, synth.bf16_to_f32(x).astype(np.float64))
    got = y.cpu().numpy().reshape(T, H)
    for t in range(T):
        assert_close(got[t], ref[t], msg=f"G={Gs} token {t}")


def test_small_batches_keep_the_persistent_path(pm, mid):
    """Fewer than 8 tokens (or no expert with 8 shallow pairs): no tensor-core unit."""
    R, O = mid
    k = 4
    for T in (1, 6):
        ids, w, dep, x = _batch(T, k, np.random.default_rng(T))
        y = torch.empty(T * H, dtype=torch.float32, device="cuda")
        nb = pm.layer_workspace_bytes(T, k, E, H, I)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        pm.moe_layer_fwd(R.layer, torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(ids).cuda(),
                         torch.from_numpy(w).cuda(), torch.from_numpy(dep).cuda(), T, k, y, ws, nb)
        torch.cuda.synchronize()
        assert pm.layer_counts(ws)[2] == 0
        ref = O.run(E, ids, w, dep, synth.bf16_to_f32(x).astype(np.float64))
        got = y.cpu().numpy().reshape(T, H)
        for t in range(T):
            assert_close(got[t], ref[t], msg=f"T={T} token {t}")


def test_deep_pairs_only_keep_the_persistent_path(pm, mid):
    """An expert hit by many pairs all deeper than 4 bits stays with the persistent kernel."""
    R, O = mid
    T, k = 16, 4
    ids, w, dep, x = _batch(T, k, np.random.default_rng(7))
    dep[:, :3] = 5 + (np.arange(T) % 4)[:, None]
    y = torch.empty(T * H, dtype=torch.float32, device="cuda")
    nb = pm.layer_workspace_bytes(T, k, E, H, I)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    pm.moe_layer_fwd(R.layer, torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(ids).cuda(),
                     torch.from_numpy(w).cuda(), torch.from_numpy(dep).cuda(), T, k, y, ws, nb)
    torch.cuda.synchronize()
    assert pm.layer_counts(ws)[2] == 0
    ref = O.run(E, ids, w, dep, synth.bf16_to_f32(x).astype(np.float64))
    got = y.cpu().numpy().reshape(T, H)
    for t in range(T):
        assert_close(got[t], ref[t], msg=f"token {t}")
