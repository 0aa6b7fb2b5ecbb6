"""The fused MoE layer (route, select, group, gate/up, SwiGLU, down, combine)
against the oracle on seeded synthetic layers of the pages' shapes."""
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


def run_step(pm, R, logits, xb, sens, k, avg):
    T, E = logits.shape
    H = R.H
    d_logits = torch.from_numpy(logits).cuda()
    d_x = torch.from_numpy(xb.view(np.int16)).cuda()
    d_sens = torch.from_numpy(sens).cuda()
    y = torch.empty(T * H, dtype=torch.float32, device="cuda")
    ids = torch.empty(T * k, dtype=torch.int32, device="cuda")
    w = torch.empty(T * k, dtype=torch.float32, device="cuda")
    dep = torch.empty(T * k, dtype=torch.uint8, device="cuda")
    nbytes = pm.layer_workspace_bytes(T, k, E, H, R.I)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    pm.moe_decode_step(R.layer, d_logits, d_sens, d_x, T, k, avg, y, ids, w, dep, ws, nbytes)
    torch.cuda.synchronize()
    assert pm.layer_error(ws) == (0, 0)
    return (y.cpu().numpy().reshape(T, H), ids.cpu().numpy().reshape(T, k),
            w.cpu().numpy().reshape(T, k), dep.cpu().numpy().reshape(T, k))


def check_layer(pm, seed, E, H, I, G, k, T, avg=2.5, bias=None, token0=0):
    R = ResidentLayer(E, H, I, G, device_fill(seed))
    O = OracleExperts(seed, H, I, G)
    sens = synth.sensitivities(seed, 0, E)
    logits, xb = tokens(seed, T, E, H, token0=token0, bias=bias)
    y, ids, w, dep = run_step(pm, R, logits, xb, sens, k, avg)
    ids_ref, w_ref = oracle.route(logits, k)
    np.testing.assert_array_equal(ids, ids_ref)
    np.testing.assert_array_equal(w, w_ref)
    dep_ref = oracle.select(w_ref, ids_ref, sens, avg)
    np.testing.assert_array_equal(dep, dep_ref)
    x64 = synth.bf16_to_f32(xb).astype(np.float64)
    ref = O.run(E, ids_ref, w_ref, dep_ref, x64)
    errs = [assert_close(y[t], ref[t], msg=f"token {t}")[0] for t in range(T)]
    return R, O, max(errs), dep


def test_small_layer_batch1(pm):
    """64 experts, top-8, hidden 2048, intermediate 768, group 128, batch-1 tokens."""
    for t in range(3):
        _, _, err, dep = check_layer(pm, 21, 64, 2048, 768, 128, 8, 1, token0=t)
        assert dep.mean() == 2.5
        assert err < 3e-4


def test_small_layer_batched_shares_experts(pm):
    """8 tokens over 64 experts: several tokens per expert, mixed depths."""
    check_layer(pm, 22, 64, 2048, 768, 128, 8, 8)


def test_large_shape_few_experts(pm):
    """Hidden 4096, intermediate 1024, top-10, but only 16 experts resident (T=5)."""
    check_layer(pm, 23, 16, 4096, 1024, 128, 10, 5)


def test_batched_zipf_ragged_blocks(pm):
    """32 tokens, Zipf(1.1) popularity bias over 24 experts: many tokens per expert,
    column blocks of 1-4 members, units split at 8 blocks."""
    E = 24
    bias = synth.zipf_bias(31, E)
    check_layer(pm, 31, E, 2048, 768, 128, 8, 32, bias=bias)


@pytest.mark.parametrize("avg", [1.0, 4.0, 8.0])
def test_budget_extremes(pm, avg):
    """avg 1 and 8 force every expert to 1 and 8 bits; avg 4 spends exactly 4 bits per expert."""
    _, _, _, dep = check_layer(pm, 41, 32, 2048, 768, 128, 8, 2, avg=avg)
    assert np.all(dep.sum(axis=1) == int(avg) * 8)
    if avg in (1.0, 8.0):
        assert np.all(dep == int(avg))


@pytest.mark.parametrize("b", [4, 1, 8])
def test_uniform_depth_layer(pm, b):
    """Uniform b-bit requests through pmoe_moe_layer_fwd (the uniform 4-bit run of the large layer)."""
    seed, E, H, I, G, k, T = 43, 16, 4096, 1024, 128, 10, 2
    R = ResidentLayer(E, H, I, G, device_fill(seed))
    O = OracleExperts(seed, H, I, G)
    logits, xb = tokens(seed, T, E, H)
    ids, w = oracle.route(logits, k)
    dep = np.full((T, k), b, np.uint8)
    y = torch.empty(T * H, dtype=torch.float32, device="cuda")
    nbytes = pm.layer_workspace_bytes(T, k, E, H, I)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    pm.moe_layer_fwd(R.layer, torch.from_numpy(xb.view(np.int16)).cuda(), torch.from_numpy(ids).cuda(),
                     torch.from_numpy(w).cuda(), torch.from_numpy(dep).cuda(), T, k, y, ws, nbytes)
    torch.cuda.synchronize()
    assert pm.layer_error(ws) == (0, 0)
    ref = O.run(E, ids, w, dep, synth.bf16_to_f32(xb).astype(np.float64))
    got = y.cpu().numpy().reshape(T, H)
    for t in range(T):
        assert_close(got[t], ref[t], msg=f"b={b} token {t}")


@pytest.mark.parametrize("G,T", [(64, 3), (32, 1), (32, 3)])
def test_group_sizes_64_and_32(pm, G, T):
    """Scale groups of 64 and 32 columns (two and four groups per 128-column tile), batch 1 and a
    3-token batch."""
    check_layer(pm, 42, 16, 1024, 512, G, 4, T)


@pytest.mark.parametrize("T,k", [(1, 4), (3, 4), (24, 10)])
def test_host_buffer_decode_step_matches_device_buffers(pm, T, k):
    """pmoe_moe_decode_step_host (logits, x and y in pinned host memory, one call per step) gives
    the device-buffer decode step's output bit for bit; pageable host buffers give it too. 24
    tokens of top-10 over 16 experts put pairs on the tensor-core units, whose operand kernel then
    reads x from the host buffer."""
    seed, E, H, I, G = 33, 16, 1024, 256, 128
    R = ResidentLayer(E, H, I, G, device_fill(seed))
    sens = synth.sensitivities(seed, 0, E)
    logits, xb = tokens(seed, T, E, H)
    pm.set_tc_min_tokens(8)  # (the default) tensor-core units from 8 pairs
    try:
        y_dev, _, _, _ = run_step(pm, R, logits, xb, sens, k, 2.5)
        nb = pm.decode_host_workspace_bytes(T, k, E, H, I)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        d_sens = torch.from_numpy(sens).cuda()
        lg = torch.from_numpy(logits).pin_memory()
        x = torch.from_numpy(xb.view(np.int16)).pin_memory()
        y = torch.full((T * H,), float("nan"), dtype=torch.float32).pin_memory()
        pm.moe_decode_step_host(R.layer, lg, d_sens, x, T, k, 2.5, y, ws, nb)
        torch.cuda.synchronize()
        assert pm.layer_error(ws) == (0, 0)
        np.testing.assert_array_equal(y.numpy().reshape(T, H), y_dev)
        if T >= 24:
            assert pm.layer_counts(ws)[2] > 0  # tensor-core units were formed
        y_np = np.full(T * H, np.nan, np.float32)
        pm.moe_decode_step_host(R.layer, np.ascontiguousarray(logits), d_sens, xb.view(np.int16).copy(), T, k, 2.5,
                                y_np, ws, nb)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(y_np.reshape(T, H), y_dev)
    finally:
        pm.set_tc_min_tokens(8)


def test_zero_tokens_is_a_no_op(pm):
    R = ResidentLayer(8, 1024, 256, 128, device_fill(1))
    y = torch.full((4,), 7.0, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    pm.moe_layer_fwd(R.layer, torch.zeros(8, dtype=torch.int16, device="cuda"),
                     torch.zeros(1, dtype=torch.int32, device="cuda"), torch.zeros(1, device="cuda"),
                     torch.ones(1, dtype=torch.uint8, device="cuda"), 0, 2, y, ws, 256)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)


def test_workspace_too_small_is_rejected(pm):
    R = ResidentLayer(8, 1024, 256, 128, device_fill(1))
    need = pm.layer_workspace_bytes(1, 2, 8, 1024, 256)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    with pytest.raises(pm.PmoeError) as ei:
        pm.moe_layer_fwd(R.layer, torch.zeros(1024, dtype=torch.int16, device="cuda"),
                         torch.zeros(2, dtype=torch.int32, device="cuda"), torch.zeros(2, device="cuda"),
                         torch.ones(2, dtype=torch.uint8, device="cuda"), 1, 2,
                         torch.empty(1024, device="cuda"), ws, need - 256)
    assert ei.value.code == 5


def test_materialise_ablation(pm):
    """Decode-to-bf16-then-GEMV equals the oracle with bf16-rounded weights."""
    seed, E, H, I, G, k, T = 51, 16, 2048, 768, 128, 8, 2
    R = ResidentLayer(E, H, I, G, device_fill(seed))
    O = OracleExperts(seed, H, I, G)
    sens = synth.sensitivities(seed, 0, E)
    logits, xb = tokens(seed, T, E, H)
    ids, w = oracle.route(logits, k)
    dep = oracle.select(w, ids, sens, 2.5)
    y = torch.empty(T * H, dtype=torch.float32, device="cuda")
    nbytes = pm.materialise_workspace_bytes(T, k, E, H, I)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    pm.materialise_layer_fwd(R.layer, torch.from_numpy(xb.view(np.int16)).cuda(), torch.from_numpy(ids).cuda(),
                             torch.from_numpy(w).cuda(), torch.from_numpy(dep).cuda(), T, k, y, ws, nbytes)
    torch.cuda.synchronize()
    x64 = synth.bf16_to_f32(xb).astype(np.float64)
    ref_bf16 = O.run(E, ids, w, dep, x64, bf16_weights=True)
    got = y.cpu().numpy().reshape(T, H)
    for t in range(T):
        assert_close(got[t], ref_bf16[t], msg=f"token {t}")


def test_missing_plane_is_reported_not_hung(pm):
    """A selected expert whose plane has no slot: the call completes and records error 2."""
    seed, E, H, I, G, k, T = 61, 8, 1024, 256, 128, 2, 1
    R = ResidentLayer(E, H, I, G, device_fill(seed))
    ids = np.array([[3, 5]], np.int32)
    w = np.array([[0.5, 0.5]], np.float32)
    dep = np.array([[2, 1]], np.uint8)
    R.slot_of[3 * 8 + 1] = -1  # plane 1 of expert 3 is absent
    y = torch.empty(T * H, dtype=torch.float32, device="cuda")
    nbytes = pm.layer_workspace_bytes(T, k, E, H, I)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    xb = synth.activation_bf16(seed, 0, 0, H)
    pm.moe_layer_fwd(R.layer, torch.from_numpy(xb.view(np.int16)).cuda(), torch.from_numpy(ids).cuda(),
                     torch.from_numpy(w).cuda(), torch.from_numpy(dep).cuda(), T, k, y, ws, nbytes)
    code, detail = pm.layer_error(ws)
    assert code == 2 and detail == 3 * 8 + 1
    # a complete layer reports no error
    R.slot_of[3 * 8 + 1] = 3 * 8 + 1
    pm.moe_layer_fwd(R.layer, torch.from_numpy(xb.view(np.int16)).cuda(), torch.from_numpy(ids).cuda(),
                     torch.from_numpy(w).cuda(), torch.from_numpy(dep).cuda(), T, k, y, ws, nbytes)
    assert pm.layer_error(ws) == (0, 0)


def test_unsupported_shapes_are_rejected(pm):
    R = ResidentLayer(4, 1536, 256, 128, device_fill(1), experts=[])
    need = pm.layer_workspace_bytes(1, 2, 4, 1536, 256)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    with pytest.raises(pm.PmoeError) as ei:
        pm.moe_layer_fwd(R.layer, torch.zeros(1536, dtype=torch.int16, device="cuda"),
                         torch.zeros(2, dtype=torch.int32, device="cuda"), torch.zeros(2, device="cuda"),
                         torch.ones(2, dtype=torch.uint8, device="cuda"), 1, 2,
                         torch.empty(1536, device="cuda"), ws, need)
    assert ei.value.code == 7
