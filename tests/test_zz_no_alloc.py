"""The allocation-free layer call against the workspace one.

pmoe_moe_layer_fwd_noalloc serves callers that cannot give the library a
device allocation for scratch (an engine that owns all device memory, a
fixed memory budget): its scratch is a fixed array inside the library that
every call shares and that keeps the last call's contents. This checks,
through the C ABI, that calls of different sizes in a row on one stream (so
that what an earlier, larger call left in the array is there for the next)
give the same output as pmoe_moe_layer_fwd within the tolerance of the other
layer tests, that one of them matches the oracle, that errors the kernels
record in the array can be read back, and that sizes beyond the array are
rejected. The file sorts last so that a stop-at-first-failure run has run
every other test.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from bitplane_mixed_precision_b200.store import ResidentLayer
from gpu_common import OracleExperts, assert_close, device_fill, tokens

pytestmark = pytest.mark.gpu

SEED, E, H, I, G, K = 71, 16, 4096, 1024, 128, 10


@pytest.fixture(scope="module")
def layer():
    return ResidentLayer(E, H, I, G, device_fill(SEED))


def _inputs(T, token0, sens):
    logits, xb = tokens(SEED, T, E, H, token0=token0)
    ids, w = oracle.route(logits, K)
    dep = oracle.select(w, ids, sens, 2.5)
    return xb, ids, w, dep


def test_noalloc_matches_workspace_call_over_changing_sizes(layer):
    import bitplane_mixed_precision_b200 as pm
    sens = synth.sensitivities(SEED, 0, E)
    O = OracleExperts(SEED, H, I, G)
    for call, T in enumerate((6, 1, 3, 1, 2)):
        nbytes = pm.layer_workspace_bytes(T, K, E, H, I)
        assert nbytes <= pm.noalloc_scratch_bytes()
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        xb, ids, w, dep = _inputs(T, 10 * call, sens)
        xd = torch.from_numpy(xb.view(np.int16)).cuda()
        idd, wd, dd = torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), torch.from_numpy(dep).cuda()
        y_ref = torch.empty(T * H, dtype=torch.float32, device="cuda")
        y = torch.full((T * H,), float("nan"), dtype=torch.float32, device="cuda")
        pm.moe_layer_fwd(layer.layer, xd, idd, wd, dd, T, K, y_ref, ws, nbytes)
        pm.moe_layer_fwd_noalloc(layer.layer, xd, idd, wd, dd, T, K, y)
        torch.cuda.synchronize()
        assert pm.noalloc_layer_error() == (0, 0)
        got, ref = y.cpu().numpy().reshape(T, H), y_ref.cpu().numpy().reshape(T, H)
        for t in range(T):
            assert_close(got[t], ref[t], msg=f"call {call} (T={T}) token {t}")
        if call == 2:
            o = O.run(E, ids, w, dep, synth.bf16_to_f32(xb).astype(np.float64))
            for t in range(T):
                assert_close(got[t], o[t], msg=f"call {call} token {t} vs oracle")


def test_noalloc_reports_a_missing_plane(layer):
    import bitplane_mixed_precision_b200 as pm
    sens = synth.sensitivities(SEED, 0, E)
    xb, ids, w, dep = _inputs(1, 500, sens)
    e = int(ids[0, 0])
    dep[0, 0] = 2
    saved = int(layer.slot_of[e * 8 + 1])
    layer.slot_of[e * 8 + 1] = -1
    try:
        y = torch.empty(H, dtype=torch.float32, device="cuda")
        pm.moe_layer_fwd_noalloc(layer.layer, torch.from_numpy(xb.view(np.int16)).cuda(),
                                 torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(),
                                 torch.from_numpy(dep).cuda(), 1, K, y)
        assert pm.noalloc_layer_error() == (2, e * 8 + 1)
    finally:
        layer.slot_of[e * 8 + 1] = saved
    pm.moe_layer_fwd_noalloc(layer.layer, torch.from_numpy(xb.view(np.int16)).cuda(), torch.from_numpy(ids).cuda(),
                             torch.from_numpy(w).cuda(), torch.from_numpy(dep).cuda(), 1, K, y)
    assert pm.noalloc_layer_error() == (0, 0)


def test_noalloc_rejects_requests_beyond_its_array(layer):
    import bitplane_mixed_precision_b200 as pm
    T = 2
    while pm.layer_workspace_bytes(T, K, E, H, I) <= pm.noalloc_scratch_bytes():
        T += 1
    x = torch.zeros(T * H, dtype=torch.int16, device="cuda")
    ids = torch.arange(K, dtype=torch.int32, device="cuda").repeat(T)
    with pytest.raises(pm.PmoeError) as ei:
        pm.moe_layer_fwd_noalloc(layer.layer, x, ids, torch.full((T * K,), 0.1, device="cuda"),
                                 torch.ones(T * K, dtype=torch.uint8, device="cuda"), T, K,
                                 torch.empty(T * H, device="cuda"))
    assert ei.value.code == 5
