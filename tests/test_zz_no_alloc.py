"""The allocation-free layer call against the workspace one.

pmoe_moe_layer_fwd_noalloc serves callers that cannot give the library a
device allocation for scratch (an engine that owns all device memory, a
fixed memory budget): its scratch is a fixed array inside the library. This
checks, through the C ABI, that two calls in a row give the same output as
pmoe_moe_layer_fwd within the tolerance of the other layer tests. The file
sorts last so that a stop-at-first-failure run has run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from bitplane_mixed_precision_b200.store import ResidentLayer
from gpu_common import assert_close, device_fill, tokens

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_call_twice():
    import bitplane_mixed_precision_b200 as pm
    seed, E, H, I, G, k, T = 71, 16, 4096, 1024, 128, 10, 2
    assert pm.layer_workspace_bytes(T, k, E, H, I) <= pm.noalloc_scratch_bytes()
    R = ResidentLayer(E, H, I, G, device_fill(seed))
    sens = synth.sensitivities(seed, 0, E)
    nbytes = pm.layer_workspace_bytes(T, k, E, H, I)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    for call in range(2):
        logits, xb = tokens(seed, T, E, H, token0=10 * call)
        ids, w = oracle.route(logits, k)
        dep = oracle.select(w, ids, sens, 2.5)
        xd = torch.from_numpy(xb.view(np.int16)).cuda()
        idd, wd, dd = torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), torch.from_numpy(dep).cuda()
        y_ref = torch.empty(T * H, dtype=torch.float32, device="cuda")
        y = torch.full((T * H,), float("nan"), dtype=torch.float32, device="cuda")
        pm.moe_layer_fwd(R.layer, xd, idd, wd, dd, T, k, y_ref, ws, nbytes)
        pm.moe_layer_fwd_noalloc(R.layer, xd, idd, wd, dd, T, k, y)
        torch.cuda.synchronize()
        got, ref = y.cpu().numpy().reshape(T, H), y_ref.cpu().numpy().reshape(T, H)
        for t in range(T):
            assert_close(got[t], ref[t], msg=f"call {call} token {t}")


def test_noalloc_rejects_requests_beyond_its_array():
    import bitplane_mixed_precision_b200 as pm
    E, H, I, k = 16, 4096, 1024, 10
    T = 1
    while pm.layer_workspace_bytes(T, k, E, H, I) <= pm.noalloc_scratch_bytes():
        T += 1
    R = ResidentLayer(E, H, I, 128, device_fill(1), experts=[])
    x = torch.zeros(T * H, dtype=torch.int16, device="cuda")
    ids = torch.arange(k, dtype=torch.int32, device="cuda").repeat(T)
    with pytest.raises(pm.PmoeError) as ei:
        pm.moe_layer_fwd_noalloc(R.layer, x, ids, torch.full((T * k,), 0.1, device="cuda"),
                                 torch.ones(T * k, dtype=torch.uint8, device="cuda"), T, k,
                                 torch.empty(T * H, device="cuda"))
    assert ei.value.code == 5
