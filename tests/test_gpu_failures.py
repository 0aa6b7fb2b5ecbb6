"""Failure detection on the GPU without a fault: a bounded device wait that runs
out is reported and the context stays usable.

The layer kernels bound every wait by one deadline per launch. With the limit
set to 1 ns, a wait that is not already satisfied when it is first polled
gives up (the down items' wait for h tiles published by other CTAs always is
at that point), the kernel records error 3 and finishes; the copies it has
issued are still awaited with a separate, long bound before it exits. The
next call with the default limit gives the same output as before, bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from bitplane_mixed_precision_b200.store import ResidentLayer
from gpu_common import device_fill, tokens

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [1, 4])
def test_wait_limit_runs_out_and_the_next_call_is_exact(T):
    import bitplane_mixed_precision_b200 as pm
    seed, E, H, I, G, k = 81, 16, 4096, 1024, 128, 10
    R = ResidentLayer(E, H, I, G, device_fill(seed))
    sens = synth.sensitivities(seed, 0, E)
    logits, xb = tokens(seed, T, E, H)
    ids, w = oracle.route(logits, k)
    dep = oracle.select(w, ids, sens, 2.5)
    args = [torch.from_numpy(xb.view(np.int16)).cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(),
            torch.from_numpy(dep).cuda()]
    nb = pm.layer_workspace_bytes(T, k, E, H, I)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    y_ref = torch.empty(T * H, dtype=torch.float32, device="cuda")
    pm.moe_layer_fwd(R.layer, *args, T, k, y_ref, ws, nb)
    torch.cuda.synchronize()
    assert pm.layer_error(ws) == (0, 0)
    y = torch.empty_like(y_ref)
    pm.set_wait_limit_ns(1)
    try:
        pm.moe_layer_fwd(R.layer, *args, T, k, y, ws, nb)
        torch.cuda.synchronize()
        code, where = pm.layer_error(ws)
    finally:
        pm.set_wait_limit_ns(0)
    assert code == 3, (code, where)
    y.fill_(float("nan"))
    pm.moe_layer_fwd(R.layer, *args, T, k, y, ws, nb)
    torch.cuda.synchronize()
    assert pm.layer_error(ws) == (0, 0)
    assert torch.equal(y, y_ref)
