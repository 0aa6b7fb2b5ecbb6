"""GPU routing and prefix selection against the oracle (bit-exact)."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pm():
    import bitplane_mixed_precision_b200 as pm
    return pm


@pytest.mark.parametrize("T,E,k", [(256, 512, 10), (64, 64, 8), (7, 4096, 32), (1, 16, 1)])
def test_route_bit_exact(pm, T, E, k):
    logits = np.stack([synth.router_logits(11, t, 0, E) for t in range(T)])
    ids_ref, w_ref = oracle.route(logits, k)
    d = torch.from_numpy(logits).cuda()
    ids = torch.empty(T * k, dtype=torch.int32, device="cuda")
    w = torch.empty(T * k, dtype=torch.float32, device="cuda")
    pm.route(d, T, E, k, ids, w)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ids.cpu().numpy().reshape(T, k), ids_ref)
    np.testing.assert_array_equal(w.cpu().numpy().reshape(T, k), w_ref)


def test_route_ties_go_to_lower_id(pm):
    logits = np.zeros((2, 40), np.float32)
    logits[0, [3, 9, 17, 30]] = 1.0
    ids_ref, w_ref = oracle.route(logits, 6)
    d = torch.from_numpy(logits).cuda()
    ids = torch.empty(12, dtype=torch.int32, device="cuda")
    w = torch.empty(12, dtype=torch.float32, device="cuda")
    pm.route(d, 2, 40, 6, ids, w)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ids.cpu().numpy().reshape(2, 6), ids_ref)
    np.testing.assert_array_equal(ids_ref[0], [3, 9, 17, 30, 0, 1])
    np.testing.assert_array_equal(w.cpu().numpy().reshape(2, 6), w_ref)


@pytest.mark.parametrize("k,avg", [(10, 2.5), (8, 2.5), (10, 4.0), (32, 1.5), (4, 8.0), (6, 1.0)])
def test_select_bit_exact(pm, k, avg):
    E, T = 512, 400
    sens = synth.sensitivities(7, 0, E)
    logits = np.stack([synth.router_logits(7, t, 0, E) for t in range(T)])
    ids, w = oracle.route(logits, k)
    ref = oracle.select(w, ids, sens, avg)
    out = torch.empty(T * k, dtype=torch.uint8, device="cuda")
    pm.select_prefix(torch.from_numpy(w).cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(sens).cuda(),
                     T, k, avg, out, on_device=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.cpu().numpy().reshape(T, k), ref)
