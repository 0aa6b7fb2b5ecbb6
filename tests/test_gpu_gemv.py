"""pmoe_expert_gemv against the oracle's dequantise-then-matvec (single-matrix case:
K=256 inputs, N=128 outputs, group 64, b swept 1..8), plus other shapes and edges."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pm():
    import bitplane_mixed_precision_b200 as pm
    return pm


def _matrix(pm, seed, N, K, G):
    w = synth.expert_weights(seed, 0, 0, 0, N, K)
    s_ref, c_ref = oracle.quantize(w, G)
    s = torch.empty(N * (K // G), dtype=torch.float32, device="cuda")
    c = torch.empty(N * K, dtype=torch.uint8, device="cuda")
    pm.quantize(torch.from_numpy(w).cuda(), N, K, G, s, c)
    planes = torch.empty(8 * N * K // 32, dtype=torch.int32, device="cuda")
    pm.pack_bitplanes(c, N, K, 8, planes, N * K // 32, on_device=True)
    cb = torch.from_numpy(oracle.tree_codebook_f32()).cuda()
    torch.cuda.synchronize()
    assert np.array_equal(c.cpu().numpy().reshape(N, K), c_ref)
    m = pm.make_matrix(planes, N * K // 32, s, cb, N, K, G)
    return m, (planes, s, cb), (c_ref, s_ref)


@pytest.mark.parametrize("b", range(1, 9))
def test_single_matrix_sweep(pm, b):
    N, K, G = 128, 256, 64
    m, keep, (c_ref, s_ref) = _matrix(pm, 1, N, K, G)
    x = synth.activation_f32(1, 0, 0, K)
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    pm.expert_gemv(m, b, torch.from_numpy(x).cuda(), False, y)
    torch.cuda.synchronize()
    ref = oracle.gemv(c_ref, s_ref, oracle.tree_codebook_f32(), G, b, x.astype(np.float64))
    err, _ = assert_close(y.cpu().numpy(), ref, msg=f"b={b}")
    assert err < 2e-4  # 16-bit fixed-point operands: far inside the bound


@pytest.mark.parametrize("N,K,G,bf16", [(48, 640, 128, True), (16, 128, 32, False), (256, 4096, 128, True),
                                        (1024, 1024, 64, True)])
@pytest.mark.parametrize("b", [1, 2, 3, 4, 5, 8])
def test_shapes(pm, N, K, G, bf16, b):
    m, keep, (c_ref, s_ref) = _matrix(pm, N + K, N, K, G)
    if bf16:
        xb = synth.activation_bf16(2, 0, 0, K)
        xd = torch.from_numpy(xb.view(np.int16)).cuda()
        x64 = synth.bf16_to_f32(xb).astype(np.float64)
    else:
        xf = synth.activation_f32(2, 0, 0, K)
        xd = torch.from_numpy(xf).cuda()
        x64 = xf.astype(np.float64)
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    pm.expert_gemv(m, b, xd, bf16, y)
    torch.cuda.synchronize()
    ref = oracle.gemv(c_ref, s_ref, oracle.tree_codebook_f32(), G, b, x64)
    assert_close(y.cpu().numpy(), ref, msg=f"{N}x{K} G={G} b={b}")


def test_zero_and_unit_inputs(pm):
    N, K, G = 64, 256, 64
    m, keep, (c_ref, s_ref) = _matrix(pm, 5, N, K, G)
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    pm.expert_gemv(m, 3, torch.zeros(K, dtype=torch.float32, device="cuda"), False, y)
    torch.cuda.synchronize()
    assert torch.all(y == 0)
    x = np.zeros(K, np.float32)
    x[200] = 1.0
    pm.expert_gemv(m, 3, torch.from_numpy(x).cuda(), False, y)
    torch.cuda.synchronize()
    ref = oracle.gemv(c_ref, s_ref, oracle.tree_codebook_f32(), G, 3, x.astype(np.float64))
    assert_close(y.cpu().numpy(), ref)


def test_rejects_bad_arguments(pm):
    N, K, G = 16, 128, 64
    m, keep, _ = _matrix(pm, 6, N, K, G)
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    x = torch.zeros(K, dtype=torch.float32, device="cuda")
    for b in (0, 9):
        with pytest.raises(pm.PmoeError):
            pm.expert_gemv(m, b, x, False, y)
    bad = pm.make_matrix(keep[0], N * K // 32, keep[1], keep[2], N, K, 48)
    with pytest.raises(pm.PmoeError):
        pm.expert_gemv(bad, 2, x, False, y)
