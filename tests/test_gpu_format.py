"""GPU format path against the oracle: bit-exact quantiser, packing and prefix extraction."""
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


def test_device_generator_matches_host():
    for stream, start, n in ((synth.stream_id(1, 0, 3, 1), 0, 100000), (77, 5, 3001), (12345, 1, 1)):
        ref = synth.normal_f32(9, stream, n, 0.02, start=start)
        d = torch.empty(n, dtype=torch.float32, device="cuda")
        synth.normal_f32_device(9, stream, n, 0.02, d.data_ptr(), 0, start=start)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(d.cpu().numpy(), ref)


@pytest.mark.parametrize("N,K,G", [(128, 256, 64), (48, 640, 128), (16, 128, 32), (1024, 4096, 128)])
def test_quantize_bit_exact(pm, N, K, G):
    w = synth.expert_weights(3, 0, N % 7, 1, N, K)
    s_ref, c_ref = oracle.quantize(w, G)
    wd = torch.from_numpy(w).cuda()
    s = torch.empty(N * (K // G), dtype=torch.float32, device="cuda")
    c = torch.empty(N * K, dtype=torch.uint8, device="cuda")
    pm.quantize(wd, N, K, G, s, c)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(s.cpu().numpy().reshape(N, K // G), s_ref)
    got = c.cpu().numpy().reshape(N, K)
    bad = np.argwhere(got != c_ref)
    if len(bad):
        # only a weight within rounding distance of a threshold may differ
        t = oracle.thresholds()
        for n, k in bad:
            z = float(w[n, k]) / float(s_ref[n, k // G])
            assert np.min(np.abs(t[1:] - z)) < 1e-12, (n, k, z)


@pytest.mark.parametrize("N,K,depth", [(16, 128, 8), (48, 384, 3), (128, 256, 8), (64, 640, 5),
                                       (1024, 4096, 8)])
def test_device_pack_bit_exact(pm, N, K, depth):
    rng = np.random.default_rng(N * K + depth)
    codes = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    ref = oracle.pack(codes, depth)
    stride = N * K // 32 + 32
    out = torch.full((stride * depth,), -1, dtype=torch.int32, device="cuda")
    pm.pack_bitplanes(torch.from_numpy(codes).cuda(), N, K, depth, out, stride, on_device=True)
    torch.cuda.synchronize()
    o = out.cpu().numpy().view(np.uint32)
    for p in range(depth):
        np.testing.assert_array_equal(o[p * stride: p * stride + N * K // 32], ref[p])
        assert np.all(o[p * stride + N * K // 32: (p + 1) * stride] == 0xFFFFFFFF)


@pytest.mark.parametrize("b", range(1, 9))
def test_extract_prefix_bit_exact(pm, b):
    N, K = 96, 512
    rng = np.random.default_rng(b)
    codes = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    planes = oracle.pack(codes, 8)
    ref = oracle.unpack(planes, N, K, b)
    dp = torch.from_numpy(planes.view(np.int32).reshape(-1)).cuda()
    idx = torch.empty(N * K, dtype=torch.uint8, device="cuda")
    pm.extract_prefix(dp, N * K // 32, N, K, b, idx)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx.cpu().numpy().reshape(N, K), ref)
    np.testing.assert_array_equal(ref, codes >> (8 - b))
