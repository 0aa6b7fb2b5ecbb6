"""Pins for the oracle's quantiser and bitplane layout.

Layout: plane p holds bit (7-p) of every 8-bit index, MSB first, so a depth-b
request reads exactly planes 0..b-1 (PagedMoE podcast transcript, cue 25;
arxivlens Abstract). The position of a weight's bit inside a plane is this
format's choice; the test at the bottom checks it against its purpose, the
operand-fragment layout of the m16n8k32 8-bit MMA as the PTX ISA documents it.
"""
import numpy as np
import pytest
from scipy import stats

from conftest import read_golden


def test_thresholds_against_library_ppf(oracle_mod):
    t = oracle_mod.thresholds()
    ref = stats.norm.ppf(np.arange(1, 256) / 256.0)
    np.testing.assert_allclose(t[1:], ref, rtol=1e-12, atol=1e-14)
    assert t[128] == 0.0
    np.testing.assert_allclose(t[1:128], -t[255:128:-1], rtol=0, atol=1e-14)


def test_scale_is_population_std(oracle_mod, synth_mod):
    w = synth_mod.expert_weights(7, 0, 3, 0, 32, 256)
    scales, _ = oracle_mod.quantize(w, 64)
    ref = w.astype(np.float64).reshape(32, 4, 64).std(axis=2, ddof=0).astype(np.float32)
    # numpy sums pairwise, the oracle sequentially: equal up to one float ulp
    assert np.all(np.abs(scales - ref) <= np.spacing(ref))


def test_zero_group_and_threshold_tie(oracle_mod):
    """A constant group has zero std -> scale 1; z = 0 sits on t_128 and goes up (half-open bins)."""
    w = np.zeros((16, 128), dtype=np.float32)
    scales, codes = oracle_mod.quantize(w, 64)
    assert np.all(scales == 1.0)
    assert np.all(codes == 128)


def test_codes_monotone_and_bins_equiprobable(oracle_mod, synth_mod):
    w = synth_mod.expert_weights(11, 0, 0, 0, 256, 1024)
    scales, codes = oracle_mod.quantize(w, 128)
    z = w.astype(np.float64) / np.repeat(scales.astype(np.float64), 128, axis=1)
    order = np.argsort(z.ravel(), kind="stable")
    assert np.all(np.diff(codes.ravel()[order].astype(int)) >= 0)
    hist = np.bincount(codes.ravel(), minlength=256)
    chi2 = stats.chisquare(hist)
    assert chi2.pvalue > 1e-4


@pytest.mark.parametrize("b", range(1, 9))
def test_distortion_matches_codebook(oracle_mod, synth_mod, b):
    """Relative weight error at depth b ~ sqrt(1 - 2^-b sum C_b^2) on Gaussian weights."""
    w = synth_mod.expert_weights(3, 0, 1, 0, 256, 2048)
    scales, codes = oracle_mod.quantize(w, 128)
    cb = oracle_mod.tree_codebook_f32().astype(np.float64)
    lv = oracle_mod.level(cb, b)
    wh = np.repeat(scales.astype(np.float64), 128, axis=1) * lv[codes >> (8 - b)]
    rel = np.linalg.norm(wh - w) / np.linalg.norm(w)
    d = 1.0 - np.sum(lv ** 2) / (1 << b)
    # per-group std normalisation thins the tails a little: 0.95-1.0 of sqrt(D_b)
    assert 0.94 * np.sqrt(d) < rel < 1.005 * np.sqrt(d)


def test_pack_roundtrip_and_prefix_invariant(oracle_mod, synth_mod):
    rng = np.random.default_rng(0)
    codes = rng.integers(0, 256, size=(48, 384), dtype=np.uint8)
    planes = oracle_mod.pack(codes, 8)
    assert planes.shape == (8, 48 * 384 // 32)
    np.testing.assert_array_equal(oracle_mod.unpack(planes, 48, 384, 8), codes)
    for b in range(1, 9):
        np.testing.assert_array_equal(oracle_mod.unpack(planes, 48, 384, b), codes >> (8 - b))
        # packing at depth b writes exactly the first b planes of the 8-plane packing
        np.testing.assert_array_equal(oracle_mod.pack(codes, b), planes[:b])
    for p in range(8):
        ones = int(np.unpackbits(planes[p].view(np.uint8)).sum())
        assert ones == int(((codes >> (7 - p)) & 1).sum())


def test_prefix_invariant_exhaustive(oracle_mod):
    """Every 8-bit code at every depth: the depth-b read is the code's top b bits."""
    codes = np.tile(np.arange(256, dtype=np.uint8), 16).reshape(16, 256)
    planes = oracle_mod.pack(codes, 8)
    for b in range(1, 9):
        np.testing.assert_array_equal(oracle_mod.unpack(planes, 16, 256, b), codes >> (8 - b))


def test_pack_rejects_bad_shapes(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.pack(np.zeros((15, 128), np.uint8), 8)
    with pytest.raises(ValueError):
        oracle_mod.pack(np.zeros((16, 100), np.uint8), 8)


def _rotl(x, r):
    return ((x << r) | (x >> (32 - r))) & 0xFFFFFFFF if r else x


def _rotr(x, r):
    return ((x >> r) | (x << (32 - r))) & 0xFFFFFFFF if r else x


@pytest.mark.parametrize("b", [1, 2, 3])
def test_layout_serves_mma_fragments(oracle_mod, b):
    """Reading the planes lane by lane gives the m16n8k32 A fragments.

    PTX ISA, mma.m16n8k32 with .s8 operands: lane = 4*groupID + threadID_in_group;
    register a_i (i = 0..3) holds 4 bytes; byte m of a_i is element
    (row = groupID + 8*(i%2), col = 4*threadID_in_group + m + 16*(i//2)).
    Per lane and 128-column tile, word h of plane p is read, masked with
    rotl(0x11111111 << p, r), OR-ed over planes and rotated right by r, giving
    t-word q = 4h + r = 2s + u whose nibble j holds the b-bit prefix with plane p
    at nibble bit p. Nibbles 0-3 are bytes of a_u, nibbles 4-7 bytes of a_{2+u},
    for k-step s (columns 32s..32s+31).
    """
    rng = np.random.default_rng(b)
    N, K = 32, 256
    codes = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    planes = oracle_mod.pack(codes, 8).astype(np.uint64)
    prefix = codes >> (8 - b)
    ktiles = K // 128
    for R in range(N // 16):
        for Q in range(ktiles):
            tile = R * ktiles + Q
            for lane in range(32):
                g, t = lane // 4, lane % 4
                for q in range(8):
                    h, r = q // 4, q % 4
                    s, u = q // 2, q % 2
                    acc = 0
                    for p in range(b):
                        word = int(planes[p, tile * 64 + 2 * lane + h])
                        acc |= word & _rotl((0x11111111 << p) & 0xFFFFFFFF, r)
                    tw = _rotr(acc, r)
                    for j in range(8):
                        nib = (tw >> (4 * j)) & 0xF
                        # nibble bit p holds plane p (the index's bit b-1-p)
                        idx = 0
                        for p in range(b):
                            idx = (idx << 1) | ((nib >> p) & 1)
                        assert nib >> b == 0
                        reg = u if j < 4 else 2 + u
                        m = j % 4
                        row = g + 8 * (reg % 2)
                        col = 4 * t + m + 16 * (reg // 2)
                        n = 16 * R + row
                        k = 128 * Q + 32 * s + col
                        assert idx == prefix[n, k], (R, Q, lane, q, j)


def test_storage_accounting_golden():
    """Transcript cues 11 and 27: the 8-bit prefix store is 2x a 4-bit copy; independent
    1..8-bit copies cost 36 bits per weight, 9x a 4-bit copy."""
    rows = {r[0]: (int(r[1]), int(r[2])) for r in read_golden("storage_accounting.txt")}
    planes_bits = 8  # one bit per plane per weight, 8 planes
    assert rows["prefix_store"] == (planes_bits, planes_bits // 4)
    indep = sum(range(1, 9))
    assert rows["independent_1_to_8"] == (indep, indep // 4)


def test_codes_equal_threshold_count(oracle_mod, synth_mod):
    """code = #{i in 1..255 : t_i <= w/scale}, checked with numpy's searchsorted."""
    w = synth_mod.expert_weights(21, 0, 2, 1, 64, 512)
    scales, codes = oracle_mod.quantize(w, 128)
    t = oracle_mod.thresholds()[1:]
    z = w.astype(np.float64) / np.repeat(scales.astype(np.float64), 128, axis=1)
    ref = np.searchsorted(t, z, side="right")
    np.testing.assert_array_equal(codes, ref.astype(np.uint8))
