"""Pins for the oracle's tree codebook (Gaussian closed form, tree property).

The codebook follows the PagedMoE podcast transcript, cues 19 and 21: sorted
codewords at the leaves of a binary tree whose parents are frequency-weighted
means of their children, so truncating an index lands on its ancestor.
"""
import math

import numpy as np
import pytest
from scipy import integrate, stats

from conftest import read_golden


def test_depth1_closed_form(oracle_mod):
    cb = oracle_mod.tree_codebook()
    c1 = oracle_mod.level(cb, 1)
    # E[Z | Z >= 0] = 2 phi(0) = sqrt(2/pi)
    assert c1[1] == pytest.approx(math.sqrt(2.0 / math.pi), rel=1e-14)
    assert c1[0] == pytest.approx(-math.sqrt(2.0 / math.pi), rel=1e-14)


def test_every_entry_against_numerical_integration(oracle_mod):
    """C[d][i] = E[Z | Z in [Phi^-1(i/2^d), Phi^-1((i+1)/2^d))], by quadrature."""
    cb = oracle_mod.tree_codebook()
    for d in range(1, 9):
        n = 1 << d
        lv = oracle_mod.level(cb, d)
        for i in range(n):
            a = stats.norm.ppf(i / n)
            b = stats.norm.ppf((i + 1) / n)
            num, _ = integrate.quad(lambda z: z * stats.norm.pdf(z), a, b, epsabs=1e-14, epsrel=1e-12)
            ref = num * n
            assert lv[i] == pytest.approx(ref, rel=2e-9, abs=1e-11), (d, i)


def test_parent_is_mean_of_children(oracle_mod):
    """Parent = frequency-weighted mean of its two children (equal mass here)."""
    cb = oracle_mod.tree_codebook()
    for d in range(2, 9):
        child = oracle_mod.level(cb, d)
        parent = oracle_mod.level(cb, d - 1)
        np.testing.assert_allclose(parent, 0.5 * (child[0::2] + child[1::2]), rtol=0, atol=1e-13)


def test_antisymmetric_sorted_zero_mean(oracle_mod):
    cb = oracle_mod.tree_codebook()
    cbf = oracle_mod.tree_codebook_f32()
    for d in range(1, 9):
        lv = oracle_mod.level(cb, d)
        assert np.all(np.diff(lv) > 0)
        np.testing.assert_allclose(lv, -lv[::-1], rtol=0, atol=1e-13)
        assert abs(lv.sum()) < 1e-12
        lf = oracle_mod.level(cbf, d)
        # float32 table: antisymmetric up to one ulp
        assert np.all(np.abs(lf + lf[::-1]) <= np.spacing(np.abs(lf)))


def test_float_table_is_rounded_double(oracle_mod):
    np.testing.assert_array_equal(oracle_mod.tree_codebook_f32(),
                                  oracle_mod.tree_codebook().astype(np.float32))


def test_distortion_depth1(oracle_mod):
    """1-bit reconstruction MSE of N(0,1) with the sign/conditional-mean quantiser is 1 - 2/pi."""
    cb = oracle_mod.tree_codebook()
    c1 = oracle_mod.level(cb, 1)
    d1 = 1.0 - 0.5 * float(np.sum(c1 ** 2))
    assert d1 == pytest.approx(1.0 - 2.0 / math.pi, rel=1e-12)


def test_golden_truncation_example(oracle_mod):
    """Transcript cues 20-21: index 01 reads its leaf at 2 bits and its parent at 1 bit."""
    cb = oracle_mod.tree_codebook()
    rows = read_golden("tree_truncation_example.txt")
    for bits, leaf, parent in rows:
        code2 = int(bits, 2)
        assert code2 == int(leaf)
        # an 8-bit code whose top two bits are `bits`; its 1-bit prefix is the parent node
        code8 = code2 << 6 | 0b010101
        assert code8 >> 6 == int(leaf)
        assert code8 >> 7 == int(parent)
        # the parent's value is the mean of the two leaves under it
        c2 = oracle_mod.level(cb, 2)
        c1 = oracle_mod.level(cb, 1)
        p = int(parent)
        assert c1[p] == pytest.approx(0.5 * (c2[2 * p] + c2[2 * p + 1]), abs=1e-14)


# Tree from sorted leaves with frequencies (transcript cues 19, 21): every parent is the
# frequency-weighted mean of its children.

def test_tree_from_leaves_equal_mass_is_the_gaussian_tree(oracle_mod):
    """Equal leaf frequencies on the Gaussian conditional-mean leaves: each parent is the plain
    mean of its children, which is the closed-form conditional mean of the merged bin."""
    cb = oracle_mod.tree_codebook()
    t = oracle_mod.tree_from_leaves(oracle_mod.level(cb, 8), np.ones(256))
    np.testing.assert_allclose(t, cb, rtol=0, atol=1e-13)


def test_tree_from_leaves_nodes_are_subtree_weighted_averages(oracle_mod, synth_mod):
    """Every depth-d node equals the frequency-weighted average of the 2^(8-d) leaves below it,
    computed directly from the leaves (numpy's weighted average), not level by level."""
    leaves, freq = synth_mod.tree_leaves(5)
    freq = freq.astype(np.float64)
    t = oracle_mod.tree_from_leaves(leaves, freq)
    for d in range(1, 9):
        lv = oracle_mod.level(t, d)
        span = 1 << (8 - d)
        for i in range(1 << d):
            sl = slice(i * span, (i + 1) * span)
            if freq[sl].sum() > 0:
                want = np.average(leaves[sl].astype(np.float64), weights=freq[sl])
                assert lv[i] == pytest.approx(want, rel=1e-13, abs=1e-14)
    # leaves 7 and 8 have zero frequency: the depth-7 node above leaves 6, 7 is leaf 6, the one
    # above 8, 9 is leaf 9
    assert oracle_mod.level(t, 7)[3] == pytest.approx(float(leaves[6]), rel=1e-15)
    assert oracle_mod.level(t, 7)[4] == pytest.approx(float(leaves[9]), rel=1e-15)


def test_tree_from_leaves_zero_mass_pair_is_plain_mean(oracle_mod):
    leaves = np.linspace(-2.0, 2.0, 256)
    freq = np.ones(256)
    freq[10] = freq[11] = 0.0
    t = oracle_mod.tree_from_leaves(leaves, freq)
    assert oracle_mod.level(t, 7)[5] == pytest.approx(0.5 * (leaves[10] + leaves[11]), rel=1e-15)
    # its parent weighs it by zero mass: the parent is its sibling pair's mean
    assert oracle_mod.level(t, 6)[2] == pytest.approx(0.5 * (leaves[8] + leaves[9]), rel=1e-15)


def test_library_tree_from_leaves_equals_oracle(oracle_mod, synth_mod):
    """The library's host builder (float output) against the oracle rounded to float."""
    import bitplane_mixed_precision_b200 as pm
    for seed in (1, 2, 3):
        leaves, freq = synth_mod.tree_leaves(seed)
        out = np.empty(510, np.float32)
        pm.tree_codebook_from_leaves(leaves, freq, out)
        ref = oracle_mod.tree_from_leaves(leaves, freq.astype(np.float64)).astype(np.float32)
        np.testing.assert_array_equal(out, ref)
    bad = np.empty(510, np.float32)
    with pytest.raises(pm.PmoeError):
        pm.tree_codebook_from_leaves(np.linspace(1, -1, 256).astype(np.float32), np.ones(256, np.float32), bad)
    with pytest.raises(pm.PmoeError):
        fr = np.ones(256, np.float32)
        fr[3] = -1
        pm.tree_codebook_from_leaves(np.linspace(-1, 1, 256).astype(np.float32), fr, bad)
