"""The seeded input generators: determinism and distribution (no method arithmetic here)."""
import numpy as np
from scipy import stats


def test_deterministic_and_stream_separated(synth_mod):
    a = synth_mod.normal_f32(1, 5, 1000)
    b = synth_mod.normal_f32(1, 5, 1000)
    c = synth_mod.normal_f32(1, 6, 1000)
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, c)
    # counter-based: any window of the stream can be generated on its own
    np.testing.assert_array_equal(synth_mod.normal_f32(1, 5, 10, start=333), a[333:343])


def test_normal_distribution(synth_mod):
    z = synth_mod.normal_f64(3, 1, 200000)
    assert abs(z.mean()) < 0.01
    assert abs(z.std() - 1.0) < 0.01
    assert stats.kstest(z, "norm").pvalue > 1e-3


def test_bf16_is_rounded_float(synth_mod):
    f = synth_mod.normal_f32(4, 2, 5000)
    h = synth_mod.normal_bf16(4, 2, 5000)
    back = synth_mod.bf16_to_f32(h)
    assert np.all(np.abs(back - f) <= np.abs(f) * 2.0 ** -8)


def test_workload_helpers(synth_mod):
    s = synth_mod.sensitivities(0, 0, 512)
    assert s.dtype == np.float32 and np.all(s > 0)
    assert abs(np.log(s).std() - 0.5) < 0.06
    p = synth_mod.permutation(0, 77, 512)
    assert sorted(p.tolist()) == list(range(512))
    zb = synth_mod.zipf_bias(0, 512)
    assert zb.max() == 0.0 and abs(zb.min() + 1.1 * np.log(512)) < 1e-5
    ar = synth_mod.ar1_logits(0, 0, 400, 64)
    r = np.corrcoef(ar[:-1].ravel(), ar[1:].ravel())[0, 1]
    assert abs(r - 0.8) < 0.05
