"""The seeded input generator: determinism, slicing, distributions, bf16 rounding."""
import numpy as np

import synth


def test_deterministic_and_sliceable():
    a = synth.normal(7, synth.TID_W_GATE, (1000,), std=0.02)
    b = synth.normal(7, synth.TID_W_GATE, (1000,), std=0.02)
    assert np.array_equal(a, b)
    part = synth.normal(7, synth.TID_W_GATE, (300,), std=0.02, start=501)
    assert np.array_equal(a[501:801], part)
    c = synth.normal(8, synth.TID_W_GATE, (1000,), std=0.02)
    d = synth.normal(7, synth.TID_W_UP, (1000,), std=0.02)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)


def test_distributions():
    z = synth.normal(3, 1, (400_000,)).astype(np.float64)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01
    # fourth moment of a normal is 3
    assert abs((z ** 4).mean() - 3.0) < 0.1
    u = synth.uniform(3, 2, (400_000,)).astype(np.float64)
    assert u.min() >= 0.0 and u.max() < 1.0 and abs(u.mean() - 0.5) < 0.01


def test_permutation_and_subset():
    p = synth.permutation(5, 9, 256)
    assert sorted(p.tolist()) == list(range(256))
    s = synth.subset(5, 8, 4096, 20)
    assert len(set(s.tolist())) == 20 and np.all(np.diff(s) > 0) and s.max() < 4096


def test_bf16_rounding_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, 1.0 + 2 ** -9, -1.0 - 2 ** -9,
                     3.0e38, 1e-40], dtype=np.float32)
    bits = synth.f32_to_bf16_bits(vals)
    back = (bits.astype(np.uint32) << 16).view(np.float32)
    # bf16 keeps 7 fraction bits: the ulp at 1 is 2^-7, so 1 + 2^-8 is an exact tie (-> even, 1.0)
    assert back[0] == 1.0
    assert back[1] == 1.0
    assert back[2] == np.float32(1.0 + 2 ** -7)
    assert back[3] == 1.0 and back[4] == -1.0
    # rounding error is at most half a bf16 ulp everywhere on a random draw
    x = synth.normal(1, 1, (100_000,))
    xb = (synth.f32_to_bf16_bits(x).astype(np.uint32) << 16).view(np.float32)
    ulp = np.ldexp(1.0, np.frexp(np.abs(x))[1] - 8)
    assert np.all(np.abs(xb.astype(np.float64) - x) <= ulp / 2 + 1e-45)


def test_activations_outliers_and_bf16():
    w = synth.WORKLOADS["decode"]
    oc = w.outlier_channels()
    assert len(oc) == 20
    x, xb = synth.activations(w.data_seed, 64, w.d, oc, w.outlier_factor, True)
    assert np.array_equal((xb.astype(np.uint32) << 16).view(np.float32), x)
    amax = np.abs(x).max(axis=0)
    normal = np.setdiff1d(np.arange(w.d), oc)
    assert amax[oc].min() > amax[normal].max()
    # row slices regenerate the same rows
    x2, _ = synth.activations(w.data_seed, 8, w.d, oc, w.outlier_factor, True, row0=40)
    assert np.array_equal(x2, x[40:48])


def test_zipf_bias():
    b = synth.zipf_bias(3, 256, 1.1)
    assert b.max() == 0.0 and np.isclose(b.min(), -1.1 * np.log(256.0))
    assert len(np.unique(b)) == 256
